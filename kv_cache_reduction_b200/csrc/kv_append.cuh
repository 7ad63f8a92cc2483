// kv_append.cuh -- scatter new K/V tokens into the full-head cache and the
// sink + ring cache of streaming (or sliding-window) heads.
//
// DuoAttention Laguna Adapter card, sections Summary and Why It Works: a
// full-context head keeps every token; a streaming head keeps a sink of the
// first `sink` tokens and the `recent` most recent ones.  A sliding-window
// layer keeps the last `window` tokens (a ring with no sink).  The ring is
// filled in position order; only tokens that are still in the ring after the
// whole append are written, which gives the same bytes as appending the
// tokens one at a time.
#pragma once

#include "ptx.cuh"

namespace duo {

struct HeadTable {
    int8_t is_full[64];   // per KV head
    int8_t rank[64];      // slot of the head among heads of its kind
};

struct AppendArgs {
    const uint4 *k;       // [B][n_new][Hkv][D] bf16, as 16-byte vectors
    const uint4 *v;
    uint4 *full_k, *full_v;   // [B][n_full][capacity][D]
    uint4 *strm_k, *strm_v;   // [B][n_ring][slots][D]
    const int32_t *seq_len;
    const int32_t *ring_head;
    int64_t capacity;
    int32_t batch, n_new, hkv, n_full, n_ring;
    int32_t sink, ring, slots;    // ring = recent (Duo) or window (sliding)
    HeadTable heads;
};

constexpr int kVecPerRow = 128 * 2 / 16;   // 16 x 16-byte vectors per head row

// One thread copies one 16-byte vector of K and of V.  Rows are
// (b, t, g) triples in input order, so reads are fully coalesced.
__global__ void __launch_bounds__(256) kv_append_scatter(AppendArgs a) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = (int64_t)a.batch * a.n_new * a.hkv;
    if (idx >= rows * kVecPerRow) return;
    const int vec = (int)(idx % kVecPerRow);
    const int64_t row = idx / kVecPerRow;
    const int g = (int)(row % a.hkv);
    const int64_t t = (row / a.hkv) % a.n_new;
    const int b = (int)(row / a.hkv / a.n_new);
    const int64_t n_old = a.seq_len[b];
    const int64_t pos = n_old + t;
    uint4 *dk, *dv;
    if (a.heads.is_full[g]) {
        if (pos >= a.capacity) {
            record_status(-6 /* DUO_ERR_CAPACITY */);
            return;
        }
        const int64_t r = ((int64_t)b * a.n_full + a.heads.rank[g]) * a.capacity + pos;
        dk = a.full_k + r * kVecPerRow;
        dv = a.full_v + r * kVecPerRow;
    } else {
        int64_t slot;
        if (pos < a.sink) {
            slot = pos;
        } else {
            const int64_t n_end = n_old + a.n_new;
            if (pos < n_end - a.ring) return;          // overwritten later in this append
            const int64_t first = n_old > a.sink ? n_old : a.sink;   // first ring position written
            slot = a.sink + ((int64_t)a.ring_head[b] + (pos - first)) % a.ring;
        }
        const int64_t r = ((int64_t)b * a.n_ring + a.heads.rank[g]) * a.slots + slot;
        dk = a.strm_k + r * kVecPerRow;
        dv = a.strm_v + r * kVecPerRow;
    }
    dk[vec] = a.k[idx];
    dv[vec] = a.v[idx];
}

// Moves seq_len and ring_head forward once the scatter has read them.
__global__ void kv_append_commit(int32_t *seq_len, int32_t *ring_head, int32_t batch,
                                 int32_t n_new, int32_t sink, int32_t ring) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    const int64_t n_old = seq_len[b];
    const int64_t n_end = n_old + n_new;
    const int64_t first = n_old > sink ? n_old : sink;
    const int64_t ring_writes = n_end > first ? n_end - first : 0;
    ring_head[b] = (int32_t)(((int64_t)ring_head[b] + ring_writes) % ring);
    seq_len[b] = (int32_t)n_end;
}

}  // namespace duo
