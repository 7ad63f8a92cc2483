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
    int32_t *seq_len;     // read by the copies, moved forward by the commit
    int32_t *ring_head;
    int64_t capacity;
    int32_t batch, n_new, hkv, n_full, n_ring;
    int32_t sink, ring, slots;    // ring = recent (Duo) or window (sliding)
    HeadTable heads;
};

constexpr int kVecPerRow = 128 * 2 / 16;   // 16 x 16-byte vectors per head row

// Where the append of a sequence that holds n_old tokens ends: n_old + n_new,
// or the full cache's capacity when the layer has full heads and the append
// would pass it.  The tokens from there on are dropped for every head (the
// scatter records DUO_ERR_CAPACITY), so that seq_len never exceeds the
// capacity and a later decode never reads past a full head's rows.
__device__ __forceinline__ int64_t append_end(int64_t n_old, int32_t n_new, int32_t n_full, int64_t capacity) {
    const int64_t n_end = n_old + n_new;
    if (n_full == 0 || n_end <= capacity) return n_end;
    return n_old > capacity ? n_old : capacity;
}

// Cache row that token t of sequence b writes for KV head g (*full tells
// which cache), or -1 when it writes none: a ring position that a later token
// of the same append overwrites, or a token past the capacity (status set).
__device__ __forceinline__ int64_t append_row(const AppendArgs &a, int b, int g, int64_t t, bool *full) {
    const int64_t n_old = a.seq_len[b];
    const int64_t pos = n_old + t;
    const int64_t n_end = append_end(n_old, a.n_new, a.n_full, a.capacity);
    *full = a.heads.is_full[g] != 0;
    if (pos >= n_end) {
        record_status(-6 /* DUO_ERR_CAPACITY */);
        return -1;
    }
    if (*full) return ((int64_t)b * a.n_full + a.heads.rank[g]) * a.capacity + pos;
    int64_t slot;
    if (pos < a.sink) {
        slot = pos;
    } else {
        if (pos < n_end - a.ring) return -1;               // overwritten later in this append
        const int64_t first = n_old > a.sink ? n_old : a.sink;   // first ring position written
        slot = a.sink + ((int64_t)a.ring_head[b] + (pos - first)) % a.ring;
    }
    return ((int64_t)b * a.n_ring + a.heads.rank[g]) * a.slots + slot;
}

// One thread copies one 16-byte vector of K and of V.  Rows are
// (b, t, g) triples in input order, so reads are fully coalesced.
__global__ void __launch_bounds__(256) kv_append_scatter(AppendArgs a) {
    pdl_wait();        // launched as a programmatic dependent of the previous kernel
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = (int64_t)a.batch * a.n_new * a.hkv;
    if (idx >= rows * kVecPerRow) return;
    const int vec = (int)(idx % kVecPerRow);
    const int64_t row = idx / kVecPerRow;
    const int g = (int)(row % a.hkv);
    const int64_t t = (row / a.hkv) % a.n_new;
    const int b = (int)(row / a.hkv / a.n_new);
    bool full = false;
    const int64_t r = append_row(a, b, g, t, &full);
    if (r < 0) return;
    uint4 *dk = (full ? a.full_k : a.strm_k) + r * kVecPerRow;
    uint4 *dv = (full ? a.full_v : a.strm_v) + r * kVecPerRow;
    dk[vec] = a.k[idx];
    dv[vec] = a.v[idx];
}

// Moves sequence b's seq_len and ring_head forward (to the append's end, which
// stops at the capacity as append_end says); every read of them is done.
__device__ __forceinline__ void commit_sequence(int32_t *seq_len, int32_t *ring_head, int b, int32_t n_new,
                                                int32_t sink, int32_t ring, int32_t n_full, int64_t capacity) {
    const int64_t n_old = seq_len[b];
    const int64_t n_end = append_end(n_old, n_new, n_full, capacity);
    const int64_t first = n_old > sink ? n_old : sink;
    const int64_t ring_writes = n_end > first ? n_end - first : 0;
    ring_head[b] = (int32_t)(((int64_t)ring_head[b] + ring_writes) % ring);
    seq_len[b] = (int32_t)n_end;
}

// Moves seq_len and ring_head forward once the scatter has read them.
__global__ void kv_append_commit(int32_t *seq_len, int32_t *ring_head, int32_t batch, int32_t n_new,
                                 int32_t sink, int32_t ring, int32_t n_full, int64_t capacity) {
    pdl_wait();        // the scatter has read seq_len and ring_head
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    commit_sequence(seq_len, ring_head, b, n_new, sink, ring, n_full, capacity);
}

// A short append (a decode step, a verify block) in one launch: one CTA per
// sequence copies that sequence's n_new x Hkv rows (16-byte vectors in input
// order, as the scatter does) and then moves its seq_len and ring_head
// forward itself: no other CTA reads them, so the commit needs no second
// kernel.
constexpr int kAppendSmallThreads = 256;
constexpr int kAppendSmallMaxVecs = 4096;     // n_new x Hkv x 16 vectors of a sequence, at most

__global__ void __launch_bounds__(kAppendSmallThreads) kv_append_small(AppendArgs a) {
    pdl_wait();        // launched as a programmatic dependent of the previous kernel
    const int b = blockIdx.x;
    const int per_seq = a.n_new * a.hkv * kVecPerRow;
    const int64_t base = (int64_t)b * per_seq;
    for (int i = threadIdx.x; i < per_seq; i += kAppendSmallThreads) {
        const int vec = i % kVecPerRow;
        const int row = i / kVecPerRow;            // t * Hkv + g
        const int g = row % a.hkv;
        const int64_t t = row / a.hkv;
        bool full = false;
        const int64_t r = append_row(a, b, g, t, &full);
        if (r < 0) continue;
        (full ? a.full_k : a.strm_k)[r * kVecPerRow + vec] = a.k[base + i];
        (full ? a.full_v : a.strm_v)[r * kVecPerRow + vec] = a.v[base + i];
    }
    __syncthreads();   // this CTA's reads of seq_len[b] and ring_head[b] are done
    if (threadIdx.x == 0)
        commit_sequence(a.seq_len, a.ring_head, b, a.n_new, a.sink, a.ring, a.n_full, a.capacity);
}

}  // namespace duo
