// prefill.cuh -- causal / banded FlashAttention-style prefill on tcgen05.
//
// What each query row attends to (DuoAttention Laguna Adapter card, Summary
// and Why It Works; Laguna sliding-window articles): a full-context KV head
// every key j <= i; a streaming head the sink j < sink plus the recent keys
// i - recent < j <= i; a sliding-window layer the keys i - window < j <= i.
// An optional per-query-head sink logit (Laguna XS 2.1 article, attention
// sinks) joins the softmax denominator with a zero value vector.
//
// A CTA computes 128-row query tiles for two query heads of one GQA group,
// so both heads share every K/V tile in shared memory.  CTAs are persistent
// (one per SM) and take (sequence, head pair, query tile) work tiles from a
// list ordered heaviest first: each claims its next one from an atomic
// counter when it is ready for it.  Keys come in 128-key tiles.
//   warps 0-3  softmax of head 0, warps 4-7 softmax of head 1: one thread per
//              query row holds the row's 128 scores of a key tile, so the row
//              max needs no exchange between threads; they write P (bf16)
//              back over the first 64 columns of S, rescale O in TMEM only when
//              the running max grew by more than 2^8, and at the end of each
//              work tile write O / l (times the output gate, if any) by TMA
//              stores and the log-sum-exp.  A share of the exponentials runs
//              on the FMA pipe (ex2_poly2) beside the MUFU units
//   warp 8     TMA producer: claims the work tiles (an atomic counter in the
//              caller's workspace, else a static stride over the list) and
//              hands them on through a shared-memory ring; loads Q of both
//              heads per work tile, K and V tiles into a two-stage ring
//              (128-byte swizzled, no multicast)
//   warp 9     TMEM allocator and MMA issuer (one thread), in the order
//                PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ...
//              with S_h = Q_h K^T (both operands in shared memory) and
//              O_h += P_h V (P_h read from tensor memory).  S_h(j+1) overwrites
//              the columns PV_h(j) reads; the tcgen05 MMAs of one thread execute
//              in issue order, so it is issued right behind it without a wait.
//              The same holds across work tiles: the next work tile's first
//              S_h follows this one's last PV_h.
// TMEM: S0 | S1 | O0 | O1, 128 fp32 columns each (512 in total).  Key tiles
// that no row of a query tile attends to are never loaded.
#pragma once

#include <cuda.h>

#include <atomic>

#include "ptx.cuh"

namespace duo {

constexpr int kPfM = 128;                  // query rows per tile
constexpr int kPfN = 128;                  // keys per tile
constexpr int kPfThreads = 512;            // 16 warps
constexpr int kPfEpiWarp0 = 8, kPfProducerWarp = 12, kPfMmaWarp = 13;   // warps 14, 15 only balance the split
// Register split (setmaxnreg): the block launches with 128 registers per thread;
// the 8 softmax warps take 192, the 4 epilogue warps keep 80, the producer, the
// MMA issuer and the two spare warps 48: 8*32*192 + 4*32*80 + 4*32*48 = 512*128,
// and each SM sub-partition (warps k, k+4, k+8, k+12) holds 192+192+80+48 = 512
// registers per lane, its whole register file.
constexpr int kPfLaunchRegs = 128, kPfSoftmaxRegs = 192, kPfEpiRegs = 80, kPfOtherRegs = 48;
static_assert(8 * 32 * kPfSoftmaxRegs + 4 * 32 * kPfEpiRegs + 4 * 32 * kPfOtherRegs == kPfThreads * kPfLaunchRegs,
              "register split");
// Pairs of each 16-pair chunk of a row whose exponentials run on the FMA pipe
// (ex2_poly2) instead of the MUFU units.
#ifndef DUO_PF_POLY_PAIRS
#define DUO_PF_POLY_PAIRS 0
#endif
constexpr int kPfPolyPairs = DUO_PF_POLY_PAIRS;
// The two heads take turns for their exponentials (1: on), so that the MUFU
// units serve one head while the tensor core runs the other head's products.
#ifndef DUO_PF_TURNS
#define DUO_PF_TURNS 0
#endif
constexpr bool kPfTurns = DUO_PF_TURNS != 0;
constexpr int kPfStages = 2;
constexpr int kPfSlots = 4;                // work-tile ring between the producer and the consumers
constexpr uint32_t kQTileBytes = kPfM * 128 * 2;     // 32 KB: one head's Q tile
constexpr uint32_t kQHalfBytes = kQTileBytes / 2;    // 64-column swizzled box
constexpr uint32_t kKVTileBytes = kPfN * 128 * 2;    // 32 KB: one K or V tile
constexpr uint32_t kKVHalfBytes = kKVTileBytes / 2;
constexpr uint32_t kPfStageBytes = 2 * kKVTileBytes;
constexpr uint32_t kOStageBytes = 32 * 16 * 2;    // one O chunk of a softmax warp: 32 rows x 16 columns
// each softmax warp stages its O chunks in two alternating buffers
constexpr size_t kPfSmem = 1024 + 2 * kQTileBytes + kPfStages * kPfStageBytes + 4 * 2 * kOStageBytes;

enum : int { kKindFull = 0, kKindStreaming = 1, kKindSliding = 2 };

struct PrefillArgs {
    CUtensorMap tm_q;      // [B][L][Hq][128] bf16, box 64 x 1 x 128 x 1
    CUtensorMap tm_k;      // [B][L][Hkv][128]
    CUtensorMap tm_v;
    CUtensorMap tm_o;      // out [B][L][Hq][128] bf16, box 16 x 1 x 32 x 1, no swizzle
    float *lse;            // [B][Hq][L] or null
    const float *sink_logit;
    int32_t *work_counter; // zeroed before the launch, or null for the static order
    const __nv_bfloat16 *gate;  // output gate pre-activations or null
    // gate layout: kGate 1 [B][L][Hq][128], kGate 2 [B][L][Hq]
    int32_t L, hq, hkv, n_qtiles, n_work, batch_pairs;
    int32_t sink, recent, window;
    int32_t withhold_tile; // failure-injection hook: CTA 0 issues no K/V load from this tile on (-1: off)
    float scale_log2;
    int8_t kind[64];       // per KV head
    // The block's keys: in prompt mode, seq_len (or null) gives the position each
    // sequence's block starts at, which shifts the sink.  In cache mode (the block's
    // queries against the cache as it stands before the block), tm_k / tm_v map the
    // full caches [B][n_full][capacity][128] as (128, capacity, n_full, B) and
    // tm_k2 / tm_v2 the sink + ring caches [B][n_ring][slots][128] as
    // (128, slots, n_ring, B); seq_len holds each sequence's cached tokens.
    CUtensorMap tm_k2, tm_v2;
    const int32_t *seq_len, *ring_head;
    int32_t capacity;
    // cache mode: a full head's cached key tiles are cut into kv_splits chunks of
    // split_tiles tiles, each its own work tile writing O and the LSE to slice s
    // of out ([S][B][L][Hq][128]) and lse ([S][B][Hq][L]); ring heads use slice 0
    // only.  Prompt mode: 1.
    int32_t kv_splits, split_tiles, batch;
    int8_t rank[64];       // cache mode: per KV head, its rank among heads of its kind
};

// Key tiles of query tile t for one head kind: an optional run of sink
// tiles [0, n_sink_tiles) followed by the band [band_lo, last].
struct TileList {
    int n_sink_tiles, band_lo, last;
    __device__ int count() const { return n_sink_tiles + (last - band_lo + 1); }
    __device__ int at(int j) const { return j < n_sink_tiles ? j : band_lo + (j - n_sink_tiles); }
};

__device__ __forceinline__ TileList tile_list(int kind, int t, int L, int sink, int recent, int window) {
    // keys past the last query of the tile, or past the sequence, are never attended
    TileList tl{0, 0, min((t * kPfM + kPfM - 1) / kPfN, (L - 1) / kPfN)};
    if (kind == kKindFull) return tl;
    const int span = kind == kKindStreaming ? recent : window;
    const int first = t * kPfM - span + 1;           // lowest key of the band (row t*128)
    tl.band_lo = first <= 0 ? 0 : first / kPfN;
    if (kind == kKindStreaming && sink > 0) {
        const int st = (sink + kPfN - 1) / kPfN;
        if (st < tl.band_lo) tl.n_sink_tiles = st;
        else tl.band_lo = 0;                           // sink and band tiles merge
    }
    return tl;
}

// Bits lo..hi of a 64-bit column mask (clamped to 0..63; empty when lo > hi).
__device__ __forceinline__ uint64_t col_range_bits(int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, 63);
    if (lo > hi) return 0ull;
    const uint64_t upto = hi == 63 ? ~0ull : ((1ull << (hi + 1)) - 1ull);
    return upto & (~0ull << lo);
}

// True when every (row, key) pair of the tile is attended.
__device__ __forceinline__ bool tile_dense(int kind, int r0, int c0, int sink, int recent, int window) {
    const int r1 = r0 + kPfM - 1, c1 = c0 + kPfN - 1;
    if (c1 > r0) return false;                         // crosses the diagonal
    if (kind == kKindFull) return true;
    if (kind == kKindStreaming) return c1 < sink || c0 > r1 - recent;
    return c0 > r1 - window;
}

// The key tiles of a work tile.  Prompt mode: the TileList of its query tile
// (with this sequence's sink).  Cache mode: tiles [0, count) of the head's
// cache (a full head's rows, a ring head's slots), never empty: a work tile with
// no cached key gets one tile in which every key is masked.
struct PfKeys {
    TileList tl;
    int sink;              // prompt mode: the sink keys among the block's keys
    int n, ns, cnt, rh;    // cache mode: cached tokens, sink slots and ring slots holding
                           // one, ring cursor
    __device__ int count() const { return tl.count(); }
    __device__ int at(int j) const { return tl.at(j); }
};

// Work tile w: query tile t (heaviest first) of head pair p of sequence b.
struct PfWork {
    int b, h0, g, t, s;    // s: the split of the cached keys (cache mode)
};

__device__ __forceinline__ PfWork work_of(const PrefillArgs &a, int w) {
    const int pairs = a.hq / 2;
    const int per_t = a.batch_pairs * a.kv_splits;
    PfWork wk;
    wk.t = a.n_qtiles - 1 - w / per_t;
    const int bp = (w % per_t) / a.kv_splits;
    wk.s = w % a.kv_splits;
    wk.b = bp / pairs;
    wk.h0 = (bp % pairs) * 2;
    wk.g = wk.h0 / (a.hq / a.hkv);
    return wk;
}

template <bool kCache>
__device__ __forceinline__ PfKeys pf_keys(const PrefillArgs &a, const PfWork &wk) {
    PfKeys k{};
    const int kind = a.kind[wk.g];
    if (!kCache) {
        k.sink = a.seq_len != nullptr ? max(0, a.sink - a.seq_len[wk.b]) : a.sink;
        k.tl = tile_list(kind, wk.t, a.L, k.sink, a.recent, a.window);
        return k;
    }
    k.n = max(a.seq_len[wk.b], 0);
    int tiles;
    if (kind == kKindFull) {
        k.n = min(k.n, a.capacity);                    // a full head's rows end at the capacity
        tiles = (k.n + kPfN - 1) / kPfN;
        if (wk.s > 0 || tiles > a.split_tiles) {
            // split s: tiles [s * split_tiles, ...); empty past the head's rows
            // (split 0 of an empty cache keeps its one masked tile)
            const int lo = wk.s * a.split_tiles, hi = min(tiles, lo + a.split_tiles);
            k.tl = TileList{0, lo, hi - 1};
            if (hi <= lo) k.tl = TileList{0, 0, wk.s == 0 ? 0 : -1};
            return k;
        }
    } else {
        // R = a.recent (the window on a sliding layer, whose sink is 0)
        k.ns = min(k.n, a.sink);
        k.cnt = min(max(k.n - a.sink, 0), a.recent);
        k.rh = a.ring_head[wk.b];
        // rows i >= R - 1 of the block see no ring slot, only the sink
        const bool ring_seen = k.cnt > 0 && wk.t * kPfM < a.recent - 1;
        tiles = ring_seen ? (a.sink + a.recent + kPfN - 1) / kPfN : (k.ns + kPfN - 1) / kPfN;
        if (wk.s > 0) tiles = -1;                      // ring heads: split 0 only
    }
    k.tl = TileList{0, 0, tiles < 0 ? -1 : max(tiles, 1) - 1};
    return k;
}

// Cache mode: the attended columns of key tile c0 for block row i, as 128 bits
// (w[0] columns 0-31 ... w[3] columns 96-127).  A full head sees its cached rows;
// a ring head its sink slots holding a token and the ring slots holding one of
// positions n - 1 - d > n + i - R, i.e. d < R - 1 - i (d-th to last written): a
// cyclic run of slots ending before the ring cursor.
__device__ __forceinline__ void cache_mask(const PrefillArgs &a, const PfKeys &k, int kind, int i, int c0,
                                           uint32_t (&w)[4]) {
    int lo[3] = {1, 1, 1}, hi[3] = {0, 0, 0};       // up to three ranges of columns
    if (kind == kKindFull) {
        lo[0] = -c0;
        hi[0] = k.n - 1 - c0;
    } else {
        lo[0] = -c0;
        hi[0] = k.ns - 1 - c0;
        const int R = a.recent, S = a.sink;
        const int len = min(k.cnt, R - 1 - i);
        if (len > 0) {
            const int r_end = (k.rh - 1 + R) % R, r_start = r_end - len + 1;
            if (r_start >= 0) {
                lo[1] = S + r_start - c0;
                hi[1] = S + r_end - c0;
            } else {
                lo[1] = S - c0;
                hi[1] = S + r_end - c0;
                lo[2] = S + R + r_start - c0;
                hi[2] = S + R - 1 - c0;
            }
        }
    }
    uint64_t m0 = 0, m1 = 0;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        m0 |= col_range_bits(lo[q], hi[q]);
        m1 |= col_range_bits(lo[q] - 64, hi[q] - 64);
    }
    w[0] = (uint32_t)m0;
    w[1] = (uint32_t)(m0 >> 32);
    w[2] = (uint32_t)m1;
    w[3] = (uint32_t)(m1 >> 32);
}

// Cache mode: does key e (a full head's row, a ring head's slot) hold a token?
// (Rows past the cache's end are zero-filled by the tensor map.)
__device__ __forceinline__ bool cache_key_valid(const PrefillArgs &a, const PfKeys &k, int kind, int e) {
    if (kind == kKindFull) return e < k.n || e >= a.capacity;
    const int S = a.sink, R = a.recent;
    if (e < S) return e < k.ns;
    if (e >= S + R) return true;
    const int d = ((k.rh - 1 - (e - S)) % R + R) % R;
    return d < k.cnt;
}

// kGate: 0 no output gate, 1 one gate per (head, channel), 2 one gate per head
// kCache: the block's queries against the cache (see PrefillArgs), else a prompt
template <int kGate, bool kCache>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_fwd(const __grid_constant__ PrefillArgs a) {
    extern __shared__ __align__(16) char psmem_base[];
    char *smem = psmem_base + ((1024u - (smem_u32(psmem_base) & 1023u)) & 1023u);
    char *sQ = smem;                                   // [2 heads][32 KB]
    char *sKV = smem + 2 * kQTileBytes;                // [stages][K 32 KB | V 32 KB]
    char *sO = sKV + kPfStages * kPfStageBytes;        // [epilogue warp][2][32 rows][16 columns] bf16
    __shared__ uint64_t q_full, q_empty, kv_full[kPfStages], kv_empty[kPfStages];
    __shared__ uint64_t vprep[kPfStages];             // cache mode: the stage's invalid V rows are zeroed
    __shared__ uint64_t s_full[2], p_full[2], o_done[2], mma_drained;
    // a work tile's rows handed from the softmax to the epilogue warps: (running
    // max, sum) per row, double-buffered by work tile; O of a head is free again
    // once the epilogue has read it
    // ml_full alternates with the work tile's parity like row_ml: the softmax
    // may finish a one-tile work tile before the epilogue has waited for the
    // one before it, and must not complete two phases of one barrier
    __shared__ uint64_t ml_full[2][2], o_free[2];     // [work tile parity][head], [head]
    __shared__ uint64_t turn[2];                      // the heads' turns on the MUFU units
    __shared__ float4 row_ml[2][2][kPfM];             // [work tile parity][head][row]: m, l, l exact
    // work tiles claimed by the producer, read by the MMA issuer and the softmax warps
    __shared__ uint64_t work_full[kPfSlots], work_empty[kPfSlots];
    __shared__ int work_slot[kPfSlots];
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&q_full, 1);
        mbar_init(&q_empty, 1);
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&vprep[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&s_full[h], 1);
            mbar_init(&p_full[h], 4);           // the head's four softmax warps
            mbar_init(&o_done[h], 1);
            mbar_init(&ml_full[0][h], 4);
            mbar_init(&ml_full[1][h], 4);
            mbar_init(&o_free[h], 4);           // the four epilogue warps
            mbar_init(&turn[h], 4);
        }
        for (int w4 = 0; w4 < 4; ++w4) mbar_arrive(&turn[0]);   // head 0 takes the first turn
        for (int sl = 0; sl < kPfSlots; ++sl) {
            mbar_init(&work_full[sl], 1);
            // the MMA issuer, 8 softmax and 4 epilogue warps (and the V preparation warp)
            mbar_init(&work_empty[sl], kCache ? 14 : 13);
        }
        mbar_init(&mma_drained, 1);
        fence_mbar_init();
    }
    if (warp == kPfMmaWarp) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    __syncwarp();      // reconverge before the CTA barrier (bar.sync is warp-aligned)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // cache mode: the next grid (the block's own keys) may take each SM this CTA
    // leaves; it does not read what this grid writes
    if (kCache) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = tmem_base;
    // each role sets its register budget first thing in its own branch, so that
    // the compiler allocates that branch's code within it
    if (warp == kPfProducerWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfOtherRegs));
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&a.tm_q);
            prefetch_tmap(&a.tm_o);
            if (!kCache) {             // (in cache mode a layer may lack one kind's maps)
                prefetch_tmap(&a.tm_k);
                prefetch_tmap(&a.tm_v);
            }
            int jg = 0;
            bool ok = true;
            // cache mode: work tiles with no key tile (a ring head's splits past the
            // first, a split past a full head's rows) are passed over, unpublished
            auto claim = [&](int wn) {
                while (kCache && wn < a.n_work && pf_keys<kCache>(a, work_of(a, wn)).count() == 0)
                    wn = a.work_counter != nullptr ? (int)gridDim.x + atomicAdd(a.work_counter, 1)
                                                   : wn + (int)gridDim.x;
                return wn;
            };
            int w = claim(blockIdx.x);
            for (int wc = 0; ok; ++wc) {
                // publish the work tile (an index >= n_work tells the consumers to stop)
                const int sl = wc % kPfSlots;
                if (wc >= kPfSlots && !(ok = mbar_wait(&work_empty[sl], ((wc / kPfSlots) - 1) & 1))) break;
                work_slot[sl] = w;
                mbar_arrive(&work_full[sl]);
                if (w >= a.n_work) break;
                // claim the next one now: the atomic's latency hides behind this tile's loads.
                // Claims follow the heaviest-first order, so every CTA takes the next
                // tile when it is free (longest-processing-time-first scheduling)
                const int w_next = claim(a.work_counter != nullptr ? (int)gridDim.x + atomicAdd(a.work_counter, 1)
                                                                   : w + (int)gridDim.x);
                const PfWork wk = work_of(a, w);
                const PfKeys tl = pf_keys<kCache>(a, wk);
                // Q of the previous work tile must no longer be read by the MMA
                if (wc > 0 && !(ok = mbar_wait(&q_empty, (wc - 1) & 1))) break;
                mbar_expect_tx(&q_full, 2 * kQTileBytes);
                for (int h = 0; h < 2; ++h)
                    for (int half = 0; half < 2; ++half)
                        tma_load_4d(sQ + h * kQTileBytes + half * kQHalfBytes, &a.tm_q, half * 64,
                                    wk.h0 + h, wk.t * kPfM, wk.b, &q_full);
                const int n_kv = tl.count();
                for (int j = 0; j < n_kv; ++j, ++jg) {
                    const int st = jg % kPfStages;
                    if (jg >= kPfStages && !(ok = mbar_wait(&kv_empty[st], ((jg / kPfStages) - 1) & 1))) break;
                    // failure-detection test: stop feeding this CTA so that its
                    // consumers' bounded waits expire (nothing stays in flight)
                    if (blockIdx.x == 0 && jg == a.withhold_tile) { ok = false; break; }
                    const int row = tl.at(j) * kPfN;
                    char *kst = sKV + st * kPfStageBytes;
                    mbar_expect_tx(&kv_full[st], kPfStageBytes);
                    if (kCache) {
                        // the head's cache: (channel, row, rank, sequence)
                        const bool full = a.kind[wk.g] == kKindFull;
                        const CUtensorMap *mk = full ? &a.tm_k : &a.tm_k2, *mv = full ? &a.tm_v : &a.tm_v2;
                        for (int half = 0; half < 2; ++half) {
                            tma_load_4d(kst + half * kKVHalfBytes, mk, half * 64, row, a.rank[wk.g], wk.b, &kv_full[st]);
                            tma_load_4d(kst + kKVTileBytes + half * kKVHalfBytes, mv, half * 64, row, a.rank[wk.g],
                                        wk.b, &kv_full[st]);
                        }
                    } else {
                        for (int half = 0; half < 2; ++half) {
                            tma_load_4d(kst + half * kKVHalfBytes, &a.tm_k, half * 64, wk.g, row, wk.b, &kv_full[st]);
                            tma_load_4d(kst + kKVTileBytes + half * kKVHalfBytes, &a.tm_v, half * 64, wk.g, row,
                                        wk.b, &kv_full[st]);
                        }
                    }
                }
                w = w_next;
            }
        }
        __syncwarp();  // lanes 1..31 wait for the producer lane before the CTA barrier
    } else if (warp == kPfMmaWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfOtherRegs));
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16_f32(kPfM, kPfN, 0, 0);
            const uint32_t id_pv = idesc_bf16_f32(kPfM, 128, 0, 1);
            const uint32_t q_addr = smem_u32(sQ), kv_addr = smem_u32(sKV);
            auto issue_qk = [&](int h, int st) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t qoff = h * kQTileBytes + (k >> 2) * kQHalfBytes + (k & 3) * 32;
                    const uint32_t koff = st * kPfStageBytes + (k >> 2) * kKVHalfBytes + (k & 3) * 32;
                    mma_ss(tmem + h * 128, smem_desc_sw128(q_addr + qoff, 16, 1024),
                           smem_desc_sw128(kv_addr + koff, 16, 1024), id_qk, k > 0);
                }
                mma_commit(&s_full[h]);
            };
            auto issue_pv = [&](int h, int st, bool first) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(tmem + 256 + h * 128, tmem + h * 128 + k * 8,
                           smem_desc_sw128(kv_addr + st * kPfStageBytes + kKVTileBytes + k * 2048,
                                           kKVHalfBytes, 1024),
                           id_pv, (first && k == 0) ? 0u : 1u);
                mma_commit(&o_done[h]);
            };
            // the work tile index of slot wc (an index >= n_work ends the list)
            auto fetch = [&](int wcx, int *wout) -> bool {
                const int sl = wcx % kPfSlots;
                if (!mbar_wait(&work_full[sl], (wcx / kPfSlots) & 1)) return false;
                *wout = work_slot[sl];
                mbar_arrive(&work_empty[sl]);
                return true;
            };
            auto kv_count = [&](int w) {
                const PfWork wk = work_of(a, w);
                return pf_keys<kCache>(a, wk).count();
            };
            int jg = 0, wc = 0, w = 0;
            bool ok = fetch(0, &w);
            int n_kv = 0;
            if (ok && w < a.n_work) {
                n_kv = kv_count(w);
                ok = mbar_wait(&q_full, 0) && mbar_wait(&kv_full[0], 0);
                if (ok) {
                    tc_fence_after();
                    issue_qk(0, 0);
                    issue_qk(1, 0);
                    if (n_kv == 1) mma_commit(&q_empty);
                }
            }
            // Each work tile's first S products are issued right behind the previous
            // work tile's last PV of the same head, so that the tensor core has them
            // while the softmax warps run that work tile's epilogue.
            while (ok && w < a.n_work) {
                int w_next = a.n_work, n_kv_next = 0;
                for (int j = 0; j < n_kv && ok; ++j, ++jg) {
                    const int st = jg % kPfStages;
                    const int st1 = (jg + 1) % kPfStages;
                    const bool last = j + 1 == n_kv;
                    if (last) {
                        if (!(ok = fetch(wc + 1, &w_next))) break;
                        if (w_next < a.n_work) n_kv_next = kv_count(w_next);
                    }
                    const bool more = !last || w_next < a.n_work;
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!(ok = mbar_wait(&p_full[h], jg & 1))) break;
                        // the first PV of a work tile overwrites O: the epilogue of the
                        // previous one must have read it
                        if (j == 0 && wc > 0 && !(ok = mbar_wait(&o_free[h], (wc - 1) & 1))) break;
                        // cache mode: the V rows of keys that hold no token are zeroed first
                        if (kCache && h == 0 && !(ok = mbar_wait(&vprep[st], (jg / kPfStages) & 1))) break;
                        tc_fence_after();
                        issue_pv(h, st, j == 0);
                        if (more) {
                            if (h == 0) {
                                if (last && !(ok = mbar_wait(&q_full, (wc + 1) & 1))) break;   // next Q
                                if (!(ok = mbar_wait(&kv_full[st1], ((jg + 1) / kPfStages) & 1))) break;
                            }
                            tc_fence_after();
                            issue_qk(h, st1);
                        }
                    }
                    if (!ok) break;
                    mma_commit(&kv_empty[st]);
                    // Q of a work tile is free once its last S products are issued
                    if (!last && j + 2 == n_kv) mma_commit(&q_empty);
                    if (last && more && n_kv_next == 1) mma_commit(&q_empty);
                }
                w = w_next;
                n_kv = n_kv_next;
                ++wc;
            }
            // every product issued has completed before the tensor memory is freed
            // (on an early exit some may still run)
            mma_commit(&mma_drained);
            mbar_wait(&mma_drained, 0);
        }
        __syncwarp();  // lanes 1..31 wait for the MMA lane before the CTA barrier
    } else if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPfSoftmaxRegs));
        // ------------------------------------------------------------ softmax
        const int h = warp >> 2;                       // head of the pair
        const int quarter = warp & 3;                  // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;             // query row within the tile
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_tmem = tmem + h * 128 + lane_base;
        const uint32_t o_tmem = tmem + 256 + h * 128 + lane_base;
        const float c = a.scale_log2;
        int jg = 0;
        bool ok = true;
        for (int wc = 0; ok; ++wc) {
            const int sl = wc % kPfSlots;
            const bool have = mbar_wait(&work_full[sl], (wc / kPfSlots) & 1);
            __syncwarp();
            if (!__all_sync(0xffffffffu, have)) { ok = false; break; }
            const int w = work_slot[sl];
            __syncwarp();
            if (lane == 0) mbar_arrive(&work_empty[sl]);
            if (w >= a.n_work) break;
            const PfWork wk = work_of(a, w);
            const int kind = a.kind[wk.g];
            const PfKeys tl = pf_keys<kCache>(a, wk);
            const int n_kv = tl.count();
            const int i = wk.t * kPfM + r;             // query position
            const int hq = wk.h0 + h;
            // running max (log2 units) and two sums: of the bf16 weights the PV
            // product uses (it normalises O) and of the unrounded ones (the
            // log-sum-exp); a sink logit starts them at (sigma, 1, 1)
            float m_run = -INFINITY, l_run = 0.f, l_exact = 0.f;
            if (a.sink_logit != nullptr) {
                m_run = a.sink_logit[hq] * kLog2eF;
                l_run = 1.f;
                l_exact = 1.f;
            }
            for (int j = 0; j < n_kv; ++j, ++jg) {
                const bool got = mbar_wait(&s_full[h], jg & 1);
                __syncwarp();      // tcgen05.ld below is warp-collective
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[128];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    tmem_ld32(s_tmem + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[q4 * 32]));
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[q4 * 32]));
                const int c0 = tl.at(j) * kPfN;
                if (kCache) {
                    if (!(kind == kKindFull && c0 + kPfN <= tl.n)) {
                        uint32_t mw[4];
                        cache_mask(a, tl, kind, i, c0, mw);
#pragma unroll
                        for (int cc = 0; cc < 128; ++cc)
                            if (!((mw[cc >> 5] >> (cc & 31)) & 1u)) sr[cc] = __float_as_uint(-INFINITY);
                    }
                } else if (!tile_dense(kind, wk.t * kPfM, c0, tl.sink, a.recent, a.window)) {
                    // the row's attended keys among the tile's 128 columns as two
                    // 64-bit masks built from their one or two ranges
                    const int di = i - c0;                     // the diagonal's column
                    int lo0, hi0, lo1 = 1, hi1 = 0;            // attended columns [lo0, hi0] u [lo1, hi1]
                    if (kind == kKindFull) {
                        lo0 = 0;
                        hi0 = di;
                    } else if (kind == kKindStreaming) {
                        lo0 = 0;
                        hi0 = min(di, tl.sink - 1 - c0);
                        lo1 = di - a.recent + 1;
                        hi1 = di;
                    } else {
                        lo0 = di - a.window + 1;
                        hi0 = di;
                    }
                    const uint64_t m0 = col_range_bits(lo0, hi0) | col_range_bits(lo1, hi1);
                    const uint64_t m1 = col_range_bits(lo0 - 64, hi0 - 64) | col_range_bits(lo1 - 64, hi1 - 64);
                    const uint32_t mw[4] = {(uint32_t)m0, (uint32_t)(m0 >> 32), (uint32_t)m1, (uint32_t)(m1 >> 32)};
                    // a warp's 32 consecutive rows have their range ends within 32
                    // columns of one another: a 16-column chunk that every row keeps
                    // (or none does) is passed over (or cleared) whole, and only the
                    // few chunks in between are masked column by column
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t bits = (mw[k >> 1] >> (16 * (k & 1))) & 0xffffu;
                        if (!__all_sync(0xffffffffu, bits == 0xffffu)) {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (!((bits >> e) & 1u)) sr[16 * k + e] = __float_as_uint(-INFINITY);
                        }
                    }
                }
                // the row max over the tile, eight independent chains of 3-input max
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[e]);
#pragma unroll
                for (int cc = 8; cc < 128; cc += 16)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        mx8[e] = fmax3(mx8[e], __uint_as_float(sr[cc + e]), __uint_as_float(sr[cc + 8 + e]));
                const float m_tile = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                           fmaxf(mx8[6], mx8[7])) * c;
                // keep the stale max unless the new one is more than 2^8 larger
                float m_use = m_run, alpha = 1.f;
                if (m_tile > m_run + 8.f) {
                    m_use = m_tile;
                    alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_tile);
                }
                const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
                // score * c - max on the packed f32x2 pipe, two columns per
                // instruction; the row sum adds the bf16 weights the PV product
                // uses, so that numerator and denominator agree
                if (kPfTurns) {
                    const bool my_turn = mbar_wait(&turn[h], jg & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, my_turn)) { ok = false; break; }
                }
                const f2 c2 = f2_splat(c), ms2 = f2_splat(-m_sub);
                f2 lx0 = f2_splat(0.f), lx1 = f2_splat(0.f);
                float lsa = 0.f, lsb = 0.f, lsc = 0.f, lsd = 0.f;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t pw[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cc = ch * 16 + 2 * e;
                        const f2 x = f2_fma(f2_make(__uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1])), c2, ms2);
                        f2 pe;
                        if ((ch & 1) * 8 + e < kPfPolyPairs) {
                            pe = ex2_poly2(x);
                        } else {
                            pe.x = ex2_approx(x.x);
                            pe.y = ex2_approx(x.y);
                        }
                        const uint32_t wv = pack_bf16x2(pe.x, pe.y);
                        pw[e] = wv;
                        if (e & 1) {
                            add_bf16x2_f32(lsc, lsd, wv);
                            lx1 = f2_add(lx1, pe);
                        } else {
                            add_bf16x2_f32(lsa, lsb, wv);
                            lx0 = f2_add(lx0, pe);
                        }
                    }
                    // P of keys [16 ch, 16 ch + 16) -> TMEM columns [8 ch, 8 ch + 8)
                    tmem_st8(s_tmem + ch * 8, pw);
                }
                if (kPfTurns) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&turn[h ^ 1]);
                }
                l_run = l_run * alpha + ((lsa + lsb) + (lsc + lsd));
                l_exact = l_exact * alpha + ((lx0.x + lx0.y) + (lx1.x + lx1.y));
                m_run = m_use;
                // O holds the previous key tiles' sum (its PV is complete: this S
                // was computed after it); rescale the row when the max moved
                if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int cb = 0; cb < 128; cb += 32) {
                        uint32_t orr[32];
                        tmem_ld32(o_tmem + cb, orr);
                        tmem_ld_wait();
                        reg_fence32(orr);
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                        tmem_st32(o_tmem + cb, orr);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[h]);
            }
            if (!ok) break;
            // hand the row's (max, sum) to the epilogue warps and go on with the
            // next work tile; they read O once its last PV is done
            row_ml[wc & 1][h][r] = make_float4(m_run, l_run, l_exact, 0.f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&ml_full[wc & 1][h]);
        }
        __syncwarp();
    } else if (warp >= kPfEpiWarp0 && warp < kPfEpiWarp0 + 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfEpiRegs));
        // ------------------------------------------------------------ work-tile epilogue
        const int quarter = warp & 3;                  // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;             // query row within the tile
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int jg = 0;
        bool ok = true;
        for (int wc = 0; ok; ++wc) {
            const int sl = wc % kPfSlots;
            const bool have = mbar_wait(&work_full[sl], (wc / kPfSlots) & 1);
            __syncwarp();
            if (!__all_sync(0xffffffffu, have)) { ok = false; break; }
            const int w = work_slot[sl];
            __syncwarp();
            if (lane == 0) mbar_arrive(&work_empty[sl]);
            if (w >= a.n_work) break;
            const PfWork wk = work_of(a, w);
            jg += pf_keys<kCache>(a, wk).count();
            const int i = wk.t * kPfM + r;             // query position
            const int row0 = wk.t * kPfM + quarter * 32;   // first row of this warp's boxes
            for (int h = 0; h < 2 && ok; ++h) {
                const int hq = wk.h0 + h;
                const uint32_t o_tmem = tmem + 256 + h * 128 + lane_base;
                // the output gate of this row's channels (16 at a time, one chunk
                // ahead) or of its head; the first loads overlap the waits below
                const uint4 *gp = reinterpret_cast<const uint4 *>(
                    a.gate + (((size_t)wk.b * a.L + i) * a.hq + hq) * 128);
                uint4 g0 = make_uint4(0, 0, 0, 0), g1 = g0;
                float g_head = 0.f;
                if (kGate == 1 && i < a.L) {
                    g0 = __ldg(gp);
                    g1 = __ldg(gp + 1);
                } else if (kGate == 2 && i < a.L) {
                    g_head = __bfloat162float(a.gate[((size_t)wk.b * a.L + i) * a.hq + hq]);
                }
                const bool ready = mbar_wait(&ml_full[wc & 1][h], (wc >> 1) & 1) &&
                                   mbar_wait(&o_done[h], (jg - 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
                tc_fence_after();
                const float4 ml = row_ml[wc & 1][h][r];
                const float m_run = ml.x, l_run = ml.y, l_exact = ml.z;
                const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                // o * sigmoid(g): one factor per row, or one per channel below
                const float row_mul = kGate == 2 ? inv_l / (1.f + ex2_approx(-g_head * kLog2eF)) : inv_l;
                // O / l leaves through this warp's two 1 KB staging buffers as 32-row x
                // 16-column TMA stores (rows past L are clipped by the tensor map)
                for (int chunk = 0; chunk < 8 && row0 < a.L; ++chunk) {
                    uint32_t orr[16];
                    tmem_ld16(o_tmem + chunk * 16, orr);
                    tmem_ld_wait();
                    reg_fence16(orr);
                    uint4 n0 = g0, n1 = g1;                // the next chunk's gates
                    if (kGate == 1 && chunk + 1 < 8 && i < a.L) {
                        n0 = __ldg(gp + 2 * (chunk + 1));
                        n1 = __ldg(gp + 2 * (chunk + 1) + 1);
                    }
                    char *stage = sO + ((warp - kPfEpiWarp0) * 2 + (chunk & 1)) * kOStageBytes;
                    // the store that last used this buffer (two chunks ago) has read it
                    if (lane == 0) bulk_wait_read_1();
                    __syncwarp();
                    auto nb = [&](int e) {
                        float m0 = row_mul, m1 = row_mul;
                        if (kGate == 1) {
                            const uint4 q4 = e < 8 ? g0 : g1;
                            const uint32_t gw = (e & 7) < 2 ? q4.x : (e & 7) < 4 ? q4.y : (e & 7) < 6 ? q4.z : q4.w;
                            m0 = inv_l / (1.f + ex2_approx(-__uint_as_float(gw << 16) * kLog2eF));
                            m1 = inv_l / (1.f + ex2_approx(-__uint_as_float(gw & 0xffff0000u) * kLog2eF));
                        }
                        return pack_bf16x2(__uint_as_float(orr[e]) * m0, __uint_as_float(orr[e + 1]) * m1);
                    };
                    const uint4 v0 = make_uint4(nb(0), nb(2), nb(4), nb(6));
                    const uint4 v1 = make_uint4(nb(8), nb(10), nb(12), nb(14));
                    uint4 *row = reinterpret_cast<uint4 *>(stage + lane * 32);
                    row[0] = v0;
                    row[1] = v1;
                    fence_proxy_async_smem();              // visible to the copy engine
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_4d(&a.tm_o, stage, chunk * 16, hq, row0, wk.s * a.batch + wk.b);
                        bulk_commit_group();
                    }
                    g0 = n0;
                    g1 = n1;
                }
                if (a.lse != nullptr && i < a.L)
                    a.lse[((size_t)(wk.s * a.batch + wk.b) * a.hq + hq) * a.L + i] =
                        l_exact > 0.f ? (m_run + __log2f(l_exact)) * kLn2F : -INFINITY;
                // O of this head has been read: the next work tile's first PV may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[h]);
            }
        }
        if (lane == 0) bulk_wait_all();                    // this warp's O stores have landed
        __syncwarp();
    } else {
        // warps 14 and 15 give up their registers; in cache mode warp 14 zeroes,
        // in each loaded stage, the V rows of keys that hold no token (cache memory
        // past a sequence's tokens is never written, and 0 x NaN would reach O)
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfOtherRegs));
        if (kCache && warp == 14) {
            int jg = 0;
            bool ok = true;
            for (int wc = 0; ok; ++wc) {
                const int sl = wc % kPfSlots;
                const bool have = mbar_wait(&work_full[sl], (wc / kPfSlots) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, have)) break;
                const int w = work_slot[sl];
                __syncwarp();
                if (lane == 0) mbar_arrive(&work_empty[sl]);
                if (w >= a.n_work) break;
                const PfWork wk = work_of(a, w);
                const int kind = a.kind[wk.g];
                const PfKeys tl = pf_keys<kCache>(a, wk);
                const int n_kv = tl.count();
                for (int j = 0; j < n_kv; ++j, ++jg) {
                    const int st = jg % kPfStages;
                    const bool got = mbar_wait(&kv_full[st], (jg / kPfStages) & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                    char *vt = sKV + st * kPfStageBytes + kKVTileBytes;
                    const int c0 = tl.at(j) * kPfN;
#pragma unroll 1
                    for (int k = lane; k < kPfN; k += 32) {
                        if (cache_key_valid(a, tl, kind, c0 + k)) continue;
                        // row k of V: 128 bytes in each 64-column half (swizzled within the row)
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            reinterpret_cast<uint4 *>(vt + k * 128)[q] = make_uint4(0, 0, 0, 0);
                            reinterpret_cast<uint4 *>(vt + kKVHalfBytes + k * 128)[q] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_proxy_async_smem();       // the zeroed rows, for the tensor core
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&vprep[st]);
                }
            }
            __syncwarp();
        }
    }
    // launched as a programmatic dependent (the block's own keys after the pass over
    // the cache): the grid completes only after the one before it, whose results
    // the next kernel reads (a no-op otherwise)
    if (!kCache) pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == kPfMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// [B][L][H][128] bf16 viewed as a 4-D tensor (128, H, L, B), loaded as
// 64-column x `rows`-row boxes with the 128-byte swizzle.
// The output [B][L][Hq][128] bf16 as 16-column x 32-row boxes, no swizzle
// (the layout a softmax warp stages: row r at byte 32 r).
inline bool make_out_tmap(CUtensorMap *m, void *base, int B, int L, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)L * H * 256};
    const cuuint32_t box[4] = {16, 1, 32, 1};
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool make_tmap(CUtensorMap *m, const void *base, int B, int L, int H, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)L * H * 256};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The cache as a 4-D tensor (128, rows, heads of the kind, B) loaded in
// 64-column x 128-row boxes with the 128-byte swizzle: (channel, row, rank, b).
inline bool make_cache_tmap(CUtensorMap *m, const void *base, int B, int heads, int64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, (cuuint64_t)rows * 256, (cuuint64_t)rows * heads * 256};
    const cuuint32_t box[4] = {64, (cuuint32_t)kPfN, 1, 1};
    const cuuint32_t elem[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches prefill_fwd<kGate, kCache> for the arguments a (maps, geometry and
// pointers set; the work list is filled in here).
// zero: zero the work counter on the stream first (else the caller has);
// pdl: launch as a programmatic dependent of the previous kernel.
template <int kGate, bool kCache>
inline int launch_prefill_kernel(PrefillArgs &a, int B, int32_t *work_counter, cudaStream_t stream, char *err,
                                 size_t err_len, bool zero = true, bool pdl = false) {
    void (*kernel)(PrefillArgs) = prefill_fwd<kGate, kCache>;
    // set once per device and instantiation (atomic: host threads may launch concurrently)
    static std::atomic<bool> smem_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !smem_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPfSmem) !=
            cudaSuccess) {
            snprintf(err, err_len, "cudaFuncSetAttribute(prefill_fwd) failed");
            return DUO_ERR_CUDA;
        }
        // the warps' register split adds up to exactly the launch allocation: a
        // build with another register count would leave a setmaxnreg.inc waiting
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || fa.numRegs != kPfLaunchRegs) {
            snprintf(err, err_len, "prefill_fwd was built with %d registers per thread, not %d",
                     fa.numRegs, kPfLaunchRegs);
            return DUO_ERR_CUDA;
        }
        if (dev >= 0 && dev < 64) smem_set[dev].store(true, std::memory_order_release);
    }
    a.batch = B;
    if (a.kv_splits < 1) {                 // prompt mode: one split holding every key tile
        a.kv_splits = 1;
        a.split_tiles = INT32_MAX / 2;
    }
    a.batch_pairs = B * (a.hq / 2);
    const int64_t n_work = (int64_t)a.batch_pairs * a.n_qtiles * a.kv_splits;
    // the counter runs up to n_work + 2 * grid
    if (n_work > INT32_MAX - 4096) {
        snprintf(err, err_len, "too many query tiles for one prefill launch");
        return DUO_ERR_INVALID_ARG;
    }
    a.n_work = (int32_t)n_work;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)std::min<int64_t>(n_work, sms);
    a.work_counter = work_counter;
    if (zero && work_counter != nullptr && cudaMemsetAsync(work_counter, 0, sizeof(int32_t), stream) != cudaSuccess) {
        snprintf(err, err_len, "zeroing the prefill work counter failed");
        return DUO_ERR_CUDA;
    }
    if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kPfThreads);
        cfg.dynamicSmemBytes = kPfSmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaLaunchKernelEx(&cfg, kernel, a);
    } else {
        kernel<<<grid, kPfThreads, kPfSmem, stream>>>(a);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(err, err_len, "prefill_fwd launch: %s", cudaGetErrorString(e));
        return DUO_ERR_CUDA;
    }
    return DUO_OK;
}

// Prompt mode: q, k, v [B][L][H][128].  block_start (device, [B]) or null: the
// position each sequence's keys start at, which shifts the sink (a block of
// queries continuing cached tokens); the sink logit, if any, is included.
inline int launch_prefill(const duo_params *p, bool sliding, const int8_t *is_full, int sink,
                          int ring, const void *q, const void *k, const void *v, int32_t L, void *out,
                          float *lse, int32_t *work_counter, int gate_mode, const void *gate,
                          int withhold_tile, cudaStream_t stream, char *err, size_t err_len,
                          const int32_t *block_start = nullptr, bool zero = true, bool pdl = false) {
    PrefillArgs a;
    memset(&a, 0, sizeof a);
    const int B = p->batch;
    if (!make_tmap(&a.tm_q, q, B, L, p->num_q_heads, kPfM) ||
        !make_tmap(&a.tm_k, k, B, L, p->num_kv_heads, kPfN) ||
        !make_tmap(&a.tm_v, v, B, L, p->num_kv_heads, kPfN) ||
        !make_out_tmap(&a.tm_o, out, B, L, p->num_q_heads)) {
        snprintf(err, err_len, "cuTensorMapEncodeTiled failed (driver entry point unavailable?)");
        return DUO_ERR_CUDA;
    }
    a.lse = lse;
    a.sink_logit = p->sink_logit;
    a.gate = (const __nv_bfloat16 *)gate;
    a.L = L;
    a.hq = p->num_q_heads;
    a.hkv = p->num_kv_heads;
    a.n_qtiles = (L + kPfM - 1) / kPfM;
    a.sink = sliding ? 0 : sink;
    a.recent = sliding ? 0 : ring;
    a.window = sliding ? ring : 0;
    a.scale_log2 = p->softmax_scale * kLog2eF;
    a.withhold_tile = withhold_tile;
    a.seq_len = block_start;
    for (int g = 0; g < p->num_kv_heads; ++g)
        a.kind[g] = sliding ? kKindSliding : (is_full[g] ? kKindFull : kKindStreaming);
    if (gate_mode == 1) return launch_prefill_kernel<1, false>(a, B, work_counter, stream, err, err_len, zero, pdl);
    if (gate_mode == 2) return launch_prefill_kernel<2, false>(a, B, work_counter, stream, err, err_len, zero, pdl);
    return launch_prefill_kernel<0, false>(a, B, work_counter, stream, err, err_len, zero, pdl);
}

// Cache mode: the block q [B][L][Hq][128] against the cache as it stands (no
// output gate, no sink logit: those are folded in once the block's own keys
// are added).  full_k/v [B][n_full][capacity][128], strm_k/v [B][n_ring][slots][128].
// A full head's cached key tiles are cut into kv_splits runs of split_tiles
// tiles: out [kv_splits][B][L][Hq][128], lse [kv_splits][B][Hq][L] (ring heads:
// slice 0 only).
inline int launch_prefill_cache(const duo_params *p, bool sliding, const int8_t *is_full, const int8_t *rank,
                                int n_full, int n_ring, int sink, int ring, int64_t capacity,
                                const void *full_k, const void *full_v, const void *strm_k, const void *strm_v,
                                const int32_t *seq_len, const int32_t *ring_head, const void *q, int32_t L,
                                int kv_splits, int split_tiles, void *out, float *lse, int32_t *work_counter,
                                int withhold_tile, cudaStream_t stream, char *err, size_t err_len) {
    PrefillArgs a;
    memset(&a, 0, sizeof a);
    const int B = p->batch;
    const int slots = (sliding ? 0 : sink) + ring;
    // out holds one [B][L][Hq][128] slice per split: the map sees kv_splits * B sequences
    bool okm = make_tmap(&a.tm_q, q, B, L, p->num_q_heads, kPfM) &&
               make_out_tmap(&a.tm_o, out, B * kv_splits, L, p->num_q_heads);
    if (n_full > 0)
        okm = okm && make_cache_tmap(&a.tm_k, full_k, B, n_full, capacity) &&
              make_cache_tmap(&a.tm_v, full_v, B, n_full, capacity);
    if (n_ring > 0)
        okm = okm && make_cache_tmap(&a.tm_k2, strm_k, B, n_ring, slots) &&
              make_cache_tmap(&a.tm_v2, strm_v, B, n_ring, slots);
    if (!okm) {
        snprintf(err, err_len, "cuTensorMapEncodeTiled failed (driver entry point unavailable?)");
        return DUO_ERR_CUDA;
    }
    a.lse = lse;
    a.L = L;
    a.hq = p->num_q_heads;
    a.hkv = p->num_kv_heads;
    a.n_qtiles = (L + kPfM - 1) / kPfM;
    // ring heads: sink S and ring R (a sliding layer: no sink, R = the window)
    a.sink = sliding ? 0 : sink;
    a.recent = ring;
    a.scale_log2 = p->softmax_scale * kLog2eF;
    a.withhold_tile = withhold_tile;
    a.seq_len = seq_len;
    a.ring_head = ring_head;
    a.capacity = (int32_t)std::min<int64_t>(capacity, INT32_MAX);
    a.kv_splits = kv_splits;
    a.split_tiles = split_tiles;
    for (int g = 0; g < p->num_kv_heads; ++g) {
        a.kind[g] = sliding ? kKindSliding : (is_full[g] ? kKindFull : kKindStreaming);
        a.rank[g] = rank[g];
    }
    return launch_prefill_kernel<0, true>(a, B, work_counter, stream, err, err_len, false);   // zeroed by the caller
}

}  // namespace duo
