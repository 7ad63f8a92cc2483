// decode_block.cuh -- a block of q_len query tokens (a speculative-decoding
// verify block) against the hybrid cache as it stands BEFORE the block is
// appended, on tcgen05.
//
// Laguna-XS-2.1 cookbook, section 3.1 (DFlash): the target model checks a
// whole drafted block in one forward pass, and only the tokens it accepts are
// kept.  Query t of sequence b sits at position i = seq_len[b] + t and
// attends to what its head's rule allows at i (DuoAttention Laguna Adapter
// card, Summary and Why It Works; the sliding-window articles):
//   - cached keys: a full head every cached row; a ring head its sink slots
//     and the ring slots whose position j satisfies j > i - recent (the slot
//     written d-th to last holds position seq_len - 1 - d), so that the
//     block's later queries drop the ring's oldest entries;
//   - the block's own keys u <= t under the same rule (passed in, not read
//     from the cache: rejected draft tokens must never evict ring slots).
// The cache is not modified; the caller appends the accepted tokens with
// duo_kv_append afterwards.
//
// Work items are (sequence, KV head, split) as in the one-token decode, with
// one more 128-row tile for the block's own keys on each head's last split
// (rows past q_len are zero-filled by the tensor map).  Persistent CTAs claim
// items from a counter, heaviest first.  The NR = 6 * q_len query rows of an
// item (row t*6 + h: block token t, head h of the group) sit in the M
// dimension of the products, spread over the four TMEM lane quarters
// (RQ = ceil(NR / 4) rows each), so that one thread holds one query row and
// its 128 scores of a key tile:
//   S[128 x 128 keys] = Q . K_tile^T     (Q in tensor memory, K from shared)
//   O[128 x 128 d]   += P . V_tile       (P over S in tensor memory)
// with the rows past NR padding.  Two S buffers let the product of tile j + 1
// run while the softmax works on tile j.
//   warps 0-3  softmax and epilogue: stage the next item's Q into tensor
//              memory, read S, mask, exponentials, P back over S, the item's
//              partial (O, running max, sum) to the workspace
//   warp 4     key preparation: per tile, the range of block queries each key
//              serves, as one 128-bit key mask per block token, and zeroes the
//              V rows no query keeps (stale cache memory never reaches the PV
//              product)
//   warp 5     TMA producer (K and V tiles, three stages; claims the items)
//   warp 6     TMEM owner and MMA issuer
// TMEM: S_a | S_b | O (128 fp32 columns each) | Q_0 | Q_1 (64 columns each).
#pragma once

#include <cuda.h>

#include "decode.cuh"

namespace duo {

template <int kQ>
struct BlockCfg {
    static constexpr int NR = kGroup * kQ;                       // query rows per item
    static constexpr int RQ = (NR + 3) / 4;                      // rows per TMEM lane quarter
    static_assert(RQ <= 16, "an M = 64 product holds 16 rows per lane quarter");
    static constexpr int Stages = 3;
    static constexpr size_t Smem = 1024 + Stages * kDecStageBytes;
    static_assert(Smem + 2048 <= 232448, "shared memory");
    static constexpr int PartFloats = NR * (kD + 2);             // m[NR], l[NR], acc[NR][D]
    static constexpr int Threads = 7 * 32;
};

// Query row r of an item <-> TMEM lane (quarter r / RQ, lane r % RQ).
template <int kQ>
__device__ __forceinline__ int blk_lane_of_row(int r) {
    return (r / BlockCfg<kQ>::RQ) * 32 + r % BlockCfg<kQ>::RQ;
}

struct BlockArgs {
    DecodeArgs d;                   // cache maps, geometry, splits (d.q, d.out, d.lse unused)
    CUtensorMap tm_bk, tm_bv;       // block K / V [B][q_len][Hkv][D] as 4-D (128, Hkv, q_len, B)
    const __nv_bfloat16 *q;         // [B][q_len][Hq][D]
    __nv_bfloat16 *out;             // [B][q_len][Hq][D]
    float *lse;                     // [B][q_len][Hq] or null
    int32_t q_len, n_cache_items, part_slots;   // part_slots = the most splits of a head
    int32_t *work_counter;          // zeroed before the launch: items claimed so far
};

struct BlockItem {
    Item it;                        // the cache item; n_tiles includes the block's tile
    int cache_tiles;                // tiles of cached keys; the block's tile, if any, follows
    bool has_block;                 // the last split of its (sequence, KV head): carries the block's keys
};

__device__ __forceinline__ BlockItem block_item_of(const BlockArgs &a, int w) {
    BlockItem bi;
    bi.it = item_of(a.d, w);
    bi.cache_tiles = bi.it.n_tiles;
    const int splits = bi.it.ring ? a.d.splits_ring : a.d.splits_full;
    bi.has_block = bi.it.split == splits - 1;
    if (bi.has_block) bi.it.n_tiles += 1;
    return bi;
}

// The block queries [t_lo, t_hi] that may attend to key e of the item (empty
// when t_lo > t_hi); on the block's tile e is the block token u.
__device__ __forceinline__ void key_query_range(const BlockArgs &a, const BlockItem &bi, bool block_tile,
                                                int32_t e, int *t_lo, int *t_hi) {
    const Item &it = bi.it;
    const int never_lo = 1, never_hi = 0, all = 1 << 20;
    *t_lo = never_lo;
    *t_hi = never_hi;
    if (block_tile) {
        // block key u = e at position n + u: causal from query u on; a ring
        // head keeps it while it is within `ring` of the query (or a sink key)
        if (e >= a.q_len) return;
        const int32_t n = a.d.seq_len[it.b];
        *t_lo = e;
        *t_hi = (!it.ring || n + e < a.d.sink) ? all : e + a.d.ring - 1;
        return;
    }
    if (e >= it.e_end) return;
    if (!it.ring || e < a.d.sink) {
        // full head rows, sink slots: every query (sink slots only once written)
        if (!it.ring || e < it.n_sink) {
            *t_lo = 0;
            *t_hi = all;
        }
        return;
    }
    int32_t r = e - a.d.sink - it.ring_base;       // 0 = the oldest written ring slot
    if (r < 0) r += a.d.ring;
    if (r >= it.cnt) return;
    // the slot holds position n - cnt + r; query t keeps it while
    // n - cnt + r > n + t - ring, i.e. t <= r + ring - cnt - 1
    *t_lo = 0;
    *t_hi = r + a.d.ring - it.cnt - 1;
}

template <int kQ>
__global__ void __launch_bounds__(BlockCfg<kQ>::Threads, 1) decode_block_split(const __grid_constant__ BlockArgs a) {
    using C = BlockCfg<kQ>;
    constexpr int NR = C::NR, RQ = C::RQ, ST = C::Stages;
    constexpr int kPrep = 4, kProducer = 5, kMma = 6;
    const DecodeArgs &d = a.d;
    extern __shared__ __align__(16) char bsmem_base[];
    char *smem = bsmem_base + ((1024u - (smem_u32(bsmem_base) & 1023u)) & 1023u);
    char *sKV = smem;                                         // [stages][K 32 KB | V 32 KB]
    __shared__ uint64_t kv_full[ST], kv_empty[ST], prep_full[ST];
    // s_full, p_full and o_done alternate with the tile parity, like the S
    // buffers: with the look-ahead QK^T, the softmax can finish a tile while
    // the PVs of the two tiles before it are still outstanding, and a wait by
    // parity on one barrier would then see an older phase as this one
    __shared__ uint64_t s_full[2], p_full[2], o_done[2], q_ready[2], mma_drained;
    // items claimed by the producer, read by the MMA issuer, the key preparation and the softmax warps
    constexpr int kSlots = 4;
    __shared__ uint64_t work_full[kSlots], work_empty[kSlots];
    __shared__ int work_slot[kSlots];
    __shared__ __align__(16) uint32_t key_mask[ST][kQ][4];   // per stage and block token: keys it attends
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = a.n_cache_items;
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
            mbar_init(&prep_full[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&q_ready[i], 4);
            mbar_init(&p_full[i], 4);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(&mma_drained, 1);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&work_full[i], 1);
            mbar_init(&work_empty[i], 6);      // the MMA issuer, the key preparation, 4 softmax warps
        }
        fence_mbar_init();
    }
    if (warp == kMma) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t tm_s = tmem, tm_o = tmem + 256, tm_q = tmem + 384;
    pdl_wait();

    // Reads item slot icx (once per reading warp).
    auto read_slot = [&](int icx, int *wout) -> bool {
        const int sl = icx % kSlots;
        const bool got = mbar_wait(&work_full[sl], (icx / kSlots) & 1);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) return false;
        *wout = work_slot[sl];
        __syncwarp();
        if (lane == 0) mbar_arrive(&work_empty[sl]);
        return true;
    };

    if (warp == kProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (d.n_full > 0) {
                prefetch_tmap(&d.tm_fk);
                prefetch_tmap(&d.tm_fv);
            }
            if (d.n_ring > 0) {
                prefetch_tmap(&d.tm_rk);
                prefetch_tmap(&d.tm_rv);
            }
            prefetch_tmap(&a.tm_bk);
            prefetch_tmap(&a.tm_bv);
            int jg = 0;
            bool ok = true;
            int w = blockIdx.x;
            for (int ic = 0; ok; ++ic) {
                // publish the item (an index >= n_items tells the others to stop)
                const int sl = ic % kSlots;
                if (ic >= kSlots && !(ok = mbar_wait(&work_empty[sl], ((ic / kSlots) - 1) & 1))) break;
                work_slot[sl] = w;
                mbar_arrive(&work_full[sl]);
                if (w >= n_items) break;
                // the next claim, heaviest items first: a CTA takes the next one when it
                // is ready for it, so unequal items do not pile up on a few CTAs
                const int w_next = (int)gridDim.x + atomicAdd(a.work_counter, 1);
                const BlockItem bi = block_item_of(a, w);
                const Item &it = bi.it;
                for (int t = 0; t < it.n_tiles; ++t, ++jg) {
                    const int st = jg % ST;
                    if (jg >= ST && !(ok = mbar_wait(&kv_empty[st], ((jg / ST) - 1) & 1))) break;
                    // failure-detection test: stop feeding this CTA so that its
                    // consumers' bounded waits expire (nothing stays in flight)
                    if (blockIdx.x == 0 && jg == d.withhold_tile) { ok = false; break; }
                    char *ks = sKV + st * kDecStageBytes;
                    mbar_expect_tx(&kv_full[st], kDecStageBytes);
                    if (t == bi.cache_tiles) {
                        // the block's keys; rows u >= q_len are outside the tensor: zero-filled
                        tma_load_4d(ks, &a.tm_bk, 0, it.g, 0, it.b, &kv_full[st]);
                        tma_load_4d(ks + kDecHalfBytes, &a.tm_bk, 64, it.g, 0, it.b, &kv_full[st]);
                        tma_load_4d(ks + kDecTileBytes, &a.tm_bv, 0, it.g, 0, it.b, &kv_full[st]);
                        tma_load_4d(ks + kDecTileBytes + kDecHalfBytes, &a.tm_bv, 64, it.g, 0, it.b,
                                    &kv_full[st]);
                    } else {
                        const CUtensorMap *tk = it.ring ? &d.tm_rk : &d.tm_fk;
                        const CUtensorMap *tv = it.ring ? &d.tm_rv : &d.tm_fv;
                        const int row = it.row0 + it.e_begin + t * kTok;
                        tma_load_2d(ks, tk, 0, row, &kv_full[st]);
                        tma_load_2d(ks + kDecHalfBytes, tk, 64, row, &kv_full[st]);
                        tma_load_2d(ks + kDecTileBytes, tv, 0, row, &kv_full[st]);
                        tma_load_2d(ks + kDecTileBytes + kDecHalfBytes, tv, 64, row, &kv_full[st]);
                    }
                }
                w = w_next;
            }
        }
        __syncwarp();
    } else if (warp == kPrep) {
        // ------------------------------------------------------------ key preparation
        int jg = 0, w = 0;
        bool ok = true;
        for (int ic = 0; ok; ++ic) {
            if (!(ok = read_slot(ic, &w))) break;
            if (w >= n_items) break;
            const BlockItem bi = block_item_of(a, w);
            for (int t = 0; t < bi.it.n_tiles; ++t, ++jg) {
                const int st = jg % ST;
                const bool got = mbar_wait(&kv_full[st], (jg / ST) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                const bool block_tile = t == bi.cache_tiles;
                char *vt = sKV + st * kDecStageBytes + kDecTileBytes;
#pragma unroll
                for (int grp = 0; grp < 4; ++grp) {
                    const int k = grp * 32 + lane;         // key row of the tile
                    const int32_t e = block_tile ? k : bi.it.e_begin + t * kTok + k;
                    int t_lo, t_hi;
                    key_query_range(a, bi, block_tile, e, &t_lo, &t_hi);
                    if (t_lo > t_hi) {
                        // a key no query keeps: its V row must not reach the PV product
                        // (V is MN-major: row k is 128 bytes in each 64-column half)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            reinterpret_cast<uint4 *>(vt + k * 128)[i] = make_uint4(0, 0, 0, 0);
                            reinterpret_cast<uint4 *>(vt + kDecHalfBytes + k * 128)[i] = make_uint4(0, 0, 0, 0);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < kQ; ++q) {
                        const uint32_t bits = __ballot_sync(0xffffffffu, q >= t_lo && q <= t_hi);
                        if (lane == 0) key_mask[st][q][grp] = bits;
                    }
                }
                fence_proxy_async_smem();       // the zeroed rows, for the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&prep_full[st]);
            }
        }
        __syncwarp();
    } else if (warp == kMma) {
        // ------------------------------------------------------------ MMA issuer
        // Two cursors walk the items' tiles in order.  Before PV(j) the issuer
        // issues S(j+1) = Q K(j+1)^T (the look-ahead, so that the softmax finds
        // the next S ready), then PV(j) once the softmax's P(j) and the key
        // preparation of tile j are there.  Both waits suspend the thread until
        // the barrier's phase completes (bounded), so the issuer reacts as soon
        // as its inputs land and takes no issue slots from the softmax warp on
        // its sub-partition meanwhile.
        if (lane == 0) {
            // M = 64: the product's 64 rows sit in lanes 0-15 of each 32-lane
            // quarter of tensor memory, where the item's (at most 12 per quarter)
            // query rows are: half the multiply-adds of M = 128
            const uint32_t id_qk = idesc_bf16_f32(64, kTok, 0, 0);
            const uint32_t id_pv = idesc_bf16_f32(64, kD, 0, 1);
            const uint32_t kv_addr = smem_u32(sKV);
            constexpr int kInfo = 8;
            __shared__ int info_w[kInfo], info_n[kInfo];   // items by fetch order: work index, tiles
            int fetched = 0;
            bool ok = true;
            auto fetch = [&]() {
                const int sl = fetched % kSlots;
                if (!(ok = mbar_wait(&work_full[sl], (fetched / kSlots) & 1))) return;
                const int w = work_slot[sl];
                mbar_arrive(&work_empty[sl]);
                info_w[fetched % kInfo] = w;
                info_n[fetched % kInfo] = w < n_items ? block_item_of(a, w).it.n_tiles : 0;
                ++fetched;
            };
            int pi = 0, pt = 0, jp = 0;                // PV cursor: item, tile, products
            int qi = 0, qt = 0, jq = 0, nq = 0;        // QK cursor: item, tile, products, non-empty items
            bool q_end = false;
            // issues the next S product; false at the end of the list, on a failed
            // wait, or while the item ring holds kInfo - 1 items ahead of the PV cursor
            auto next_qk = [&]() -> bool {
                while (!q_end && ok) {
                    if (qi == fetched) {
                        if (fetched - pi >= kInfo - 1) return false;
                        fetch();
                        if (!ok) return false;
                    }
                    if (info_w[qi % kInfo] >= n_items) {
                        q_end = true;
                        return false;
                    }
                    const int n = info_n[qi % kInfo];
                    if (qt >= n) {
                        if (n > 0) ++nq;
                        ++qi;
                        qt = 0;
                        continue;
                    }
                    // the item's Q (staged by the softmax warps), then the key tile
                    if (qt == 0 && !(ok = mbar_wait(&q_ready[nq & 1], (nq >> 1) & 1))) return false;
                    const int st = jq % ST;
                    if (!(ok = mbar_wait(&kv_full[st], (jq / ST) & 1))) return false;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_ts(tm_s + (jq & 1) * 128, tm_q + (nq & 1) * 64 + k * 8,
                               smem_desc_sw128(kv_addr + st * kDecStageBytes + (k >> 2) * kDecHalfBytes +
                                                   (k & 3) * 32, 16, 1024),
                               id_qk, k > 0);
                    mma_commit(&s_full[jq & 1]);
                    ++jq;
                    ++qt;
                    return true;
                }
                return false;
            };
            next_qk();                                 // S(0)
            while (ok) {
                // the PV cursor's next tile: past finished and empty items
                while (true) {
                    if (pi == fetched) fetch();
                    if (!ok || info_w[pi % kInfo] >= n_items || pt < info_n[pi % kInfo]) break;
                    ++pi;
                    pt = 0;
                }
                if (!ok || info_w[pi % kInfo] >= n_items) break;
                // S(jp) and the look-ahead S(jp + 1) before PV(jp) (S(jp + 2) would
                // overwrite P(jp))
                while (ok && jq < jp + 2 && next_qk()) {
                }
                if (!ok || jq <= jp) break;
                const int st = jp % ST;
                if (!(ok = mbar_wait(&p_full[jp & 1], (jp >> 1) & 1) && mbar_wait(&prep_full[st], (jp / ST) & 1)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ts(tm_o, tm_s + (jp & 1) * 128 + k * 8,
                           smem_desc_sw128(kv_addr + st * kDecStageBytes + kDecTileBytes + k * 2048,
                                           kDecHalfBytes, 1024),
                           id_pv, (pt == 0 && k == 0) ? 0u : 1u);
                mma_commit(&o_done[jp & 1]);
                mma_commit(&kv_empty[st]);
                ++jp;
                ++pt;
            }
            // every product issued has completed before the tensor memory is freed
            // (on an early exit some may still run)
            mma_commit(&mma_drained);
            mbar_wait(&mma_drained, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quarter = warp;                            // TMEM lane quarter
        const int r = quarter * RQ + lane;                   // query row of this thread
        const bool has_row = lane < RQ && r < NR;
        const int tq = has_row ? r / kGroup : 0;             // its block token
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        // The softmax reads S and writes P with the 16-lane shapes: the quad of
        // threads 4L..4L+3 shares rows A (lane L of the quarter) and B (lane L + 8),
        // thread qd of the quad holding columns 8k + 2 qd and 8k + 2 qd + 1 of each,
        // so that all 32 threads work on the quarter's (at most 16) query rows.
        const int qd = lane & 3, rl = lane >> 2;
        const int rowA = quarter * RQ + rl, rowB = rowA + 8;
        const bool hasA = rl < RQ && rowA < NR, hasB = rl + 8 < RQ && rowB < NR;
        const int tqA = hasA ? rowA / kGroup : 0, tqB = hasB ? rowB / kGroup : 0;
        const float c = d.scale_log2;
        // Stages the query rows of item wq into Q buffer buf (zeros in the padding rows).
        auto stage_q = [&](int wq, int buf) {
            uint32_t qv[64];
            const bool real = has_row;
            const uint4 *src = nullptr;
            if (real) {
                const BlockItem nx = block_item_of(a, wq);
                src = reinterpret_cast<const uint4 *>(
                    a.q + (((size_t)nx.it.b * kQ + tq) * d.hkv * kGroup + nx.it.g * kGroup + r % kGroup) * kD);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint4 v = real ? src[i] : make_uint4(0, 0, 0, 0);
                qv[4 * i] = v.x;
                qv[4 * i + 1] = v.y;
                qv[4 * i + 2] = v.z;
                qv[4 * i + 3] = v.w;
            }
            tmem_st32(tm_q + buf * 64 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&qv[0]));
            tmem_st32(tm_q + buf * 64 + 32 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&qv[32]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready[buf]);
        };
        // Q buffers alternate over the items that have tiles (an empty item needs
        // no Q), in the order the MMA issuer counts them
        int n_staged = 0;
        auto stage_if_needed = [&](int wx) {
            if (wx < n_items && block_item_of(a, wx).it.n_tiles > 0) {
                stage_q(wx, n_staged & 1);
                ++n_staged;
            }
        };
        int jg = 0, ic = 0, w = 0;
        bool ok = read_slot(0, &w);
        if (ok) stage_if_needed(w);
        for (; ok && w < n_items; ++ic) {
            const BlockItem bi = block_item_of(a, w);
            const Item &it = bi.it;
            // rows A, B of this thread: running max and its share of the row sum
            float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
            for (int t = 0; t < it.n_tiles; ++t, ++jg) {
                const bool got = mbar_wait(&s_full[jg & 1], (jg >> 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                const uint32_t s_tm = tm_s + (jg & 1) * 128 + lane_base;
                // sr[4k..4k+3]: (A, c), (A, c + 1), (B, c), (B, c + 1) with c = 8k + 2 qd
                uint32_t sr[64];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    tmem_ld_q16(s_tm + q4 * 32, *reinterpret_cast<uint32_t(*)[16]>(&sr[q4 * 16]));
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) reg_fence16(*reinterpret_cast<uint32_t(*)[16]>(&sr[q4 * 16]));
                const bool block_tile = t == bi.cache_tiles;
                // a full head's tile inside the cached length: every key for every query
                const bool dense = !block_tile && !it.ring && it.e_begin + (t + 1) * kTok <= it.e_end;
                if (!dense) {
                    const int st = jg % ST;
                    const bool prepped = mbar_wait(&prep_full[st], (jg / ST) & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, prepped)) { ok = false; break; }
                    const uint4 ka = *reinterpret_cast<const uint4 *>(key_mask[st][tqA]);
                    const uint4 kb = *reinterpret_cast<const uint4 *>(key_mask[st][tqB]);
                    const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int sh = 8 * (k & 3) + 2 * qd;   // bit of column 8k + 2 qd in its word
                        const uint32_t ba = wa[k >> 2] >> sh, bb = wb[k >> 2] >> sh;
                        if (!(ba & 1u)) sr[4 * k] = __float_as_uint(-INFINITY);
                        if (!(ba & 2u)) sr[4 * k + 1] = __float_as_uint(-INFINITY);
                        if (!(bb & 1u)) sr[4 * k + 2] = __float_as_uint(-INFINITY);
                        if (!(bb & 2u)) sr[4 * k + 3] = __float_as_uint(-INFINITY);
                    }
                }
                // the rows' maxima: this thread's 32 columns of each, then its quad
                float xa[4], xb[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xa[e] = fmaxf(__uint_as_float(sr[4 * e]), __uint_as_float(sr[4 * e + 1]));
                    xb[e] = fmaxf(__uint_as_float(sr[4 * e + 2]), __uint_as_float(sr[4 * e + 3]));
                }
#pragma unroll
                for (int k = 4; k < 16; k += 4)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        xa[e] = fmax3(xa[e], __uint_as_float(sr[4 * (k + e)]), __uint_as_float(sr[4 * (k + e) + 1]));
                        xb[e] = fmax3(xb[e], __uint_as_float(sr[4 * (k + e) + 2]), __uint_as_float(sr[4 * (k + e) + 3]));
                    }
                float ta = fmaxf(fmaxf(xa[0], xa[1]), fmaxf(xa[2], xa[3]));
                float tb = fmaxf(fmaxf(xb[0], xb[1]), fmaxf(xb[2], xb[3]));
                ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 1));
                tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 1));
                ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 2)) * c;
                tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 2)) * c;
                // keep the stale max unless the new one is more than 2^8 larger
                float alA = 1.f, alB = 1.f;
                if (ta > mA + 8.f) {
                    alA = (mA == -INFINITY) ? 0.f : ex2_approx(mA - ta);
                    mA = ta;
                }
                if (tb > mB + 8.f) {
                    alB = (mB == -INFINITY) ? 0.f : ex2_approx(mB - tb);
                    mB = tb;
                }
                const f2 c2 = f2_splat(c);
                const f2 msA = f2_splat(mA == -INFINITY ? 0.f : -mA), msB = f2_splat(mB == -INFINITY ? 0.f : -mB);
                f2 sa = f2_splat(0.f), sb = f2_splat(0.f);
                // P: keys (c, c + 1) of each row packed into column 4k + qd of this S buffer
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pw[16];
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int k = half * 8 + kk;
                        const f2 x0 = f2_fma(f2_make(__uint_as_float(sr[4 * k]), __uint_as_float(sr[4 * k + 1])), c2, msA);
                        const f2 x1 = f2_fma(f2_make(__uint_as_float(sr[4 * k + 2]), __uint_as_float(sr[4 * k + 3])), c2, msB);
                        const f2 pa = f2_make(ex2_approx(x0.x), ex2_approx(x0.y));
                        const f2 pb = f2_make(ex2_approx(x1.x), ex2_approx(x1.y));
                        pw[2 * kk] = pack_bf16x2(pa.x, pa.y);     // bf16 for the PV product
                        pw[2 * kk + 1] = pack_bf16x2(pb.x, pb.y);
                        sa = f2_add(sa, pa);
                        sb = f2_add(sb, pb);
                    }
                    tmem_st_p16(s_tm + half * 32, pw);
                }
                lA = lA * alA + (sa.x + sa.y);
                lB = lB * alB + (sb.x + sb.y);
                if (t > 0 && __any_sync(0xffffffffu, alA != 1.f || alB != 1.f)) {
                    // O must hold every earlier tile's product before it is scaled
                    const bool prev = mbar_wait(&o_done[(jg - 1) & 1], ((jg - 1) >> 1) & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, prev)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int cb = 0; cb < 128; cb += 32) {
                        uint32_t orr[16];
                        tmem_ld_q16(tm_o + cb + lane_base, orr);
                        tmem_ld_wait();
                        reg_fence16(orr);
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            orr[e] = __float_as_uint(__uint_as_float(orr[e]) * ((e & 2) ? alB : alA));
                        tmem_st_q16(tm_o + cb + lane_base, orr);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[jg & 1]);
            }
            if (!ok) break;
            // The next item's Q goes into the other buffer now, before this item's
            // epilogue, so that its first products can run meanwhile (the item
            // with tiles before this one, which used that buffer, has had all its
            // products read).  Its slot is read only now: the producer publishes
            // it after loading all of this item's tiles, which needs this
            // item's tiles to have gone through the softmax.
            int w_next = n_items;
            if (!(ok = read_slot(ic + 1, &w_next))) break;
            stage_if_needed(w_next);
            // ------------------------------------------------------------ item epilogue
            float *part = d.part + (((size_t)it.b * d.hkv + it.g) * a.part_slots + it.split) * C::PartFloats;
            if (it.n_tiles > 0) {
                const bool done = mbar_wait(&o_done[(jg - 1) & 1], ((jg - 1) >> 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, done)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < 128; cb += 32) {
                    uint32_t orr[16];
                    tmem_ld_q16(tm_o + cb + lane_base, orr);
                    tmem_ld_wait();
                    reg_fence16(orr);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int col = cb + 8 * k + 2 * qd;
                        if (hasA)
                            *reinterpret_cast<float2 *>(part + 2 * NR + rowA * kD + col) =
                                make_float2(__uint_as_float(orr[4 * k]), __uint_as_float(orr[4 * k + 1]));
                        if (hasB)
                            *reinterpret_cast<float2 *>(part + 2 * NR + rowB * kD + col) =
                                make_float2(__uint_as_float(orr[4 * k + 2]), __uint_as_float(orr[4 * k + 3]));
                    }
                }
            } else {
#pragma unroll 1
                for (int k = 0; k < 16; ++k) {
                    const int col = 8 * k + 2 * qd;
                    if (hasA) *reinterpret_cast<float2 *>(part + 2 * NR + rowA * kD + col) = make_float2(0.f, 0.f);
                    if (hasB) *reinterpret_cast<float2 *>(part + 2 * NR + rowB * kD + col) = make_float2(0.f, 0.f);
                }
            }
            // each row's sum over its quad, in a fixed order
            lA += __shfl_xor_sync(0xffffffffu, lA, 1);
            lB += __shfl_xor_sync(0xffffffffu, lB, 1);
            lA += __shfl_xor_sync(0xffffffffu, lA, 2);
            lB += __shfl_xor_sync(0xffffffffu, lB, 2);
            if (qd == 0 && hasA) {
                part[rowA] = mA;
                part[NR + rowA] = lA;
            }
            if (qd == 0 && hasB) {
                part[rowB] = mB;
                part[NR + rowB] = lB;
            }
            // O is read before this warp's first p_full arrival of the next item
            tc_fence_before();
            w = w_next;
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Folds the splits (the last one holds the block's keys too) and the sink
// logit of the six query heads of one (sequence, block token, KV head): one
// warp per head, four output dimensions per thread (few threads: how fast they
// launch is what bounds a merge this short).  Each fold runs in split order.
template <int kQ>
__global__ void __launch_bounds__(kMergeThreads) decode_block_merge(const __grid_constant__ BlockArgs a) {
    using C = BlockCfg<kQ>;
    constexpr int NR = C::NR;
    pdl_wait();
    const DecodeArgs &d = a.d;
    const int grp = blockIdx.x;                      // (b * q_len + t) * Hkv + g
    const int g = grp % d.hkv;
    const int t = (grp / d.hkv) % kQ;
    const int b = grp / d.hkv / kQ;
    const int hh = threadIdx.x >> 5, c4 = (threadIdx.x & 31) * 4;
    const int h = g * kGroup + hh;
    const size_t idx = ((size_t)b * kQ + t) * d.hkv * kGroup + h;   // (b, t, query head)
    const int row = t * kGroup + hh;
    const int splits = d.heads.is_full[g] ? d.splits_full : d.splits_ring;
    const float *part = d.part + ((size_t)b * d.hkv + g) * a.part_slots * C::PartFloats;
    const bool has_sink = d.sink_logit != nullptr;
    const float sig = has_sink ? d.sink_logit[h] * kLog2eF : -INFINITY;
    float M = sig, den = 0.f;
    float4 num;
    fold_splits4<2>(part, C::PartFloats, splits, row, NR + row, 2 * NR + row * kD + c4, &M, &den, &num);
    if (M != -INFINITY && has_sink) den += ex2_approx(sig - M);
    const float g_head = d.gate_mode == 2 ? __bfloat162float(d.gate[idx]) : 0.f;
    *reinterpret_cast<uint2 *>(a.out + idx * kD + c4) =
        fold_out4(num, den, d.gate_mode, d.gate_mode == 1 ? d.gate + idx * kD + c4 : nullptr, g_head);
    if (a.lse != nullptr && c4 == 0)
        a.lse[idx] = den > 0.f ? (M + __log2f(den)) * kLn2F : -INFINITY;
}

// A block longer than the verify kernel takes is computed in two passes: its
// queries against the cached keys (prefill_fwd's cache mode; a full head's keys
// in kv_splits runs, each written as its own slice) and against its own keys
// (prefill_fwd's prompt mode, which also adds the sink logit).  Each part is
// normalised by its own sum and rounded to bf16; they are folded here by their
// sums: O = sum_p e^Lp Op / sum_p e^Lp, LSE = ln sum_p e^Lp.
constexpr int kMaxLongSplits = 8;     // slices of a full head's cached keys in a long block

struct CombineArgs {
    const __nv_bfloat16 *oa, *ob;   // [S][B][C][Hq][D], [B][C][Hq][D]
    const float *lse_a, *lse_b;     // [S][B][Hq][C], [B][Hq][C]
    __nv_bfloat16 *out;             // [B][C][Hq][D]
    float *lse;                     // [B][C][Hq] or null
    const __nv_bfloat16 *gate;      // output gate pre-activations or null
    int32_t gate_mode, C, hq, batch, kv_splits, split_tiles, capacity;
    const int32_t *seq_len;         // cached tokens per sequence
    int8_t is_full[64];             // per KV head: its cached keys come in split slices (else one)
};

// kCombineDims output dimensions per thread, 128 / kCombineDims threads per
// output row (sequence, block token, query head): the per-row work (indices,
// the parts' log-sum-exps and weights) is shared by a row's threads, and every
// part's 16-byte loads are issued at once.  Rows are (b * C + t) * Hq + h,
// fewer than 2^31 (the host checks), so the index arithmetic stays 32-bit.
#ifndef DUO_COMBINE_DIMS
#define DUO_COMBINE_DIMS 8
#endif
constexpr int kCombineDims = DUO_COMBINE_DIMS, kCombineVec = kCombineDims / 8;
constexpr int kCombineRowThreads = kD / kCombineDims, kCombineThreads = 256;
constexpr int kCombineRows = kCombineThreads / kCombineRowThreads;

__global__ void __launch_bounds__(kCombineThreads) block_combine(const __grid_constant__ CombineArgs a) {
    const uint32_t rows = (uint32_t)a.batch * (uint32_t)a.C * (uint32_t)a.hq;
    const uint32_t row = blockIdx.x * kCombineRows + threadIdx.x / kCombineRowThreads;
    const int c16 = (threadIdx.x % kCombineRowThreads) * kCombineDims;
    if (row >= rows) return;
    const uint32_t h = row % (uint32_t)a.hq, bt = row / (uint32_t)a.hq;
    const uint32_t t = bt % (uint32_t)a.C, b = bt / (uint32_t)a.C;
    // a full head's slices: as many as its cached rows fill (prefill_fwd passes
    // over the rest unwritten); split 0 always, maybe with no key
    int parts = 1;
    if (a.is_full[h / kGroup]) {
        const int tiles = (min(max(a.seq_len[b], 0), a.capacity) + 127) / 128;
        parts = min(a.kv_splits, max(1, (tiles + a.split_tiles - 1) / a.split_tiles));
    }
    const size_t slice_o = (size_t)rows * kD, slice_l = rows;
    const size_t li = ((size_t)b * a.hq + h) * a.C + t;
    const size_t oi = (size_t)row * kD + c16;
    // every part's log-sum-exp and outputs (part kMaxLongSplits is the block's own)
    float l[kMaxLongSplits + 1];
    uint4 ov[kMaxLongSplits + 1][kCombineVec];
#pragma unroll
    for (int s = 0; s <= kMaxLongSplits; ++s) {
        const bool own = s == kMaxLongSplits;
        l[s] = -INFINITY;
#pragma unroll
        for (int v = 0; v < kCombineVec; ++v) ov[s][v] = make_uint4(0u, 0u, 0u, 0u);
        if (own || s < parts) {
            l[s] = (own ? a.lse_b[li] : a.lse_a[s * slice_l + li]) * kLog2eF;
            const uint4 *src = reinterpret_cast<const uint4 *>((own ? a.ob : a.oa + s * slice_o) + oi);
#pragma unroll
            for (int v = 0; v < kCombineVec; ++v) ov[s][v] = src[v];
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s <= kMaxLongSplits; ++s) M = fmaxf(M, l[s]);
    float den = 0.f, num[kCombineDims];
#pragma unroll
    for (int e = 0; e < kCombineDims; ++e) num[e] = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int s = 0; s <= kMaxLongSplits; ++s) {
            if (l[s] == -INFINITY) continue;
            const float wgt = ex2_approx(l[s] - M);
            den += wgt;
#pragma unroll
            for (int e = 0; e < kCombineDims / 2; ++e) {
                const uint4 &q = ov[s][e >> 2];
                const uint32_t wv = (e & 3) == 0 ? q.x : (e & 3) == 1 ? q.y : (e & 3) == 2 ? q.z : q.w;
                num[2 * e] = fmaf(wgt, __uint_as_float(wv << 16), num[2 * e]);
                num[2 * e + 1] = fmaf(wgt, __uint_as_float(wv & 0xffff0000u), num[2 * e + 1]);
            }
        }
    }
    // O = num / den, times the sigmoid of the output gate (per channel or per head)
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int e = 0; e < kCombineDims; ++e) num[e] *= inv;
    if (a.gate_mode == 1) {
        const uint4 *gp = reinterpret_cast<const uint4 *>(a.gate + oi);
#pragma unroll
        for (int v = 0; v < kCombineVec; ++v) {
            const uint4 g = gp[v];
            const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gx = __uint_as_float(e & 1 ? (gv[e >> 1] & 0xffff0000u) : (gv[e >> 1] << 16));
                num[8 * v + e] = __fdividef(num[8 * v + e], 1.f + ex2_approx(-gx * kLog2eF));
            }
        }
    } else if (a.gate_mode == 2) {
        const float gs = 1.f / (1.f + ex2_approx(-__bfloat162float(a.gate[row]) * kLog2eF));
#pragma unroll
        for (int e = 0; e < kCombineDims; ++e) num[e] *= gs;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(a.out + oi);
#pragma unroll
    for (int v = 0; v < kCombineVec; ++v)
        dst[v] = make_uint4(pack_bf16x2(num[8 * v], num[8 * v + 1]), pack_bf16x2(num[8 * v + 2], num[8 * v + 3]),
                            pack_bf16x2(num[8 * v + 4], num[8 * v + 5]), pack_bf16x2(num[8 * v + 6], num[8 * v + 7]));
    if (a.lse != nullptr && c16 == 0) a.lse[row] = den > 0.f ? (M + __log2f(den)) * kLn2F : -INFINITY;
}

}  // namespace duo
