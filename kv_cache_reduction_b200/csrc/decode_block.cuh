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
// The structure is the one-token decode's (decode.cuh): persistent CTAs over
// (sequence, KV head, split) items, "swap AB" products with the tokens of a
// 128-token tile in M and the query rows in N:
//   S^T[128 tok x NP] = K_tile . Q^T,   O^T[128 d x NP] += V_tile^T . P^T
// with NR = 6 * q_len query rows (row t*6 + h: block token t, head h of the
// group) padded to NP = 16, 32 or 48.  Each (sequence, KV head) has one
// more tile for the block's keys: one 128-row tile of the block's K/V (rows
// past q_len are zero-filled by the tensor map and masked), the last tile of
// that head's last split item.  Every key token
// carries the range [t_lo, t_hi] of block queries that may attend to it.
// The softmax of a tile is split over two or three warps per TMEM lane
// quarter (at most 16 query rows per thread), and one vote across them
// (bar.red.or) skips the row-max reduction on tiles where no score exceeds its
// row's running max by more than 2^8 -- the same result as reducing.
#pragma once

#include <cuda.h>

#include "decode.cuh"

namespace duo {

__device__ __forceinline__ void blk_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void blk_reg_fence16(uint32_t (&r)[16]) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

template <int kQ>
struct BlockCfg {
    static constexpr int NR = kGroup * kQ;                       // query rows per item
    static constexpr int NP = (NR + 15) / 16 * 16;               // MMA N
    static constexpr uint32_t OpBytes = NP * kD * 2;             // Q or P^T operand
    static constexpr uint32_t OpHalf = NP * 128;                 // one 64-column half of it
    // three K/V stages keep two tiles in flight behind the one being scored;
    // the operand buffers give way when the query rows grow
#ifndef DUO_BLK_WIDE_STAGES
#define DUO_BLK_WIDE_STAGES 3
#endif
#ifndef DUO_BLK_WIDE_PB
#define DUO_BLK_WIDE_PB 1
#endif
    static constexpr int Stages = NP <= 32 ? 3 : DUO_BLK_WIDE_STAGES;
    static constexpr int QB = NP <= 32 ? 2 : 1;                  // Q buffers (next item's Q staged early)
    static constexpr int PB = NP <= 16 ? 2 : NP <= 32 ? 1 : DUO_BLK_WIDE_PB;   // P^T buffers
    static constexpr size_t Smem = 1024 + Stages * kDecStageBytes + (QB + PB) * OpBytes;
    static_assert(Smem + 4096 <= 232448, "shared memory");
    static constexpr int PartFloats = NR * (kD + 2);             // m[NR], l[NR], acc[NR][D]
    static constexpr uint32_t TmemCols = 3 * NP <= 64 ? 64 : 3 * NP <= 128 ? 128 : 256;
    // softmax warps per TMEM lane quarter, each with NH of the query rows: more
    // of them for wide blocks, so that no thread holds more than 16 rows
    static constexpr int NPART = NP == 48 ? 3 : 2;
    static constexpr int NH = NP / NPART;                        // 8 or 16 rows
    static constexpr int RP = NH <= 4 ? 4 : NH <= 8 ? 8 : NH <= 16 ? 16 : 32;   // NH padded to 2^k
    static constexpr int SoftmaxThreads = 128 * NPART;
    // softmax warps 0 .. 4*NPART-1, then the producer warp and the MMA warp
    static constexpr int Threads = SoftmaxThreads + 64;
};

__device__ __forceinline__ void blk_tmem_ld4(uint32_t taddr, uint32_t *r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}

__device__ __forceinline__ void blk_tmem_st4(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void blk_reg_fence4(uint32_t *r) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]));
}

// Per-row reduction of v[RP] over the 32 lanes of a warp that leaves row
// (lane >> (5 - log2 RP)) with each lane: at every step a lane keeps half of
// its rows and hands the other half to its partner, so RP - 1 shuffles do the
// work of RP * 5 butterflies.  op: 0 max, 1 sum.
template <int RP, int OP>
__device__ __forceinline__ float lane_row_reduce(float (&v)[RP], int lane) {
    int cnt = RP;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        if (cnt >= 2) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < RP / 2; ++i) {
                if (i < cnt / 2) {
                    const float keep = up ? v[cnt / 2 + i] : v[i];
                    const float give = up ? v[i] : v[cnt / 2 + i];
                    const float got = __shfl_xor_sync(0xffffffffu, give, o);
                    v[i] = OP == 0 ? fmaxf(keep, got) : keep + got;
                }
            }
            cnt >>= 1;
        } else {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], o);
            v[0] = OP == 0 ? fmaxf(v[0], got) : v[0] + got;
        }
    }
    return v[0];
}

// OR of a predicate over the `nthreads` softmax threads (named barrier 1).
__device__ __forceinline__ bool softmax_vote_any(bool v, int nthreads) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(nthreads)
        : "memory");
    return r != 0;
}

template <int RP>
__host__ __device__ constexpr int rp_bits() { return RP == 4 ? 2 : RP == 8 ? 3 : RP == 16 ? 4 : 5; }

template <int RP>
__device__ __forceinline__ int lane_row(int lane) { return lane >> (5 - rp_bits<RP>()); }

struct BlockArgs {
    DecodeArgs d;                   // cache maps, geometry, splits (d.q, d.out, d.lse unused)
    CUtensorMap tm_bk, tm_bv;       // block K / V [B][q_len][Hkv][D] as 4-D (128, Hkv, q_len, B)
    const __nv_bfloat16 *q;         // [B][q_len][Hq][D]
    __nv_bfloat16 *out;             // [B][q_len][Hq][D]
    float *lse;                     // [B][q_len][Hq] or null
    int32_t q_len, n_cache_items, part_slots;   // part_slots = the most splits of a head
    int32_t *work_counter;          // zeroed before the launch: items claimed so far
};

// Byte offset of element (row, k) in an [NP rows][128] bf16 K-major operand
// stored as two 64-column halves with the 128-byte swizzle.
template <int NP>
__device__ __forceinline__ uint32_t blk_op_offset(int row, int k) {
    const int half = k >> 6, kk = k & 63;
    return half * (NP * 128) + (row >> 3) * 1024 + (row & 7) * 128 + ((((kk >> 3) ^ (row & 7))) << 4) +
           (kk & 7) * 2;
}

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
    constexpr int NR = C::NR, NP = C::NP, ST = C::Stages, NH = C::NH, RP = C::RP;
    constexpr int NSM = C::SoftmaxThreads, NSW = NSM / 32;    // softmax threads / warps
    constexpr int kProducer = NSW, kMma = NSW + 1;
    const DecodeArgs &d = a.d;
    extern __shared__ __align__(16) char bsmem_base[];
    char *smem = bsmem_base + ((1024u - (smem_u32(bsmem_base) & 1023u)) & 1023u);
    char *sKV = smem;                                         // [stages][K 32 KB | V 32 KB]
    char *sQ = smem + ST * kDecStageBytes;                    // [2 items][OpBytes]
    char *sP = sQ + C::QB * C::OpBytes;                       // [PB tiles][OpBytes]
    __shared__ uint64_t kv_full[ST], kv_empty[ST];
    // P^T is double-buffered: PV of tile j commits o_done[j & 1]
    __shared__ uint64_t s_full[2], p_full, o_done[2], q_ready[2];
    // items claimed by the producer, read by the MMA issuer and the softmax warps
    constexpr int kSlots = 4;
    __shared__ uint64_t work_full[kSlots], work_empty[kSlots];
    __shared__ int work_slot[kSlots];
    __shared__ uint32_t tmem_base;
    __shared__ __align__(16) float red_max[2][4][NP];
    __shared__ float red_sum[4][NP];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = a.n_cache_items;
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&q_ready[i], NSW);
        }
        mbar_init(&p_full, NSW);
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&work_full[i], 1);
            mbar_init(&work_empty[i], 1 + NSW);        // the MMA issuer and every softmax warp
        }
        fence_mbar_init();
    }
    if (warp < NSW) {
        // operand rows NR..NP-1 stay zero for the whole kernel
        for (int i = threadIdx.x; i < (C::QB + C::PB) * (int)C::OpBytes / 16; i += NSM)
            reinterpret_cast<uint4 *>(sQ)[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == kMma) {
        tmem_alloc(&tmem_base, C::TmemCols);
        tmem_relinquish();
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

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
                // publish the item (an index >= n_items tells the consumers to stop)
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
    } else if (warp == kMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16_f32(kTok, NP, 0, 0);
            const uint32_t id_pv = idesc_bf16_f32(kD, NP, 1, 0);
            const uint32_t kv_addr = smem_u32(sKV), q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            const uint32_t o_tmem = tmem + 2 * NP;
            auto issue_pv_blk = [&](int st, int pbuf, bool first) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss(o_tmem, smem_desc_sw128(kv_addr + st * kDecStageBytes + kDecTileBytes + k * 2048,
                                                   kDecHalfBytes, 1024),
                           smem_desc_sw128(p_addr + (C::PB == 2 ? pbuf : 0) * C::OpBytes + (k >> 2) * C::OpHalf +
                                               (k & 3) * 32,
                                           16, 1024),
                           id_pv, (first && k == 0) ? 0u : 1u);
            };
            int jg = 0, ic = 0;
            bool ok = true, pend = false, pend_first = false;
            int pend_st = 0;
            for (; ok; ++ic) {
                const int sl = ic % kSlots;
                if (!(ok = mbar_wait(&work_full[sl], (ic / kSlots) & 1))) break;
                const int w = work_slot[sl];
                mbar_arrive(&work_empty[sl]);
                if (w >= n_items) break;
                const BlockItem bi = block_item_of(a, w);
                const Item &it = bi.it;
                // every item's Q is staged (an empty item's only signals), so the
                // staging and this wait pair up item by item
                if (!(ok = mbar_wait(&q_ready[ic & 1], (ic >> 1) & 1))) break;
                if (it.n_tiles == 0) continue;
                for (int t = 0; t < it.n_tiles && ok; ++t, ++jg) {
                    const int st = jg % ST;
                    if (!(ok = mbar_wait(&kv_full[st], (jg / ST) & 1))) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * kDecHalfBytes + (k & 3) * 32;
                        const uint32_t qoff = (C::QB == 2 ? (ic & 1) : 0) * C::OpBytes + (k >> 2) * C::OpHalf + (k & 3) * 32;
                        mma_ss(tmem + (jg & 1) * NP, smem_desc_sw128(kv_addr + st * kDecStageBytes + off, 16, 1024),
                               smem_desc_sw128(q_addr + qoff, 16, 1024), id_qk, k > 0);
                    }
                    mma_commit(&s_full[jg & 1]);
                    if (pend) {
                        if (!(ok = mbar_wait(&p_full, (jg - 1) & 1))) break;
                        tc_fence_after();
                        issue_pv_blk(pend_st, (jg - 1) & 1, pend_first);
                        mma_commit(&o_done[(jg - 1) & 1]);
                        mma_commit(&kv_empty[pend_st]);
                    }
                    pend = true;
                    pend_st = st;
                    pend_first = (t == 0);
                }
            }
            if (ok && pend && mbar_wait(&p_full, (jg - 1) & 1)) {
                tc_fence_after();
                issue_pv_blk(pend_st, (jg - 1) & 1, pend_first);
                mma_commit(&o_done[(jg - 1) & 1]);
                mma_commit(&kv_empty[pend_st]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;                        // TMEM lane quarter: tokens / dims
        const int part = warp >> 2;                          // query rows [part * NH, part * NH + NH)
        const int r = quarter * 32 + lane;                   // token row / output dimension
        const int q0 = part * NH;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t o_tmem = tmem + 2 * NP + q0 + lane_base;
        const float c = d.scale_log2;
        const int tid = threadIdx.x;                         // 0 .. NSM - 1
        auto sm_sync = [] { asm volatile("bar.sync 1, %0;" ::"r"(NSM) : "memory"); };
        // Reads item slot icx (each softmax warp once per slot).
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
        // Stages the NR query rows of item w as the Q operand in buffer `buf`
        // (nothing to copy for an empty item, but the MMA warp is still told).
        auto stage_q = [&](int w, int buf) {
            if (w >= n_items) return;
            {
                const BlockItem nx = block_item_of(a, w);
                if (nx.it.n_tiles > 0)
                for (int i = tid; i < NR * 16; i += NSM) {
                    const int row = i >> 4, ch = i & 15;
                    const int t = row / kGroup, h = row % kGroup;
                    const uint4 v = reinterpret_cast<const uint4 *>(
                        a.q + (((size_t)nx.it.b * kQ + t) * d.hkv * kGroup + nx.it.g * kGroup + h) * kD)[ch];
                    *reinterpret_cast<uint4 *>(sQ + (C::QB == 2 ? buf : 0) * C::OpBytes + blk_op_offset<NP>(row, ch * 8)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&q_ready[buf]);
            }
        };
        int jg = 0, ic = 0, w = 0;
        bool ok = read_slot(0, &w);
        if (ok) stage_q(w, 0);
        for (; ok && w < n_items; ++ic) {
            const BlockItem bi = block_item_of(a, w);
            const Item &it = bi.it;
            float m_run[NH], l_part[NH];
#pragma unroll
            for (int q = 0; q < NH; ++q) {
                m_run[q] = -INFINITY;
                l_part[q] = 0.f;
            }
            for (int t = 0; t < it.n_tiles; ++t, ++jg) {
                const bool got = mbar_wait(&s_full[jg & 1], (jg >> 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[NH];
#pragma unroll
                for (int cb = 0; cb < NH; cb += 4) blk_tmem_ld4(tmem + (jg & 1) * NP + q0 + cb + lane_base, &sr[cb]);
                tmem_ld_wait();
#pragma unroll
                for (int cb = 0; cb < NH; cb += 4) blk_reg_fence4(&sr[cb]);
                const bool block_tile = t == bi.cache_tiles;
                const int32_t e = block_tile ? r : it.e_begin + t * kTok + r;
                int t_lo, t_hi;
                key_query_range(a, bi, block_tile, e, &t_lo, &t_hi);
                // a full head's tile inside the cached length: every key for every query
                const bool dense = !block_tile && !it.ring && it.e_begin + (t + 1) * kTok <= it.e_end;
                float s[NH];
                bool exceed = false;
#pragma unroll
                for (int q = 0; q < NH; ++q) {
                    const int tq = (q0 + q) / kGroup;
                    const bool keep = q0 + q < NR && (dense || (tq >= t_lo && tq <= t_hi));
                    s[q] = keep ? __uint_as_float(sr[q]) : -INFINITY;
                    exceed |= s[q] * c > m_run[q] + 8.f;
                }
                // The running max of a row moves only when some score exceeds it by
                // more than 2^8.  One vote over the eight warps settles whether any
                // row of this tile does; if none does, the tile's max is not needed
                // and every row keeps its max (the same result as computing it).
                if (softmax_vote_any(exceed, NSM)) {
                    float mx[RP];
#pragma unroll
                    for (int q = 0; q < RP; ++q) mx[q] = q < NH ? s[q] : -INFINITY;
                    const float mrow = lane_row_reduce<RP, 0>(mx, lane);
                    if (lane == (lane_row<RP>(lane) << (5 - rp_bits<RP>())) && lane_row<RP>(lane) < NH)
                        red_max[jg & 1][quarter][q0 + lane_row<RP>(lane)] = mrow;
                    sm_sync();
                    float alpha[NH];
                    bool rescale = false;
#pragma unroll
                    for (int q = 0; q < NH; q += 4) {
                        float4 v4[4];
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4)
                            v4[w4] = *reinterpret_cast<const float4 *>(&red_max[jg & 1][w4][q0 + q]);
                        const float mj[4] = {fmaxf(fmaxf(v4[0].x, v4[1].x), fmaxf(v4[2].x, v4[3].x)),
                                             fmaxf(fmaxf(v4[0].y, v4[1].y), fmaxf(v4[2].y, v4[3].y)),
                                             fmaxf(fmaxf(v4[0].z, v4[1].z), fmaxf(v4[2].z, v4[3].z)),
                                             fmaxf(fmaxf(v4[0].w, v4[1].w), fmaxf(v4[2].w, v4[3].w))};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float m_tile = mj[u] * c;
                            alpha[q + u] = 1.f;
                            if (m_tile > m_run[q + u] + 8.f) {
                                alpha[q + u] = (m_run[q + u] == -INFINITY) ? 0.f : ex2_approx(m_run[q + u] - m_tile);
                                m_run[q + u] = m_tile;
                                l_part[q + u] *= alpha[q + u];
                                rescale = true;
                            }
                        }
                    }
                    if (t > 0 && __any_sync(0xffffffffu, rescale)) {
                        // O^T must hold every earlier tile's product before it is scaled
                        const bool prev = mbar_wait(&o_done[(jg - 1) & 1], ((jg - 1) >> 1) & 1);
                        __syncwarp();
                        if (!__all_sync(0xffffffffu, prev)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int cb = 0; cb < NH; cb += 4) {
                            uint32_t orr[4];
                            blk_tmem_ld4(o_tmem + cb, orr);
                            tmem_ld_wait();
                            blk_reg_fence4(orr);
#pragma unroll
                            for (int q = 0; q < 4; ++q) orr[q] = __float_as_uint(__uint_as_float(orr[q]) * alpha[cb + q]);
                            blk_tmem_st4(o_tmem + cb, orr);
                        }
                        tmem_st_wait();
                    }
                }
                float p[NH];
#pragma unroll
                for (int q = 0; q < NH; ++q) {
                    // rounded to bf16 here: the PV product and the row sum use the same weights
                    p[q] = __bfloat162float(__float2bfloat16_rn(
                        ex2_approx(fmaf(s[q], c, m_run[q] == -INFINITY ? 0.f : -m_run[q]))));
                    l_part[q] += p[q];
                }
                // the P^T buffer was last read by the PV of tile jg - PB
                if (jg >= C::PB) {
                    const int pj = jg - C::PB;
                    const bool prev = mbar_wait(&o_done[pj & 1], (pj >> 1) & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, prev)) { ok = false; break; }
                    tc_fence_after();
                }
                if (t_lo > t_hi && part == 0) {
                    // a key no query keeps: its V row must not reach the PV product
                    char *vrow = sKV + (jg % ST) * kDecStageBytes + kDecTileBytes + r * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        reinterpret_cast<uint4 *>(vrow)[i] = make_uint4(0, 0, 0, 0);
                        reinterpret_cast<uint4 *>(vrow + kDecHalfBytes)[i] = make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int q = 0; q < NH; ++q)
                    if (q0 + q < NR)
                        *reinterpret_cast<__nv_bfloat16 *>(sP + (C::PB == 2 ? (jg & 1) : 0) * C::OpBytes +
                                                           blk_op_offset<NP>(q0 + q, r)) =
                            __float2bfloat16_rn(p[q]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full);
            }
            if (!ok) break;
            // the next item: its Q may be staged now (this item's S products are all read)
            int w_next = n_items;
            if (!(ok = read_slot(ic + 1, &w_next))) break;
            stage_q(w_next, (ic + 1) & 1);
            // ------------------------------------------------------------ item epilogue
            float acc[NH];
#pragma unroll
            for (int q = 0; q < NH; ++q) acc[q] = 0.f;
            if (it.n_tiles > 0) {
                const bool done = mbar_wait(&o_done[(jg - 1) & 1], ((jg - 1) >> 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, done)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < NH; cb += 4) {
                    uint32_t orr[4];
                    blk_tmem_ld4(o_tmem + cb, orr);
                    tmem_ld_wait();
                    blk_reg_fence4(orr);
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[cb + q] = __uint_as_float(orr[q]);
                }
            }
            // l: this warp's 32 tokens per row, then the four quarters in a fixed order
            float lsum[RP];
#pragma unroll
            for (int q = 0; q < RP; ++q) lsum[q] = q < NH ? l_part[q] : 0.f;
            const float lrow = lane_row_reduce<RP, 1>(lsum, lane);
            const int my_row = lane_row<RP>(lane);
            const bool row_writer = lane == (my_row << (5 - rp_bits<RP>()));
            if (row_writer && my_row < NH) red_sum[quarter][q0 + my_row] = lrow;
            sm_sync();
            float *part = d.part + (((size_t)it.b * d.hkv + it.g) * a.part_slots + it.split) * C::PartFloats;
#pragma unroll
            for (int q = 0; q < NH; ++q)
                if (q0 + q < NR) part[2 * NR + (q0 + q) * kD + r] = acc[q];
            if (quarter == 0 && row_writer && my_row < NH && q0 + my_row < NR) {
                const int q = q0 + my_row;
                float mq = -INFINITY;
#pragma unroll
                for (int i = 0; i < NH; ++i)
                    if (i == my_row) mq = m_run[i];
                part[q] = mq;
                part[NR + q] = (red_sum[0][q] + red_sum[1][q]) + (red_sum[2][q] + red_sum[3][q]);
            }
            sm_sync();
            w = w_next;
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TmemCols);
    }
}

// Folds the splits (the last one holds the block's keys too) and the sink
// logit of every (sequence, block token, query head).
template <int kQ>
__global__ void __launch_bounds__(kD) decode_block_merge(const __grid_constant__ BlockArgs a) {
    using C = BlockCfg<kQ>;
    constexpr int NR = C::NR;
    pdl_wait();
    const DecodeArgs &d = a.d;
    const int hq_all = d.hkv * kGroup;
    const int idx = blockIdx.x;                      // (b * q_len + t) * Hq + h
    const int h = idx % hq_all;
    const int t = (idx / hq_all) % kQ;
    const int b = idx / hq_all / kQ;
    const int g = h / kGroup, row = t * kGroup + h % kGroup;
    const int splits = d.heads.is_full[g] ? d.splits_full : d.splits_ring;
    const float *part = d.part + ((size_t)b * d.hkv + g) * a.part_slots * C::PartFloats;
    const bool has_sink = d.sink_logit != nullptr;
    const float sig = has_sink ? d.sink_logit[h] * kLog2eF : -INFINITY;
    float M = sig;
    for (int i = 0; i < splits; ++i) M = fmaxf(M, part[i * C::PartFloats + row]);
    float den = 0.f, num = 0.f;
    if (M != -INFINITY) {
        for (int i = 0; i < splits; ++i) {
            const float *ps = part + i * C::PartFloats;
            const float ms = ps[row];
            if (ms == -INFINITY) continue;
            const float f = ex2_approx(ms - M);
            den += f * ps[NR + row];
            num += f * ps[2 * NR + row * kD + threadIdx.x];
        }
        if (has_sink) den += ex2_approx(sig - M);
    }
    float o = den > 0.f ? num / den : 0.f;
    if (d.gate_mode != 0) {
        const float gv = __bfloat162float(d.gate[d.gate_mode == 1 ? (size_t)idx * kD + threadIdx.x : (size_t)idx]);
        o = o / (1.f + ex2_approx(-gv * kLog2eF));
    }
    a.out[(size_t)idx * kD + threadIdx.x] = __float2bfloat16_rn(o);
    if (a.lse != nullptr && threadIdx.x == 0)
        a.lse[idx] = den > 0.f ? (M + __log2f(den)) * kLn2F : -INFINITY;
}

}  // namespace duo
