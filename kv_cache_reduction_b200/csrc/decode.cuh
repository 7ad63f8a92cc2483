// decode.cuh -- one-token split-KV decode over the hybrid cache, on tcgen05.
//
// DuoAttention Laguna Adapter card (Summary, Why It Works): a full-context
// KV head attends over every cached token, a streaming head over its sink
// slots plus its ring of recent tokens; sliding-window layers (Laguna
// sliding-window articles) over a ring of the last `window` tokens, with an
// optional per-query-head sink logit (Laguna XS 2.1 article, attention-sink
// item).  The six query heads of a GQA group share every K/V row read.
//
// Work items are (sequence, KV head, split).  One persistent CTA per SM
// walks its share of the items (a balanced static split):
//   warps 0-3  softmax and epilogue; thread r owns token r of a 128-token tile
//              (and dimension r of the output)
//   warp 4     producer: TMA loads of 128-token K and V tiles (2-D tensor
//              maps, 64-column boxes, 128-byte swizzle, no multicast) into a
//              three-stage ring
//   warp 5     TMEM owner and MMA issuer, "swap AB" so that tokens fill M:
//                S^T[128 tok x 16] = K_tile[128 x 128] . Q^T   (Q: 6 heads + zero rows)
//                O^T[128 d  x 16] += V_tile^T . P^T            (P^T written by the softmax)
//              QK of tile t+1 is issued before PV of tile t.
// Ring heads load their whole slot array in slot order and mask the slots
// that hold no valid token (attention does not depend on key order, keys are
// stored after RoPE).  Rows of V that belong to invalid tokens are zeroed in
// shared memory before the PV product, so stale cache memory never reaches
// it.  Each item leaves (m, l, acc) in log2 units in the workspace;
// decode_merge folds the splits and the sink logit.  Every reduction has a
// fixed order, so the result is bitwise reproducible.
#pragma once

#include <cuda.h>

#include "kv_append.cuh"
#include "ptx.cuh"

namespace duo {

constexpr int kD = 128;
constexpr int kGroup = 6;                  // query heads per KV head
constexpr int kNPad = 16;                  // MMA N: the group's heads padded with zero rows
constexpr int kTok = 128;                  // tokens per tile (MMA M)
constexpr int kDecStages = 3;
constexpr uint32_t kDecTileBytes = kTok * kD * 2;        // 32 KB: one K or V tile
constexpr uint32_t kDecHalfBytes = kDecTileBytes / 2;    // one 64-column swizzled box
constexpr uint32_t kDecStageBytes = 2 * kDecTileBytes;   // K + V
constexpr uint32_t kOpBytes = kNPad * kD * 2;            // 4 KB: Q or P^T operand
constexpr size_t kDecSmem = 1024 + kDecStages * kDecStageBytes + 3 * kOpBytes;
constexpr int kDecThreads = 192;
constexpr int kPartFloats = kGroup * (kD + 2);           // m[6], l[6], acc[6][128]
constexpr uint32_t kDecTmemCols = 64;                    // S^T x2 (16 each) + O^T (16)

struct DecodeArgs {
    CUtensorMap tm_fk, tm_fv;       // full caches as 2-D (128, B*n_full*capacity)
    CUtensorMap tm_rk, tm_rv;       // ring caches as 2-D (128, B*n_ring*slots)
    const int32_t *seq_len, *ring_head;
    const __nv_bfloat16 *q;         // [B][Hq][D]
    const float *sink_logit;        // [Hq] or null
    float *part;                    // [B][Hkv][max_splits][kPartFloats]
    __nv_bfloat16 *out;             // [B][Hq][D]
    float *lse;                     // [B][Hq] or null
    int64_t capacity;
    int32_t batch, hkv, n_full, n_ring;
    int32_t sink, ring, slots;
    int32_t chunk_full, splits_full, chunk_ring, splits_ring, max_splits, n_items;
    float scale_log2;               // softmax_scale * log2(e)
    const __nv_bfloat16 *gate;      // output gate pre-activations or null
    int32_t gate_mode;              // 0 none, 1 per (head, channel) [B][Hq][D], 2 per head [B][Hq]
    int32_t withhold_tile;          // failure-injection hook: CTA 0 issues no load from this tile on (-1: off)
    int8_t full_head[64];           // full rank -> KV head
    int8_t ring_head_of[64];        // ring rank -> KV head
    HeadTable heads;
};

// One work item: rows [row0 + e_begin, row0 + e_end) of a cache tensor map.
// For a ring item the index e is the slot; slot validity follows the ring
// state (sink slots below n_sink; ring slots among the cnt written last).
struct Item {
    int b, g, split;
    bool ring;
    int32_t row0, e_begin, e_end;
    int32_t n_sink, cnt, ring_base;
    int n_tiles;
};

__device__ __forceinline__ Item item_of(const DecodeArgs &a, int w) {
    Item it;
    const int n_full_items = a.batch * a.n_full * a.splits_full;
    if (w < n_full_items) {
        const int unit = w / a.splits_full;
        it.split = w % a.splits_full;
        it.b = unit / a.n_full;
        const int r = unit % a.n_full;
        it.g = a.full_head[r];
        it.ring = false;
        it.row0 = (int32_t)(((int64_t)it.b * a.n_full + r) * a.capacity);
        // a full head's rows end at the capacity, whatever seq_len says
        const int32_t n = (int32_t)min((int64_t)a.seq_len[it.b], a.capacity);
        it.e_begin = it.split * a.chunk_full;
        it.e_end = min(n, it.e_begin + a.chunk_full);
        it.n_sink = 0;
        it.cnt = 0;
        it.ring_base = 0;
    } else {
        w -= n_full_items;
        const int unit = w / a.splits_ring;
        it.split = w % a.splits_ring;
        it.b = unit / a.n_ring;
        const int r = unit % a.n_ring;
        it.g = a.ring_head_of[r];
        it.ring = true;
        it.row0 = (int32_t)(((int64_t)it.b * a.n_ring + r) * a.slots);
        const int32_t n = a.seq_len[it.b];
        it.n_sink = min(n, a.sink);
        it.cnt = min(max(n - a.sink, 0), a.ring);
        int32_t base = (a.ring_head[it.b] - it.cnt) % a.ring;
        it.ring_base = base < 0 ? base + a.ring : base;
        it.e_begin = it.split * a.chunk_ring;
        // nothing valid past the sink while the ring is empty
        const int32_t last = (it.cnt == 0) ? it.n_sink : a.slots;
        it.e_end = min(last, it.e_begin + a.chunk_ring);
    }
    it.n_tiles = it.e_end > it.e_begin ? (it.e_end - it.e_begin + kTok - 1) / kTok : 0;
    return it;
}

__device__ __forceinline__ bool token_valid(const Item &it, int32_t e, int32_t sink, int32_t ring) {
    if (e >= it.e_end) return false;
    if (!it.ring) return true;
    if (e < sink) return e < it.n_sink;
    int32_t r = e - sink - it.ring_base;
    if (r < 0) r += ring;
    return r < it.cnt;
}

// Byte offset of element (row, k) in a [16 rows][128] bf16 K-major operand
// stored as two 64-column halves with the 128-byte swizzle.
__device__ __forceinline__ uint32_t op_offset(int row, int k) {
    const int half = k >> 6, kk = k & 63;
    return half * 2048 + (row >> 3) * 1024 + (row & 7) * 128 + ((((kk >> 3) ^ (row & 7))) << 4) +
           (kk & 7) * 2;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void reg_fence8(uint32_t (&r)[8]) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]));
}

// Named barrier over the four softmax warps (threads 0..127).
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t v_addr, uint32_t p_addr,
                                         uint32_t idesc, bool first) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
        mma_ss(o_tmem, smem_desc_sw128(v_addr + k * 2048, kDecHalfBytes, 1024),
               smem_desc_sw128(p_addr + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024), idesc,
               (first && k == 0) ? 0u : 1u);
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_split(const __grid_constant__ DecodeArgs a) {
    extern __shared__ __align__(16) char dsmem_base[];
    char *smem = dsmem_base + ((1024u - (smem_u32(dsmem_base) & 1023u)) & 1023u);
    char *sKV = smem;                                         // [stages][K 32 KB | V 32 KB]
    char *sQ = smem + kDecStages * kDecStageBytes;            // [2 items][4 KB]
    char *sP = sQ + 2 * kOpBytes;                             // 4 KB
    __shared__ uint64_t kv_full[kDecStages], kv_empty[kDecStages];
    __shared__ uint64_t s_full[2], p_full, o_done, q_ready[2], mma_drained;
    __shared__ uint32_t tmem_base;
    __shared__ float red_max[2][4][kGroup], red_sum[4][kGroup];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecStages; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&q_ready[i], 4);
        }
        mbar_init(&p_full, 4);
        mbar_init(&o_done, 1);
        mbar_init(&mma_drained, 1);
        fence_mbar_init();
    }
    if (warp < 4) {
        // operand rows 6..15 stay zero for the whole kernel
        for (int i = threadIdx.x; i < 3 * (int)kOpBytes / 16; i += 128)
            reinterpret_cast<uint4 *>(sQ)[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(&tmem_base, kDecTmemCols);
        tmem_relinquish();
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    // launched as a programmatic dependent: the set-up above overlapped the
    // previous kernel (an append, or the last call's merge, which reads the
    // workspace this kernel writes); nothing global is touched before this
    pdl_wait();

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (a.n_full > 0) {
                prefetch_tmap(&a.tm_fk);
                prefetch_tmap(&a.tm_fv);
            }
            if (a.n_ring > 0) {
                prefetch_tmap(&a.tm_rk);
                prefetch_tmap(&a.tm_rv);
            }
            int jg = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < a.n_items && ok; w += gridDim.x) {
                const Item it = item_of(a, w);
                const CUtensorMap *tk = it.ring ? &a.tm_rk : &a.tm_fk;
                const CUtensorMap *tv = it.ring ? &a.tm_rv : &a.tm_fv;
                for (int t = 0; t < it.n_tiles; ++t, ++jg) {
                    const int st = jg % kDecStages;
                    if (jg >= kDecStages && !(ok = mbar_wait(&kv_empty[st], ((jg / kDecStages) - 1) & 1))) break;
                    // failure-detection test: stop feeding this CTA so that the
                    // consumers' bounded waits expire (nothing stays in flight)
                    if (blockIdx.x == 0 && jg == a.withhold_tile) { ok = false; break; }
                    char *ks = sKV + st * kDecStageBytes;
                    const int row = it.row0 + it.e_begin + t * kTok;
                    mbar_expect_tx(&kv_full[st], kDecStageBytes);
                    tma_load_2d(ks, tk, 0, row, &kv_full[st]);
                    tma_load_2d(ks + kDecHalfBytes, tk, 64, row, &kv_full[st]);
                    tma_load_2d(ks + kDecTileBytes, tv, 0, row, &kv_full[st]);
                    tma_load_2d(ks + kDecTileBytes + kDecHalfBytes, tv, 64, row, &kv_full[st]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16_f32(kTok, kNPad, 0, 0);
            const uint32_t id_pv = idesc_bf16_f32(kD, kNPad, 1, 0);
            const uint32_t kv_addr = smem_u32(sKV), q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            const uint32_t o_tmem = tmem + 2 * kNPad;
            int jg = 0, ic = 0;            // tiles and non-empty items so far
            bool ok = true;
            bool pend = false;             // a PV is owed for the previous tile
            int pend_st = 0;
            bool pend_first = false;
            for (int w = blockIdx.x; w < a.n_items && ok; w += gridDim.x) {
                const Item it = item_of(a, w);
                if (it.n_tiles == 0) continue;
                if (!(ok = mbar_wait(&q_ready[ic & 1], (ic >> 1) & 1))) break;
                for (int t = 0; t < it.n_tiles && ok; ++t, ++jg) {
                    const int st = jg % kDecStages;
                    if (!(ok = mbar_wait(&kv_full[st], (jg / kDecStages) & 1))) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * kDecHalfBytes + (k & 3) * 32;
                        const uint32_t qoff = (ic & 1) * kOpBytes + (k >> 2) * 2048 + (k & 3) * 32;
                        mma_ss(tmem + (jg & 1) * kNPad,
                               smem_desc_sw128(kv_addr + st * kDecStageBytes + off, 16, 1024),
                               smem_desc_sw128(q_addr + qoff, 16, 1024), id_qk, k > 0);
                    }
                    mma_commit(&s_full[jg & 1]);
                    if (pend) {
                        // PV of the previous tile, one tile behind its QK
                        if (!(ok = mbar_wait(&p_full, (jg - 1) & 1))) break;
                        tc_fence_after();
                        issue_pv(o_tmem, kv_addr + pend_st * kDecStageBytes + kDecTileBytes, p_addr,
                                 id_pv, pend_first);
                        mma_commit(&o_done);
                        mma_commit(&kv_empty[pend_st]);
                    }
                    pend = true;
                    pend_st = st;
                    pend_first = (t == 0);
                }
                ++ic;
            }
            if (ok && pend && mbar_wait(&p_full, (jg - 1) & 1)) {
                tc_fence_after();
                issue_pv(o_tmem, kv_addr + pend_st * kDecStageBytes + kDecTileBytes, p_addr, id_pv,
                         pend_first);
                mma_commit(&o_done);
                mma_commit(&kv_empty[pend_st]);
            }
            // every product issued has completed before the tensor memory is freed
            // (on an early exit some may still run)
            mma_commit(&mma_drained);
            mbar_wait(&mma_drained, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int r = threadIdx.x;                           // token row / output dimension
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t o_tmem = tmem + 2 * kNPad + lane_base;
        const float c = a.scale_log2;
        // Stages the 6 query rows of the first non-empty item at or after w
        // as the swizzled K-major Q operand in buffer `buf`.
        auto stage_q = [&](int w, int buf) {
            for (; w < a.n_items; w += gridDim.x) {
                const Item nx = item_of(a, w);
                if (nx.n_tiles == 0) continue;
                if (r < kGroup * 16) {
                    const int h = r >> 4, ch = r & 15;
                    const uint4 v = reinterpret_cast<const uint4 *>(
                        a.q + ((size_t)nx.b * a.hkv * kGroup + nx.g * kGroup + h) * kD)[ch];
                    *reinterpret_cast<uint4 *>(sQ + buf * kOpBytes + op_offset(h, ch * 8)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&q_ready[buf]);
                return;
            }
        };
        int jg = 0, ic = 0;                // tiles and non-empty items so far
        bool ok = true;
        stage_q(blockIdx.x, 0);
        for (int w = blockIdx.x; w < a.n_items && ok; w += gridDim.x) {
            const Item it = item_of(a, w);
            float m_run[kGroup], l_part[kGroup];
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                m_run[h] = -INFINITY;
                l_part[h] = 0.f;
            }
            for (int t = 0; t < it.n_tiles; ++t, ++jg) {
                const bool got = mbar_wait(&s_full[jg & 1], (jg >> 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[8];
                tmem_ld8(tmem + (jg & 1) * kNPad + lane_base, sr);
                tmem_ld_wait();
                reg_fence8(sr);
                const int32_t e = it.e_begin + t * kTok + r;
                const bool valid = token_valid(it, e, a.sink, a.ring);
                float s[kGroup], mx[kGroup];
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    s[h] = valid ? __uint_as_float(sr[h]) : -INFINITY;
                    mx[h] = s[h];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], off));
                if (lane == 0)
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) red_max[jg & 1][warp][h] = mx[h];
                softmax_sync();
                float alpha[kGroup], m_sub[kGroup];
                bool rescale = false;
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    const float m_tile = fmaxf(fmaxf(red_max[jg & 1][0][h], red_max[jg & 1][1][h]),
                                               fmaxf(red_max[jg & 1][2][h], red_max[jg & 1][3][h])) * c;
                    alpha[h] = 1.f;
                    // keep the stale max unless the new one is more than 2^8 larger
                    if (m_tile > m_run[h] + 8.f) {
                        alpha[h] = (m_run[h] == -INFINITY) ? 0.f : ex2_approx(m_run[h] - m_tile);
                        m_run[h] = m_tile;
                        rescale = true;
                    }
                    m_sub[h] = (m_run[h] == -INFINITY) ? 0.f : m_run[h];
                }
                float p[kGroup];
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    p[h] = ex2_approx(fmaf(s[h], c, -m_sub[h]));
                    l_part[h] = fmaf(l_part[h], alpha[h], p[h]);
                }
                // the previous PV must be done with P^T and with O^T
                if (jg > 0) {
                    const bool prev = mbar_wait(&o_done, (jg - 1) & 1);
                    __syncwarp();
                    if (!__all_sync(0xffffffffu, prev)) { ok = false; break; }
                    tc_fence_after();
                }
                if (t > 0 && rescale) {
                    uint32_t orr[8];
                    tmem_ld8(o_tmem, orr);
                    tmem_ld_wait();
                    reg_fence8(orr);
#pragma unroll
                    for (int h = 0; h < kGroup; ++h) orr[h] = __float_as_uint(__uint_as_float(orr[h]) * alpha[h]);
                    tmem_st8(o_tmem, orr);
                    tmem_st_wait();
                }
                if (!valid) {
                    // stale cache rows must not reach the PV product (0 x NaN)
                    char *vrow = sKV + (jg % kDecStages) * kDecStageBytes + kDecTileBytes + r * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        reinterpret_cast<uint4 *>(vrow)[i] = make_uint4(0, 0, 0, 0);
                        reinterpret_cast<uint4 *>(vrow + kDecHalfBytes)[i] = make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int h = 0; h < kGroup; ++h)
                    *reinterpret_cast<__nv_bfloat16 *>(sP + op_offset(h, r)) = __float2bfloat16_rn(p[h]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full);
            }
            if (!ok) break;
            if (it.n_tiles > 0) {
                // the MMA warp may start the next item's QK while this epilogue runs
                ++ic;
                stage_q(w + gridDim.x, ic & 1);
            }
            // ------------------------------------------------------------ item epilogue
            float acc[kGroup];
#pragma unroll
            for (int h = 0; h < kGroup; ++h) acc[h] = 0.f;
            if (it.n_tiles > 0) {
                const bool done = mbar_wait(&o_done, (jg - 1) & 1);
                __syncwarp();
                if (!__all_sync(0xffffffffu, done)) { ok = false; break; }
                tc_fence_after();
                uint32_t orr[8];
                tmem_ld8(o_tmem, orr);
                tmem_ld_wait();
                reg_fence8(orr);
#pragma unroll
                for (int h = 0; h < kGroup; ++h) acc[h] = __uint_as_float(orr[h]);
            }
            // l: sum of the 128 per-token partials, in a fixed order
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int h = 0; h < kGroup; ++h) l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], off);
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < kGroup; ++h) red_sum[warp][h] = l_part[h];
            softmax_sync();
            float *part = a.part + (((size_t)it.b * a.hkv + it.g) * a.max_splits + it.split) * kPartFloats;
#pragma unroll
            for (int h = 0; h < kGroup; ++h) part[2 * kGroup + h * kD + r] = acc[h];
            if (r < kGroup) {
                part[r] = m_run[r];
                part[kGroup + r] = (red_sum[0][r] + red_sum[1][r]) + (red_sum[2][r] + red_sum[3][r]);
            }
            softmax_sync();    // red_sum is reused by the next item
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    // this CTA's partials are written: the merge grid may start launching
    // (it still waits for the whole grid before reading them)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kDecTmemCols);
    }
}

// The split fold of one output element in one pass: with M entering as the
// sink logit (log2 units) or -inf and den = num = 0, it leaves
// M = max(M, m_s) over the splits, den = sum_s 2^(m_s - M) l_s and
// num = sum_s 2^(m_s - M) acc_s (splits with m_s = -inf skipped).  m_s, l_s,
// acc_s sit at floats m_off, l_off, a_off of split s's record of `stride`
// floats.  The partials were written by the previous grid and sit in L2: the
// loads go out kFoldBatch splits at a time (only real records are read), the
// running max rises batch by batch and the sums so far are rescaled when it
// does, so a fold costs one L2 round trip per batch.
template <int kFoldBatch>
__device__ __forceinline__ void fold_splits(const float *part, int stride, int splits, int m_off, int l_off,
                                            int a_off, float *M_io, float *den_io, float *num_io) {
    float M = *M_io, den = 0.f, num = 0.f;
    for (int s0 = 0; s0 < splits; s0 += kFoldBatch) {
        float mv[kFoldBatch], lv[kFoldBatch], av[kFoldBatch];
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) {
            mv[i] = -INFINITY;
            lv[i] = av[i] = 0.f;
            if (s0 + i < splits) {
                const float *ps = part + (s0 + i) * stride;
                mv[i] = ps[m_off];
                lv[i] = ps[l_off];
                av[i] = ps[a_off];
            }
        }
        float Mb = M;
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) Mb = fmaxf(Mb, mv[i]);
        if (Mb == -INFINITY) continue;
        if (Mb > M) {
            const float r = ex2_approx(M - Mb);       // 0 while M is -inf (the sums are 0 then)
            den *= r;
            num *= r;
            M = Mb;
        }
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) {
            if (mv[i] == -INFINITY) continue;
            const float f = ex2_approx(mv[i] - M);
            den += f * lv[i];
            num += f * av[i];
        }
    }
    *M_io = M;
    *den_io = den;
    *num_io = num;
}

// fold_splits for four consecutive output elements (acc_s a float4 at a_off).
template <int kFoldBatch>
__device__ __forceinline__ void fold_splits4(const float *part, int stride, int splits, int m_off, int l_off,
                                             int a_off, float *M_io, float *den_io, float4 *num_io) {
    float M = *M_io, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < splits; s0 += kFoldBatch) {
        float mv[kFoldBatch], lv[kFoldBatch];
        float4 av[kFoldBatch];
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) {
            mv[i] = -INFINITY;
            lv[i] = 0.f;
            av[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s0 + i < splits) {
                const float *ps = part + (s0 + i) * stride;
                mv[i] = ps[m_off];
                lv[i] = ps[l_off];
                av[i] = *reinterpret_cast<const float4 *>(ps + a_off);
            }
        }
        float Mb = M;
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) Mb = fmaxf(Mb, mv[i]);
        if (Mb == -INFINITY) continue;
        if (Mb > M) {
            const float r = ex2_approx(M - Mb);
            den *= r;
            num.x *= r;
            num.y *= r;
            num.z *= r;
            num.w *= r;
            M = Mb;
        }
#pragma unroll
        for (int i = 0; i < kFoldBatch; ++i) {
            if (mv[i] == -INFINITY) continue;
            const float f = ex2_approx(mv[i] - M);
            den += f * lv[i];
            num.x += f * av[i].x;
            num.y += f * av[i].y;
            num.z += f * av[i].z;
            num.w += f * av[i].w;
        }
    }
    *M_io = M;
    *den_io = den;
    *num_io = num;
}

// Four bf16 (two packed words) to floats.
__device__ __forceinline__ void unpack_bf16x4(uint2 w, float (&f)[4]) {
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xffff0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xffff0000u);
}

// O = num / den for four output elements, times sigmoid of the output gate
// (per channel: the four gates at gate4; per head: g_head), as four bf16.
__device__ __forceinline__ uint2 fold_out4(float4 num, float den, int gate_mode, const __nv_bfloat16 *gate4,
                                           float g_head) {
    float o[4] = {num.x, num.y, num.z, num.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = den > 0.f ? o[e] / den : 0.f;
    if (gate_mode == 1) {
        const uint2 gw = *reinterpret_cast<const uint2 *>(gate4);
        const uint32_t gv[2] = {gw.x, gw.y};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float gx = __uint_as_float(e & 1 ? (gv[e >> 1] & 0xffff0000u) : (gv[e >> 1] << 16));
            o[e] = o[e] / (1.f + ex2_approx(-gx * kLog2eF));
        }
    } else if (gate_mode == 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = o[e] / (1.f + ex2_approx(-g_head * kLog2eF));
    }
    return make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
}

constexpr int kMergeThreads = kGroup * 32;      // decode_block_merge: a warp per query head

// Folds the splits of every (sequence, query head) and the sink logit:
// O = sum_s 2^(m_s - M) acc_s / (sum_s 2^(m_s - M) l_s + 2^(sigma*log2e - M)).
// One CTA per (sequence, KV head), thread (hh, r) giving dimension r of head
// hh: six times fewer CTAs than one per head (the launch of many small CTAs
// bounds a merge this short).
__global__ void __launch_bounds__(kD * kGroup) decode_merge(const __grid_constant__ DecodeArgs a) {
    // launched as a programmatic dependent of decode_split: wait until that
    // grid has completed and its partials are visible
    pdl_wait();
    const int b = blockIdx.x / a.hkv, g = blockIdx.x % a.hkv;
    const int hh = threadIdx.x / kD, r = threadIdx.x % kD;
    const int h = g * kGroup + hh;
    const size_t bh = (size_t)b * a.hkv * kGroup + h;
    const int splits = a.heads.is_full[g] ? a.splits_full : a.splits_ring;
    const float *part = a.part + ((size_t)b * a.hkv + g) * a.max_splits * kPartFloats;
    const bool has_sink = a.sink_logit != nullptr;
    const float sig = has_sink ? a.sink_logit[h] * kLog2eF : -INFINITY;
    float M = sig, den = 0.f, num = 0.f;
    fold_splits<4>(part, kPartFloats, splits, hh, kGroup + hh, 2 * kGroup + hh * kD + r, &M, &den, &num);
    if (M != -INFINITY && has_sink) den += ex2_approx(sig - M);
    float o = den > 0.f ? num / den : 0.f;
    if (a.gate_mode != 0) {
        // output gate: o * sigmoid(g), g per channel or per head
        const float gv = __bfloat162float(a.gate[a.gate_mode == 1 ? bh * kD + r : bh]);
        o = o / (1.f + ex2_approx(-gv * kLog2eF));
    }
    a.out[bh * kD + r] = __float2bfloat16_rn(o);
    if (a.lse != nullptr && r == 0) a.lse[bh] = den > 0.f ? (M + log2f(den)) * kLn2F : -INFINITY;
}

}  // namespace duo
