// decode.cuh -- one-token split-KV decode over the hybrid cache.
//
// DuoAttention Laguna Adapter card (Summary, Why It Works): a full-context
// KV head attends over every cached token, a streaming head over its sink
// slots plus its ring of recent tokens; sliding-window layers (Laguna
// sliding-window articles) over a ring of the last `window` tokens, with an
// optional per-query-head sink logit (Laguna XS 2.1 article, attention-sink
// item).  The six query heads of a GQA group share every K/V row read.
//
// Work items are (sequence, KV head, split).  A CTA streams its split's K
// and V rows from HBM into shared memory with bulk async copies (a
// dedicated producer warp, STAGES-deep mbarrier ring), and eight compute
// warps run the dot products and the online softmax in fp32 registers.
// Its partial result (running max, sum, unnormalised output, in log2
// units) goes to the workspace; decode_merge folds the splits and the sink
// logit into the final output and log-sum-exp.
#pragma once

#include "kv_append.cuh"
#include "ptx.cuh"

namespace duo {

constexpr int kD = 128;
constexpr int kGroup = 6;                 // query heads per KV head
constexpr int kHalf = kGroup / 2;         // heads per compute group
constexpr int kDecTile = 64;              // tokens per pipeline stage
constexpr int kDecStages = 4;
constexpr int kDecComputeWarps = 8;
constexpr int kDecThreads = (kDecComputeWarps + 1) * 32;
constexpr int kRowBytes = kD * 2;         // one token of one head, bf16
constexpr int kStageBytes = kDecTile * kRowBytes * 2;   // K + V
constexpr int kPartFloats = kGroup * (kD + 2);          // m[6], l[6], acc[6][128]
constexpr size_t kDecSmem = (size_t)kDecStages * kStageBytes + 1024;

struct DecodeArgs {
    const __nv_bfloat16 *full_k, *full_v, *strm_k, *strm_v;
    const int32_t *seq_len, *ring_head;
    const __nv_bfloat16 *q;         // [B][Hq][D]
    const float *sink_logit;        // [Hq] or null
    float *part;                    // [B][Hkv][max_splits][kPartFloats]
    __nv_bfloat16 *out;             // [B][Hq][D]
    float *lse;                     // [B][Hq] or null
    int64_t capacity;
    int32_t batch, hkv, n_full, n_ring;
    int32_t sink, ring, slots;
    int32_t chunk_full, splits_full, chunk_ring, splits_ring, max_splits;
    float scale_log2;               // softmax_scale * log2(e)
    int8_t full_head[64];           // full rank -> KV head
    int8_t ring_head_of[64];        // ring rank -> KV head
    HeadTable heads;
};

// Tokens of one work item: logical index e in [e_begin, e_end) maps to a
// cache row.  Full heads: row e.  Ring heads: sink slot e for e < n_sink,
// else ring slot sink + (ring_base + e - n_sink) mod ring.
struct Span {
    const char *k_base;
    const char *v_base;
    int32_t e_begin, e_end;
    int32_t n_sink, ring_base;
    bool ring;
};

__device__ __forceinline__ int32_t span_slot(const Span &s, int32_t e, int32_t sink, int32_t ring) {
    if (!s.ring || e < s.n_sink) return e;
    int32_t r = s.ring_base + (e - s.n_sink);
    if (r >= ring) r -= ring;
    return sink + r;
}

// Issues the copies for tokens [e0, e0 + count) into one stage.
__device__ __forceinline__ void issue_tile(const Span &s, int32_t e0, int32_t count, char *stage,
                                           uint64_t *bar, int32_t sink, int32_t ring) {
    mbar_expect_tx(bar, (uint32_t)count * kRowBytes * 2);
    int32_t e = e0;
    const int32_t e1 = e0 + count;
    while (e < e1) {
        // extend a run of consecutive slots
        const int32_t slot0 = span_slot(s, e, sink, ring);
        int32_t run = 1;
        while (e + run < e1 && span_slot(s, e + run, sink, ring) == slot0 + run) ++run;
        const uint32_t bytes = (uint32_t)run * kRowBytes;
        char *dk = stage + (size_t)(e - e0) * kRowBytes;
        char *dv = stage + kDecTile * kRowBytes + (size_t)(e - e0) * kRowBytes;
        bulk_g2s(dk, s.k_base + (size_t)slot0 * kRowBytes, bytes, bar);
        bulk_g2s(dv, s.v_base + (size_t)slot0 * kRowBytes, bytes, bar);
        e += run;
    }
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_split(const DecodeArgs a) {
    extern __shared__ __align__(1024) char dsmem_raw[];
    char *smem = (char *)(((uintptr_t)dsmem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full_bar[kDecStages], empty_bar[kDecStages];
    __shared__ float red_m[32][kHalf], red_l[32][kHalf];

    // ---------------------------------------------------------------- work item
    const int32_t n_full_items = a.batch * a.n_full * a.splits_full;
    int32_t w = blockIdx.x;
    int b, g, split;
    Span s;
    if (w < n_full_items) {
        const int unit = w / a.splits_full;
        split = w % a.splits_full;
        b = unit / a.n_full;
        const int r = unit % a.n_full;
        g = a.full_head[r];
        const int32_t n = a.seq_len[b];
        const size_t base = (((size_t)b * a.n_full + r) * a.capacity) * kRowBytes;
        s.k_base = (const char *)a.full_k + base;
        s.v_base = (const char *)a.full_v + base;
        s.e_begin = split * a.chunk_full;
        s.e_end = min(n, s.e_begin + a.chunk_full);
        s.ring = false;
        s.n_sink = 0;
        s.ring_base = 0;
    } else {
        w -= n_full_items;
        const int unit = w / a.splits_ring;
        split = w % a.splits_ring;
        b = unit / a.n_ring;
        const int r = unit % a.n_ring;
        g = a.ring_head_of[r];
        const int32_t n = a.seq_len[b];
        const int32_t n_sink = min(n, a.sink);
        const int32_t cnt = min(max(n - a.sink, 0), a.ring);
        int32_t base_r = (a.ring_head[b] - cnt) % a.ring;
        if (base_r < 0) base_r += a.ring;
        const size_t base = (((size_t)b * a.n_ring + r) * a.slots) * kRowBytes;
        s.k_base = (const char *)a.strm_k + base;
        s.v_base = (const char *)a.strm_v + base;
        s.e_begin = split * a.chunk_ring;
        s.e_end = min(n_sink + cnt, s.e_begin + a.chunk_ring);
        s.ring = true;
        s.n_sink = n_sink;
        s.ring_base = base_r;
    }
    const int32_t total = max(s.e_end - s.e_begin, 0);
    const int32_t n_tiles = (total + kDecTile - 1) / kDecTile;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], kDecComputeWarps);
        }
        fence_mbar_init();
    }
    __syncwarp();      // reconverge before the CTA barrier (bar.sync is warp-aligned)
    __syncthreads();

    // ---------------------------------------------------------------- producer warp
    if (warp == kDecComputeWarps) {
        if (lane == 0) {
            for (int t = 0; t < n_tiles; ++t) {
                const int st = t % kDecStages;
                if (t >= kDecStages && !mbar_wait(&empty_bar[st], ((t / kDecStages) - 1) & 1)) break;
                const int32_t e0 = s.e_begin + t * kDecTile;
                issue_tile(s, e0, min(kDecTile, s.e_end - e0), smem + (size_t)st * kStageBytes,
                           &full_bar[st], a.sink, a.ring);
            }
        }
        __syncwarp();  // lanes 1..31 wait for the producer lane before any CTA barrier
        // the producer warp joins the final reduction below
    }

    // ---------------------------------------------------------------- compute warps
    // 32 groups of 8 lanes: group j handles heads [3*(j/16), 3*(j/16)+3) for
    // tokens j%16, j%16+16, ... of every tile; lane l of the group owns the
    // d-slices [8l, 8l+8) and [64+8l, 64+8l+8).  Pairs of adjacent d are
    // held packed and multiplied with the f32x2 FMA.
    const int grp = threadIdx.x >> 3;          // 0..31 for compute warps
    const int l8 = threadIdx.x & 7;
    const int half = grp >> 4;
    const int tok0 = grp & 15;
    // groups of one warp may run different trip counts on a short tile, so
    // every shuffle names only the 8 lanes of its own group
    const unsigned gmask = 0xFFu << (lane & 24);
    f2 qf[kHalf][8];
    f2 acc[kHalf][8];
    float m[kHalf], lsum[kHalf];
#pragma unroll
    for (int h = 0; h < kHalf; ++h) {
        m[h] = -INFINITY;
        lsum[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = f2_splat(0.f);
    }
    bool ok = true;
    if (warp < kDecComputeWarps) {
        const int hq0 = g * kGroup + half * kHalf;
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
            const uint4 *qrow = (const uint4 *)(a.q + ((size_t)b * a.hkv * kGroup + hq0 + h) * kD);
            const uint4 c0 = qrow[l8], c1 = qrow[l8 + 8];
            const uint32_t qw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                qf[h][i] = f2_make(bf16lo(qw[i]) * a.scale_log2, bf16hi(qw[i]) * a.scale_log2);
        }
        for (int t = 0; t < n_tiles && ok; ++t) {
            const int st = t % kDecStages;
            if (!mbar_wait(&full_bar[st], (t / kDecStages) & 1)) { ok = false; break; }
            const char *kt = smem + (size_t)st * kStageBytes;
            const char *vt = kt + kDecTile * kRowBytes;
            const int count = min(kDecTile, s.e_end - (s.e_begin + t * kDecTile));
#pragma unroll 1
            for (int tt = tok0; tt < count; tt += 16) {
                const uint4 k0 = *(const uint4 *)(kt + tt * kRowBytes + l8 * 16);
                const uint4 k1 = *(const uint4 *)(kt + tt * kRowBytes + (l8 + 8) * 16);
                const uint4 v0 = *(const uint4 *)(vt + tt * kRowBytes + l8 * 16);
                const uint4 v1 = *(const uint4 *)(vt + tt * kRowBytes + (l8 + 8) * 16);
                const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                f2 x[kHalf];
#pragma unroll
                for (int h = 0; h < kHalf; ++h) x[h] = f2_splat(0.f);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const f2 kf = f2_make(bf16lo(kw[i]), bf16hi(kw[i]));
#pragma unroll
                    for (int h = 0; h < kHalf; ++h) x[h] = f2_fma(qf[h][i], kf, x[h]);
                }
                float sc[kHalf];
#pragma unroll
                for (int h = 0; h < kHalf; ++h) sc[h] = f2_sum(x[h]);
#pragma unroll
                for (int off = 1; off < 8; off <<= 1)
#pragma unroll
                    for (int h = 0; h < kHalf; ++h) sc[h] += __shfl_xor_sync(gmask, sc[h], off);
                f2 pp[kHalf];
#pragma unroll
                for (int h = 0; h < kHalf; ++h) {
                    if (sc[h] > m[h]) {
                        const f2 alpha = f2_splat(ex2_approx(m[h] - sc[h]));
                        lsum[h] *= alpha.x;
                        m[h] = sc[h];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[h][i] = f2_mul(acc[h][i], alpha);
                    }
                    const float p = ex2_approx(sc[h] - m[h]);
                    lsum[h] += p;
                    pp[h] = f2_splat(p);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const f2 vf = f2_make(bf16lo(vw[i]), bf16hi(vw[i]));
#pragma unroll
                    for (int h = 0; h < kHalf; ++h) acc[h][i] = f2_fma(pp[h], vf, acc[h][i]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        __syncwarp();
    }
    __syncthreads();   // every copy has landed and been consumed; stages are free

    // ---------------------------------------------------------------- combine the 32 groups
    float *red_acc = (float *)smem;              // [kGroup][kD]
    for (int i = threadIdx.x; i < kGroup * kD; i += blockDim.x) red_acc[i] = 0.f;
    if (warp < kDecComputeWarps && l8 == 0) {
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
            red_m[grp][h] = m[h];
            red_l[grp][h] = lsum[h];
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp < kDecComputeWarps) {
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
            float M = -INFINITY;
            for (int j = 0; j < 16; ++j) M = fmaxf(M, red_m[half * 16 + j][h]);
            const float f = (m[h] == -INFINITY) ? 0.f : ex2_approx(m[h] - M);
            float *dst = red_acc + (half * kHalf + h) * kD;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int d = (i < 4 ? 8 * l8 : 64 + 8 * l8) + 2 * (i & 3);
                atomicAdd(dst + d, acc[h][i].x * f);
                atomicAdd(dst + d + 1, acc[h][i].y * f);
            }
        }
    }
    __syncthreads();
    float *part = a.part + (((size_t)b * a.hkv + g) * a.max_splits + split) * kPartFloats;
    if (threadIdx.x < kGroup) {
        const int hh = threadIdx.x, hf = hh / kHalf, h = hh % kHalf;
        float M = -INFINITY;
        for (int j = 0; j < 16; ++j) M = fmaxf(M, red_m[hf * 16 + j][h]);
        float L = 0.f;
        if (M != -INFINITY)
            for (int j = 0; j < 16; ++j) {
                const float mj = red_m[hf * 16 + j][h];
                if (mj != -INFINITY) L += red_l[hf * 16 + j][h] * ex2_approx(mj - M);
            }
        part[hh] = M;
        part[kGroup + hh] = L;
    }
    for (int i = threadIdx.x; i < kGroup * kD; i += blockDim.x) part[2 * kGroup + i] = red_acc[i];
}

// Folds the splits of every (sequence, query head) and the sink logit:
// O = sum_s 2^(m_s - M) acc_s / (sum_s 2^(m_s - M) l_s + 2^(sigma*log2e - M)).
__global__ void __launch_bounds__(kD) decode_merge(const DecodeArgs a) {
    const int bh = blockIdx.x;
    const int b = bh / (a.hkv * kGroup);
    const int h = bh % (a.hkv * kGroup);
    const int g = h / kGroup, hh = h % kGroup;
    const int splits = a.heads.is_full[g] ? a.splits_full : a.splits_ring;
    const float *part = a.part + ((size_t)b * a.hkv + g) * a.max_splits * kPartFloats;
    const bool has_sink = a.sink_logit != nullptr;
    const float sig = has_sink ? a.sink_logit[h] * kLog2eF : -INFINITY;
    float M = sig;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part[s * kPartFloats + hh]);
    float den = 0.f, num = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ms = part[s * kPartFloats + hh];
            if (ms == -INFINITY) continue;
            const float f = ex2_approx(ms - M);
            den += f * part[s * kPartFloats + kGroup + hh];
            num += f * part[s * kPartFloats + 2 * kGroup + hh * kD + threadIdx.x];
        }
        if (has_sink) den += ex2_approx(sig - M);
    }
    const float o = den > 0.f ? num / den : 0.f;
    a.out[(size_t)bh * kD + threadIdx.x] = __float2bfloat16_rn(o);
    if (a.lse != nullptr && threadIdx.x == 0)
        a.lse[bh] = den > 0.f ? (M + log2f(den)) * kLn2F : -INFINITY;
}

}  // namespace duo
