// qk_prep.cuh -- RMSNorm + YaRN rotary embedding of the new queries and keys,
// fused with the append of the prepared keys (and the values) to the cache.
//
// Laguna attention article, section on YaRN dynamic RoPE (rope parameters of
// the full-attention layers); Laguna XS 2.1 sliding-window article, section on
// its attention optimisations (queries and keys are RMS-normalised before the
// rotary embedding).  One CTA per (sequence, token): 64 threads compute the
// token's cos / sin table once (the angle p * inv_freq in double precision and
// reduced modulo 2 pi in double, so that positions up to 2^30 keep their
// phase), then 16 threads per head row
// normalise it, rotate the pairs (i, i + 64) and write it back in place; key
// rows also go to the cache with their values, with the append's survivor
// rule for ring heads.
#pragma once

#include "kv_append.cuh"

namespace duo {

struct PrepArgs {
    uint4 *q;                       // [B][n_new][Hq][D] bf16, rewritten in place
    AppendArgs app;                 // k (rewritten in place through kw), v, caches, geometry
    uint4 *kw;                      // == app.k, writable
    const __nv_bfloat16 *q_w, *k_w; // norm weights [D] or null
    double inv_freq[64];
    float attention_factor, rms_eps;
    int32_t hq;
};

__device__ __forceinline__ void unpack8(const uint4 u, float *x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

constexpr int kPrepThreads = 128;   // 8 head rows at a time, 16 threads each

constexpr int kPrepBatch = 8;       // head rows a 16-thread group has in flight at once

__global__ void __launch_bounds__(kPrepThreads) qk_prep_append(const __grid_constant__ PrepArgs a) {
    const AppendArgs &ap = a.app;
    const int tok = blockIdx.x;
    const int b = tok / ap.n_new;
    const int64_t t = tok % ap.n_new;
    const int64_t tok_row = (int64_t)b * ap.n_new + t;
    const int rows = a.hq + ap.hkv;
    const int grp = (int)(threadIdx.x >> 4);        // head rows grp, grp + 8, ...
    const int j = threadIdx.x & 15;                 // channels [8j, 8j + 8) of a row
    auto row_ptr = [&](int r) -> uint4 * {
        return r < a.hq ? a.q + (tok_row * a.hq + r) * kVecPerRow
                        : a.kw + (tok_row * ap.hkv + (r - a.hq)) * kVecPerRow;
    };
    const int step = kPrepThreads / 16;
    // first batch of rows in flight before the cos / sin table is built
    uint4 xin[kPrepBatch];
#pragma unroll
    for (int u = 0; u < kPrepBatch; ++u) {
        const int r = grp + u * step;
        xin[u] = r < rows ? row_ptr(r)[j] : make_uint4(0, 0, 0, 0);
    }
    const int64_t pos = (int64_t)ap.seq_len[b] + t;
    __shared__ float cs[64], sn[64];
    if (threadIdx.x < 64) {
        // angle p * f in double, reduced to [-pi, pi] by Cody and Waite's
        // two-constant method (2 pi = kC1 + kC2 with kC1 exact in 24 bits, so
        // n * kC1 is exact in double for |n| < 2^29), then sin and cos of the
        // small remainder in double
        constexpr double kC1 = 6.2831854820251465;             // float(2 pi)
        constexpr double kC2 = -1.748455600074497e-07;         // 2 pi - kC1, rounded to double
        constexpr double kInv2Pi = 0.15915494309189535;
        const double x = (double)pos * a.inv_freq[threadIdx.x];
        const double n = rint(x * kInv2Pi);
        const double r = fma(-n, kC2, fma(-n, kC1, x));
        double s, c;
        sincos(r, &s, &c);          // |r| <= pi: no large-argument reduction inside
        cs[threadIdx.x] = (float)c * a.attention_factor;
        sn[threadIdx.x] = (float)s * a.attention_factor;
    }
    __syncthreads();
    const int f0 = (j & 7) * 8;                     // frequency index of channel 8j (mod 64)
    const bool lo = j < 8;                          // first half of the (i, i + 64) pairs
    float wq[8], wk[8], c8[8], s8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        wq[e] = a.q_w ? __bfloat162float(a.q_w[8 * j + e]) : 1.f;
        wk[e] = a.k_w ? __bfloat162float(a.k_w[8 * j + e]) : 1.f;
        c8[e] = cs[f0 + e];
        s8[e] = lo ? -sn[f0 + e] : sn[f0 + e];      // out = y cos -/+ partner sin
    }
    for (int rb = 0; rb < rows; rb += kPrepBatch * step) {
        if (rb > 0) {
#pragma unroll
            for (int u = 0; u < kPrepBatch; ++u) {
                const int r = rb + grp + u * step;
                xin[u] = r < rows ? row_ptr(r)[j] : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kPrepBatch; ++u) {
            const int r = rb + grp + u * step;
            const bool active = r < rows;
            const bool is_q = r < a.hq;
            float x[8];
            unpack8(xin[u], x);
            // pairs of channels through the packed f32x2 pipe
            f2 ss2 = f2_mul(f2_make(x[0], x[1]), f2_make(x[0], x[1]));
#pragma unroll
            for (int e = 2; e < 8; e += 2) ss2 = f2_fma(f2_make(x[e], x[e + 1]), f2_make(x[e], x[e + 1]), ss2);
            float ss = f2_sum(ss2);
            // the 16 threads of a row are 16 consecutive lanes: reduce within them
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const f2 inv2 = f2_splat(rsqrtf(ss * (1.f / 128.f) + a.rms_eps));
            f2 y2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                y2[e] = f2_mul(f2_mul(f2_make(x[2 * e], x[2 * e + 1]), inv2),
                               is_q ? f2_make(wq[2 * e], wq[2 * e + 1]) : f2_make(wk[2 * e], wk[2 * e + 1]));
            f2 p2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                p2[e].x = __shfl_xor_sync(0xffffffffu, y2[e].x, 8);   // channel +-64
                p2[e].y = __shfl_xor_sync(0xffffffffu, y2[e].y, 8);
            }
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f2 r2 = f2_fma(p2[e], f2_make(s8[2 * e], s8[2 * e + 1]),
                                     f2_mul(y2[e], f2_make(c8[2 * e], c8[2 * e + 1])));
                o[e] = pack_bf16x2(r2.x, r2.y);
            }
            if (!active) continue;
            const uint4 out = make_uint4(o[0], o[1], o[2], o[3]);
            row_ptr(r)[j] = out;
            if (!is_q) {
                const int g = r - a.hq;
                bool full = false;
                const int64_t row = append_row(ap, b, g, t, &full);
                if (row >= 0) {
                    const uint4 vv = ap.v[(tok_row * ap.hkv + g) * kVecPerRow + j];
                    if (full) {
                        ap.full_k[row * kVecPerRow + j] = out;
                        ap.full_v[row * kVecPerRow + j] = vv;
                    } else {
                        ap.strm_k[row * kVecPerRow + j] = out;
                        ap.strm_v[row * kVecPerRow + j] = vv;
                    }
                }
            }
        }
    }
}

}  // namespace duo
