// qk_prep.cuh -- RMSNorm + YaRN rotary embedding of the new queries and keys,
// fused with the append of the prepared keys (and the values) to the cache.
//
// Laguna attention article, section on YaRN dynamic RoPE (rope parameters of
// the full-attention layers); Laguna XS 2.1 sliding-window article, section on
// its attention optimisations (queries and keys are RMS-normalised before the
// rotary embedding).  One CTA per (sequence, token): 64 threads compute the
// token's cos / sin table once (the angle p * inv_freq in double precision and
// reduced modulo 2 pi in double, so that positions up to 2^30 keep their
// phase), then 8 threads per head row normalise it, rotate the pairs
// (i, i + 64) and write it back in place; key rows also go to the cache, and
// so do the values (loaded when the CTA starts), with the append's survivor
// rule for ring heads.  A one-token append is committed by its CTA.
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

constexpr int kPrepThreads = 128;   // 16 head rows at a time, 8 threads each
constexpr int kPrepBatch = 4;       // head rows an 8-thread group has in flight at once

// One CTA per (sequence, token).  Thread j of a row's group of 8 holds the
// channels [8j, 8j + 8) and their rotation partners [64 + 8j, 64 + 8j + 8), so
// that the rotation needs no exchange between threads and every load and store
// is 16 bytes wide; the sum of squares is reduced over the 8 threads.
__global__ void __launch_bounds__(kPrepThreads, 4) qk_prep_append(const __grid_constant__ PrepArgs a) {
    pdl_wait();        // launched as a programmatic dependent of the previous kernel
    const AppendArgs &ap = a.app;
    const int tok = blockIdx.x;
    const int b = tok / ap.n_new;
    const int64_t t = tok % ap.n_new;
    const int64_t tok_row = (int64_t)b * ap.n_new + t;
    const int rows = a.hq + ap.hkv;
    const int grp = (int)(threadIdx.x >> 3);        // head rows grp, grp + 16, ...
    const int j = threadIdx.x & 7;                  // channels [8j, 8j + 8) and [64 + 8j, 64 + 8j + 8)
    constexpr int step = kPrepThreads / 8;
    auto row_ptr = [&](int r) -> uint4 * {
        return r < a.hq ? a.q + (tok_row * a.hq + r) * kVecPerRow
                        : a.kw + (tok_row * ap.hkv + (r - a.hq)) * kVecPerRow;
    };
    // the value rows that survive the append go straight to the cache: thread c
    // of the first pass holds chunk c % 16 of head c / 16, loaded first so that
    // the load overlaps the table and the rotation (heads past the first pass
    // are copied at the end)
    const int vc = threadIdx.x;
    uint4 vpre = make_uint4(0, 0, 0, 0);
    uint4 *vdst = nullptr;
    if (vc < ap.hkv * kVecPerRow) {
        const int g = vc / kVecPerRow;
        bool full = false;
        const int64_t row = append_row(ap, b, g, t, &full);
        if (row >= 0) {
            vpre = ap.v[(tok_row * ap.hkv + g) * kVecPerRow + vc % kVecPerRow];
            vdst = (full ? ap.full_v : ap.strm_v) + row * kVecPerRow + vc % kVecPerRow;
        }
    }
    // the first batch of rows in flight before the cos / sin table is built
    uint4 xlo[kPrepBatch], xhi[kPrepBatch];
#pragma unroll
    for (int u = 0; u < kPrepBatch; ++u) {
        const int r = grp + u * step;
        xlo[u] = r < rows ? row_ptr(r)[j] : make_uint4(0, 0, 0, 0);
        xhi[u] = r < rows ? row_ptr(r)[8 + j] : make_uint4(0, 0, 0, 0);
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
    float wq[16], wk[16], c8[8], s8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        wq[e] = a.q_w ? __bfloat162float(a.q_w[8 * j + e]) : 1.f;
        wq[8 + e] = a.q_w ? __bfloat162float(a.q_w[64 + 8 * j + e]) : 1.f;
        wk[e] = a.k_w ? __bfloat162float(a.k_w[8 * j + e]) : 1.f;
        wk[8 + e] = a.k_w ? __bfloat162float(a.k_w[64 + 8 * j + e]) : 1.f;
        c8[e] = cs[8 * j + e];
        s8[e] = sn[8 * j + e];
    }
    for (int rb = 0; rb < rows; rb += kPrepBatch * step) {
        if (rb > 0) {
#pragma unroll
            for (int u = 0; u < kPrepBatch; ++u) {
                const int r = rb + grp + u * step;
                xlo[u] = r < rows ? row_ptr(r)[j] : make_uint4(0, 0, 0, 0);
                xhi[u] = r < rows ? row_ptr(r)[8 + j] : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kPrepBatch; ++u) {
            const int r = rb + grp + u * step;
            const bool active = r < rows;
            const bool is_q = r < a.hq;
            float lo[8], hi[8];
            unpack8(xlo[u], lo);
            unpack8(xhi[u], hi);
            // pairs of channels through the packed f32x2 pipe
            f2 ss2 = f2_mul(f2_make(lo[0], lo[1]), f2_make(lo[0], lo[1]));
#pragma unroll
            for (int e = 2; e < 8; e += 2) ss2 = f2_fma(f2_make(lo[e], lo[e + 1]), f2_make(lo[e], lo[e + 1]), ss2);
#pragma unroll
            for (int e = 0; e < 8; e += 2) ss2 = f2_fma(f2_make(hi[e], hi[e + 1]), f2_make(hi[e], hi[e + 1]), ss2);
            float ss = f2_sum(ss2);
            // the 8 threads of a row are 8 consecutive lanes: reduce within them
#pragma unroll
            for (int m = 1; m < 8; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const f2 inv2 = f2_splat(rsqrtf(ss * (1.f / 128.f) + a.rms_eps));
            uint32_t olo[4], ohi[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const f2 wlo = is_q ? f2_make(wq[e], wq[e + 1]) : f2_make(wk[e], wk[e + 1]);
                const f2 whi = is_q ? f2_make(wq[8 + e], wq[9 + e]) : f2_make(wk[8 + e], wk[9 + e]);
                const f2 ylo = f2_mul(f2_mul(f2_make(lo[e], lo[e + 1]), inv2), wlo);
                const f2 yhi = f2_mul(f2_mul(f2_make(hi[e], hi[e + 1]), inv2), whi);
                const f2 cc = f2_make(c8[e], c8[e + 1]), sc = f2_make(s8[e], s8[e + 1]);
                // (y_i, y_{i+64}) rotated by the angle of pair i
                const f2 rlo = f2_fma(yhi, f2_make(-sc.x, -sc.y), f2_mul(ylo, cc));
                const f2 rhi = f2_fma(ylo, sc, f2_mul(yhi, cc));
                olo[e / 2] = pack_bf16x2(rlo.x, rlo.y);
                ohi[e / 2] = pack_bf16x2(rhi.x, rhi.y);
            }
            if (!active) continue;
            const uint4 out_lo = make_uint4(olo[0], olo[1], olo[2], olo[3]);
            const uint4 out_hi = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
            uint4 *rp = row_ptr(r);
            rp[j] = out_lo;
            rp[8 + j] = out_hi;
            if (!is_q) {
                const int g = r - a.hq;
                bool full = false;
                const int64_t row = append_row(ap, b, g, t, &full);
                if (row >= 0) {
                    uint4 *kd = (full ? ap.full_k : ap.strm_k) + row * kVecPerRow;
                    kd[j] = out_lo;
                    kd[8 + j] = out_hi;
                }
            }
        }
    }
    if (vdst != nullptr) *vdst = vpre;
    for (int c = vc + kPrepThreads; c < ap.hkv * kVecPerRow; c += kPrepThreads) {
        const int g = c / kVecPerRow;
        bool full = false;
        const int64_t row = append_row(ap, b, g, t, &full);
        if (row >= 0)
            ((full ? ap.full_v : ap.strm_v) + row * kVecPerRow)[c % kVecPerRow] =
                ap.v[(tok_row * ap.hkv + g) * kVecPerRow + c % kVecPerRow];
    }
    // a one-token append (a decode step): this CTA is its sequence's only one, so
    // it moves seq_len and ring_head forward itself once all its reads are done
    if (ap.n_new == 1) {
        __syncthreads();
        if (threadIdx.x == 0) commit_sequence(ap.seq_len, ap.ring_head, b, 1, ap.sink, ap.ring, ap.n_full, ap.capacity);
    }
}

}  // namespace duo
