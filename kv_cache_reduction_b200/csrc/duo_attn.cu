// duo_attn.cu -- the C ABI of libduoattn.so: argument checks, work
// planning and kernel launches.  Every check runs on the host before the
// first launch, so a call that returns an error has launched nothing.
#include <atomic>
#include <utility>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "duo_attn.h"
#include "duo_attn_testing.h"
#include "decode.cuh"
#include "decode_block.cuh"
#include "kv_append.cuh"
#include "plan.h"
#include "prefill.cuh"
#include "ptx.cuh"
#include "qk_prep.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// The output gate, if any: mode in range, values present and 16-byte aligned.
int check_gate(const duo_gate *g, int *mode, const void **values) {
    *mode = DUO_GATE_NONE;
    *values = nullptr;
    if (g == nullptr || g->mode == DUO_GATE_NONE) return DUO_OK;
    if (g->mode != DUO_GATE_PER_ELEMENT && g->mode != DUO_GATE_PER_HEAD)
        return fail(DUO_ERR_INVALID_ARG, "gate mode %d is not DUO_GATE_NONE / PER_ELEMENT / PER_HEAD",
                    (int)g->mode);
    if (g->values == nullptr || !aligned16(g->values))
        return fail(DUO_ERR_INVALID_ARG, "gate values must be a 16-byte aligned device pointer");
    *mode = g->mode;
    *values = g->values;
    return DUO_OK;
}

// The failure-injection setting of each kernel (duo_attn_testing.h): the
// tile from which CTA 0's producer stops, or -1.
std::atomic<int> g_withhold[4] = {{-1}, {-1}, {-1}, {-1}};

int withhold_tile(int kernel) { return g_withhold[kernel].load(std::memory_order_relaxed); }

constexpr int kMaxHkv = 64;
constexpr int kMaxWindow = 8192;
constexpr int kMaxRing = 8192;
constexpr int64_t kMaxPos = (int64_t)1 << 30;
constexpr size_t kPrefillWorkspaceBytes = 16;   // the prefill work-tile counter

struct Layout {
    bool sliding;
    int n_full, n_ring;
    int sink, ring, slots;     // ring cache geometry
    duo::HeadTable heads;
    int8_t full_head[64], ring_head_of[64];
};

int check_device(int *sm_count) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(DUO_ERR_CUDA, "cudaGetDevice failed");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(DUO_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                    major, minor);
    if (sm_count) cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev);
    return DUO_OK;
}

int check_params(const duo_params *p, Layout *lay) {
    if (!p) return fail(DUO_ERR_INVALID_ARG, "params is NULL");
    if (p->batch < 1) return fail(DUO_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", p->batch);
    if (p->head_dim != duo::kD)
        return fail(DUO_ERR_UNSUPPORTED, "head_dim must be 128 (got %d)", p->head_dim);
    if (p->num_kv_heads < 1 || p->num_kv_heads > kMaxHkv)
        return fail(DUO_ERR_UNSUPPORTED, "num_kv_heads must be in [1, %d]", kMaxHkv);
    if (p->num_q_heads != duo::kGroup * p->num_kv_heads)
        return fail(DUO_ERR_UNSUPPORTED, "num_q_heads must be 6 * num_kv_heads (got %d, %d)",
                    p->num_q_heads, p->num_kv_heads);
    if (!(p->softmax_scale > 0.f) || !std::isfinite(p->softmax_scale))
        return fail(DUO_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (p->window < 0 || p->window > kMaxWindow)
        return fail(DUO_ERR_INVALID_ARG, "window must be in [0, %d]", kMaxWindow);
    if (p->sink_logit && !aligned16(p->sink_logit))
        return fail(DUO_ERR_INVALID_ARG, "sink_logit must be 16-byte aligned");
    Layout L{};
    L.sliding = p->window > 0;
    if (L.sliding) {
        L.sink = 0;
        L.ring = p->window;
    } else {
        if (!p->full_mask) return fail(DUO_ERR_INVALID_ARG, "full_mask is NULL on a DuoAttention layer");
        if (p->sink < 0 || p->recent < 1 || (int64_t)p->sink + p->recent > kMaxRing)
            return fail(DUO_ERR_INVALID_ARG, "need sink >= 0, recent >= 1, sink + recent <= %d",
                        kMaxRing);
        L.sink = p->sink;
        L.ring = p->recent;
    }
    L.slots = L.sink + L.ring;
    for (int g = 0; g < p->num_kv_heads; ++g) {
        const bool full = !L.sliding && p->full_mask[g] != 0;
        if (!L.sliding && p->full_mask[g] > 1)
            return fail(DUO_ERR_INVALID_ARG, "full_mask[%d] must be 0 or 1", g);
        L.heads.is_full[g] = full ? 1 : 0;
        if (full) {
            L.heads.rank[g] = (int8_t)L.n_full;
            L.full_head[L.n_full++] = (int8_t)g;
        } else {
            L.heads.rank[g] = (int8_t)L.n_ring;
            L.ring_head_of[L.n_ring++] = (int8_t)g;
        }
    }
    *lay = L;
    return DUO_OK;
}

int check_cache(const duo_cache *c, const Layout &L) {
    if (!c) return fail(DUO_ERR_INVALID_ARG, "cache is NULL");
    if (!c->seq_len || !c->ring_head) return fail(DUO_ERR_INVALID_ARG, "seq_len / ring_head is NULL");
    if (L.n_full > 0) {
        if (!c->full_k || !c->full_v) return fail(DUO_ERR_INVALID_ARG, "full_k / full_v is NULL");
        if (!aligned16(c->full_k) || !aligned16(c->full_v))
            return fail(DUO_ERR_INVALID_ARG, "full_k / full_v must be 16-byte aligned");
        if (c->capacity < 1 || c->capacity > kMaxPos)
            return fail(DUO_ERR_INVALID_ARG, "capacity must be in [1, 2^30]");
    }
    if (L.n_ring > 0) {
        if (!c->strm_k || !c->strm_v) return fail(DUO_ERR_INVALID_ARG, "strm_k / strm_v is NULL");
        if (!aligned16(c->strm_k) || !aligned16(c->strm_v))
            return fail(DUO_ERR_INVALID_ARG, "strm_k / strm_v must be 16-byte aligned");
    }
    if (((uintptr_t)c->seq_len & 3u) || ((uintptr_t)c->ring_head & 3u))
        return fail(DUO_ERR_INVALID_ARG, "seq_len / ring_head must be 4-byte aligned");
    return DUO_OK;
}

int launch_status(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DUO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return DUO_OK;
}

// Launches kernel<<<grid, block, smem, st>>>(args...) as a programmatic
// dependent of the kernel before it on the stream: it is scheduled while that
// one drains, and waits for it on the device (pdl_wait) before touching
// global memory, so that short kernels in a row overlap their launch and set-up
// with the previous kernel's tail.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per device.  The flags
// are atomic because host threads may launch concurrently; two threads that
// both see a flag clear both set the attribute, which is harmless.
template <typename Kernel>
int set_smem_once(Kernel kernel, size_t bytes, const char *name, std::atomic<bool> (&done)[64]) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return DUO_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return fail(DUO_ERR_CUDA, "cudaFuncSetAttribute(%s) failed", name);
    if (dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_release);
    return DUO_OK;
}

// ------------------------------------------------------------------ decode plan
struct DecodePlan {
    int chunk_full = duo::kTok, splits_full = 0;
    int chunk_ring = duo::kTok, splits_ring = 0;
    int max_splits = 1;
    int64_t items = 0;
    int grid = 0;
};

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Items are processed by one persistent CTA per SM, round robin.  Full-head
// caches are cut into equal chunks of whole 128-token tiles; the chunk count
// is the one that minimises the estimated makespan (tiles of the busiest
// CTA plus a per-item cost).  Ring heads take one item each unless
// there are too few of them to occupy the SMs.
DecodePlan plan_decode(const duo_params *p, const Layout &L, int64_t max_n, int sms) {
    DecodePlan d;
    const int64_t ring_units = (int64_t)p->batch * L.n_ring;
    const int64_t full_units = (int64_t)p->batch * L.n_full;
    const int64_t ring_tiles = cdiv(L.slots, duo::kTok);
    // pipeline fill and epilogue, in tiles: the value that fits the measured
    // decode times over split counts (B=32 at 32768 tokens: 9, 16, 20, 32 and
    // 12 splits rank as the model ranks them)
    const double item_cost = 1.5;
    if (ring_units > 0) {
        int64_t want = 1;
        if (full_units == 0 || max_n <= 4 * L.slots)
            want = std::min<int64_t>(ring_tiles, std::max<int64_t>(1, cdiv(sms, ring_units)));
        d.chunk_ring = (int)(cdiv(ring_tiles, want) * duo::kTok);
        d.splits_ring = (int)cdiv(L.slots, d.chunk_ring);
    }
    const int64_t ring_items = ring_units * d.splits_ring;
    const double ring_cost = ring_items > 0 ? (double)cdiv(d.chunk_ring, duo::kTok) + item_cost : 0.0;
    if (full_units > 0) {
        const int64_t n = std::max<int64_t>(max_n, 1);
        const int64_t tiles = cdiv(n, duo::kTok);
        double best = 1e300;
        for (int64_t s = 1; s <= std::min<int64_t>(tiles, 1024); ++s) {
            const int64_t chunk_tiles = cdiv(tiles, s);
            const int64_t splits = cdiv(tiles, chunk_tiles);
            const int64_t items = full_units * splits;
            const double cost = (double)cdiv(items, sms) * ((double)chunk_tiles + item_cost) +
                                (double)cdiv(ring_items, sms) * ring_cost;
            if (cost < best - 1e-9) {
                best = cost;
                d.chunk_full = (int)(chunk_tiles * duo::kTok);
                d.splits_full = (int)splits;
            }
        }
    }
    d.max_splits = std::max(1, std::max(d.splits_full, d.splits_ring));
    d.items = full_units * d.splits_full + ring_items;
    d.grid = (int)std::min<int64_t>(d.items, sms);
    return d;
}

// The block decode's plan.  Each item (split of a full head, ring head; the
// last split of each also takes the block's own tile) carries a fixed cost
// that grows with the query rows it holds (staging their Q, filling the
// pipeline, writing their partials), so the full heads' split count is chosen
// on the makespan of the persistent CTAs' round-robin share of all the items,
// in tiles plus that cost.
#ifndef DUO_BLK_ITEM_COST
#define DUO_BLK_ITEM_COST 3.0
#endif
DecodePlan plan_block(const duo_params *p, const Layout &L, int64_t max_n, int sms, int rows) {
    DecodePlan d = plan_decode(p, L, max_n, sms);
    (void)rows;
    // per-item cost in tiles: staging the item's Q into tensor memory and
    // writing its partials; the pipeline runs on across items
    const double item = DUO_BLK_ITEM_COST;
    const int64_t full_units = (int64_t)p->batch * L.n_full;
    const int64_t ring_items = (int64_t)p->batch * L.n_ring * d.splits_ring;
    if (full_units > 0) {
        // (the block's own tile rides on each full head's last split: no items of its own)
        const int64_t tiles = cdiv(std::max<int64_t>(max_n, 1), duo::kTok);
        const double c_ring = (double)cdiv(d.chunk_ring, duo::kTok) + item;
        double best = 1e300;
        for (int64_t s = 1; s <= std::min<int64_t>(tiles, 64); ++s) {
            const int64_t chunk = cdiv(tiles, s), splits = cdiv(tiles, chunk);
            const int64_t nf = full_units * splits, total = nf + ring_items;
            const int64_t g = std::min<int64_t>(total, sms);
            // the full heads' splits come first in the item list, the ring heads after
            const double span = duo::round_robin_makespan(nf, (double)chunk + item, ring_items, c_ring, g);
            if (span < best - 1e-9) {
                best = span;
                d.chunk_full = (int)(chunk * duo::kTok);
                d.splits_full = (int)splits;
            }
        }
        d.max_splits = std::max(1, std::max(d.splits_full, d.splits_ring));
        d.items = full_units * d.splits_full + ring_items;
        d.grid = (int)std::min<int64_t>(d.items, sms);
    }
    return d;
}

// A cache viewed as a 2-D tensor (128 columns, rows) loaded in 64-column x
// 128-row boxes with the 128-byte swizzle.
bool cache_tmap(CUtensorMap *m, void *base, int64_t rows) {
    duo::EncodeTiledFn fn = duo::encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {duo::kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {duo::kD * 2};
    const cuuint32_t box[2] = {64, duo::kTok};
    const cuuint32_t elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Checks an append's arguments and fills the scatter arguments (nothing is
// launched); DUO_OK with n_new == 0 means there is nothing to do.
int append_args(const duo_params *params, const duo_cache *cache, const void *k, const void *v,
                int32_t n_new, Layout *L, duo::AppendArgs *a) {
    int rc = check_params(params, L);
    if (rc) return rc;
    if ((rc = check_cache(cache, *L))) return rc;
    if (n_new < 0 || n_new > kMaxPos) return fail(DUO_ERR_INVALID_ARG, "n_new must be in [0, 2^30]");
    if (n_new == 0) return DUO_OK;
    if (!k || !v) return fail(DUO_ERR_INVALID_ARG, "k / v is NULL");
    if (!aligned16(k) || !aligned16(v)) return fail(DUO_ERR_INVALID_ARG, "k / v must be 16-byte aligned");
    if ((rc = check_device(nullptr))) return rc;
    a->k = (const uint4 *)k;
    a->v = (const uint4 *)v;
    a->full_k = (uint4 *)cache->full_k;
    a->full_v = (uint4 *)cache->full_v;
    a->strm_k = (uint4 *)cache->strm_k;
    a->strm_v = (uint4 *)cache->strm_v;
    a->seq_len = cache->seq_len;
    a->ring_head = cache->ring_head;
    a->capacity = L->n_full > 0 ? cache->capacity : 0;
    a->batch = params->batch;
    a->n_new = n_new;
    a->hkv = params->num_kv_heads;
    a->n_full = L->n_full;
    a->n_ring = L->n_ring;
    a->sink = L->sink;
    a->ring = L->ring;
    a->slots = L->slots;
    a->heads = L->heads;
    return DUO_OK;
}

size_t workspace_bytes(const duo_params *p, const DecodePlan &d) {
    return (size_t)p->batch * p->num_kv_heads * d.max_splits * duo::kPartFloats * sizeof(float);
}

constexpr int kMaxBlock = 8;     // block decode: query tokens per call

template <int kQ>
int launch_block(duo::BlockArgs &a, int grid, cudaStream_t st, int64_t merge_blocks) {
    static std::atomic<bool> smem_set[64] = {};
    int rc;
    if ((rc = set_smem_once(duo::decode_block_split<kQ>, duo::BlockCfg<kQ>::Smem, "decode_block_split",
                            smem_set)))
        return rc;
    duo::decode_block_split<kQ><<<(unsigned)grid, duo::BlockCfg<kQ>::Threads, duo::BlockCfg<kQ>::Smem, st>>>(a);
    if ((rc = launch_status("decode_block_split"))) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)merge_blocks);
    cfg.blockDim = dim3(duo::kMergeThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, duo::decode_block_merge<kQ>, a) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "decode_block_merge launch: %s", cudaGetErrorString(cudaGetLastError()));
    return launch_status("decode_block_merge");
}

// y = 2^x by the prefill's FMA-pipe exponential, two values per thread.
__global__ void ex2_poly_kernel(const float *x, float *y, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const duo::f2 r = duo::ex2_poly2(duo::f2_make(x[i], i + 1 < n ? x[i + 1] : 0.f));
    y[i] = r.x;
    if (i + 1 < n) y[i + 1] = r.y;
}

}  // namespace

extern "C" {

const char *duo_last_error(void) { return g_err; }

const char *duo_status_string(int code) {
    switch (code) {
    case DUO_OK: return "ok";
    case DUO_ERR_INVALID_ARG: return "invalid argument";
    case DUO_ERR_UNSUPPORTED: return "unsupported geometry";
    case DUO_ERR_CUDA: return "CUDA error";
    case DUO_ERR_WORKSPACE: return "workspace missing or too small";
    case DUO_ERR_TIMEOUT: return "a bounded device wait expired";
    case DUO_ERR_CAPACITY: return "append past the full-cache capacity";
    case DUO_ERR_DEVICE: return "device is not sm_100";
    default: return "unknown status";
    }
}

int duo_kv_append(const duo_params *params, const duo_cache *cache, const void *k, const void *v,
                  int32_t n_new, void *stream) {
    Layout L;
    duo::AppendArgs a{};
    int rc = append_args(params, cache, k, v, n_new, &L, &a);
    if (rc || n_new == 0) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    if ((int64_t)n_new * params->num_kv_heads * duo::kVecPerRow <= duo::kAppendSmallMaxVecs) {
        // a short append: copy and commit in one launch, one CTA per sequence
        if (launch_pdl(duo::kv_append_small, dim3((unsigned)params->batch), dim3(duo::kAppendSmallThreads), 0, st,
                       a) != cudaSuccess)
            return launch_status("kv_append_small");
        return launch_status("kv_append_small");
    }
    const int64_t vecs = (int64_t)params->batch * n_new * params->num_kv_heads * duo::kVecPerRow;
    const int64_t blocks = (vecs + 255) / 256;
    if (blocks > INT32_MAX) return fail(DUO_ERR_INVALID_ARG, "append too large for one launch");
    if (launch_pdl(duo::kv_append_scatter, dim3((unsigned)blocks), dim3(256), 0, st, a) != cudaSuccess)
        return launch_status("kv_append_scatter");
    if (launch_pdl(duo::kv_append_commit, dim3((params->batch + 127) / 128), dim3(128), 0, st, cache->seq_len,
                   cache->ring_head, params->batch, n_new, L.sink, L.ring, L.n_full, a.capacity) != cudaSuccess)
        return launch_status("kv_append_commit");
    return launch_status("kv_append_commit");
}

// YaRN inverse frequencies ("NTK-by-parts"), in double: f_i = theta^(-2i/D);
// the dimensions between the correction bounds of beta_fast and beta_slow blend
// f_i (extrapolation) and f_i / factor (interpolation) along a linear ramp.
static void yarn_inv_freq(const duo_qk_prep *p, double *inv) {
    const double d = duo::kD, theta = p->rope_theta, s = p->rope_factor;
    const double orig = p->original_max_position;
    const double two_pi = 6.283185307179586476925286766559;
    auto bound = [&](double beta) { return d * std::log(orig / (beta * two_pi)) / (2.0 * std::log(theta)); };
    double low = std::floor(bound(p->beta_fast)), high = std::ceil(bound(p->beta_slow));
    low = std::max(low, 0.0);
    high = std::min(high, d - 1.0);
    if (high == low) high += 0.001;
    for (int i = 0; i < duo::kD / 2; ++i) {
        const double f = std::pow(theta, -2.0 * i / d);
        const double ramp = std::min(1.0, std::max(0.0, (i - low) / (high - low)));
        const double keep = 1.0 - ramp;             // share of the unscaled frequency
        inv[i] = f / s * (1.0 - keep) + f * keep;
    }
}

int duo_kv_append_prep(const duo_params *params, const duo_cache *cache, const duo_qk_prep *prep,
                       void *q, void *k, const void *v, int32_t n_new, void *stream) {
    if (!prep) return fail(DUO_ERR_INVALID_ARG, "prep is NULL");
    if (!(prep->rope_theta > 1.f) || !(prep->rope_factor >= 1.f) || prep->original_max_position < 1 ||
        !(prep->beta_slow > 0.f) || !(prep->beta_fast >= prep->beta_slow) || !(prep->rms_eps >= 0.f) ||
        !std::isfinite(prep->attention_factor) || !std::isfinite(prep->rope_theta) ||
        !std::isfinite(prep->rope_factor) || !std::isfinite(prep->beta_fast))
        return fail(DUO_ERR_INVALID_ARG, "rope / norm parameters out of range");
    if ((prep->q_norm_weight && !aligned16(prep->q_norm_weight)) ||
        (prep->k_norm_weight && !aligned16(prep->k_norm_weight)))
        return fail(DUO_ERR_INVALID_ARG, "norm weights must be 16-byte aligned");
    Layout L;
    duo::PrepArgs a{};
    int rc = append_args(params, cache, k, v, n_new, &L, &a.app);
    if (rc || n_new == 0) return rc;
    if (!q || !aligned16(q)) return fail(DUO_ERR_INVALID_ARG, "q must be a 16-byte aligned pointer");
    const int64_t blocks = (int64_t)params->batch * n_new;
    if (blocks > INT32_MAX) return fail(DUO_ERR_INVALID_ARG, "append too large for one launch");
    a.q = (uint4 *)q;
    a.kw = (uint4 *)k;
    a.q_w = (const __nv_bfloat16 *)prep->q_norm_weight;
    a.k_w = (const __nv_bfloat16 *)prep->k_norm_weight;
    yarn_inv_freq(prep, a.inv_freq);
    a.attention_factor = prep->attention_factor;
    a.rms_eps = prep->rms_eps;
    a.hq = params->num_q_heads;
    cudaStream_t st = (cudaStream_t)stream;
    if (launch_pdl(duo::qk_prep_append, dim3((unsigned)blocks), dim3(duo::kPrepThreads), 0, st, a) != cudaSuccess)
        return launch_status("qk_prep_append");
    if (n_new == 1) return launch_status("qk_prep_append");     // it committed the one token itself
    if (launch_pdl(duo::kv_append_commit, dim3((params->batch + 127) / 128), dim3(128), 0, st, cache->seq_len,
                   cache->ring_head, params->batch, n_new, L.sink, L.ring, L.n_full, a.app.capacity) != cudaSuccess)
        return launch_status("kv_append_commit");
    return launch_status("kv_append_commit");
}

size_t duo_decode_workspace_bytes(const duo_params *params, int32_t max_seq_len) {
    Layout L;
    if (check_params(params, &L) || max_seq_len < 0) return 0;
    int sms = 148;
    if (check_device(&sms)) sms = 148;
    return workspace_bytes(params, plan_decode(params, L, max_seq_len, sms));
}

int duo_attn_decode(const duo_params *params, const duo_cache *cache, const void *q,
                    int32_t max_seq_len, void *out, float *lse, void *workspace,
                    size_t workspace_size, const duo_gate *gate, void *stream) {
    Layout L;
    int rc = check_params(params, &L);
    if (rc) return rc;
    int gate_mode = 0;
    const void *gate_values = nullptr;
    if ((rc = check_gate(gate, &gate_mode, &gate_values))) return rc;
    if ((rc = check_cache(cache, L))) return rc;
    if (max_seq_len < 0 || max_seq_len > kMaxPos)
        return fail(DUO_ERR_INVALID_ARG, "max_seq_len must be in [0, 2^30]");
    if (L.n_full > 0 && max_seq_len > cache->capacity)
        return fail(DUO_ERR_INVALID_ARG, "max_seq_len %d exceeds capacity %lld", max_seq_len,
                    (long long)cache->capacity);
    if (!q || !out) return fail(DUO_ERR_INVALID_ARG, "q / out is NULL");
    if (!aligned16(q) || !aligned16(out) || (lse && !aligned16(lse)))
        return fail(DUO_ERR_INVALID_ARG, "q / out / lse must be 16-byte aligned");
    if ((int64_t)params->batch * L.n_full * (L.n_full ? cache->capacity : 0) > INT32_MAX ||
        (int64_t)params->batch * L.n_ring * L.slots > INT32_MAX)
        return fail(DUO_ERR_UNSUPPORTED, "cache rows exceed 2^31 (tensor-map coordinates are 32-bit)");
    int sms = 148;
    if ((rc = check_device(&sms))) return rc;
    const DecodePlan d = plan_decode(params, L, max_seq_len, sms);
    const size_t need = workspace_bytes(params, d);
    if (!workspace || workspace_size < need || ((uintptr_t)workspace & 255u))
        return fail(DUO_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need,
                    workspace_size);
    duo::DecodeArgs a;
    memset(&a, 0, sizeof a);
    if (L.n_full > 0 &&
        (!cache_tmap(&a.tm_fk, cache->full_k, (int64_t)params->batch * L.n_full * cache->capacity) ||
         !cache_tmap(&a.tm_fv, cache->full_v, (int64_t)params->batch * L.n_full * cache->capacity)))
        return fail(DUO_ERR_CUDA, "cuTensorMapEncodeTiled failed for the full cache");
    if (L.n_ring > 0 &&
        (!cache_tmap(&a.tm_rk, cache->strm_k, (int64_t)params->batch * L.n_ring * L.slots) ||
         !cache_tmap(&a.tm_rv, cache->strm_v, (int64_t)params->batch * L.n_ring * L.slots)))
        return fail(DUO_ERR_CUDA, "cuTensorMapEncodeTiled failed for the ring cache");
    a.seq_len = cache->seq_len;
    a.ring_head = cache->ring_head;
    a.q = (const __nv_bfloat16 *)q;
    a.sink_logit = params->sink_logit;
    a.part = (float *)workspace;
    a.out = (__nv_bfloat16 *)out;
    a.lse = lse;
    a.capacity = L.n_full > 0 ? cache->capacity : 0;
    a.batch = params->batch;
    a.hkv = params->num_kv_heads;
    a.n_full = L.n_full;
    a.n_ring = L.n_ring;
    a.sink = L.sink;
    a.ring = L.ring;
    a.slots = L.slots;
    a.chunk_full = d.chunk_full;
    a.splits_full = d.splits_full;
    a.chunk_ring = d.chunk_ring;
    a.splits_ring = d.splits_ring;
    a.max_splits = d.max_splits;
    a.n_items = (int32_t)d.items;
    a.scale_log2 = params->softmax_scale * duo::kLog2eF;
    a.gate = (const __nv_bfloat16 *)gate_values;
    a.gate_mode = gate_mode;
    a.withhold_tile = withhold_tile(DUO_TESTING_DECODE);
    memcpy(a.full_head, L.full_head, sizeof a.full_head);
    memcpy(a.ring_head_of, L.ring_head_of, sizeof a.ring_head_of);
    a.heads = L.heads;
    cudaStream_t st = (cudaStream_t)stream;
    static std::atomic<bool> smem_set[64] = {};
    if ((rc = set_smem_once(duo::decode_split, duo::kDecSmem, "decode_split", smem_set))) return rc;
    if (d.items > 0) {
        if (launch_pdl(duo::decode_split, dim3((unsigned)d.grid), dim3(duo::kDecThreads), duo::kDecSmem, st, a) !=
            cudaSuccess)
            return launch_status("decode_split");
        if ((rc = launch_status("decode_split"))) return rc;
    }
    // the merge is a programmatic dependent launch: it is scheduled while
    // decode_split drains and waits on the device for its results
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)params->batch * params->num_kv_heads));   // one per (b, KV head)
    cfg.blockDim = dim3(duo::kD * duo::kGroup);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, duo::decode_merge, a) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "decode_merge launch: %s", cudaGetErrorString(cudaGetLastError()));
    return launch_status("decode_merge");
}

size_t duo_prefill_workspace_bytes(void) { return kPrefillWorkspaceBytes; }

int duo_attn_prefill(const duo_params *params, const void *q, const void *k, const void *v,
                     int32_t seq_len, void *out, float *lse, void *workspace, size_t workspace_bytes,
                     const duo_gate *gate, void *stream) {
    Layout L;
    int rc = check_params(params, &L);
    if (rc) return rc;
    int gate_mode = 0;
    const void *gate_values = nullptr;
    if ((rc = check_gate(gate, &gate_mode, &gate_values))) return rc;
    if (workspace && (workspace_bytes < kPrefillWorkspaceBytes || !aligned16(workspace)))
        return fail(DUO_ERR_WORKSPACE, "prefill workspace: need %zu bytes, 16-byte aligned (got %zu)",
                    kPrefillWorkspaceBytes, workspace_bytes);
    if (seq_len < 0 || seq_len > kMaxPos) return fail(DUO_ERR_INVALID_ARG, "seq_len must be in [0, 2^30]");
    if (seq_len == 0) return DUO_OK;
    if (!q || !k || !v || !out) return fail(DUO_ERR_INVALID_ARG, "q / k / v / out is NULL");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned16(lse)))
        return fail(DUO_ERR_INVALID_ARG, "q / k / v / out / lse must be 16-byte aligned");
    if ((rc = check_device(nullptr))) return rc;
    return duo::launch_prefill(params, L.sliding, L.heads.is_full, L.sink, L.ring, q, k, v, seq_len,
                               out, lse, (int32_t *)workspace, gate_mode, gate_values,
                               withhold_tile(DUO_TESTING_PREFILL), (cudaStream_t)stream, g_err, sizeof g_err);
}

int duo_cache_bytes(const duo_params *params, int64_t capacity, int64_t seq_len,
                    duo_cache_stats *out) {
    Layout L;
    const int rc = check_params(params, &L);
    if (rc) return rc;
    if (capacity < 0 || seq_len < 0 || !out)
        return fail(DUO_ERR_INVALID_ARG, "need capacity >= 0, seq_len >= 0 and a non-NULL out");
    const uint64_t row = (uint64_t)params->head_dim * 2u * 2u;   // K and V, bf16
    const uint64_t B = (uint64_t)params->batch;
    const uint64_t full_rows = (uint64_t)L.n_full * (uint64_t)capacity;
    const uint64_t ring_rows = (uint64_t)L.n_ring * (uint64_t)L.slots;
    out->duo_bytes = B * (full_rows + ring_rows) * row;
    out->full_cache_bytes = B * (uint64_t)params->num_kv_heads * (uint64_t)capacity * row;
    const uint64_t act_full = (uint64_t)L.n_full * (uint64_t)std::min(seq_len, capacity);
    const uint64_t act_ring = (uint64_t)L.n_ring * (uint64_t)std::min<int64_t>(seq_len, L.slots);
    out->active_bytes = B * (act_full + act_ring) * row;
    out->utilization = out->duo_bytes ? (double)out->active_bytes / (double)out->duo_bytes : 0.0;
    return DUO_OK;
}

// ------------------------------------------------------------------ block decode
// A block longer than kMaxBlock tokens.  The full heads' cached keys are cut
// into kv_splits runs (at most kMaxLongSplits: block_combine reads one slice per
// run) so that the pass over the cache has enough work tiles for the SMs: the
// count minimises the estimated makespan of the persistent CTAs, all work spread
// evenly plus the last work tile (a work tile costs its key tiles plus two for
// its fill and epilogue; a ring head's about five).
struct LongBlockPlan {
    int kv_splits, split_tiles;
    size_t o_bytes, l_bytes, total;     // one bf16 [B][q_len][Hq][D] slice, one fp32 [B][Hq][q_len] slice
};

LongBlockPlan long_block_plan(const duo_params *p, const Layout &L, int64_t q_len, int64_t max_seq_len, int sms) {
    LongBlockPlan w;
    const int64_t qtiles = (q_len + duo::kPfM - 1) / duo::kPfM;
    const int64_t tiles = std::max<int64_t>(1, (max_seq_len + duo::kPfN - 1) / duo::kPfN);
    const int64_t units = (int64_t)p->batch * L.n_full * (duo::kGroup / 2) * qtiles;    // full head pairs x query tiles
    const int64_t ring_units = (int64_t)p->batch * L.n_ring * (duo::kGroup / 2) * qtiles;
    w.kv_splits = 1;
    w.split_tiles = (int)tiles;
    if (units > 0) {
        double best = 1e300;
        for (int64_t s = 1; s <= std::min<int64_t>(tiles, duo::kMaxLongSplits); ++s) {
            const int64_t chunk = (tiles + s - 1) / s;
            const double span = ((double)units * s * (chunk + 2) + 5.0 * ring_units) / sms + (double)(chunk + 2);
            if (span < best - 1e-9) {
                best = span;
                w.kv_splits = (int)s;
                w.split_tiles = (int)chunk;
            }
        }
    }
    w.o_bytes = ((size_t)p->batch * q_len * p->num_q_heads * duo::kD * 2 + 255) / 256 * 256;
    w.l_bytes = ((size_t)p->batch * p->num_q_heads * q_len * sizeof(float) + 255) / 256 * 256;
    // the cache pass's slices, the block pass's output and LSE, two work-tile counters
    w.total = (size_t)(w.kv_splits + 1) * (w.o_bytes + w.l_bytes) + 2 * 256;
    return w;
}

size_t duo_decode_block_workspace_bytes(const duo_params *params, int32_t q_len, int32_t max_seq_len) {
    Layout L;
    if (check_params(params, &L) || q_len < 1 || q_len > kMaxPos || max_seq_len < 0 || max_seq_len > kMaxPos)
        return 0;
    int sms = 148;
    if (check_device(&sms)) sms = 148;
    if (q_len > kMaxBlock) return long_block_plan(params, L, q_len, max_seq_len, sms).total;
    const DecodePlan d = plan_block(params, L, max_seq_len, sms, duo::kGroup * q_len);
    const size_t slots = (size_t)std::max(d.splits_full, d.splits_ring);
    const size_t partials = (size_t)params->batch * params->num_kv_heads * slots *
                            (size_t)(duo::kGroup * q_len) * (duo::kD + 2) * sizeof(float);
    return (partials + 255) / 256 * 256 + 256;       // + the work-item counter
}

// The block q [B][q_len][Hq][D] (q_len > kMaxBlock) against the cache before it is
// appended, plus its own keys: prefill_fwd in cache mode over the cached keys,
// prefill_fwd in prompt mode over the block's keys (its sink shifted by each
// sequence's cached length; the sink logit joins here), then block_combine.
int long_block(const duo_params *params, const Layout &L, const duo_cache *cache, const void *q,
               const void *k_new, const void *v_new, int32_t q_len, int32_t max_seq_len, void *out, float *lse,
               void *workspace, int gate_mode, const void *gate_values, int sms, cudaStream_t st) {
    const LongBlockPlan pl = long_block_plan(params, L, q_len, max_seq_len, sms);
    if ((int64_t)params->batch * q_len * params->num_q_heads > INT32_MAX)
        return fail(DUO_ERR_UNSUPPORTED, "batch x q_len x query heads must be below 2^31 for a block of %d tokens",
                    q_len);
    char *w = (char *)workspace;
    void *oa = w;                                                  // [S][B][q_len][Hq][D]
    void *ob = w + (size_t)pl.kv_splits * pl.o_bytes;              // [B][q_len][Hq][D]
    float *la = (float *)(w + (size_t)(pl.kv_splits + 1) * pl.o_bytes);   // [S][B][Hq][q_len]
    float *lb = (float *)((char *)la + (size_t)pl.kv_splits * pl.l_bytes);
    int32_t *ca = (int32_t *)((char *)lb + pl.l_bytes), *cb = ca + 64;
    char err[256];
    // both passes' work counters at once: no memset between the passes, so that the
    // second can start on the SMs the first leaves
    if (cudaMemsetAsync(ca, 0, 2 * 256, st) != cudaSuccess) return fail(DUO_ERR_CUDA, "zeroing the work counters failed");
    int rc = duo::launch_prefill_cache(params, L.sliding, L.heads.is_full, L.heads.rank, L.n_full, L.n_ring,
                                       L.sink, L.ring, L.n_full > 0 ? cache->capacity : 0, cache->full_k,
                                       cache->full_v, cache->strm_k, cache->strm_v, cache->seq_len, cache->ring_head,
                                       q, q_len, pl.kv_splits, pl.split_tiles, oa, la, ca, -1, st, err, sizeof err);
    if (rc) return fail(rc, "%s", err);
    rc = duo::launch_prefill(params, L.sliding, L.heads.is_full, L.sink, L.ring, q, k_new, v_new, q_len, ob, lb,
                             cb, 0, nullptr, -1, st, err, sizeof err, cache->seq_len, false, true);
    if (rc) return fail(rc, "%s", err);
    duo::CombineArgs c;
    memset(&c, 0, sizeof c);
    c.oa = (const __nv_bfloat16 *)oa;
    c.ob = (const __nv_bfloat16 *)ob;
    c.lse_a = la;
    c.lse_b = lb;
    c.out = (__nv_bfloat16 *)out;
    c.lse = lse;
    c.gate = (const __nv_bfloat16 *)gate_values;
    c.gate_mode = gate_mode;
    c.C = q_len;
    c.hq = params->num_q_heads;
    c.batch = params->batch;
    c.kv_splits = pl.kv_splits;
    c.split_tiles = pl.split_tiles;
    c.capacity = L.n_full > 0 ? (int32_t)std::min<int64_t>(cache->capacity, INT32_MAX) : 0;
    c.seq_len = cache->seq_len;
    for (int g = 0; g < params->num_kv_heads; ++g) c.is_full[g] = L.heads.is_full[g];
    const int64_t rows = (int64_t)params->batch * q_len * params->num_q_heads;
    duo::block_combine<<<(unsigned)((rows + duo::kCombineRows - 1) / duo::kCombineRows), duo::kCombineThreads, 0,
                         st>>>(c);
    return launch_status("block_combine");
}

int duo_attn_decode_block(const duo_params *params, const duo_cache *cache, const void *q,
                          const void *k_new, const void *v_new, int32_t q_len, int32_t max_seq_len,
                          void *out, float *lse, void *workspace, size_t workspace_size,
                          const duo_gate *gate, void *stream) {
    Layout L;
    int rc = check_params(params, &L);
    if (rc) return rc;
    if ((rc = check_cache(cache, L))) return rc;
    if (q_len < 1 || q_len > kMaxPos)
        return fail(DUO_ERR_UNSUPPORTED, "q_len must be in [1, 2^30] (got %d)", q_len);
    int gate_mode = 0;
    const void *gate_values = nullptr;
    if ((rc = check_gate(gate, &gate_mode, &gate_values))) return rc;
    if (max_seq_len < 0 || max_seq_len > kMaxPos)
        return fail(DUO_ERR_INVALID_ARG, "max_seq_len must be in [0, 2^30]");
    if (L.n_full > 0 && max_seq_len > cache->capacity)
        return fail(DUO_ERR_INVALID_ARG, "max_seq_len %d exceeds capacity %lld", max_seq_len,
                    (long long)cache->capacity);
    if (!q || !out || !k_new || !v_new) return fail(DUO_ERR_INVALID_ARG, "q / k_new / v_new / out is NULL");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_new) || !aligned16(v_new) || (lse && !aligned16(lse)))
        return fail(DUO_ERR_INVALID_ARG, "q / k_new / v_new / out / lse must be 16-byte aligned");
    if ((int64_t)params->batch * L.n_full * (L.n_full ? cache->capacity : 0) > INT32_MAX ||
        (int64_t)params->batch * L.n_ring * L.slots > INT32_MAX)
        return fail(DUO_ERR_UNSUPPORTED, "cache rows exceed 2^31 (tensor-map coordinates are 32-bit)");
    int sms = 148;
    if ((rc = check_device(&sms))) return rc;
    const size_t need = duo_decode_block_workspace_bytes(params, q_len, max_seq_len);
    if (!workspace || workspace_size < need || ((uintptr_t)workspace & 255u))
        return fail(DUO_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need,
                    workspace_size);
    if (q_len > kMaxBlock) {
        if ((int64_t)params->batch * params->num_q_heads / 2 * ((q_len + duo::kPfM - 1) / duo::kPfM) > INT32_MAX - 4096)
            return fail(DUO_ERR_UNSUPPORTED, "too many query tiles for one block");
        return long_block(params, L, cache, q, k_new, v_new, q_len, max_seq_len, out, lse, workspace, gate_mode,
                          gate_values, sms, (cudaStream_t)stream);
    }
    const DecodePlan d = plan_block(params, L, max_seq_len, sms, duo::kGroup * q_len);
    duo::BlockArgs a;
    memset(&a, 0, sizeof a);
    duo::DecodeArgs &da = a.d;
    if (L.n_full > 0 &&
        (!cache_tmap(&da.tm_fk, cache->full_k, (int64_t)params->batch * L.n_full * cache->capacity) ||
         !cache_tmap(&da.tm_fv, cache->full_v, (int64_t)params->batch * L.n_full * cache->capacity)))
        return fail(DUO_ERR_CUDA, "cuTensorMapEncodeTiled failed for the full cache");
    if (L.n_ring > 0 &&
        (!cache_tmap(&da.tm_rk, cache->strm_k, (int64_t)params->batch * L.n_ring * L.slots) ||
         !cache_tmap(&da.tm_rv, cache->strm_v, (int64_t)params->batch * L.n_ring * L.slots)))
        return fail(DUO_ERR_CUDA, "cuTensorMapEncodeTiled failed for the ring cache");
    if (!duo::make_tmap(&a.tm_bk, k_new, params->batch, q_len, params->num_kv_heads, duo::kTok) ||
        !duo::make_tmap(&a.tm_bv, v_new, params->batch, q_len, params->num_kv_heads, duo::kTok))
        return fail(DUO_ERR_CUDA, "cuTensorMapEncodeTiled failed for the block keys");
    da.seq_len = cache->seq_len;
    da.ring_head = cache->ring_head;
    da.sink_logit = params->sink_logit;
    da.part = (float *)workspace;
    da.capacity = L.n_full > 0 ? cache->capacity : 0;
    da.batch = params->batch;
    da.hkv = params->num_kv_heads;
    da.n_full = L.n_full;
    da.n_ring = L.n_ring;
    da.sink = L.sink;
    da.ring = L.ring;
    da.slots = L.slots;
    da.chunk_full = d.chunk_full;
    da.splits_full = d.splits_full;
    da.chunk_ring = d.chunk_ring;
    da.splits_ring = d.splits_ring;
    da.max_splits = std::max(d.splits_full, d.splits_ring);
    da.n_items = (int32_t)d.items;
    da.scale_log2 = params->softmax_scale * duo::kLog2eF;
    da.gate = (const __nv_bfloat16 *)gate_values;
    da.gate_mode = gate_mode;
    da.withhold_tile = withhold_tile(DUO_TESTING_DECODE_BLOCK);
    memcpy(da.full_head, L.full_head, sizeof da.full_head);
    memcpy(da.ring_head_of, L.ring_head_of, sizeof da.ring_head_of);
    da.heads = L.heads;
    a.q = (const __nv_bfloat16 *)q;
    a.out = (__nv_bfloat16 *)out;
    a.lse = lse;
    a.q_len = q_len;
    a.n_cache_items = (int32_t)d.items;
    a.part_slots = da.max_splits;
    // the work-item counter sits behind the partials, zeroed on the stream
    a.work_counter = (int32_t *)((char *)workspace + (need - 256));
    if (cudaMemsetAsync(a.work_counter, 0, sizeof(int32_t), (cudaStream_t)stream) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "zeroing the block decode's work counter failed");
    const int64_t items = d.items;
    const int grid = (int)std::min<int64_t>(items, sms);
    const int64_t merge_blocks = (int64_t)params->batch * q_len * params->num_kv_heads;   // one per (b, t, KV head)
    cudaStream_t st = (cudaStream_t)stream;
    switch (q_len) {
        case 1: return launch_block<1>(a, grid, st, merge_blocks);
        case 2: return launch_block<2>(a, grid, st, merge_blocks);
        case 3: return launch_block<3>(a, grid, st, merge_blocks);
        case 4: return launch_block<4>(a, grid, st, merge_blocks);
        case 5: return launch_block<5>(a, grid, st, merge_blocks);
        case 6: return launch_block<6>(a, grid, st, merge_blocks);
        case 7: return launch_block<7>(a, grid, st, merge_blocks);
        default: return launch_block<8>(a, grid, st, merge_blocks);
    }
}

int duo_testing_withhold_tile(int32_t kernel, int32_t tile) {
    if (kernel < DUO_TESTING_DECODE || kernel > DUO_TESTING_DECODE_BLOCK || tile < -1)
        return fail(DUO_ERR_INVALID_ARG, "unknown kernel %d or tile %d", (int)kernel, (int)tile);
    g_withhold[kernel].store(tile, std::memory_order_relaxed);
    return DUO_OK;
}

int duo_testing_ex2(const float *x, float *y, int64_t n, void *stream) {
    if (n < 0 || (n > 0 && (!x || !y || !aligned16(x) || !aligned16(y))))
        return fail(DUO_ERR_INVALID_ARG, "x / y must be 16-byte aligned device pointers and n >= 0");
    if (n == 0) return DUO_OK;
    int rc;
    if ((rc = check_device(nullptr))) return rc;
    const int64_t blocks = ((n + 1) / 2 + 255) / 256;
    if (blocks > INT32_MAX) return fail(DUO_ERR_INVALID_ARG, "n too large for one launch");
    ex2_poly_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(x, y, n);
    return launch_status("ex2_poly_kernel");
}

int duo_get_device_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "stream synchronize failed: %s", cudaGetErrorString(cudaGetLastError()));
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, duo::g_status, sizeof v) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "reading the status word failed");
    const int zero = 0;
    if (cudaMemcpyToSymbol(duo::g_status, &zero, sizeof zero) != cudaSuccess)
        return fail(DUO_ERR_CUDA, "clearing the status word failed");
    return v;
}

}  // extern "C"
