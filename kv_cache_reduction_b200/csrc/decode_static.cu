// decode_static.cu -- one-token decode that never allocates device memory.
//
// duo_attn_decode needs a caller-provided workspace for its split partials.
// Some callers cannot allocate one: a plugin or custom op run by an
// inference engine that owns all device memory and forbids allocation
// inside its execute hook; a serving process that reserved a fixed memory
// budget at start-up and cannot grow it per request; a latency-critical
// loop that cannot afford cudaMalloc, which may synchronise the whole
// device.  duo_attn_decode_static serves them: its scratch lives in the
// fixed-size array below, which every GPU that loads the library holds
// until the process exits.  Nothing here calls cudaMalloc, cudaFree or any
// allocating library routine.
//
// Every call on a device uses the same array and leaves its contents
// behind.  Nothing in it has to start at zero (each split writes its whole
// partial before the merge reads it), but two calls whose kernels can run at
// the same time on one GPU (different streams or threads) overwrite each
// other's partials: issue them on one stream, or use duo_attn_decode with
// separate workspaces.
#include <cuda_runtime.h>

#include <atomic>

#include "duo_attn.h"

// 16 MiB of split partials: enough for B=32 at context 32768 or B=16 at
// context 131072 with 2 of 8 full heads (any layer whose workspace, as
// duo_decode_workspace_bytes reports it, fits).
constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
// Per-device address of the array.  Host threads may make their first call
// at the same time: both look the address up and store the same value, so
// relaxed atomics are enough.  A cached address does not survive
// cudaDeviceReset (the device's module, and the array with it, is reloaded).
std::atomic<void *> g_scratch_addr[kMaxDevices] = {};

// In host code the array's name is only a stand-in, not a device address.
// The device address is looked up once per device, with that device
// current, on the first call made there (so make that first call before
// any stream capture starts).
int scratch_for_current_device(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DUO_ERR_CUDA;
    void *p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) return DUO_ERR_CUDA;
        g_scratch_addr[dev].store(p, std::memory_order_relaxed);
    }
    *addr = p;
    return DUO_OK;
}

}  // namespace

extern "C" {

// Same contract as duo_attn_decode, with the split partials kept in
// g_decode_scratch instead of a caller workspace.  A layer whose workspace
// (duo_decode_workspace_bytes) exceeds the array is rejected by the regular
// workspace check: DUO_ERR_WORKSPACE, nothing launched, and duo_last_error()
// gives the bytes needed and available.
DUO_API int duo_attn_decode_static(const duo_params *params, const duo_cache *cache, const void *q,
                                   int32_t max_seq_len, void *out, float *lse,
                                   const duo_gate *gate, void *stream) {
    void *scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != DUO_OK) return rc;
    return duo_attn_decode(params, cache, q, max_seq_len, out, lse, scratch, kStaticScratchBytes,
                           gate, stream);
}

}  // extern "C"
