// fa_noalloc.cu -- fa_kvcache_fwd for callers that cannot allocate device
// memory: the scratch the call needs comes from a fixed array inside the
// library instead of a caller-supplied workspace.
//
// Who needs this: code that may not call cudaMalloc (or any allocator) at
// the point where it runs attention -- a plug-in whose host application
// owns every device allocation and exposes no allocator to it, or a
// latency-critical loop that must never enter the CUDA allocator (which can
// synchronise the device).  Such a caller still passes its own inputs and
// outputs; only the scratch moves into the library.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

// Scratch shared by every call on a device.  Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array on the current device, looked up once
// per device with that device current (in host code the array's name is only
// a host-side stand-in, not a device address).
void *scratch_address(int *status) {
    static void *addr[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *status = fa::set_last_error(FA_ERR_CUDA, "no usable CUDA device");
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            *status = fa::set_last_error(FA_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed");
            return nullptr;
        }
        addr[dev] = p;
    }
    *status = FA_OK;
    return addr[dev];
}

}  // namespace

extern "C" int fa_kvcache_fwd_noalloc(const fa_tensor *q, const fa_tensor *k_cache, const fa_tensor *v_cache,
                                      const fa_tensor *k_new, const fa_tensor *v_new, const fa_tensor *cos,
                                      const fa_tensor *sin, const int32_t *cache_seqlens, int32_t rotary_dim,
                                      int32_t interleaved, int32_t causal, float scale, const fa_tensor *out,
                                      float *lse, int32_t cache_seqlens_scalar, void *stream) {
    size_t need = 0;
    int rc = fa_kvcache_workspace_size(q, k_cache, v_cache, k_new, cos ? rotary_dim : 0, &need);
    if (rc != FA_OK) return rc;
    if (need > kScratchBytes) {
        char msg[160];
        snprintf(msg, sizeof(msg), "these shapes need %zu bytes of scratch; the built-in scratch holds %zu", need,
                 kScratchBytes);
        return fa::set_last_error(FA_ERR_WORKSPACE, msg);
    }
    int st = FA_OK;
    void *scratch = scratch_address(&st);
    if (!scratch) return st;
    // The scratch keeps whatever the previous call left in it; the kernels
    // write every scratch word before they read it, so nothing is cleared.
    return fa_kvcache_fwd(q, k_cache, v_cache, k_new, v_new, cos, sin, cache_seqlens, rotary_dim, interleaved,
                          causal, scale, out, lse, cache_seqlens_scalar, scratch, kScratchBytes, stream);
}
