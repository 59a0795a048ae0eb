// decode_noalloc.cu -- a decode entry point that allocates no device memory.
//
// relbias_attn_decode needs a scratch workspace for its split partials, and the
// caller allocates it.  Some callers cannot: a plugin hosted by an inference
// runtime that owns every device allocation and hands its plugins no allocator,
// a serving loop that must not call cudaFree (which can synchronise the whole
// device) between steps, or a process whose device-memory budget is fixed once at
// start-up.  relbias_attn_decode_noalloc serves them from a scratch array that is
// part of this library's device image: it is created when the library's module is
// loaded on a device and lives until the process exits, so every GPU that loads
// the library holds RELBIAS_DECODE_NOALLOC_SCRATCH_BYTES for it.
//
// In host code the array's name is only a host-side stand-in for the symbol, not
// a device address: handing it to a kernel would fault, or on systems where the
// GPU can reach host memory silently use the wrong memory.  The real device
// address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "relbias_attn.h"

namespace relbias {
namespace {

constexpr size_t kNoAllocScratchBytes = RELBIAS_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The shared scratch: partial (max, sum, output) records of the split-KV kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(RELBIAS_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return RELBIAS_OK;
}

}  // namespace
}  // namespace relbias

extern "C" int relbias_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const float* r,
                                           const float* w, void* o, float* lse, int B, int n_ctx, int Hq, int Hkv,
                                           int d, int window, int R, float scale, int temp_n0, int dtype,
                                           void* stream) {
    using namespace relbias;
    t_err.clear();
    // Argument errors first, exactly as the regular entry point reports them.
    int rc = check_common(B, n_ctx, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (B == 0)
        return relbias_attn_decode(q, k_cache, v_cache, r, w, o, lse, B, n_ctx, Hq, Hkv, d, window, R, scale,
                                   temp_n0, dtype, nullptr, 0, stream);
    void* ws = nullptr;
    if ((rc = noalloc_scratch(&ws)) != RELBIAS_OK) return rc;
    const size_t need = relbias_attn_decode_workspace_size(B, Hq, Hkv, n_ctx, d, window);
    if (need > kNoAllocScratchBytes)
        return fail(RELBIAS_ERR_UNSUPPORTED,
                    "this decode needs %zu bytes of scratch, more than the %zu-byte static scratch of "
                    "relbias_attn_decode_noalloc; call relbias_attn_decode with a workspace instead",
                    need, kNoAllocScratchBytes);
    // The split partials are written before they are read: nothing needs clearing.
    return relbias_attn_decode(q, k_cache, v_cache, r, w, o, lse, B, n_ctx, Hq, Hkv, d, window, R, scale, temp_n0,
                               dtype, ws, kNoAllocScratchBytes, stream);
}
