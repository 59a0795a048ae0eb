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
// address is looked up with cudaGetSymbolAddress, with the caller's device and
// context current, on every call.  The lookup is a host-side table query that
// allocates nothing; doing it per call keeps the address right after a
// cudaDeviceReset (which unloads and reloads the library's device image) and when
// a caller switches between contexts of the same device.  The first call on a
// device may load the library's device image there (lazy module loading), so it
// should come before any stream capture.
#include <cuda_runtime.h>

#include "relbias_attn.h"

namespace relbias {
namespace {

constexpr size_t kNoAllocScratchBytes = RELBIAS_DECODE_NOALLOC_SCRATCH_BYTES;

// The shared scratch: partial (max, sum, output) records of the split-KV kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current context.
int noalloc_scratch(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
        cudaGetLastError();   // do not leave the failed lookup pending for the caller's next check
        return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(decode scratch)");
    }
    *out = p;
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
    // Argument and device checks first, with the same codes and messages as
    // relbias_attn_decode: a bad call never reaches the symbol lookup.
    bool nothing_to_do = false;
    DeviceInfo dev;
    int rc = decode_check_args(q, k_cache, v_cache, r, w, 0, o, lse, B, n_ctx, Hq, Hkv, d, R, scale, dtype,
                               false, nullptr, &nothing_to_do, &dev);
    if (rc != RELBIAS_OK || nothing_to_do) return rc;
    const int nsplit = decode_num_splits(B, Hkv, n_ctx, window > 0 ? window : 0, dev.sms);
    const size_t need = decode_workspace_bytes(B, Hq, nsplit, d);
    if (need > kNoAllocScratchBytes)
        return fail(RELBIAS_ERR_UNSUPPORTED,
                    "this decode needs %zu bytes of scratch, more than the %zu-byte static scratch of "
                    "relbias_attn_decode_noalloc; call relbias_attn_decode with a workspace instead",
                    need, kNoAllocScratchBytes);
    void* ws = nullptr;
    if ((rc = noalloc_scratch(&ws)) != RELBIAS_OK) return rc;
    // Every split partial is written before the combine reads it: nothing needs clearing.
    return relbias_attn_decode(q, k_cache, v_cache, r, w, o, lse, B, n_ctx, Hq, Hkv, d, window, R, scale, temp_n0,
                               dtype, ws, kNoAllocScratchBytes, stream);
}
