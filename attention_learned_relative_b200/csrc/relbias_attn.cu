// relbias_attn.cu -- the C ABI of librelbias_attn.so (declared in
// include/relbias_attn.h): argument checks, TMA descriptor set-up, launch
// configuration and error reporting.  The kernels are compiled into this one
// translation unit so they share the device-side status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>

#include "relbias_attn.h"

#include "decode_sm100.cu"
#include "prefill_fp32.cu"
#include "prefill_sm100.cu"
#include "backward_fp32.cu"
#include "backward_sm100.cu"

namespace relbias {
namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(RELBIAS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(std::string& why) {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static std::string err;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || ptr == nullptr)
            err = std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(e);
        else
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    why = err;
    return fn;
}

struct DeviceInfo {
    int major = 0, minor = 0, sms = 0;
};

int device_info(DeviceInfo& info) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if ((e = cudaDeviceGetAttribute(&info.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&info.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    return RELBIAS_OK;
}

// 4-D bf16 tensor map over a [B, T, H, d] tensor, box = 64 head-dim columns x
// `rows` tokens of one head, 128-byte swizzle, zero fill outside the tensor.  With
// T_alloc > T the tensor is the first T rows of a [B, T_alloc, H, d] allocation: rows
// past T read as zeros.
int make_map(CUtensorMap* m, const void* ptr, int B, int T, int H, int d, int rows, int T_alloc = 0) {
    std::string why;
    EncodeTiledFn fn = encode_fn(why);
    if (fn == nullptr) return fail(RELBIAS_ERR_CUDA, "%s", why.c_str());
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T),
                          static_cast<cuuint64_t>(B)};
    const int Ta = T_alloc > T ? T_alloc : T;
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                             static_cast<cuuint64_t>(Ta) * H * d * 2};
    cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(RELBIAS_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", int(r));
    return RELBIAS_OK;
}

int check_common(int B, int T, int Hq, int Hkv, int d, int R, float scale, const float* w) {
    if (B < 0 || T < 0) return fail(RELBIAS_ERR_ARG, "B (%d) and T (%d) must be >= 0", B, T);
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
        return fail(RELBIAS_ERR_ARG, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq, Hkv);
    if (d < 1) return fail(RELBIAS_ERR_ARG, "d (%d) must be positive", d);
    if (R < 0) return fail(RELBIAS_ERR_ARG, "R (%d) must be >= 0", R);
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return fail(RELBIAS_ERR_ARG, "scale (%g) must be positive and finite", static_cast<double>(scale));
    if (R > 0 && (w == nullptr || !aligned4(w))) return fail(RELBIAS_ERR_ARG, "w is null or misaligned");
    return RELBIAS_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// Bytes of the bf16 bank prefill's curve workspace: [B, T, Hq] padded rows.
size_t bank_prefill_curve_bytes(int B, int T, int Hq, int R) {
    const size_t b = static_cast<size_t>(B) * T * Hq * prefill_bank_curve_stride(R) * sizeof(float);
    return (b + 255) / 256 * 256;
}

}  // namespace
}  // namespace relbias

using namespace relbias;

namespace {

// Prefill of T query rows at positions q_off ... q_off+T-1 against kv_T >= q_off+T
// key/value rows (q_off = 0, kv_T = T: a whole sequence).
// C == 0: rank-1 bias (r [B, T, Hq], w [Hq, R]); C >= 1: shared bank (r [B, T, Hq, C]
// coefficients, w [proj_heads, C, R] functions), fp32 only.
int fwd_impl(const void* q, const void* k, const void* v, const float* r, const float* w, void* o, float* lse, int B,
             int T, int q_off, int kv_T, int Hq, int Hkv, int d, int window, int R, float scale, int temp_n0,
             int dtype, void* stream, int C = 0, int proj_heads = 0, void* workspace = nullptr,
             size_t ws_bytes = 0) {
    int rc = check_common(B, T, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (q_off < 0 || static_cast<long long>(q_off) + T > kv_T)
        return fail(RELBIAS_ERR_ARG, "need 0 <= q_off (%d) and q_off + T (%lld) <= kv_T (%d)", q_off,
                    static_cast<long long>(q_off) + T, kv_T);
    if (B == 0 || T == 0) return RELBIAS_OK;
    if (!q || !k || !v || !r || !o) return fail(RELBIAS_ERR_ARG, "q, k, v, r and o must not be null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(RELBIAS_ERR_ARG, "q, k, v and o must be 16-byte aligned");
    if (!aligned4(r) || (lse && !aligned4(lse))) return fail(RELBIAS_ERR_ARG, "r and lse must be 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (dtype == RELBIAS_FP32) {
        if (d != 32 && d != 64 && d != 128 && d != 256)
            return fail(RELBIAS_ERR_UNSUPPORTED, "fp32 prefill supports d in {32, 64, 128, 256}, got %d", d);
        cudaError_t e = launch_prefill_fp32(static_cast<const float*>(q), static_cast<const float*>(k),
                                            static_cast<const float*>(v), r, w, static_cast<float*>(o), lse, B, T,
                                            q_off, kv_T, Hq, Hkv, d, window, R, scale, temp_n0, C, proj_heads, st);
        return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "fp32 prefill launch");
    }

    if (d != 64 && d != 128) return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill supports d in {64, 128}, got %d", d);
    if (R > 2048 || prefill_bf16_table_copies(d, R) == 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill stages R <= 2048 table entries, got %d", R);
    size_t curve_bytes = 0;
    if (C > 0 && R > 0) {
        curve_bytes = bank_prefill_curve_bytes(B, T, Hq, R);
        if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 31u) != 0)
            return fail(RELBIAS_ERR_ARG, "the bf16 shared-bank prefill needs a 32-byte aligned workspace");
        if (ws_bytes < curve_bytes)
            return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes is smaller than the %zu bytes of bank curves",
                        ws_bytes, curve_bytes);
    }
    DeviceInfo dev;
    if ((rc = device_info(dev)) != RELBIAS_OK) return rc;
    if (dev.major != 10 || dev.minor != 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill needs compute capability 10.0 (sm_100a), found %d.%d",
                    dev.major, dev.minor);

    CUtensorMap tq, tk, tv;
    if ((rc = make_map(&tq, q, B, T, Hq, d, 128)) != RELBIAS_OK) return rc;
    // Keys and values past the chunk's last row (q_off + T - 1) are never visible;
    // the maps end there, so tiles reaching past it read zeros, not stale cache rows
    // (a masked key still multiplies its value row by a zero weight).
    if ((rc = make_map(&tk, k, B, q_off + T, Hkv, d, 128, kv_T)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tv, v, B, q_off + T, Hkv, d, 128, kv_T)) != RELBIAS_OK) return rc;

    PrefillParams p{};
    p.r = r;
    p.w = w;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.nslots = (p.G % 2 == 0) ? 2 : 1;
    p.HP = p.G / p.nslots;
    p.window = window > 0 ? window : 0;
    p.R = R;
    p.n_qt = (T + 127) / 128;
    p.q_off = q_off;
    p.kv_T = kv_T;
    const long long items = static_cast<long long>(p.n_qt) * B * Hkv * p.HP;
    if (items > INT32_MAX) return fail(RELBIAS_ERR_UNSUPPORTED, "too many work items (%lld)", items);
    p.total_items = static_cast<int>(items);
    p.contiguous = p.window > 0 ? 1 : 0;
    p.o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    p.temp_n0 = temp_n0 > 1 ? temp_n0 : 0;
    p.inv_log_n0 = temp_n0 > 1 ? static_cast<float>(1.0 / std::log(static_cast<double>(temp_n0))) : 0.0f;
    if (C > 0 && R > 0) {
        // Shared bank: each row's curve sum_c rs[c] * proj[c, dist] first, into the workspace.
        cudaError_t e = launch_bank_rows(r, w, static_cast<float*>(workspace), B, T, Hq, q_off, C, proj_heads, R, st);
        if (e != cudaSuccess) return cuda_fail(e, "bank curve launch");
        p.curves = static_cast<const float*>(workspace);
        p.curve_stride = prefill_bank_curve_stride(R);
    }
    const int grid = static_cast<int>(std::min<long long>(items, dev.sms));
    cudaError_t e = launch_prefill_bf16_sm100(tq, tk, tv, p, d, grid, st);
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "bf16 prefill launch");
}

}  // namespace

extern "C" int relbias_attn_fwd(const void* q, const void* k, const void* v, const float* r, const float* w,
                                void* o, float* lse, int B, int T, int Hq, int Hkv, int d, int window, int R,
                                float scale, int temp_n0, int dtype, void* stream) {
    t_err.clear();
    return fwd_impl(q, k, v, r, w, o, lse, B, T, 0, T, Hq, Hkv, d, window, R, scale, temp_n0, dtype, stream);
}

extern "C" int relbias_attn_fwd_chunk(const void* q, const void* k, const void* v, const float* r, const float* w,
                                      void* o, float* lse, int B, int T, int q_off, int kv_T, int Hq, int Hkv, int d,
                                      int window, int R, float scale, int temp_n0, int dtype, void* stream) {
    t_err.clear();
    return fwd_impl(q, k, v, r, w, o, lse, B, T, q_off, kv_T, Hq, Hkv, d, window, R, scale, temp_n0, dtype,
                    stream);
}

// Chunked prefill against a paged cache: every sequence's chunk at its own offset.
extern "C" int relbias_attn_fwd_chunk_paged(const void* q, const void* k_pages, const void* v_pages,
                                            const int* block_table, const int* q_offs, const int* q_lens,
                                            const float* r, const float* w, void* o, float* lse, int B, int T,
                                            int num_pages, int page_size, int max_pages, int Hq, int Hkv, int d,
                                            int window, int R, float scale, int temp_n0, int dtype, void* stream) {
    t_err.clear();
    int rc = check_common(B, T, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (B == 0 || T == 0) return RELBIAS_OK;
    if (num_pages < 1 || max_pages < 1)
        return fail(RELBIAS_ERR_ARG, "num_pages (%d) and max_pages (%d) must be >= 1", num_pages, max_pages);
    if (page_size < 64 || page_size % 64 != 0)
        return fail(RELBIAS_ERR_ARG, "page_size (%d) must be a positive multiple of 64", page_size);
    if (!q || !k_pages || !v_pages || !block_table || !q_offs || !q_lens || !r || !o)
        return fail(RELBIAS_ERR_ARG, "q, k_pages, v_pages, block_table, q_offs, q_lens, r and o must not be null");
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o))
        return fail(RELBIAS_ERR_ARG, "q, k_pages, v_pages and o must be 16-byte aligned");
    if (!aligned4(r) || !aligned4(block_table) || !aligned4(q_offs) || !aligned4(q_lens) || (lse && !aligned4(lse)))
        return fail(RELBIAS_ERR_ARG, "r, block_table, q_offs, q_lens and lse must be 4-byte aligned");
    if (dtype != RELBIAS_BF16) return fail(RELBIAS_ERR_UNSUPPORTED, "the paged chunked prefill is bf16 only");
    if (d != 64 && d != 128) return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill supports d in {64, 128}, got %d", d);
    if (R > 2048 || prefill_bf16_table_copies(d, R) == 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill stages R <= 2048 table entries, got %d", R);
    DeviceInfo dev;
    if ((rc = device_info(dev)) != RELBIAS_OK) return rc;
    if (dev.major != 10 || dev.minor != 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "bf16 prefill needs compute capability 10.0 (sm_100a), found %d.%d",
                    dev.major, dev.minor);
    CUtensorMap tq, tk, tv;
    if ((rc = make_map(&tq, q, B, T, Hq, d, 128)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tk, k_pages, num_pages, page_size, Hkv, d, 64)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tv, v_pages, num_pages, page_size, Hkv, d, 64)) != RELBIAS_OK) return rc;
    PrefillParams p{};
    p.r = r;
    p.w = w;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.nslots = (p.G % 2 == 0) ? 2 : 1;
    p.HP = p.G / p.nslots;
    p.window = window > 0 ? window : 0;
    p.R = R;
    p.n_qt = (T + 127) / 128;
    p.q_off = 0;
    p.kv_T = T;
    const long long items = static_cast<long long>(p.n_qt) * B * Hkv * p.HP;
    if (items > INT32_MAX) return fail(RELBIAS_ERR_UNSUPPORTED, "too many work items (%lld)", items);
    p.total_items = static_cast<int>(items);
    p.contiguous = p.window > 0 ? 1 : 0;
    p.o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    p.temp_n0 = temp_n0 > 1 ? temp_n0 : 0;
    p.inv_log_n0 = temp_n0 > 1 ? static_cast<float>(1.0 / std::log(static_cast<double>(temp_n0))) : 0.0f;
    p.paged = 1;
    p.block_table = block_table;
    p.q_offs = q_offs;
    p.q_lens = q_lens;
    p.page_size = page_size;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    const int grid = static_cast<int>(std::min<long long>(items, dev.sms));
    const cudaError_t e = launch_prefill_bf16_sm100(tq, tk, tv, p, d, grid, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "paged chunked prefill launch");
}

namespace relbias {
namespace {
int check_bank(int C, int proj_heads, int Hq) {
    if (C < 1 || C > kMaxBankC) return fail(RELBIAS_ERR_ARG, "C (%d) must be in [1, %d]", C, kMaxBankC);
    if (proj_heads != 1 && proj_heads != Hq)
        return fail(RELBIAS_ERR_ARG, "proj_heads (%d) must be 1 or Hq (%d)", proj_heads, Hq);
    return RELBIAS_OK;
}
size_t bank_curve_bytes(int B, int Hq, int R) {
    const size_t b = static_cast<size_t>(B) * Hq * std::max(R, 0) * sizeof(float);
    return (b + 255) / 256 * 256;
}
}  // namespace
}  // namespace relbias

extern "C" size_t relbias_attn_fwd_bank_workspace_size(int B, int T, int Hq, int R, int dtype) {
    if (B < 0 || T < 0 || Hq < 1 || R < 0) return 0;
    if (dtype != RELBIAS_BF16 || R == 0) return 0;
    return bank_prefill_curve_bytes(B, T, Hq, R);
}

extern "C" int relbias_attn_fwd_bank(const void* q, const void* k, const void* v, const float* rs, const float* proj,
                                     void* o, float* lse, int B, int T, int Hq, int Hkv, int d, int C, int proj_heads,
                                     int window, int R, float scale, int temp_n0, int dtype, void* workspace,
                                     size_t ws_bytes, void* stream) {
    t_err.clear();
    const int rc = check_bank(C, proj_heads, Hq);
    if (rc != RELBIAS_OK) return rc;
    return fwd_impl(q, k, v, rs, proj, o, lse, B, T, 0, T, Hq, Hkv, d, window, R, scale, temp_n0, dtype, stream, C,
                    proj_heads, workspace, ws_bytes);
}

extern "C" size_t relbias_attn_decode_workspace_size(int B, int Hq, int Hkv, int n_ctx, int d, int window) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || n_ctx < 1 || d < 1) return 0;
    DeviceInfo dev;
    if (device_info(dev) != RELBIAS_OK) return 0;
    const int nsplit = decode_num_splits(B, Hkv, n_ctx, window, dev.sms);
    return decode_workspace_bytes(B, Hq, nsplit, d);
}

namespace {
// Host-side checks of a contiguous-cache decode call; the workspace pointer is
// checked only when `check_ws` (the allocation-free variant supplies its own).  Sets
// *nothing_to_do for an empty batch (after the shape checks, before any pointer
// check).  The only CUDA calls are the device queries, made after the arguments pass.
int decode_check_args(const void* q, const void* k_cache, const void* v_cache, const float* r, const float* w,
                      size_t w_bstride, const void* o, const float* lse, int B, int n_ctx, int Hq, int Hkv, int d,
                      int R, float scale, int dtype, bool check_ws, const void* workspace, bool* nothing_to_do,
                      DeviceInfo* dev) {
    *nothing_to_do = false;
    int rc = check_common(B, n_ctx, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (B == 0) {
        *nothing_to_do = true;
        return RELBIAS_OK;
    }
    if (n_ctx < 1) return fail(RELBIAS_ERR_ARG, "n_ctx (%d) must be >= 1", n_ctx);
    if (!q || !k_cache || !v_cache || (w_bstride == 0 && !r) || !o)
        return fail(RELBIAS_ERR_ARG, "q, k_cache, v_cache, r and o must not be null");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return fail(RELBIAS_ERR_ARG, "q, k_cache, v_cache and o must be 16-byte aligned");
    if (!aligned4(r) || (lse && !aligned4(lse))) return fail(RELBIAS_ERR_ARG, "r and lse must be 4-byte aligned");
    if (check_ws && (!workspace || !aligned16(workspace)))
        return fail(RELBIAS_ERR_ARG, "workspace must be non-null and 16-byte aligned");
    if (dtype != RELBIAS_BF16) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports bf16 only");
    if (d != 128) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports d == 128, got %d", d);
    if (Hq / Hkv > 8) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports up to 8 query heads per key/value head");
    if ((rc = device_info(*dev)) != RELBIAS_OK) return rc;
    if (dev->major != 10 || dev->minor != 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "decode needs compute capability 10.0 (sm_100a), found %d.%d",
                    dev->major, dev->minor);
    return RELBIAS_OK;
}

// Contiguous-cache decode.  w_bstride == 0: rank-1 tables w [Hq, R] times r [B, Hq];
// w_bstride == Hq * R: per-sequence curves w [B, Hq, R] with coefficient 1 (r unused).
int decode_impl(const void* q, const void* k_cache, const void* v_cache, const float* r, const float* w,
                size_t w_bstride, void* o, float* lse, int B, int n_ctx, int Hq, int Hkv, int d, int window, int R,
                float scale, int temp_n0, int dtype, void* workspace, size_t ws_bytes, void* stream) {
    bool nothing_to_do = false;
    DeviceInfo dev;
    int rc = decode_check_args(q, k_cache, v_cache, r, w, w_bstride, o, lse, B, n_ctx, Hq, Hkv, d, R, scale, dtype,
                               true, workspace, &nothing_to_do, &dev);
    if (rc != RELBIAS_OK || nothing_to_do) return rc;

    DecodeParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.r = w_bstride == 0 ? r : nullptr;
    p.w = w;
    p.w_bstride = w_bstride;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.part = static_cast<float*>(workspace);
    p.B = B;
    p.N = n_ctx;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.window = window > 0 ? window : 0;
    p.R = R;
    p.key_lo = p.window > 0 ? std::max(0, n_ctx - p.window) : 0;
    p.nchunks = (n_ctx - p.key_lo + kChunk - 1) / kChunk;
    p.nsplit = decode_num_splits(B, Hkv, n_ctx, p.window, dev.sms);
    p.chunks_per_split = (p.nchunks + p.nsplit - 1) / p.nsplit;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    {
        // Context-length temperature of the one query row, which sees n keys: both
        // logit terms scale by ln n / ln temp_n0 (the bias is added in units of the
        // unscaled logit, so scaling the log2 factor scales both).
        const int n = p.window > 0 ? std::min(n_ctx, p.window) : n_ctx;
        if (temp_n0 > 1 && n > temp_n0)
            p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634 *
                                              (std::log(static_cast<double>(n)) /
                                               std::log(static_cast<double>(temp_n0))));
    }
    const size_t need = decode_workspace_bytes(B, Hq, p.nsplit, d);
    if (ws_bytes < need)
        return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed", ws_bytes, need);

    CUtensorMap tk, tv;
    if ((rc = make_map(&tk, k_cache, B, n_ctx, Hkv, d, kChunk)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tv, v_cache, B, n_ctx, Hkv, d, kChunk)) != RELBIAS_OK) return rc;
    cudaError_t e = launch_decode_bf16(tk, tv, p, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "decode launch");
}
}  // namespace

extern "C" int relbias_attn_decode(const void* q, const void* k_cache, const void* v_cache, const float* r,
                                   const float* w, void* o, float* lse, int B, int n_ctx, int Hq, int Hkv, int d,
                                   int window, int R, float scale, int temp_n0, int dtype, void* workspace,
                                   size_t ws_bytes, void* stream) {
    t_err.clear();
    return decode_impl(q, k_cache, v_cache, r, w, 0, o, lse, B, n_ctx, Hq, Hkv, d, window, R, scale, temp_n0, dtype,
                       workspace, ws_bytes, stream);
}

extern "C" size_t relbias_attn_decode_bank_workspace_size(int B, int Hq, int Hkv, int n_ctx, int d, int window,
                                                          int R) {
    const size_t base = relbias_attn_decode_workspace_size(B, Hq, Hkv, n_ctx, d, window);
    if (base == 0 || R < 0) return 0;
    return bank_curve_bytes(B, Hq, R) + base;
}

extern "C" int relbias_attn_decode_bank(const void* q, const void* k_cache, const void* v_cache, const float* rs,
                                        const float* proj, void* o, float* lse, int B, int n_ctx, int Hq, int Hkv,
                                        int d, int C, int proj_heads, int window, int R, float scale, int temp_n0,
                                        int dtype, void* workspace, size_t ws_bytes, void* stream) {
    t_err.clear();
    int rc = check_bank(C, proj_heads, Hq);
    if (rc != RELBIAS_OK) return rc;
    if ((rc = check_common(B, n_ctx, Hq, Hkv, d, R, scale, proj)) != RELBIAS_OK) return rc;
    if (B == 0) return RELBIAS_OK;
    if (dtype != RELBIAS_BF16) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports bf16 only");
    if (d != 128) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports d == 128, got %d", d);
    if (!rs || !aligned4(rs)) return fail(RELBIAS_ERR_ARG, "rs is null or not 4-byte aligned");
    if (!workspace || !aligned16(workspace)) return fail(RELBIAS_ERR_ARG, "workspace is null or not 16-byte aligned");
    const size_t cb = bank_curve_bytes(B, Hq, R);
    if (ws_bytes < cb) return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes cannot hold the %zu bytes of curves",
                                   ws_bytes, cb);
    float* curves = static_cast<float*>(workspace);
    if (R > 0) {
        const cudaError_t e = launch_bank_curves(rs, proj, curves, B * Hq, Hq, C, proj_heads, R,
                                                 static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "bank curve launch");
    }
    return decode_impl(q, k_cache, v_cache, nullptr, curves, static_cast<size_t>(Hq) * R, o, lse, B, n_ctx, Hq, Hkv,
                       d, window, R, scale, temp_n0, dtype, static_cast<char*>(workspace) + cb, ws_bytes - cb,
                       stream);
}

namespace relbias {
namespace {
// Split plan for paged decode: the longest chunk run any sequence of at most
// max_seq_len rows can need (chunks aligned to multiples of 32 rows).
int paged_max_chunks(int max_seq_len, int window) {
    const int all = (max_seq_len + kChunk - 1) / kChunk;
    if (window <= 0) return all;
    return std::min(all, (window + kChunk - 1) / kChunk + 1);
}
int paged_num_splits(int B, int Hkv, int max_chunks, int num_sms) {
    const int target = num_sms * 8;
    const int pairs = std::max(1, B * Hkv);
    int nsplit = std::max(1, std::min((target + pairs - 1) / pairs, max_chunks));
    const int cps = (max_chunks + nsplit - 1) / nsplit;
    return (max_chunks + cps - 1) / cps;
}
}  // namespace
}  // namespace relbias

extern "C" size_t relbias_attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_seq_len, int d,
                                                          int window) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_seq_len < 1 || d < 1) return 0;
    DeviceInfo dev;
    if (device_info(dev) != RELBIAS_OK) return 0;
    const int nsplit = paged_num_splits(B, Hkv, paged_max_chunks(max_seq_len, window > 0 ? window : 0), dev.sms);
    return decode_workspace_bytes(B, Hq, nsplit, d);
}

extern "C" int relbias_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                         const int* block_table, const int* seq_lens, const float* r, const float* w,
                                         void* o, float* lse, int B, int num_pages, int page_size, int max_pages,
                                         int max_seq_len, int Hq, int Hkv, int d, int window, int R, float scale,
                                         int temp_n0, int dtype, void* workspace, size_t ws_bytes, void* stream) {
    t_err.clear();
    int rc = check_common(B, max_seq_len, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (B == 0) return RELBIAS_OK;
    if (max_seq_len < 1) return fail(RELBIAS_ERR_ARG, "max_seq_len (%d) must be >= 1", max_seq_len);
    if (num_pages < 1 || max_pages < 1)
        return fail(RELBIAS_ERR_ARG, "num_pages (%d) and max_pages (%d) must be >= 1", num_pages, max_pages);
    if (page_size < kChunk || page_size % kChunk != 0)
        return fail(RELBIAS_ERR_ARG, "page_size (%d) must be a positive multiple of %d", page_size, kChunk);
    if (static_cast<long long>(max_pages) * page_size < max_seq_len)
        return fail(RELBIAS_ERR_ARG, "max_pages * page_size (%lld) is shorter than max_seq_len (%d)",
                    static_cast<long long>(max_pages) * page_size, max_seq_len);
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !r || !o || !workspace)
        return fail(RELBIAS_ERR_ARG, "q, k_pages, v_pages, block_table, seq_lens, r, o and workspace must not be null");
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace))
        return fail(RELBIAS_ERR_ARG, "q, k_pages, v_pages, o and workspace must be 16-byte aligned");
    if (!aligned4(r) || !aligned4(block_table) || !aligned4(seq_lens) || (lse && !aligned4(lse)))
        return fail(RELBIAS_ERR_ARG, "r, block_table, seq_lens and lse must be 4-byte aligned");
    if (dtype != RELBIAS_BF16) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports bf16 only");
    if (d != 128) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports d == 128, got %d", d);
    if (Hq / Hkv > 8) return fail(RELBIAS_ERR_UNSUPPORTED, "decode supports up to 8 query heads per key/value head");
    DeviceInfo dev;
    if ((rc = device_info(dev)) != RELBIAS_OK) return rc;
    if (dev.major != 10 || dev.minor != 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "decode needs compute capability 10.0 (sm_100a), found %d.%d", dev.major,
                    dev.minor);

    DecodeParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.r = r;
    p.w = w;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.part = static_cast<float*>(workspace);
    p.B = B;
    p.N = max_seq_len;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.window = window > 0 ? window : 0;
    p.R = R;
    p.key_lo = 0;
    p.nchunks = paged_max_chunks(max_seq_len, p.window);
    p.nsplit = paged_num_splits(B, Hkv, p.nchunks, dev.sms);
    p.chunks_per_split = (p.nchunks + p.nsplit - 1) / p.nsplit;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.page_size = page_size;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    p.temp_n0 = temp_n0 > 1 ? temp_n0 : 0;
    p.inv_log_n0 = temp_n0 > 1 ? static_cast<float>(1.0 / std::log(static_cast<double>(temp_n0))) : 0.0f;
    const size_t need = decode_workspace_bytes(B, Hq, p.nsplit, d);
    if (ws_bytes < need)
        return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed", ws_bytes, need);

    CUtensorMap tk, tv;
    if ((rc = make_map(&tk, k_pages, num_pages, page_size, Hkv, d, kChunk)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tv, v_pages, num_pages, page_size, Hkv, d, kChunk)) != RELBIAS_OK) return rc;
    cudaError_t e = launch_decode_paged_bf16(tk, tv, p, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "paged decode launch");
}

namespace {
// The backward pass on the tcgen05 tensor cores: the dQ / dr kernel, then the
// dK / dV / dw kernel (which reads the D_i = dout_i . o_i the first one writes).
int bwd_tc_impl(const void* q, const void* k, const void* v, const float* r, const float* w, const void* o,
                const float* lse, const void* dout, float* dq, float* dk, float* dv, float* dr, float* dw, int B,
                int T, int Hq, int Hkv, int d, int window, int R, float scale, int temp_n0, float* dvec, int sms,
                cudaStream_t st, const float* curves = nullptr, float* dcv = nullptr, int curve_stride = 0) {
    int rc;
    CUtensorMap tq, tdo, tk, tv;
    if ((rc = make_map(&tq, q, B, T, Hq, d, 128)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tdo, dout, B, T, Hq, d, 128)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tk, k, B, T, Hkv, d, 128)) != RELBIAS_OK) return rc;
    if ((rc = make_map(&tv, v, B, T, Hkv, d, 128)) != RELBIAS_OK) return rc;
    PrefillParams p{};
    p.r = r;
    p.w = w;
    p.B = B;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.nslots = 1;
    p.HP = p.G;
    p.window = window > 0 ? window : 0;
    p.R = R;
    p.n_qt = (T + 127) / 128;
    p.q_off = 0;
    p.kv_T = T;
    p.contiguous = p.window > 0 ? 1 : 0;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    p.temp_n0 = temp_n0 > 1 ? temp_n0 : 0;
    p.inv_log_n0 = temp_n0 > 1 ? static_cast<float>(1.0 / std::log(static_cast<double>(temp_n0))) : 0.0f;
    PrefillParams p_dq = p, p_dkv = p;
    const long long n_dq = static_cast<long long>(p.n_qt) * B * Hq;
    const long long n_dkv = static_cast<long long>(p.n_qt) * B * Hkv;
    if (n_dq > INT32_MAX) return fail(RELBIAS_ERR_UNSUPPORTED, "too many work items (%lld)", n_dq);
    p_dq.total_items = static_cast<int>(n_dq);
    p_dkv.total_items = static_cast<int>(n_dkv);
    BwdTcParams bp{};
    bp.o = static_cast<const __nv_bfloat16*>(o);
    bp.dout = static_cast<const __nv_bfloat16*>(dout);
    bp.lse = lse;
    bp.dvec = dvec;
    bp.dq = dq;
    bp.dr = dr;
    bp.dk = dk;
    bp.dv = dv;
    bp.dw = dw;
    bp.scale = scale;
    bp.curves = curves;
    bp.dcv = dcv;
    bp.curve_stride = curve_stride;
    if (R > 0 && dw != nullptr) {
        const cudaError_t e = cudaMemsetAsync(dw, 0, static_cast<size_t>(Hq) * R * sizeof(float), st);
        if (e != cudaSuccess) return cuda_fail(e, "clearing dw");
    }
    const cudaError_t e = launch_backward_sm100(tq, tdo, tk, tv, p_dq, p_dkv, bp, d, sms, st);
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "backward launch");
}
}  // namespace

extern "C" size_t relbias_attn_bwd_workspace_size(int B, int T, int Hq) {
    if (B < 0 || T < 0 || Hq < 1) return 0;
    const size_t n = static_cast<size_t>(B) * Hq * T * sizeof(float);
    return n < 16 ? 16 : n;
}

extern "C" int relbias_attn_bwd(const void* q, const void* k, const void* v, const float* r, const float* w,
                                const void* o, const float* lse, const void* dout, float* dq, float* dk, float* dv,
                                float* dr, float* dw, int B, int T, int Hq, int Hkv, int d, int window, int R,
                                float scale, int temp_n0, int dtype, void* workspace, size_t ws_bytes, void* stream) {
    t_err.clear();
    int rc = check_common(B, T, Hq, Hkv, d, R, scale, w);
    if (rc != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (B == 0 || T == 0) return RELBIAS_OK;
    if (!q || !k || !v || !r || !o || !lse || !dout || !dq || !dk || !dv || !dr || (R > 0 && !dw) || !workspace)
        return fail(RELBIAS_ERR_ARG, "q, k, v, r, o, lse, dout, dq, dk, dv, dr, dw (R > 0) and workspace must not be "
                                     "null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return fail(RELBIAS_ERR_ARG, "q, k, v, o, dout, dq, dk, dv and workspace must be 16-byte aligned");
    if (!aligned4(r) || !aligned4(lse) || !aligned4(dr) || (dw && !aligned4(dw)))
        return fail(RELBIAS_ERR_ARG, "r, lse, dr and dw must be 4-byte aligned");
    if (d != 32 && d != 64 && d != 128 && d != 256)
        return fail(RELBIAS_ERR_UNSUPPORTED, "the backward pass supports d in {32, 64, 128, 256}, got %d", d);
    if (R > 32768) return fail(RELBIAS_ERR_UNSUPPORTED, "the backward pass stages R <= 32768 table gradients");
    if (ws_bytes < relbias_attn_bwd_workspace_size(B, T, Hq))
        return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed", ws_bytes,
                    relbias_attn_bwd_workspace_size(B, T, Hq));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == RELBIAS_BF16 && (d == 64 || d == 128) && backward_tc_supported(d, R)) {
        DeviceInfo dev;
        if ((rc = device_info(dev)) != RELBIAS_OK) return rc;
        if (dev.major == 10 && dev.minor == 0) return bwd_tc_impl(q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw,
                                                                  B, T, Hq, Hkv, d, window, R, scale, temp_n0,
                                                                  static_cast<float*>(workspace), dev.sms, st);
    }
    const cudaError_t e = launch_backward(dtype == RELBIAS_BF16, d, q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw,
                                          static_cast<float*>(workspace), B, T, Hq, Hkv, window > 0 ? window : 0, R,
                                          scale, temp_n0 > 1 ? temp_n0 : 0, st);
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "backward launch");
}

namespace {
// The bank form's backward workspace: D_i [B, Hq, T], then the per-row curves and
// their gradient, each [B, T, Hq, S] floats (S = prefill_bank_curve_stride(R)), each
// part starting on a 256-byte boundary.
size_t bwd_bank_part(size_t bytes) { return (bytes + 255) / 256 * 256; }
}  // namespace

extern "C" size_t relbias_attn_bwd_bank_workspace_size(int B, int T, int Hq, int R) {
    if (B < 0 || T < 0 || Hq < 1 || R < 1) return 0;
    const size_t rows = static_cast<size_t>(B) * T * Hq;
    return bwd_bank_part(rows * sizeof(float)) + 2 * bwd_bank_part(rows * prefill_bank_curve_stride(R) * sizeof(float));
}

extern "C" int relbias_attn_bwd_bank(const void* q, const void* k, const void* v, const float* rs, const float* proj,
                                     const void* o, const float* lse, const void* dout, float* dq, float* dk,
                                     float* dv, float* drs, float* dproj, int B, int T, int Hq, int Hkv, int d, int C,
                                     int proj_heads, int window, int R, float scale, int temp_n0, int dtype,
                                     void* workspace, size_t ws_bytes, void* stream) {
    t_err.clear();
    int rc = check_common(B, T, Hq, Hkv, d, R, scale, proj);
    if (rc != RELBIAS_OK) return rc;
    if ((rc = check_bank(C, proj_heads, Hq)) != RELBIAS_OK) return rc;
    if (dtype != RELBIAS_BF16 && dtype != RELBIAS_FP32) return fail(RELBIAS_ERR_ARG, "unknown dtype %d", dtype);
    if (B == 0 || T == 0) return RELBIAS_OK;
    if (dtype != RELBIAS_BF16 || !backward_bank_tc_supported(d))
        return fail(RELBIAS_ERR_UNSUPPORTED, "the bank-form backward runs bf16 with d in {64, 128}");
    if (R < 1) return fail(RELBIAS_ERR_UNSUPPORTED, "the bank-form backward needs R >= 1 (R = 0 has no bias)");
    if (R > 2048) return fail(RELBIAS_ERR_UNSUPPORTED, "the bank-form backward supports R <= 2048, got %d", R);
    if (static_cast<long long>(B) * T * Hq > INT32_MAX)
        return fail(RELBIAS_ERR_UNSUPPORTED, "B * T * Hq must stay below 2^31");
    if (!q || !k || !v || !rs || !proj || !o || !lse || !dout || !dq || !dk || !dv || !drs || !dproj || !workspace)
        return fail(RELBIAS_ERR_ARG, "no pointer argument may be null");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(RELBIAS_ERR_ARG, "q, k, v, o, dout, dq, dk and dv must be 16-byte aligned, workspace 256-byte");
    if (!aligned4(rs) || !aligned4(proj) || !aligned4(lse) || !aligned4(drs) || !aligned4(dproj))
        return fail(RELBIAS_ERR_ARG, "rs, proj, lse, drs and dproj must be 4-byte aligned");
    const size_t need = relbias_attn_bwd_bank_workspace_size(B, T, Hq, R);
    if (ws_bytes < need)
        return fail(RELBIAS_ERR_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed", ws_bytes, need);
    DeviceInfo dev;
    if ((rc = device_info(dev)) != RELBIAS_OK) return rc;
    if (dev.major != 10 || dev.minor != 0)
        return fail(RELBIAS_ERR_UNSUPPORTED, "the bank-form backward needs an sm_100 device");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t rows = static_cast<size_t>(B) * T * Hq;
    const int S = prefill_bank_curve_stride(R);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* dvec = reinterpret_cast<float*>(ws);
    float* curves = reinterpret_cast<float*>(ws + bwd_bank_part(rows * sizeof(float)));
    float* dcv = reinterpret_cast<float*>(ws + bwd_bank_part(rows * sizeof(float)) +
                                          bwd_bank_part(rows * S * sizeof(float)));
    cudaError_t e = launch_bank_rows(rs, proj, curves, B, T, Hq, 0, C, proj_heads, R, st);
    if (e != cudaSuccess) return cuda_fail(e, "bank curve launch");
    if ((e = cudaMemsetAsync(dcv, 0, rows * S * sizeof(float), st)) != cudaSuccess) return cuda_fail(e, "clearing dcv");
    if ((e = cudaMemsetAsync(dproj, 0, static_cast<size_t>(proj_heads) * C * R * sizeof(float), st)) != cudaSuccess)
        return cuda_fail(e, "clearing dproj");
    rc = bwd_tc_impl(q, k, v, rs, proj, o, lse, dout, dq, dk, dv, nullptr, nullptr, B, T, Hq, Hkv, d, window, R,
                     scale, temp_n0, dvec, dev.sms, st, curves, dcv, S);
    if (rc != RELBIAS_OK) return rc;
    e = launch_bank_grads(rs, proj, dcv, drs, dproj, B, T, Hq, C, proj_heads, R, S, st);
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "bank gradient launch");
}

extern "C" const char* relbias_last_error(void) { return t_err.c_str(); }

extern "C" int relbias_device_status(int reset) {
    t_err.clear();
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    unsigned int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v))) != cudaSuccess)
        return cuda_fail(e, "reading the status word");
    if (reset) {
        const unsigned int zero = 0;
        if ((e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero))) != cudaSuccess)
            return cuda_fail(e, "clearing the status word");
    }
    return static_cast<int>(v);
}

extern "C" int relbias_set_wait_limit_ns(unsigned long long ns) {
    t_err.clear();
    const unsigned long long v = ns == 0 ? kWaitLimitNs : ns;
    const cudaError_t e = cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
    return e == cudaSuccess ? RELBIAS_OK : cuda_fail(e, "setting the wait limit");
}

extern "C" int relbias_version(void) { return 701; }

// The allocation-free decode variant (its own file: it owns a static device array).
#include "decode_noalloc.cu"
