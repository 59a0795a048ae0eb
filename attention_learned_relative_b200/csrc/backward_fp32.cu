// backward_fp32.cu -- gradients of the biased attention forward pass, on CUDA cores.
//
// For one row (b, h, i) with logits l_j = tau_i * (scale * q_i.k_j + bias_ij) over
// the attended keys, p_j = exp(l_j - LSE_i) and O_i = sum_j p_j v_j, the chain rule
// gives dl_j = p_j (dO_i.v_j - D_i) with D_i = dO_i.O_i, and then
//   dq_i = tau_i scale sum_j dl_j k_j        dk_j = sum_(h,i) tau_i scale dl_j q_i
//   dv_j = sum_(h,i) p_j dO_i                 dr_i = sum_j tau_i dl_j w[h, i-j]
//   dw[h, d] = sum_i tau_i dl_(i, i-d) r_i    (bias only at 0 <= i-j < R)
// The bias is r[b,i,h] * w[h, i-j] ("Thinking Machines dropped RoPE", recipe steps
// 3-5; the pages train the model but print no backward, so this is the plain
// derivative of the forward definition).
//
// Two kernels, fp32 arithmetic, inputs in bf16 or fp32:
//   bwd_dq_kernel   one CTA per 32 query rows of (b, h): recomputes each row's
//                   logits and p against key/value tiles staged in shared memory,
//                   writes dq, dr and D_i (to the workspace).
//   bwd_dkv_kernel  one CTA per 32 keys of (b, key/value head g): loops over the
//                   group's query heads and the rows that attend to its keys,
//                   accumulates dk and dv in registers and dw in shared memory
//                   (then atomically into the [Hq, R] output).
// D/32 lanes share a row (or a key), each holding a contiguous 32-dimension chunk;
// tiles in shared memory are padded so those lanes read with conflict-free 128-bit
// loads (see BwdShape).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace relbias {

namespace {

constexpr int kBwdThreads = 128;

// Layout: a row (query or key) is shared by D/32 lanes, each holding a contiguous
// 32-dimension chunk in registers.  Tiles in shared memory keep a row's chunks 36
// floats apart (32 plus 4 of padding), so the D/32 lanes of a row read their chunks
// with conflict-free 128-bit loads while every row group of the warp reads the same
// row (a broadcast).
template <int D>
struct BwdShape {
    static constexpr int kLanes = D / 32;            // lanes per row
    static constexpr int kRows = kBwdThreads / kLanes;   // rows (or keys) per CTA
    static constexpr int kTile = 4096 / D;           // rows per shared-memory tile (16 KB)
    static constexpr int kChunk = 36;                // floats between a row's chunks
    static constexpr int kStride = kLanes * kChunk;  // floats per tile row
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <int LANES>
__device__ __forceinline__ float lane_sum(float x) {
#pragma unroll
    for (int off = 1; off < LANES; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Temperature of a row at position `pos`: tau = max(1, ln n / ln n0), n = visible keys.
__device__ __forceinline__ float row_tau(int pos, int window, int temp_n0) {
    if (temp_n0 <= 1) return 1.0f;
    const int n = window > 0 ? min(pos + 1, window) : pos + 1;
    if (n <= temp_n0) return 1.0f;
    return static_cast<float>(log(static_cast<double>(n)) / log(static_cast<double>(temp_n0)));
}

// Stage rows [r0, r0 + kTile) of a [.., rows, heads, D] tensor (head `hd`) into a
// padded fp32 tile; rows at or past `nrows` read as zeros.
template <int D, typename TI>
__device__ __forceinline__ void stage_tile(float* tile, const TI* src, int b, int r0, int nrows, int heads, int hd) {
    using S = BwdShape<D>;
    for (int x = threadIdx.x; x < S::kTile * D / 4; x += kBwdThreads) {
        const int e = 4 * x;
        const int rr = e / D, c = e % D;
        const int row = r0 + rr;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < nrows) val = ld4(src + ((static_cast<size_t>(b) * nrows + row) * heads + hd) * D + c);
        *reinterpret_cast<float4*>(tile + rr * S::kStride + (c / 32) * S::kChunk + (c % 32)) = val;
    }
}

template <int D, typename TI>
__global__ void __launch_bounds__(kBwdThreads)
    bwd_dq_kernel(const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
                  const float* __restrict__ r, const float* __restrict__ w, const TI* __restrict__ o,
                  const float* __restrict__ lse, const TI* __restrict__ dout, float* __restrict__ dq,
                  float* __restrict__ dr, float* __restrict__ dvec, int T, int Hq, int Hkv, int window, int R,
                  float scale, int temp_n0) {
    using S = BwdShape<D>;
    __shared__ __align__(16) float ks[S::kTile * S::kStride];
    __shared__ __align__(16) float vs[S::kTile * S::kStride];

    const int b = blockIdx.z, h = blockIdx.y;
    const int g = h / (Hq / Hkv);
    const int i0 = blockIdx.x * S::kRows;
    const int row = threadIdx.x / S::kLanes, part = threadIdx.x % S::kLanes;
    const int i = i0 + row;
    const bool row_ok = i < T;
    const size_t rbase = ((static_cast<size_t>(b) * T + (row_ok ? i : 0)) * Hq + h) * D + part * 32;

    float qv[32], dov[32], dqv[32];
    float dpart = 0.0f;
#pragma unroll
    for (int u = 0; u < 32; u += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), d4 = a, o4 = a;
        if (row_ok) {
            a = ld4(q + rbase + u);
            d4 = ld4(dout + rbase + u);
            o4 = ld4(o + rbase + u);
        }
        qv[u] = a.x, qv[u + 1] = a.y, qv[u + 2] = a.z, qv[u + 3] = a.w;
        dov[u] = d4.x, dov[u + 1] = d4.y, dov[u + 2] = d4.z, dov[u + 3] = d4.w;
        dpart = fmaf(d4.x, o4.x, fmaf(d4.y, o4.y, fmaf(d4.z, o4.z, fmaf(d4.w, o4.w, dpart))));
        dqv[u] = dqv[u + 1] = dqv[u + 2] = dqv[u + 3] = 0.0f;
    }
    const float Di = lane_sum<S::kLanes>(dpart);
    const size_t srow = (static_cast<size_t>(b) * Hq + h) * T + i;
    const float lse_i = row_ok ? lse[srow] : 0.0f;
    const float tau = row_tau(i, window, temp_n0);
    const float ri = row_ok ? r[(static_cast<size_t>(b) * T + i) * Hq + h] : 0.0f;
    const float* wh = w + static_cast<size_t>(h) * R;
    const float ts = tau * scale;
    float drv = 0.0f;

    int j_begin = 0;
    if (window > 0) j_begin = max(0, i0 - window + 1);
    const int j_end = min(T, i0 + S::kRows);
    for (int j0 = j_begin; j0 < j_end; j0 += S::kTile) {
        __syncthreads();
        stage_tile<D>(ks, k, b, j0, T, Hkv, g);
        stage_tile<D>(vs, v, b, j0, T, Hkv, g);
        __syncthreads();
#pragma unroll 2
        for (int jj = 0; jj < S::kTile; ++jj) {
            const float* kr = ks + jj * S::kStride + part * S::kChunk;
            const float* vr = vs + jj * S::kStride + part * S::kChunk;
            float kreg[32];
            // Four independent partial sums per product: short dependency chains.
            float dot4[4] = {0.f, 0.f, 0.f, 0.f}, dpv4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
                const float4 k4 = *reinterpret_cast<const float4*>(kr + u);
                const float4 v4 = *reinterpret_cast<const float4*>(vr + u);
                kreg[u] = k4.x, kreg[u + 1] = k4.y, kreg[u + 2] = k4.z, kreg[u + 3] = k4.w;
                dot4[0] = fmaf(qv[u], k4.x, dot4[0]);
                dot4[1] = fmaf(qv[u + 1], k4.y, dot4[1]);
                dot4[2] = fmaf(qv[u + 2], k4.z, dot4[2]);
                dot4[3] = fmaf(qv[u + 3], k4.w, dot4[3]);
                dpv4[0] = fmaf(dov[u], v4.x, dpv4[0]);
                dpv4[1] = fmaf(dov[u + 1], v4.y, dpv4[1]);
                dpv4[2] = fmaf(dov[u + 2], v4.z, dpv4[2]);
                dpv4[3] = fmaf(dov[u + 3], v4.w, dpv4[3]);
            }
            const float dot = lane_sum<S::kLanes>((dot4[0] + dot4[1]) + (dot4[2] + dot4[3]));
            const float dpv = lane_sum<S::kLanes>((dpv4[0] + dpv4[1]) + (dpv4[2] + dpv4[3]));
            const int j = j0 + jj;
            const int dist = i - j;
            const bool valid = row_ok && j < T && dist >= 0 && (window <= 0 || dist < window);
            if (!valid) continue;
            const float wd = dist < R ? __ldg(wh + dist) : 0.0f;
            const float l = tau * fmaf(scale, dot, ri * wd);
            const float p = expf(l - lse_i);
            const float dl = p * (dpv - Di);
            const float c_q = dl * ts;
#pragma unroll
            for (int u = 0; u < 32; ++u) dqv[u] = fmaf(c_q, kreg[u], dqv[u]);
            drv = fmaf(dl * tau, wd, drv);
        }
    }
    if (row_ok) {
        float* dst = dq + rbase;
#pragma unroll
        for (int u = 0; u < 32; u += 4)
            *reinterpret_cast<float4*>(dst + u) = make_float4(dqv[u], dqv[u + 1], dqv[u + 2], dqv[u + 3]);
        if (part == 0) {
            dr[(static_cast<size_t>(b) * T + i) * Hq + h] = drv;
            dvec[srow] = Di;
        }
    }
}

template <int D, typename TI>
__global__ void __launch_bounds__(kBwdThreads)
    bwd_dkv_kernel(const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
                   const float* __restrict__ r, const float* __restrict__ w, const float* __restrict__ lse,
                   const TI* __restrict__ dout, const float* __restrict__ dvec, float* __restrict__ dk,
                   float* __restrict__ dv, float* __restrict__ dw, int T, int Hq, int Hkv, int window, int R,
                   float scale, int temp_n0) {
    using S = BwdShape<D>;
    __shared__ __align__(16) float qs[S::kTile * S::kStride];
    __shared__ __align__(16) float ds[S::kTile * S::kStride];
    __shared__ float row_lse[S::kTile], row_D[S::kTile], row_r[S::kTile], row_tau_s[S::kTile];
    extern __shared__ float dw_s[];          // [R]: this CTA's dw for the current head

    const int b = blockIdx.z, g = blockIdx.y;
    const int G = Hq / Hkv;
    const int j0 = blockIdx.x * S::kRows;
    const int key = threadIdx.x / S::kLanes, part = threadIdx.x % S::kLanes;
    const int j = j0 + key;
    const bool key_ok = j < T;
    const size_t kbase = ((static_cast<size_t>(b) * T + (key_ok ? j : 0)) * Hkv + g) * D + part * 32;

    float kv_[32], vv_[32], dkv[32], dvv[32];
#pragma unroll
    for (int u = 0; u < 32; u += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c4 = a;
        if (key_ok) {
            a = ld4(k + kbase + u);
            c4 = ld4(v + kbase + u);
        }
        kv_[u] = a.x, kv_[u + 1] = a.y, kv_[u + 2] = a.z, kv_[u + 3] = a.w;
        vv_[u] = c4.x, vv_[u + 1] = c4.y, vv_[u + 2] = c4.z, vv_[u + 3] = c4.w;
        dkv[u] = dkv[u + 1] = dkv[u + 2] = dkv[u + 3] = 0.0f;
        dvv[u] = dvv[u + 1] = dvv[u + 2] = dvv[u + 3] = 0.0f;
    }
    // Query rows that attend to some key of this CTA.
    const int i_begin = j0;
    const int i_end = window > 0 ? min(T, j0 + S::kRows - 1 + window) : T;   // exclusive

    for (int hl = 0; hl < G; ++hl) {
        const int h = g * G + hl;
        const float* wh = w + static_cast<size_t>(h) * R;
        for (int x = threadIdx.x; x < R; x += kBwdThreads) dw_s[x] = 0.0f;
        for (int ib = i_begin; ib < i_end; ib += S::kTile) {
            __syncthreads();
            stage_tile<D>(qs, q, b, ib, T, Hq, h);
            stage_tile<D>(ds, dout, b, ib, T, Hq, h);
            for (int ii = threadIdx.x; ii < S::kTile; ii += kBwdThreads) {
                const int i = ib + ii;
                const bool ok = i < T;
                const size_t srow = (static_cast<size_t>(b) * Hq + h) * T + i;
                row_lse[ii] = ok ? lse[srow] : 0.0f;
                row_D[ii] = ok ? dvec[srow] : 0.0f;
                row_r[ii] = ok ? r[(static_cast<size_t>(b) * T + i) * Hq + h] : 0.0f;
                row_tau_s[ii] = row_tau(i, window, temp_n0);
            }
            __syncthreads();
            for (int ii = 0; ii < S::kTile; ++ii) {
                const float* qr = qs + ii * S::kStride + part * S::kChunk;
                const float* dr_ = ds + ii * S::kStride + part * S::kChunk;
                float qreg[32], dreg[32];
                float dot4[4] = {0.f, 0.f, 0.f, 0.f}, dpv4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int u = 0; u < 32; u += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(qr + u);
                    const float4 d4 = *reinterpret_cast<const float4*>(dr_ + u);
                    qreg[u] = q4.x, qreg[u + 1] = q4.y, qreg[u + 2] = q4.z, qreg[u + 3] = q4.w;
                    dreg[u] = d4.x, dreg[u + 1] = d4.y, dreg[u + 2] = d4.z, dreg[u + 3] = d4.w;
                    dot4[0] = fmaf(kv_[u], q4.x, dot4[0]);
                    dot4[1] = fmaf(kv_[u + 1], q4.y, dot4[1]);
                    dot4[2] = fmaf(kv_[u + 2], q4.z, dot4[2]);
                    dot4[3] = fmaf(kv_[u + 3], q4.w, dot4[3]);
                    dpv4[0] = fmaf(vv_[u], d4.x, dpv4[0]);
                    dpv4[1] = fmaf(vv_[u + 1], d4.y, dpv4[1]);
                    dpv4[2] = fmaf(vv_[u + 2], d4.z, dpv4[2]);
                    dpv4[3] = fmaf(vv_[u + 3], d4.w, dpv4[3]);
                }
                const float dot = lane_sum<S::kLanes>((dot4[0] + dot4[1]) + (dot4[2] + dot4[3]));
                const float dpv = lane_sum<S::kLanes>((dpv4[0] + dpv4[1]) + (dpv4[2] + dpv4[3]));
                const int i = ib + ii;
                const int dist = i - j;
                const bool valid = key_ok && i < T && dist >= 0 && (window <= 0 || dist < window);
                if (!valid) continue;
                const float tau = row_tau_s[ii];
                const float wd = dist < R ? __ldg(wh + dist) : 0.0f;
                const float l = tau * fmaf(scale, dot, row_r[ii] * wd);
                const float p = expf(l - row_lse[ii]);
                const float dl = p * (dpv - row_D[ii]);
                const float c_k = dl * tau * scale;
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    dvv[u] = fmaf(p, dreg[u], dvv[u]);
                    dkv[u] = fmaf(c_k, qreg[u], dkv[u]);
                }
                if (part == 0 && dist < R) atomicAdd(&dw_s[dist], dl * tau * row_r[ii]);
            }
        }
        __syncthreads();
        for (int x = threadIdx.x; x < R; x += kBwdThreads)
            if (dw_s[x] != 0.0f) atomicAdd(dw + static_cast<size_t>(h) * R + x, dw_s[x]);
        __syncthreads();
    }
    if (key_ok) {
#pragma unroll
        for (int u = 0; u < 32; u += 4) {
            *reinterpret_cast<float4*>(dk + kbase + u) = make_float4(dkv[u], dkv[u + 1], dkv[u + 2], dkv[u + 3]);
            *reinterpret_cast<float4*>(dv + kbase + u) = make_float4(dvv[u], dvv[u + 1], dvv[u + 2], dvv[u + 3]);
        }
    }
}

template <int D, typename TI>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const float* r, const float* w, const void* o,
                       const float* lse, const void* dout, float* dq, float* dk, float* dv, float* dr, float* dw,
                       float* dvec, int B, int T, int Hq, int Hkv, int window, int R, float scale, int temp_n0,
                       cudaStream_t st) {
    const TI* q_ = static_cast<const TI*>(q);
    const TI* k_ = static_cast<const TI*>(k);
    const TI* v_ = static_cast<const TI*>(v);
    const TI* o_ = static_cast<const TI*>(o);
    const TI* do_ = static_cast<const TI*>(dout);
    constexpr int kRows = BwdShape<D>::kRows;
    dim3 g1((T + kRows - 1) / kRows, Hq, B);
    bwd_dq_kernel<D, TI><<<g1, kBwdThreads, 0, st>>>(q_, k_, v_, r, w, o_, lse, do_, dq, dr, dvec, T, Hq, Hkv,
                                                      window, R, scale, temp_n0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t dyn = static_cast<size_t>(R) * sizeof(float);
    auto kern = bwd_dkv_kernel<D, TI>;
    if (dyn > 0) {
        // Static tiles (37 KB) plus the [R] table gradient may pass the 48 KB default.
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
        if (e != cudaSuccess) return e;
    }
    dim3 g2((T + kRows - 1) / kRows, Hkv, B);
    kern<<<g2, kBwdThreads, dyn, st>>>(q_, k_, v_, r, w, lse, do_, dvec, dk, dv, dw, T, Hq, Hkv, window, R, scale,
                                       temp_n0);
    return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_bwd_d(int d, const void* q, const void* k, const void* v, const float* r, const float* w,
                         const void* o, const float* lse, const void* dout, float* dq, float* dk, float* dv,
                         float* dr, float* dw, float* dvec, int B, int T, int Hq, int Hkv, int window, int R,
                         float scale, int temp_n0, cudaStream_t st) {
    switch (d) {
        case 32:
            return launch_bwd<32, TI>(q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv, window,
                                      R, scale, temp_n0, st);
        case 64:
            return launch_bwd<64, TI>(q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv, window,
                                      R, scale, temp_n0, st);
        case 128:
            return launch_bwd<128, TI>(q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv,
                                       window, R, scale, temp_n0, st);
        case 256:
            return launch_bwd<256, TI>(q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv,
                                       window, R, scale, temp_n0, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* r,
                            const float* w, const void* o, const float* lse, const void* dout, float* dq, float* dk,
                            float* dv, float* dr, float* dw, float* dvec, int B, int T, int Hq, int Hkv, int window,
                            int R, float scale, int temp_n0, cudaStream_t stream) {
    if (R > 0) {
        const cudaError_t e = cudaMemsetAsync(dw, 0, static_cast<size_t>(Hq) * R * sizeof(float), stream);
        if (e != cudaSuccess) return e;
    }
    if (bf16)
        return launch_bwd_d<__nv_bfloat16>(d, q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv,
                                           window, R, scale, temp_n0, stream);
    return launch_bwd_d<float>(d, q, k, v, r, w, o, lse, dout, dq, dk, dv, dr, dw, dvec, B, T, Hq, Hkv, window, R,
                               scale, temp_n0, stream);
}

}  // namespace relbias
