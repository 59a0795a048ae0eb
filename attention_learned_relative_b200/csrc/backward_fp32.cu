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
// Four lanes share a row (or a key); each holds a quarter of the head dimension,
// interleaved so that the four lanes read four consecutive floats.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace relbias {

namespace {

constexpr int kBwdRows = 32;     // query rows (bwd_dq) or keys (bwd_dkv) per CTA
constexpr int kBwdThreads = 128;

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

// Temperature of a row at position `pos`: tau = max(1, ln n / ln n0), n = visible keys.
__device__ __forceinline__ float row_tau(int pos, int window, int temp_n0) {
    if (temp_n0 <= 1) return 1.0f;
    const int n = window > 0 ? min(pos + 1, window) : pos + 1;
    if (n <= temp_n0) return 1.0f;
    return static_cast<float>(log(static_cast<double>(n)) / log(static_cast<double>(temp_n0)));
}

template <int D, typename TI>
__global__ void __launch_bounds__(kBwdThreads)
    bwd_dq_kernel(const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
                  const float* __restrict__ r, const float* __restrict__ w, const TI* __restrict__ o,
                  const float* __restrict__ lse, const TI* __restrict__ dout, float* __restrict__ dq,
                  float* __restrict__ dr, float* __restrict__ dvec, int T, int Hq, int Hkv, int window, int R,
                  float scale, int temp_n0) {
    constexpr int BK = D <= 128 ? 32 : 16;
    constexpr int DL = D / 4;
    __shared__ __align__(16) float ks[BK * D];
    __shared__ __align__(16) float vs[BK * D];

    const int b = blockIdx.z, h = blockIdx.y;
    const int g = h / (Hq / Hkv);
    const int i0 = blockIdx.x * kBwdRows;
    const int row = threadIdx.x >> 2, qd = threadIdx.x & 3;
    const int i = i0 + row;
    const bool row_ok = i < T;
    const size_t rbase = ((static_cast<size_t>(b) * T + (row_ok ? i : 0)) * Hq + h) * D;

    float qv[DL], dov[DL], dqv[DL];
    float dpart = 0.0f;
#pragma unroll
    for (int u = 0; u < DL; ++u) {
        const int c = 4 * u + qd;
        qv[u] = row_ok ? ld(q + rbase + c) : 0.0f;
        dov[u] = row_ok ? ld(dout + rbase + c) : 0.0f;
        dpart = fmaf(dov[u], row_ok ? ld(o + rbase + c) : 0.0f, dpart);
        dqv[u] = 0.0f;
    }
    const float Di = quad_sum(dpart);
    const size_t srow = (static_cast<size_t>(b) * Hq + h) * T + i;
    const float lse_i = row_ok ? lse[srow] : 0.0f;
    const float tau = row_tau(i, window, temp_n0);
    const float ri = row_ok ? r[(static_cast<size_t>(b) * T + i) * Hq + h] : 0.0f;
    const float* wh = w + static_cast<size_t>(h) * R;
    const float ts = tau * scale;
    float drv = 0.0f;

    int j_begin = 0;
    if (window > 0) j_begin = max(0, i0 - window + 1);
    const int j_end = min(T, i0 + kBwdRows);
    for (int j0 = j_begin; j0 < j_end; j0 += BK) {
        __syncthreads();
        for (int x = threadIdx.x; x < BK * D; x += kBwdThreads) {
            const int jj = x / D, c = x % D;
            const int j = j0 + jj;
            float kk = 0.0f, vv = 0.0f;
            if (j < T) {
                const size_t off = ((static_cast<size_t>(b) * T + j) * Hkv + g) * D + c;
                kk = ld(k + off);
                vv = ld(v + off);
            }
            ks[x] = kk;
            vs[x] = vv;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < BK; ++jj) {
            float dot = 0.0f, dpv = 0.0f;
#pragma unroll
            for (int u = 0; u < DL; ++u) {
                dot = fmaf(qv[u], ks[jj * D + 4 * u + qd], dot);
                dpv = fmaf(dov[u], vs[jj * D + 4 * u + qd], dpv);
            }
            dot = quad_sum(dot);
            dpv = quad_sum(dpv);
            const int j = j0 + jj;
            const int dist = i - j;
            const bool valid = row_ok && j < T && dist >= 0 && (window <= 0 || dist < window);
            if (!valid) continue;
            const float wd = dist < R ? __ldg(wh + dist) : 0.0f;
            const float l = tau * fmaf(scale, dot, ri * wd);
            const float p = expf(l - lse_i);
            const float dl = p * (dpv - Di);
#pragma unroll
            for (int u = 0; u < DL; ++u) dqv[u] = fmaf(dl * ts, ks[jj * D + 4 * u + qd], dqv[u]);
            drv = fmaf(dl * tau, wd, drv);
        }
    }
    if (row_ok) {
#pragma unroll
        for (int u = 0; u < DL; ++u) dq[rbase + 4 * u + qd] = dqv[u];
        if (qd == 0) {
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
    constexpr int BQ = D <= 128 ? 32 : 16;   // query rows per shared-memory tile
    constexpr int DL = D / 4;
    __shared__ __align__(16) float qs[BQ * D];
    __shared__ __align__(16) float ds[BQ * D];
    __shared__ float row_lse[BQ], row_D[BQ], row_r[BQ], row_tau_s[BQ];
    extern __shared__ float dw_s[];          // [R]: this CTA's dw for the current head

    const int b = blockIdx.z, g = blockIdx.y;
    const int G = Hq / Hkv;
    const int j0 = blockIdx.x * kBwdRows;
    const int key = threadIdx.x >> 2, qd = threadIdx.x & 3;
    const int j = j0 + key;
    const bool key_ok = j < T;
    const size_t kbase = ((static_cast<size_t>(b) * T + (key_ok ? j : 0)) * Hkv + g) * D;

    float kv_[DL], vv_[DL], dkv[DL], dvv[DL];
#pragma unroll
    for (int u = 0; u < DL; ++u) {
        kv_[u] = key_ok ? ld(k + kbase + 4 * u + qd) : 0.0f;
        vv_[u] = key_ok ? ld(v + kbase + 4 * u + qd) : 0.0f;
        dkv[u] = 0.0f;
        dvv[u] = 0.0f;
    }
    // Query rows that attend to some key of this CTA.
    const int i_begin = j0;
    const int i_end = window > 0 ? min(T, j0 + kBwdRows - 1 + window) : T;   // exclusive

    for (int hl = 0; hl < G; ++hl) {
        const int h = g * G + hl;
        const float* wh = w + static_cast<size_t>(h) * R;
        for (int x = threadIdx.x; x < R; x += kBwdThreads) dw_s[x] = 0.0f;
        for (int ib = i_begin; ib < i_end; ib += BQ) {
            __syncthreads();
            for (int x = threadIdx.x; x < BQ * D; x += kBwdThreads) {
                const int ii = x / D, c = x % D;
                const int i = ib + ii;
                float qq = 0.0f, dd = 0.0f;
                if (i < T) {
                    const size_t off = ((static_cast<size_t>(b) * T + i) * Hq + h) * D + c;
                    qq = ld(q + off);
                    dd = ld(dout + off);
                }
                qs[x] = qq;
                ds[x] = dd;
            }
            for (int ii = threadIdx.x; ii < BQ; ii += kBwdThreads) {
                const int i = ib + ii;
                const bool ok = i < T;
                const size_t srow = (static_cast<size_t>(b) * Hq + h) * T + i;
                row_lse[ii] = ok ? lse[srow] : 0.0f;
                row_D[ii] = ok ? dvec[srow] : 0.0f;
                row_r[ii] = ok ? r[(static_cast<size_t>(b) * T + i) * Hq + h] : 0.0f;
                row_tau_s[ii] = row_tau(i, window, temp_n0);
            }
            __syncthreads();
#pragma unroll 4
            for (int ii = 0; ii < BQ; ++ii) {
                float dot = 0.0f, dpv = 0.0f;
#pragma unroll
                for (int u = 0; u < DL; ++u) {
                    dot = fmaf(kv_[u], qs[ii * D + 4 * u + qd], dot);
                    dpv = fmaf(vv_[u], ds[ii * D + 4 * u + qd], dpv);
                }
                dot = quad_sum(dot);
                dpv = quad_sum(dpv);
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
                for (int u = 0; u < DL; ++u) {
                    dvv[u] = fmaf(p, ds[ii * D + 4 * u + qd], dvv[u]);
                    dkv[u] = fmaf(c_k, qs[ii * D + 4 * u + qd], dkv[u]);
                }
                if (qd == 0 && dist < R) atomicAdd(&dw_s[dist], dl * tau * row_r[ii]);
            }
        }
        __syncthreads();
        for (int x = threadIdx.x; x < R; x += kBwdThreads)
            if (dw_s[x] != 0.0f) atomicAdd(dw + static_cast<size_t>(h) * R + x, dw_s[x]);
        __syncthreads();
    }
    if (key_ok) {
#pragma unroll
        for (int u = 0; u < DL; ++u) {
            dk[kbase + 4 * u + qd] = dkv[u];
            dv[kbase + 4 * u + qd] = dvv[u];
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
    dim3 g1((T + kBwdRows - 1) / kBwdRows, Hq, B);
    bwd_dq_kernel<D, TI><<<g1, kBwdThreads, 0, st>>>(q_, k_, v_, r, w, o_, lse, do_, dq, dr, dvec, T, Hq, Hkv,
                                                      window, R, scale, temp_n0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t dyn = static_cast<size_t>(R) * sizeof(float);
    auto kern = bwd_dkv_kernel<D, TI>;
    if (dyn > 0) {
        // Static tiles (up to 33 KB) plus the [R] table gradient may pass the 48 KB default.
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
        if (e != cudaSuccess) return e;
    }
    dim3 g2((T + kBwdRows - 1) / kBwdRows, Hkv, B);
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
