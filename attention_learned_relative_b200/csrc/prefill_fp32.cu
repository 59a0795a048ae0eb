// prefill_fp32.cu -- fp32 prefill on CUDA cores.
//
// Same operation as the bf16 tensor-core kernel, in fp32 storage and arithmetic:
// logit = scale * q.k + (0 <= i-j < R ? r[b,i,h] * w[h,i-j] : 0) over the causal
// (optionally windowed) keys, softmax, weighted sum of V ("Thinking Machines
// dropped RoPE", recipe steps 3-5; "Learned Relative-Position Bias", T5-style
// formula).  The BANK instance takes the essay's shared-bank form instead: the
// bias is sum_c r[b,i,h,c] * proj[h or 0, c, i-j], C <= 16 coefficients per token
// and head times the bank's functions (recipe steps 1-2).  A CTA takes 32 query rows of one (b, h); four lanes share a row and
// each holds a quarter of the head dimension (interleaved, so the four lanes read
// four consecutive floats of a key and the eight rows of a warp share them).
// Keys and values pass through shared memory in tiles.
#include <cuda_runtime.h>

#include <cfloat>

#include "kernels.h"

namespace relbias {

namespace {

constexpr int kRows = 32;
constexpr int kThreadsF32 = 128;

template <int D, bool BANK>
__global__ void __launch_bounds__(kThreadsF32)
    prefill_fp32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                        const float* __restrict__ r, const float* __restrict__ w, float* __restrict__ o,
                        float* __restrict__ lse, int T, int q_off, int kv_T, int Hq, int Hkv, int window, int R,
                        float scale, int temp_n0, int C, int proj_heads) {
    constexpr int BK = D <= 128 ? 32 : 16;   // keys per shared-memory tile
    constexpr int DL = D / 4;                 // dims per lane
    __shared__ __align__(16) float ks[BK * D];
    __shared__ __align__(16) float vs[BK * D];

    const int b = blockIdx.z, h = blockIdx.y;
    const int g = h / (Hq / Hkv);
    const int i0 = blockIdx.x * kRows;
    const int row = threadIdx.x >> 2, qd = threadIdx.x & 3;
    const int i = i0 + row;
    const bool row_ok = i < T;
    const int pos = q_off + i;   // the row's position in the sequence (K/V have kv_T rows)
    const int kv_end = q_off + T;   // keys past the chunk's last row are never visible: never read

    float qv[DL], ov[DL];
    const float* qrow = q + ((static_cast<size_t>(b) * T + (row_ok ? i : 0)) * Hq + h) * D;
#pragma unroll
    for (int u = 0; u < DL; ++u) {
        qv[u] = row_ok ? qrow[4 * u + qd] : 0.0f;
        ov[u] = 0.0f;
    }
    // Context-length temperature: a row that sees n > temp_n0 keys has both logit
    // terms scaled by ln n / ln temp_n0.
    float tau = 1.0f;
    if (temp_n0 > 1) {
        const int n = window > 0 ? min(pos + 1, window) : pos + 1;
        if (n > temp_n0) tau = static_cast<float>(log(static_cast<double>(n)) / log(static_cast<double>(temp_n0)));
    }
    const float ri = (!BANK && row_ok) ? tau * r[(static_cast<size_t>(b) * T + i) * Hq + h] : 0.0f;
    // Shared bank: this row's coefficients (times tau) and its head's bank.
    float rc[BANK ? kMaxBankC : 1];
    const float* bank = w;
    if constexpr (BANK) {
#pragma unroll
        for (int c = 0; c < kMaxBankC; ++c)
            rc[c] = (row_ok && c < C) ? tau * r[((static_cast<size_t>(b) * T + i) * Hq + h) * C + c] : 0.0f;
        bank = w + static_cast<size_t>(proj_heads == 1 ? 0 : h) * C * R;
    }
    const float scale_row = tau * scale;
    float m = -INFINITY, l = 0.0f;

    int j_begin = 0;
    if (window > 0) j_begin = max(0, q_off + i0 - window + 1);
    const int j_end = min(kv_end, q_off + i0 + kRows);   // exclusive
    for (int j0 = j_begin; j0 < j_end; j0 += BK) {
        __syncthreads();
        for (int x = threadIdx.x; x < BK * D / 4; x += kThreadsF32) {
            const int jj = (4 * x) / D, c = (4 * x) % D;
            const int j = j0 + jj;
            float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
            if (j < kv_end) {
                const size_t off = ((static_cast<size_t>(b) * kv_T + j) * Hkv + g) * D + c;
                kk = *reinterpret_cast<const float4*>(k + off);
                vv = *reinterpret_cast<const float4*>(v + off);
            }
            *reinterpret_cast<float4*>(ks + jj * D + c) = kk;
            *reinterpret_cast<float4*>(vs + jj * D + c) = vv;
        }
        __syncthreads();

        float s[BK];
        float mt = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < BK; ++jj) {
            float part = 0.0f;
#pragma unroll
            for (int u = 0; u < DL; ++u) part = fmaf(qv[u], ks[jj * D + 4 * u + qd], part);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            const int j = j0 + jj;
            const int dist = pos - j;
            const bool valid = row_ok && j < kv_end && dist >= 0 && (window <= 0 || dist < window);
            float x = -INFINITY;
            if (valid) {
                x = part * scale_row;
                if constexpr (BANK) {
                    if (dist < R) {
#pragma unroll
                        for (int c = 0; c < kMaxBankC; ++c)
                            if (c < C) x = fmaf(rc[c], __ldg(bank + static_cast<size_t>(c) * R + dist), x);
                    }
                } else {
                    if (dist < R) x = fmaf(ri, __ldg(w + static_cast<size_t>(h) * R + dist), x);
                }
            }
            s[jj] = x;
            mt = fmaxf(mt, x);
        }
        const float m_new = fmaxf(m, mt);
        if (m_new == -INFINITY) continue;   // nothing visible yet for this row
        const float alpha = expf(m - m_new);
        l *= alpha;
#pragma unroll
        for (int u = 0; u < DL; ++u) ov[u] *= alpha;
#pragma unroll
        for (int jj = 0; jj < BK; ++jj) {
            const float pj = expf(s[jj] - m_new);
            l += pj;
#pragma unroll
            for (int u = 0; u < DL; ++u) ov[u] = fmaf(pj, vs[jj * D + 4 * u + qd], ov[u]);
        }
        m = m_new;
    }

    if (row_ok) {
        float* orow = o + ((static_cast<size_t>(b) * T + i) * Hq + h) * D;
        const float inv = 1.0f / l;
#pragma unroll
        for (int u = 0; u < DL; ++u) orow[4 * u + qd] = ov[u] * inv;
        if (lse != nullptr && qd == 0) lse[(static_cast<size_t>(b) * Hq + h) * T + i] = m + logf(l);
    }
}

template <int D>
cudaError_t launch(const float* q, const float* k, const float* v, const float* r, const float* w, float* o,
                   float* lse, int B, int T, int q_off, int kv_T, int Hq, int Hkv, int window, int R, float scale,
                   int temp_n0, int C, int proj_heads, cudaStream_t st) {
    dim3 grid((T + kRows - 1) / kRows, Hq, B);
    if (C > 0)
        prefill_fp32_kernel<D, true><<<grid, kThreadsF32, 0, st>>>(q, k, v, r, w, o, lse, T, q_off, kv_T, Hq, Hkv,
                                                                   window, R, scale, temp_n0, C, proj_heads);
    else
        prefill_fp32_kernel<D, false><<<grid, kThreadsF32, 0, st>>>(q, k, v, r, w, o, lse, T, q_off, kv_T, Hq, Hkv,
                                                                    window, R, scale, temp_n0, 0, 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_fp32(const float* q, const float* k, const float* v, const float* r, const float* w,
                                float* o, float* lse, int B, int T, int q_off, int kv_T, int Hq, int Hkv, int d,
                                int window, int R, float scale, int temp_n0, int C, int proj_heads,
                                cudaStream_t stream) {
    switch (d) {
        case 32:
            return launch<32>(q, k, v, r, w, o, lse, B, T, q_off, kv_T, Hq, Hkv, window, R, scale, temp_n0, C,
                              proj_heads, stream);
        case 64:
            return launch<64>(q, k, v, r, w, o, lse, B, T, q_off, kv_T, Hq, Hkv, window, R, scale, temp_n0, C,
                              proj_heads, stream);
        case 128:
            return launch<128>(q, k, v, r, w, o, lse, B, T, q_off, kv_T, Hq, Hkv, window, R, scale, temp_n0, C,
                               proj_heads, stream);
        case 256:
            return launch<256>(q, k, v, r, w, o, lse, B, T, q_off, kv_T, Hq, Hkv, window, R, scale, temp_n0, C,
                               proj_heads, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace relbias
