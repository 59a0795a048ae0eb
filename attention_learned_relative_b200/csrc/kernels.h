// kernels.h -- internal interface between the C-ABI host layer (relbias_attn.cu)
// and the kernels.  Not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace relbias {

// bf16 tcgen05 prefill (prefill_sm100.cu).
struct PrefillParams {
    const float* r;          // [B, T, Hq]
    const float* w;          // [Hq, R]
    __nv_bfloat16* o;        // [B, T, Hq, d]
    float* lse;              // [B, Hq, T] or nullptr
    int B, T, Hq, Hkv;
    int G;                   // Hq / Hkv
    int nslots;              // query heads per work item (2 when G is even, else 1)
    int HP;                  // G / nslots: head pairs per key/value head
    int window, R;
    int n_qt;                // ceil(T / 128)
    int q_off;               // position of query row 0 (a chunk after a cached prefix; 0 otherwise)
    int kv_T;                // rows of K/V (>= q_off + T)
    int total_items;         // n_qt * B * Hkv * HP
    int o_v8;                // 1: o is 32-byte aligned (rows are written with 32-byte stores)
    int contiguous;          // 1: each CTA takes a contiguous run of items, query tiles innermost
                             //    (sliding window: equal-cost items, the bias table is reused);
                             // 0: items dealt round-robin, heaviest query tiles first (causal)
    float scale_log2;        // scale * log2(e)
    float inv_scale;         // 1 / scale
    int temp_n0;             // > 1: logits of a row seeing n > temp_n0 keys are scaled by ln n / ln temp_n0
    float inv_log_n0;        // 1 / ln(temp_n0)
    // Shared-bank form (curves != nullptr): each row's bias curve, padded rows of
    // curve_stride floats written by launch_bank_rows; r and w are then unused.
    const float* curves;
    int curve_stride;
    // Paged chunks (paged != 0): K/V live in a page pool [num_pages, page_size, Hkv, d],
    // sequence b's logical block k in page block_table[b * max_pages + k]; sequence b's
    // chunk has q_lens[b] rows (<= T) at positions q_offs[b] ... (both on the device).
    int paged;
    const int* block_table;
    const int* q_offs;
    const int* q_lens;
    int page_size, max_pages, num_pages;
};
int prefill_bf16_table_copies(int d, int R);   // 0 if R does not fit shared memory
// Shared-bank curves of every prefill row: [B, T, Hq] rows of prefill_bank_curve_stride(R)
// floats (see bank_rows_kernel in prefill_sm100.cu).
int prefill_bank_curve_stride(int R);
cudaError_t launch_bank_rows(const float* rs, const float* proj, float* curves, int B, int T, int Hq, int q_off, int C,
                             int proj_heads, int R, cudaStream_t stream);
int prefill_bf16_smem_bytes(int d, int R, int nc);
cudaError_t launch_prefill_bf16_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                      const PrefillParams& p, int d, int grid, cudaStream_t stream);

// fp32 SIMT prefill (prefill_fp32.cu).  C == 0: rank-1 bias, r [B, T, Hq] and w [Hq, R].
// C >= 1: shared-bank bias, r [B, T, Hq, C] coefficients and w [proj_heads, C, R] curves
// (proj_heads 1: one bank for all heads; Hq: a bank per head).
cudaError_t launch_prefill_fp32(const float* q, const float* k, const float* v, const float* r, const float* w,
                                float* o, float* lse, int B, int T, int q_off, int kv_T, int Hq, int Hkv, int d,
                                int window, int R, float scale, int temp_n0, int C, int proj_heads,
                                cudaStream_t stream);
constexpr int kMaxBankC = 16;   // functions in a shared bank

// Backward pass on the tcgen05 tensor cores (backward_sm100.cu), bf16 inputs, d in {64, 128}.
// Scheduling, r, w, R, window, scale and temperature come in a PrefillParams (nslots = 1,
// HP = G; for the dK/dV kernel total_items counts (sequence, kv head, key tile)).
struct BwdTcParams {
    const __nv_bfloat16* o;     // [B, T, Hq, d] forward output
    const __nv_bfloat16* dout;  // [B, T, Hq, d]
    const float* lse;           // [B, Hq, T] forward log-sum-exp
    float* dvec;                // [B, Hq, T] D_i = dout_i . o_i (written by bwd_dvec_kernel)
    float* dq;                  // [B, T, Hq, d]
    float* dr;                  // [B, T, Hq] (nullptr in the bank form)
    float* dk;                  // [B, T, Hkv, d]
    float* dv;                  // [B, T, Hkv, d]
    float* dw;                  // [Hq, R], zeroed by the caller, accumulated atomically
    float scale;
    // Shared-bank form (curves != nullptr): the bias of row (b, i, h) at distance d is
    // curves[row * curve_stride + pad + d] (the padded layout of launch_bank_rows), and
    // the dQ kernel writes dL/dcurve, tau_i * dl(i, i-d), to dcv in the same layout
    // (zeroed by the caller) in place of dr and dw.
    const float* curves;
    float* dcv;
    int curve_stride;
};
bool backward_tc_supported(int d, int R);
bool backward_bank_tc_supported(int d);
// dL/drs[row, c] = sum_d dcv[row, d] proj[hp, c, d] and dL/dproj[hp, c, d] += sum over
// the rows of head group hp of rs[row, c] dcv[row, d] (dproj zeroed by the caller).
cudaError_t launch_bank_grads(const float* rs, const float* proj, const float* dcv, float* drs, float* dproj, int B,
                              int T, int Hq, int C, int proj_heads, int R, int S, cudaStream_t stream);
cudaError_t launch_backward_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const PrefillParams& p_dq, const PrefillParams& p_dkv,
                                  const BwdTcParams& bp, int d, int grid, cudaStream_t stream);

// Backward pass on CUDA cores (backward_fp32.cu): dq [B,T,Hq,d], dk/dv [B,T,Hkv,d], dr
// [B,T,Hq], dw [Hq,R] (zeroed here, then accumulated), all fp32; q, k, v, o, dout in
// bf16 (bf16 == true) or fp32; dvec [B,Hq,T] scratch for D_i = dout_i . o_i.
cudaError_t launch_backward(bool bf16, int d, const void* q, const void* k, const void* v, const float* r,
                            const float* w, const void* o, const float* lse, const void* dout, float* dq, float* dk,
                            float* dv, float* dr, float* dw, float* dvec, int B, int T, int Hq, int Hkv, int window,
                            int R, float scale, int temp_n0, cudaStream_t stream);

// Per-(sequence, head) bias curves of the shared bank for one query row each
// (decode_sm100.cu): curves[bh, dist] = sum_c rs[bh, c] * proj[bh % Hq or 0, c, dist].
cudaError_t launch_bank_curves(const float* rs, const float* proj, float* curves, int BH, int Hq, int C,
                               int proj_heads, int R, cudaStream_t stream);

// bf16 split-KV decode + log-sum-exp combine (decode_sm100.cu).
struct DecodeParams {
    const __nv_bfloat16* q;  // [B, Hq, d]
    const float* r;          // [B, Hq], or nullptr: coefficient 1 (w then holds whole curves)
    const float* w;          // [Hq, R] distance tables (w_bstride 0), or [B, Hq, R] curves
    size_t w_bstride;        // elements between sequences' tables: 0, or Hq * R
    __nv_bfloat16* o;        // [B, Hq, d]
    float* lse;              // [B, Hq] or nullptr
    float* part;             // [B, Hq, nsplit, d + 4] workspace records
    int B, N, Hq, Hkv, G;
    int window, R;
    int key_lo;              // first attended cache row
    int nchunks;             // kChunk-key chunks in [key_lo, N)
    int nsplit;              // CTAs per (b, key/value head)
    int chunks_per_split;
    float scale_log2;
    float inv_scale;
    // Paged, variable-length caches (decode_splitkv_kernel<true>): the cache is a pool
    // of pages [num_pages, page_size, Hkv, d]; sequence b's logical block k lives in
    // page block_table[b * max_pages + k]; its length is seq_lens[b] (<= N, the bound
    // the splits are planned for).  key_lo / nchunks are then per sequence.
    const int* block_table;
    const int* seq_lens;
    int page_size, max_pages, num_pages;
    int temp_n0;             // > 1: per-sequence context-length temperature
    float inv_log_n0;
};
int decode_num_splits(int B, int Hkv, int N, int window, int num_sms);
size_t decode_workspace_bytes(int B, int Hq, int nsplit, int d);
cudaError_t launch_decode_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                               cudaStream_t stream);
// tk/tv: tensor maps over the page pool (make_map with B = num_pages, T = page_size).
cudaError_t launch_decode_paged_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                                     cudaStream_t stream);

}  // namespace relbias
