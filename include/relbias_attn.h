/*
 * relbias_attn.h -- C ABI of librelbias_attn.so: causal grouped-query attention
 * with an additive, input-dependent, learned relative-position bias, forward
 * pass, for NVIDIA B200 (sm_100a).
 *
 * The operation (per batch b, query head h, query position i):
 *
 *   logit[j] = scale * <q[b,i,h,:], k[b,j,g,:]> + bias[j]          g = h / (Hq/Hkv)
 *   bias[j]  = r[b,i,h] * w[h, i-j]   if 0 <= i-j < R,   else 0
 *   j ranges over A_i = { j : 0 <= i-j  and  (window <= 0 or i-j < window) }
 *   o[b,i,h,:] = sum_j softmax(logit)[j] * v[b,j,g,:]
 *   lse[b,h,i] = log sum_j exp(logit[j])
 *
 * Sources.  The bias is added to the scaled logits before the softmax, next to
 * the causal mask, and is exactly zero at distances of R or more ("Thinking
 * Machines dropped RoPE", wpnews.pro essay: the five-step recipe, steps 3-5,
 * and the relative_position_bias listing).  The per-token, per-head feature r
 * comes from a fourth projection and is modulated by distance (banandre.com
 * Inkling deep dive, "No RoPE? No Problem?"); here it multiplies a learned
 * per-head distance table w.  Local layers use window = 512 and R = 512; global
 * layers use the full causal mask with R = 1024 and content-only attention
 * beyond ("Learned Relative-Position Bias", codewithdark concepts page, "Key
 * Components" and "Hybrid Attention Interaction").  The scaled-logit form is the
 * T5-style formula on that page ("Standard Relative Bias (T5-style)"); the scale
 * is a parameter because the essay's logit-scaling sentence lost its symbols.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     densely packed, and at least 16-byte aligned.  The library allocates no
 *     device memory and keeps no per-call state.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise.  Arguments are checked on the host before
 *     any launch; a rejected call launches nothing.
 *   - Return value: RELBIAS_OK (0) or a negative RELBIAS_ERR_* code.  The calls
 *     never abort the process.  relbias_last_error() describes the last failure
 *     on the calling thread.
 *   - Kernels bound every wait on an asynchronous copy or tensor-core result (2 s
 *     by default, see relbias_set_wait_limit_ns).  A wait that runs out records
 *     RELBIAS_STATUS_TIMEOUT in a device-side status word; the kernel then waits
 *     for the copies and MMAs it has itself issued, releases its tensor memory and
 *     returns, leaving the context usable.  relbias_device_status() reads the word.
 */
#ifndef RELBIAS_ATTN_H
#define RELBIAS_ATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define RELBIAS_API __attribute__((visibility("default")))
#else
#define RELBIAS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define RELBIAS_OK               0
#define RELBIAS_ERR_ARG         -1  /* null pointer, bad shape, misalignment, bad scale   */
#define RELBIAS_ERR_UNSUPPORTED -2  /* valid request the library or device cannot serve   */
#define RELBIAS_ERR_CUDA        -3  /* a CUDA runtime call or kernel launch failed        */

/* Bytes of the static scratch behind relbias_attn_decode_noalloc (8 MiB). */
#define RELBIAS_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Bits of the device-side status word (relbias_device_status). */
#define RELBIAS_STATUS_TIMEOUT   1u /* a bounded wait inside a kernel ran out             */
#define RELBIAS_STATUS_BAD_LENGTH 2u /* a device-side sequence length or page index was out of range */

/* Element type of q, k, v and o.  r, w and lse are always fp32. */
typedef enum {
    RELBIAS_BF16 = 0,   /* bf16 storage, fp32 accumulation (tensor cores)  */
    RELBIAS_FP32 = 1    /* fp32 storage and arithmetic (CUDA cores)        */
} relbias_dtype;

/*
 * Prefill: every query row of every sequence attends causally to its own
 * sequence.
 *
 *   q    [B, T, Hq,  d]   dtype
 *   k    [B, T, Hkv, d]   dtype
 *   v    [B, T, Hkv, d]   dtype
 *   r    [B, T, Hq]       fp32   per-token, per-head bias feature
 *   w    [Hq, R]          fp32   per-head distance table (may be NULL if R == 0)
 *   o    [B, T, Hq,  d]   dtype  output, written for every row
 *   lse  [B, Hq, T]       fp32   natural-log LSE of each row; may be NULL
 *
 *   B, T >= 1; Hq, Hkv >= 1 with Hq % Hkv == 0; window <= 0 means full causal;
 *   R >= 0 (R == 0: no bias); scale > 0 and finite.
 *   temp_n0: context-length temperature of global layers (the essay, "The
 *   temperature scale is dependent on context length": queries and position bias
 *   are both scaled by a factor that is flat up to 128k tokens and grows
 *   logarithmically beyond; the page's formula is garbled).  Reading taken: a
 *   row that sees n keys (n = i+1, or min(i+1, window)) has its whole logit
 *   multiplied by max(1, ln n / ln temp_n0).  temp_n0 <= 1 turns it off; the
 *   page's break point is 131072.  The LSE is that of the scaled logits.
 *   RELBIAS_BF16 needs a B200-class GPU (compute capability 10.0), d in {64, 128}
 *   and R <= 2048; RELBIAS_FP32 takes d in {32, 64, 128, 256} on any GPU.
 *   The output buffers must not overlap the inputs.
 */
RELBIAS_API int relbias_attn_fwd(const void* q, const void* k, const void* v,
                     const float* r, const float* w,
                     void* o, float* lse,
                     int B, int T, int Hq, int Hkv, int d,
                     int window, int R, float scale, int temp_n0,
                     int dtype, void* stream);

/*
 * Chunked prefill: T new query rows at positions q_off ... q_off+T-1 of each
 * sequence, against a key/value cache of kv_T >= q_off+T rows that already holds
 * the prefix (rows 0 ... q_off-1) and the chunk's own keys and values (rows
 * q_off ... q_off+T-1); rows at or past q_off+T are never read for a visible key.
 * A serving engine processes a long prompt this way, chunk by chunk against a
 * growing cache.  Same computation as
 * relbias_attn_fwd for those rows: the causal mask, the window and the bias use the
 * positions q_off + i; relbias_attn_fwd is the case q_off = 0, kv_T = T.
 *
 *   q [B, T, Hq, d], r [B, T, Hq], o [B, T, Hq, d], lse [B, Hq, T]: the chunk's rows
 *   k, v [B, kv_T, Hkv, d]: the cache
 *   q_off >= 0, q_off + T <= kv_T; other rules as for relbias_attn_fwd.
 */
RELBIAS_API int relbias_attn_fwd_chunk(const void* q, const void* k, const void* v,
                     const float* r, const float* w,
                     void* o, float* lse,
                     int B, int T, int q_off, int kv_T, int Hq, int Hkv, int d,
                     int window, int R, float scale, int temp_n0,
                     int dtype, void* stream);

/*
 * Chunked prefill against a paged, variable-length cache: the paged KV cache and
 * variable sequence lengths the essay ("Thinking Machines dropped RoPE", closing
 * section on kernel cost) lists among what a production attention kernel covers.
 * Sequence b's chunk has q_lens[b] rows (0 <= q_lens[b] <= T) at positions
 * q_offs[b] ... q_offs[b]+q_lens[b]-1; its keys and values, the prefix and the
 * chunk's own rows, are cache rows 0 ... q_offs[b]+q_lens[b]-1, where cache row t of
 * sequence b is row t % page_size of page block_table[b][t / page_size].  Same
 * computation as relbias_attn_fwd_chunk for each sequence.
 *
 *   q, o     [B, T, Hq, d]          bf16   rows >= q_lens[b] are neither read for a
 *                                          result nor written (o, lse keep their contents)
 *   r        [B, T, Hq]             fp32
 *   lse      [B, Hq, T]             fp32   may be NULL
 *   k_pages, v_pages [num_pages, page_size, Hkv, d]   bf16, the page pool
 *   block_table      [B, max_pages]  int32  (device)
 *   q_offs, q_lens   [B]             int32  (device, read by the kernel)
 *   page_size a positive multiple of 64; bf16 only, d in {64, 128}, R <= 2048.
 *   An offset or length out of range (q_offs[b] + q_lens[b] > max_pages * page_size,
 *   or q_lens[b] > T) is clamped into range, and a page index outside the pool reads
 *   zeros; either sets RELBIAS_STATUS_BAD_LENGTH.  Cache rows past a sequence's end
 *   may hold anything (they are never attended, and their values never reach a
 *   product).
 */
RELBIAS_API int relbias_attn_fwd_chunk_paged(const void* q, const void* k_pages, const void* v_pages,
                        const int* block_table, const int* q_offs, const int* q_lens,
                        const float* r, const float* w,
                        void* o, float* lse,
                        int B, int T, int num_pages, int page_size, int max_pages,
                        int Hq, int Hkv, int d,
                        int window, int R, float scale, int temp_n0,
                        int dtype, void* stream);

/*
 * Decode: one new query per sequence at position n_ctx-1 against a key/value
 * cache of n_ctx rows whose last row already holds that query's own key and
 * value (the 1,048,576-token context of the archdiff.com model card, "Context").
 * The keys are split over many CTAs; each writes a partial (max, sum, output)
 * into `workspace`, and a second kernel merges the partials by log-sum-exp.
 *
 *   q        [B, Hq, d]          bf16
 *   k_cache  [B, n_ctx, Hkv, d]  bf16
 *   v_cache  [B, n_ctx, Hkv, d]  bf16
 *   r        [B, Hq]             fp32   the new token's bias feature
 *   w        [Hq, R]             fp32   (may be NULL if R == 0)
 *   o        [B, Hq, d]          bf16
 *   lse      [B, Hq]             fp32   may be NULL
 *   workspace, ws_bytes: caller-owned device scratch of at least
 *            relbias_attn_decode_workspace_size(...) bytes, 16-byte aligned; its
 *            contents on entry do not matter and are overwritten.
 *
 *   dtype must be RELBIAS_BF16; d == 128; Hq/Hkv <= 8; n_ctx >= 1; other
 *   argument rules as for relbias_attn_fwd (the query sees n = n_ctx keys, or
 *   min(n_ctx, window), for the temperature).
 */
RELBIAS_API size_t relbias_attn_decode_workspace_size(int B, int Hq, int Hkv, int n_ctx, int d,
                                          int window);

RELBIAS_API int relbias_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                        const float* r, const float* w,
                        void* o, float* lse,
                        int B, int n_ctx, int Hq, int Hkv, int d,
                        int window, int R, float scale, int temp_n0,
                        int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Decode that allocates nothing, for callers that cannot allocate device memory
 * (e.g. a plugin inside an inference runtime that owns all device allocations, or
 * a serving loop that must not call cudaMalloc/cudaFree between steps).  The
 * paper has no counterpart; this is a property of the library, not of the method.
 *
 * Same arguments, results and rules as relbias_attn_decode, without the
 * workspace: the split partials go to a scratch array of
 * RELBIAS_DECODE_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU
 * that loads the library holds until the process exits.
 *   - A call whose partials need more than that (see
 *     relbias_attn_decode_workspace_size) is rejected with RELBIAS_ERR_UNSUPPORTED
 *     and launches nothing.
 *   - Argument errors are reported exactly as relbias_attn_decode reports them,
 *     before anything else happens.
 *   - Every call looks up the scratch's device address (cudaGetSymbolAddress, a
 *     host-side query that allocates nothing) in the device and context current
 *     at the call, so the address stays right after cudaDeviceReset or a context
 *     switch.  The first call on a device may load the library's device image
 *     there; make that first call before any stream capture.
 *   - All calls on a device share the one scratch array, which keeps the last
 *     call's contents (every value a call reads it writes first).  Calls that
 *     overlap on the GPU -- on different streams without ordering between them --
 *     race on it and must not be issued.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 */
RELBIAS_API int relbias_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                        const float* r, const float* w,
                        void* o, float* lse,
                        int B, int n_ctx, int Hq, int Hkv, int d,
                        int window, int R, float scale, int temp_n0,
                        int dtype, void* stream);

/*
 * Decode against a paged, variable-length KV cache: the "paged KV, variable seq
 * len" a production attention kernel must cover (the essay "Thinking Machines
 * dropped RoPE", closing section on kernel cost).  Same computation as
 * relbias_attn_decode for each sequence b, whose query sits at position
 * seq_lens[b]-1 and whose cache rows live in pages:
 *
 *   k_pages, v_pages [num_pages, page_size, Hkv, d]  bf16   the page pool
 *   block_table      [B, max_pages]                 int32  page of each logical
 *                    block of page_size rows (row t of sequence b is row
 *                    t % page_size of page block_table[b][t / page_size])
 *   seq_lens         [B]                            int32  rows of each sequence
 *                    (device memory, read by the kernel; 1 <= seq_lens[b] <= max_seq_len)
 *   q [B, Hq, d], r [B, Hq], w [Hq, R], o [B, Hq, d], lse [B, Hq]: as for decode.
 *
 *   page_size: a positive multiple of 32.  max_pages * page_size >= max_seq_len.
 *   max_seq_len bounds every seq_lens[b] and plans the key splits;
 *   workspace: at least relbias_attn_decode_paged_workspace_size(...) bytes.
 *   A length outside [1, max_seq_len] is clamped into it, and a page index outside
 *   the pool reads zeros; either sets RELBIAS_STATUS_BAD_LENGTH in the device
 *   status word (relbias_device_status).  Other rules as for relbias_attn_decode.
 */
RELBIAS_API size_t relbias_attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_seq_len, int d,
                                                int window);

RELBIAS_API int relbias_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                        const int* block_table, const int* seq_lens,
                        const float* r, const float* w,
                        void* o, float* lse,
                        int B, int num_pages, int page_size, int max_pages, int max_seq_len,
                        int Hq, int Hkv, int d,
                        int window, int R, float scale, int temp_n0,
                        int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Shared-bank bias.  The essay's recipe ("Thinking Machines dropped RoPE", steps
 * 1-2) keeps a small bank of C learned functions of distance, shared by the
 * heads of a layer, and gives every token and head C coefficients from a
 * projection; the bias is the coefficients times the bank:
 *
 *   bias[j] = sum_c rs[b,i,h,c] * proj[h', c, i-j]   if 0 <= i-j < R, else 0
 *
 * with h' = 0 (one bank for all heads, proj_heads = 1) or h' = h (a bank per
 * head, proj_heads = Hq).  The rank-1 form of relbias_attn_fwd is the case
 * C = 1, proj_heads = Hq.  1 <= C <= 16.
 *
 * relbias_attn_fwd_bank: prefill.
 *   rs   [B, T, Hq, C]          fp32
 *   proj [proj_heads, C, R]     fp32   (may be NULL if R == 0)
 *   workspace, ws_bytes: RELBIAS_BF16 only (NULL and 0 for RELBIAS_FP32): caller-owned
 *        device scratch of at least relbias_attn_fwd_bank_workspace_size(...) bytes,
 *        32-byte aligned.  The bf16 path first writes every row's curve
 *        sum_c rs[b,i,h,c] * proj[h', c, :] there (one padded fp32 row of R + 14..21
 *        floats per (b, i, h)), then the tensor-core kernel reads each row's curve in
 *        place of the rank-1 r * w; the fp32 path evaluates the sum per key itself.
 *   other arguments as for relbias_attn_fwd.
 *
 * relbias_attn_decode_bank: decode as relbias_attn_decode, with
 *   rs   [B, Hq, C]             fp32   the new token's coefficients
 *   proj [proj_heads, C, R]     fp32
 * The call first writes each (sequence, head) curve sum_c rs[c] * proj[c, :]
 * (B * Hq * R floats) into the front of `workspace`; the split-KV kernels then
 * read those curves.  ws_bytes must be at least
 * relbias_attn_decode_bank_workspace_size(...).
 */
RELBIAS_API size_t relbias_attn_fwd_bank_workspace_size(int B, int T, int Hq, int R, int dtype);

RELBIAS_API int relbias_attn_fwd_bank(const void* q, const void* k, const void* v,
                        const float* rs, const float* proj,
                        void* o, float* lse,
                        int B, int T, int Hq, int Hkv, int d, int C, int proj_heads,
                        int window, int R, float scale, int temp_n0,
                        int dtype, void* workspace, size_t ws_bytes, void* stream);
RELBIAS_API size_t relbias_attn_decode_bank_workspace_size(int B, int Hq, int Hkv, int n_ctx, int d,
                                          int window, int R);
RELBIAS_API int relbias_attn_decode_bank(const void* q, const void* k_cache, const void* v_cache,
                     const float* rs, const float* proj,
                     void* o, float* lse,
                     int B, int n_ctx, int Hq, int Hkv, int d, int C, int proj_heads,
                     int window, int R, float scale, int temp_n0,
                     int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward pass of relbias_attn_fwd (rank-1 bias): given dout = dL/dO, the
 * gradients of every input.  The pages train this model but print no backward;
 * these are the derivatives of the forward definition above.  With logits
 * l_j = tau_i * (scale * q_i.k_j + bias_ij), p_j = exp(l_j - lse_i) and
 * D_i = dout_i . o_i:
 *   dl_j = p_j * (dout_i . v_j - D_i)
 *   dq_i = tau_i * scale * sum_j dl_j k_j     dk_j = sum over (h, i) of tau_i * scale * dl_j q_i
 *   dv_j = sum over (h, i) of p_j dout_i      dr_i = sum_j tau_i dl_j w[h, i-j]
 *   dw[h, d] = sum_i tau_i dl_(i, i-d) r_i    (bias terms only where 0 <= i-j < R)
 *
 *   q, o, dout [B, T, Hq, d]  dtype     k, v [B, T, Hkv, d]  dtype
 *   r [B, T, Hq], w [Hq, R]   fp32      lse [B, Hq, T] fp32: the forward's log-sum-exp
 *   dq [B, T, Hq, d], dk and dv [B, T, Hkv, d], dr [B, T, Hq], dw [Hq, R]: fp32
 *     outputs, overwritten (dw may be NULL if R == 0)
 *   workspace: at least relbias_attn_bwd_workspace_size(B, T, Hq) bytes of
 *     caller-owned device scratch (D_i per row), 16-byte aligned.
 * o and lse must be the forward's outputs for the same inputs.  dtype
 * RELBIAS_BF16 or RELBIAS_FP32.  bf16 with d in {64, 128} on sm_100 runs on the
 * tensor cores (bf16 products of the recomputed P and dS, fp32 accumulation; dr and
 * dw are summed with fp32 atomics, so dw is not bitwise repeatable); fp32 and other
 * head sizes run in fp32 on CUDA cores.  d in {32, 64, 128, 256}; R <= 32768; other
 * rules as for relbias_attn_fwd.
 */
RELBIAS_API size_t relbias_attn_bwd_workspace_size(int B, int T, int Hq);
RELBIAS_API int relbias_attn_bwd(const void* q, const void* k, const void* v,
                     const float* r, const float* w,
                     const void* o, const float* lse, const void* dout,
                     float* dq, float* dk, float* dv, float* dr, float* dw,
                     int B, int T, int Hq, int Hkv, int d,
                     int window, int R, float scale, int temp_n0,
                     int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward pass of relbias_attn_fwd_bank (the shared-bank bias of the essay's
 * recipe steps 1-2, curve_i = sum_c rs[b,i,h,c] * proj[h', c, :]).  With
 * dcurve_i[d] = tau_i * dl_(i, i-d) for 0 <= d < R (the gradient of row i's curve):
 *   drs[b,i,h,c]   = sum_d dcurve_i[d] * proj[h', c, d]
 *   dproj[h', c, d] = sum over the rows (b, i, h) that use bank h' of rs[b,i,h,c] * dcurve_i[d]
 * and dq, dk, dv as for relbias_attn_bwd.
 *
 *   rs [B, T, Hq, C], proj [proj_heads, C, R] fp32 (1 <= C <= 16, proj_heads 1 or Hq)
 *   drs [B, T, Hq, C], dproj [proj_heads, C, R]: fp32 outputs, overwritten
 *   workspace: at least relbias_attn_bwd_bank_workspace_size(B, T, Hq, R) bytes of
 *     caller-owned device scratch, 256-byte aligned: D_i per row, then each row's
 *     curve and its gradient (two padded fp32 rows of R + 14..21 floats per (b, i, h)).
 * Runs the curve kernel of relbias_attn_fwd_bank, the tensor-core dQ and dK/dV
 * kernels reading each row's curve in place of r * w (the dQ kernel writing
 * dcurve), then two reductions for drs and dproj.  dproj is summed with fp32 atomics
 * and is not bitwise repeatable.  RELBIAS_BF16 with d in {64, 128} on sm_100 only
 * (RELBIAS_ERR_UNSUPPORTED otherwise); 1 <= R <= 2048; B * T * Hq < 2^31; other
 * rules as for relbias_attn_bwd.
 */
RELBIAS_API size_t relbias_attn_bwd_bank_workspace_size(int B, int T, int Hq, int R);
RELBIAS_API int relbias_attn_bwd_bank(const void* q, const void* k, const void* v,
                     const float* rs, const float* proj,
                     const void* o, const float* lse, const void* dout,
                     float* dq, float* dk, float* dv, float* drs, float* dproj,
                     int B, int T, int Hq, int Hkv, int d, int C, int proj_heads,
                     int window, int R, float scale, int temp_n0,
                     int dtype, void* workspace, size_t ws_bytes, void* stream);

/* Description of the last failed call on this thread ("" if none).  The string
 * stays valid until the next library call on the same thread. */
RELBIAS_API const char* relbias_last_error(void);

/* Synchronises the current device, returns the device-side status bits
 * accumulated since the last reset (RELBIAS_STATUS_*) and, if reset != 0,
 * clears them.  Returns a negative RELBIAS_ERR_CUDA on a CUDA failure. */
RELBIAS_API int relbias_device_status(int reset);

/* Sets the bound on a single wait inside this library's kernels on the current
 * device, in nanoseconds (0 restores the default of 2 s).  Kernels launched after
 * the call use it.  A short bound makes waits run out on purpose, which tests the
 * failure path: the kernel records RELBIAS_STATUS_TIMEOUT, winds down and returns,
 * and its outputs are then undefined.  The waits by which a kernel drains its own
 * copies and MMAs before exiting always keep the 2 s bound.  The pages have no
 * counterpart; this is a property of the library.  Synchronous with respect to the
 * host (a cudaMemcpyToSymbol); returns RELBIAS_OK or RELBIAS_ERR_CUDA. */
RELBIAS_API int relbias_set_wait_limit_ns(unsigned long long ns);

/* Library version as major*10000 + minor*100 + patch. */
RELBIAS_API int relbias_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RELBIAS_ATTN_H */
