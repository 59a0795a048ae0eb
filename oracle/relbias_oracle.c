/*
 * relbias_oracle.c -- fp64 CPU oracle for causal attention with a learned,
 * input-dependent relative-position bias.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA library is checked against.  Only the test suite, the package's smoke
 * check and the benchmark's CPU-baseline / reference leg may load it.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * What one output row computes, in the order the pages give it:
 *
 *   "Thinking Machines dropped RoPE" (wpnews.pro essay), the five-step recipe
 *   under "how this is reflected in the maths", and the NumPy function
 *   relative_position_bias printed right after it:
 *     step 1  per-token, per-head coefficients rs[i,h,0..C-1]  (an input here:
 *             the r_proj projection runs upstream)
 *     step 2  the token's curve over distance: curve[d] = sum_c rs[c]*proj[c,d]
 *     step 3  read the curve at the query-key distance i-j (one gather, with
 *             the index clipped into [0, R-1])
 *     step 4  hard zero where i-j < 0 or i-j >= R
 *     step 5  add the bias to the scaled dot-product logit before the softmax
 *   With C = 1 and a table per head this is b[h,i,j] = r[i,h] * w[h,i-j]
 *   (the per-token, per-head feature "modulated with distance" of the
 *   banandre.com deep dive, section "No RoPE? No Problem?").
 *
 *   "Learned Relative-Position Bias" (codewithdark concepts page), section
 *   "Standard Relative Bias (T5-style)": the logit is q.k/sqrt(d) + b; the
 *   scale is a parameter here (the essay's "logit scaling" paragraph lost its
 *   symbols; callers pass 1/sqrt(d) for the T5 form).
 *
 *   Attended set (causal mask, plus the 512-token sliding window of local
 *   layers from the concepts page, "Hybrid Attention Interaction"):
 *     A_i = { j : 0 <= i-j  and  (window <= 0 or i-j < window) }.
 *
 *   Context-length temperature (optional; the essay, section "The temperature
 *   scale is dependent on context length"): global layers multiply both the
 *   query (hence the content logit) and the position bias by tau(n), n = the
 *   number of keys the query can see, flat up to 128k tokens and growing
 *   logarithmically beyond.  The page's formula lost its symbols; the reading
 *   taken is the log-n scaling it names, tau(n) = max(1, ln n / ln n0), with
 *   the break point n0 a parameter (131072 on the page; n0 <= 0 turns the
 *   temperature off).  So the logit is tau(|A_i|) * (scale*q.k + bias).
 *
 *   Softmax in fp64: m = max logit, O_i = sum_j exp(l_j - m) v_j / sum exp(l - m),
 *   LSE_i = m + log(sum_j exp(l_j - m)).
 *
 * Every arithmetic step is in double precision; inputs arrive as float32
 * arrays (bf16 values are exact in float32) and are widened element by element.
 * Rows are independent and run in parallel with OpenMP; nothing inside a row
 * is blocked, fused or reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One output row.
 *   q      [d]            query vector of row i, head h
 *   rs     [C]            coefficients of (i, h)
 *   proj   [C, R]         distance table(s) seen by head h, row-major
 *   k, v   key / value row j at k + j*kv_stride (d contiguous values each)
 *   i      query position; keys 0..i are causally visible
 *   out    [d]            attention output (fp64)
 *   lse    [1]            log-sum-exp of the logits (fp64)
 * Returns 0, or -1 if scratch memory could not be allocated.
 */
static int oracle_row(const float* q, const float* rs, const float* proj, int C,
                      const float* k, const float* v, int64_t kv_stride,
                      int64_t i, int64_t window, int64_t R, double scale, int64_t temp_n0, int d,
                      double* out, double* lse)
{
    /* step 2: the token's personal curve over distances 0..R-1 */
    double* curve = NULL;
    if (R > 0) {
        curve = (double*)malloc((size_t)R * sizeof(double));
        if (!curve) return -1;
        for (int64_t dd = 0; dd < R; ++dd) {
            double acc = 0.0;
            for (int c = 0; c < C; ++c)
                acc += (double)rs[c] * (double)proj[(int64_t)c * R + dd];
            curve[dd] = acc;
        }
    }

    int64_t j_lo = 0;
    if (window > 0 && i - window + 1 > 0) j_lo = i - window + 1;
    int64_t n = i - j_lo + 1;
    /* context-length temperature: tau(n) = max(1, ln n / ln n0) */
    double tau = 1.0;
    if (temp_n0 > 1 && n > temp_n0) tau = log((double)n) / log((double)temp_n0);
    double* logit = (double*)malloc((size_t)n * sizeof(double));
    if (!logit) { free(curve); return -1; }

    double m = -INFINITY;
    for (int64_t j = j_lo; j <= i; ++j) {
        const float* kj = k + j * kv_stride;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += (double)q[c] * (double)kj[c];
        /* steps 3-4: gather at the distance, zero outside [0, R) */
        int64_t dist = i - j;
        double bias = 0.0;
        if (R > 0) {
            int64_t idx = dist < 0 ? 0 : (dist > R - 1 ? R - 1 : dist);
            bias = (dist < 0 || dist >= R) ? 0.0 : curve[idx];
        }
        /* step 5: add to the scaled logit (then the temperature, if any) */
        double l = tau * (scale * dot + bias);
        logit[j - j_lo] = l;
        if (l > m) m = l;
    }

    double den = 0.0;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int64_t j = j_lo; j <= i; ++j) {
        double p = exp(logit[j - j_lo] - m);
        den += p;
        const float* vj = v + j * kv_stride;
        for (int c = 0; c < d; ++c) out[c] += p * (double)vj[c];
    }
    for (int c = 0; c < d; ++c) out[c] /= den;
    *lse = m + log(den);

    free(logit);
    free(curve);
    return 0;
}

/* Many rows of a [B, T, Hkv, d] key/value layout.
 *
 *   q_rows [n, d]        query vector of each requested row
 *   rs_rows [n, C]       coefficients of each requested row
 *   proj   [Hp, C, R]    distance tables; head h uses table (Hp == 1 ? 0 : h)
 *   k, v   [B, T, Hkv, d]
 *   req    [n, 3]        (b, h, i) of each requested row
 *   Hq, Hkv              query heads and key/value heads; head h reads
 *                        key/value head h / (Hq / Hkv)
 *   temp_n0              temperature break point (<= 1: no temperature)
 *   o_out  [n, d], lse_out [n]
 * Returns 0 on success, -1 on a bad argument or allocation failure.
 */
int oracle_attn_rows(const float* q_rows, const float* rs_rows,
                     const float* proj, int Hp, int C,
                     const float* k, const float* v,
                     const int64_t* req, int64_t n,
                     int B, int64_t T, int Hq, int Hkv, int d,
                     int64_t window, int64_t R, double scale, int64_t temp_n0,
                     double* o_out, double* lse_out)
{
    if (n < 0 || B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || C <= 0 || R < 0)
        return -1;
    if (Hq % Hkv != 0 || !(Hp == 1 || Hp == Hq)) return -1;
    const int G = Hq / Hkv;
    int status = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n; ++u) {
        int64_t b = req[3 * u + 0], h = req[3 * u + 1], i = req[3 * u + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= T) {
#pragma omp atomic write
            status = -1;
            continue;
        }
        int64_t g = h / G;
        const float* kb = k + ((b * T) * Hkv + g) * (int64_t)d;
        const float* vb = v + ((b * T) * Hkv + g) * (int64_t)d;
        const float* table = proj + (Hp == 1 ? 0 : h) * (int64_t)C * R;
        int rc = oracle_row(q_rows + u * (int64_t)d, rs_rows + u * (int64_t)C, table, C,
                            kb, vb, (int64_t)Hkv * d, i, window, R, scale, temp_n0, d,
                            o_out + u * (int64_t)d, lse_out + u);
        if (rc != 0) {
#pragma omp atomic write
            status = -1;
        }
    }
    return status;
}

/* Gradients of the whole forward pass (the backward pass), in fp64.
 *
 * Loss-independent form: given dout = dL/dO for every output row, return dL/d of
 * every input.  For one row (b, h, i) with logits l_j = tau * (scale * q.k_j +
 * bias_j) over j in A_i, p_j = exp(l_j - LSE_i) and O_i = sum_j p_j v_j (the
 * forward above), the chain rule gives, step by step:
 *   dp_j   = dout_i . v_j                       (O is linear in p)
 *   D_i    = sum_j p_j dp_j  (= dout_i . O_i)
 *   dl_j   = p_j (dp_j - D_i)                   (softmax Jacobian)
 *   dq_i  += dl_j * tau * scale * k_j           (l_j through the dot product)
 *   dk_j  += dl_j * tau * scale * q_i
 *   dv_j  += p_j * dout_i
 *   dbias  = dl_j * tau, for 0 <= i-j < R       (step 5: the bias adds to the logit)
 *   drs[i,c]        += dbias * proj[c, i-j]     (step 2: curve = sum_c rs[c] proj[c, .])
 *   dproj[h', c, i-j] += dbias * rs[i,c]
 * Key/value gradients sum over the query heads of their group; a bank shared by
 * all heads (Hp == 1) sums over every head.  tau depends only on the number of
 * visible keys, not on any input, so it is a constant factor here.
 *
 *   q, dout [B, T, Hq, d]; k, v [B, T, Hkv, d]; rs [B, T, Hq, C]; proj [Hp, C, R]
 *   dq [B, T, Hq, d]; dk, dv [B, T, Hkv, d]; drs [B, T, Hq, C]; dproj [Hp, C, R]
 *   (all outputs fp64, overwritten).
 * Heads run in parallel (OpenMP), each into private key/value and table
 * buffers that are summed afterwards in a fixed order.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int oracle_attn_bwd(const float* q, const float* k, const float* v, const float* rs,
                    const float* proj, int Hp, int C, const float* dout,
                    int B, int64_t T, int Hq, int Hkv, int d,
                    int64_t window, int64_t R, double scale, int64_t temp_n0,
                    double* dq, double* dk, double* dv, double* drs, double* dproj)
{
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || C <= 0 || R < 0) return -1;
    if (Hq % Hkv != 0 || !(Hp == 1 || Hp == Hq)) return -1;
    const int G = Hq / Hkv;
    const int64_t kv_stride = (int64_t)Hkv * d;
    memset(dq, 0, sizeof(double) * (size_t)B * T * Hq * d);
    memset(dk, 0, sizeof(double) * (size_t)B * T * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * T * Hkv * d);
    memset(drs, 0, sizeof(double) * (size_t)B * T * Hq * C);
    memset(dproj, 0, sizeof(double) * (size_t)Hp * C * (R > 0 ? R : 0));

    /* private per-head buffers: dk/dv contributions [Hq][T][d], table grads [Hq][C][R] */
    double* dk_h = (double*)calloc((size_t)Hq * T * d, sizeof(double));
    double* dv_h = (double*)calloc((size_t)Hq * T * d, sizeof(double));
    double* dp_h = (double*)calloc((size_t)Hq * C * (R > 0 ? R : 1), sizeof(double));
    if (!dk_h || !dv_h || !dp_h) { free(dk_h); free(dv_h); free(dp_h); return -1; }
    int status = 0;

    for (int b = 0; b < B; ++b) {
        memset(dk_h, 0, sizeof(double) * (size_t)Hq * T * d);
        memset(dv_h, 0, sizeof(double) * (size_t)Hq * T * d);
#pragma omp parallel for schedule(dynamic, 1)
        for (int h = 0; h < Hq; ++h) {
            const int64_t g = h / G;
            const float* table = proj + (Hp == 1 ? 0 : h) * (int64_t)C * R;
            double* logit = (double*)malloc((size_t)T * sizeof(double));
            double* curve = (double*)malloc((size_t)(R > 0 ? R : 1) * sizeof(double));
            double* o_row = (double*)malloc((size_t)d * sizeof(double));
            if (!logit || !curve || !o_row) {
                free(logit); free(curve); free(o_row);
#pragma omp atomic write
                status = -1;
                continue;
            }
            for (int64_t i = 0; i < T; ++i) {
                const float* qi = q + ((b * T + i) * Hq + h) * (int64_t)d;
                const float* doi = dout + ((b * T + i) * Hq + h) * (int64_t)d;
                const float* rsi = rs + ((b * T + i) * Hq + h) * (int64_t)C;
                for (int64_t dd = 0; dd < R; ++dd) {
                    double acc = 0.0;
                    for (int c = 0; c < C; ++c) acc += (double)rsi[c] * (double)table[(int64_t)c * R + dd];
                    curve[dd] = acc;
                }
                int64_t j_lo = 0;
                if (window > 0 && i - window + 1 > 0) j_lo = i - window + 1;
                const int64_t n = i - j_lo + 1;
                double tau = 1.0;
                if (temp_n0 > 1 && n > temp_n0) tau = log((double)n) / log((double)temp_n0);
                /* forward recomputed: logits, max, sum, O */
                double m = -INFINITY;
                for (int64_t j = j_lo; j <= i; ++j) {
                    const float* kj = k + (b * T + j) * kv_stride + g * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += (double)qi[c] * (double)kj[c];
                    const int64_t dist = i - j;
                    const double bias = (dist < R) ? curve[dist] : 0.0;
                    logit[j] = tau * (scale * dot + bias);
                    if (logit[j] > m) m = logit[j];
                }
                double den = 0.0;
                for (int64_t j = j_lo; j <= i; ++j) den += exp(logit[j] - m);
                const double lse = m + log(den);
                for (int c = 0; c < d; ++c) o_row[c] = 0.0;
                for (int64_t j = j_lo; j <= i; ++j) {
                    const double p = exp(logit[j] - lse);
                    const float* vj = v + (b * T + j) * kv_stride + g * d;
                    for (int c = 0; c < d; ++c) o_row[c] += p * (double)vj[c];
                }
                double D = 0.0;
                for (int c = 0; c < d; ++c) D += (double)doi[c] * o_row[c];
                /* backward through softmax, dot products and bias */
                double* dqi = dq + ((b * T + i) * Hq + h) * (int64_t)d;
                double* drsi = drs + ((b * T + i) * Hq + h) * (int64_t)C;
                for (int64_t j = j_lo; j <= i; ++j) {
                    const float* kj = k + (b * T + j) * kv_stride + g * d;
                    const float* vj = v + (b * T + j) * kv_stride + g * d;
                    const double p = exp(logit[j] - lse);
                    double dp = 0.0;
                    for (int c = 0; c < d; ++c) dp += (double)doi[c] * (double)vj[c];
                    const double dl = p * (dp - D);
                    double* dkj = dk_h + ((int64_t)h * T + j) * d;
                    double* dvj = dv_h + ((int64_t)h * T + j) * d;
                    for (int c = 0; c < d; ++c) {
                        dqi[c] += dl * tau * scale * (double)kj[c];
                        dkj[c] += dl * tau * scale * (double)qi[c];
                        dvj[c] += p * (double)doi[c];
                    }
                    const int64_t dist = i - j;
                    if (dist < R) {
                        const double dbias = dl * tau;
                        double* dph = dp_h + (int64_t)h * C * R;
                        for (int c = 0; c < C; ++c) {
                            drsi[c] += dbias * (double)table[(int64_t)c * R + dist];
                            dph[(int64_t)c * R + dist] += dbias * (double)rsi[c];
                        }
                    }
                }
            }
            free(logit); free(curve); free(o_row);
        }
        /* sum the heads of each group into the key/value gradients, in head order */
        for (int h = 0; h < Hq; ++h) {
            const int64_t g = h / G;
            for (int64_t j = 0; j < T; ++j)
                for (int c = 0; c < d; ++c) {
                    dk[((b * T + j) * Hkv + g) * d + c] += dk_h[((int64_t)h * T + j) * d + c];
                    dv[((b * T + j) * Hkv + g) * d + c] += dv_h[((int64_t)h * T + j) * d + c];
                }
        }
    }
    /* table gradients: per head, or summed over all heads for a shared bank */
    for (int h = 0; h < Hq; ++h) {
        double* dst = dproj + (Hp == 1 ? 0 : h) * (int64_t)C * R;
        for (int64_t x = 0; x < (int64_t)C * R; ++x) dst[x] += dp_h[(int64_t)h * C * R + x];
    }
    free(dk_h); free(dv_h); free(dp_h);
    return status;
}

/* Threads the OpenMP loop above would use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
