// decode_sm100.cu -- single-query decode against a long bf16 KV cache: split-KV
// streaming kernel plus a log-sum-exp combine kernel.
//
// One new query per sequence sits at position n_ctx-1; its own key and value are
// the cache's last row (the 1,048,576-token context of the archdiff.com model
// card).  Logit of cache row j: scale * q.k_j + (n_ctx-1-j < R ? r * w[h, n_ctx-1-j]
// : 0) -- the bias exists only for the last R rows, content-only beyond
// ("Learned Relative-Position Bias", codewithdark, "Hybrid Attention Interaction").
//
// Work: grid (split, key/value head g, sequence b).  A CTA streams a contiguous
// range of 32-key chunks of K and V once, through a 12-stage TMA ring, and serves
// all query heads of the group from each chunk (grouped-query attention).  Keys
// sit on the M dimension of m16n8k16 tensor-core MMAs and the (up to 8) query
// heads of the group on N:  S^T = K q^T,  O^T += V^T P^T.  P^T's accumulator
// fragments become B operands through a movmatrix transpose.  The four consumer
// warps take chunks round-robin and merge their running (max, sum, output) in
// shared memory; each CTA writes one partial per query head to the workspace.  The
// combine kernel merges the partials of a (b, h) with one warp.
//
// Paged, variable-length caches (PAGED = true): keys live in a pool of pages of
// page_size rows (a multiple of the 32-key chunk), sequence b's logical block k in
// page block_table[b][k], and each sequence has its own length seq_lens[b] -- the
// paged KV cache and variable sequence lengths the essay's kernel-cost section lists
// among what a production attention kernel covers.  Chunks then start at multiples
// of 32 (so each lies in one page), keys before a window's start are masked, and a
// split that lies past a short sequence's end writes an empty partial (max -inf),
// which the combine skips.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace relbias {

namespace {

constexpr int kD = 128;
constexpr int kChunk = 32;                 // keys per stage
constexpr int kConsumers = 4;
// Chunk li lives in stage li % kDStages and is consumed by warp li % kConsumers.
// kDStages is a multiple of kConsumers, so every stage is always consumed by the
// same warp, in order: no consumer can look at a stage's barrier while it is two
// phases behind (which a parity wait could not tell apart from "ready").
constexpr int kDStages = 12;
static_assert(kDStages % kConsumers == 0, "stage ownership must be per warp");
constexpr int kDThreads = (kConsumers + 1) * 32;
constexpr int kBoxBytes = kChunk * 128;    // 32 keys x 64 bf16
constexpr int kStageBytes = 4 * kBoxBytes; // K (2 boxes) + V (2 boxes)
constexpr int kMT = kChunk / 16;           // 16-key MMA tiles per chunk
constexpr int kRec = kD + 4;               // workspace record: O[128], m, l, pad

struct DecodeBars {
    uint64_t full[kDStages];
    uint64_t empty[kDStages];
    int abort_flag;
};

struct DecodeSmem {
    uint8_t stages[kDStages][kStageBytes];
    float warp_o[kConsumers][8][kD];
    float warp_m[kConsumers][8];
    float warp_l[kConsumers][8];
    DecodeBars bars;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Byte offset of 16-byte chunk (key row, head-dim column dcol) inside a stage half
// (K or V) loaded as two 64-column boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int key, int dcol) {
    const int box = dcol >> 6;
    const int ch = (dcol & 63) >> 3;
    return box * kBoxBytes + key * 128 + ((ch ^ (key & 7)) << 4);
}

template <bool PAGED>
__global__ void __launch_bounds__(kDThreads, 1)
    decode_splitkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    DecodeSmem* sm = reinterpret_cast<DecodeSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    DecodeBars* bars = &sm->bars;
    volatile int* abort_flag = &bars->abort_flag;

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // This sequence's length, first attended row, chunk grid and logit scale.
    int N = p.N, key_lo = p.key_lo, chunk0 = p.key_lo, nchunks = p.nchunks;
    float c1 = p.scale_log2;
    if constexpr (PAGED) {
        N = p.seq_lens[b];
        if (N < 1 || N > p.N) {
            // Outside [1, max_seq_len]: clamp (block-table reads stay in bounds) and report.
            if (threadIdx.x == 0) atomicOr(&g_status, kStatusBadLength);
            N = min(max(N, 1), p.N);
        }
        key_lo = p.window > 0 ? max(0, N - p.window) : 0;
        chunk0 = (key_lo / kChunk) * kChunk;
        nchunks = (N - chunk0 + kChunk - 1) / kChunk;
        const int nk = N - key_lo;   // keys the query sees, for the temperature
        if (p.temp_n0 > 1 && nk > p.temp_n0) c1 *= __logf(static_cast<float>(nk)) * p.inv_log_n0;
    }
    const int c_begin = split * p.chunks_per_split;
    const int c_end = min(nchunks, c_begin + p.chunks_per_split);
    const int nloc = max(0, c_end - c_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumers) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int issued = 0;   // chunks whose copies were issued
            for (int li = 0; li < nloc; ++li) {
                const int st = li % kDStages;
                const uint32_t ph = (li / kDStages) & 1;
                if (!mbar_wait(&bars->empty[st], ph ^ 1, abort_flag)) break;
                const int key0 = chunk0 + (c_begin + li) * kChunk;
                int row = key0, seq = b;   // token and sequence coordinates of the chunk
                if constexpr (PAGED) {
                    // key0 < N <= max_pages * page_size, so the table read is in bounds; a
                    // page index outside the pool reads zeros (TMA fills out-of-range rows).
                    seq = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + key0 / p.page_size);
                    row = key0 % p.page_size;
                    if (seq < 0 || seq >= p.num_pages) atomicOr(&g_status, kStatusBadLength);
                }
                mbar_arrive_expect_tx(&bars->full[st], kStageBytes);
                uint8_t* base = sm->stages[st];
                tma_load_4d(base, &tm_k, &bars->full[st], 0, g, row, seq);
                tma_load_4d(base + kBoxBytes, &tm_k, &bars->full[st], 64, g, row, seq);
                tma_load_4d(base + 2 * kBoxBytes, &tm_v, &bars->full[st], 0, g, row, seq);
                tma_load_4d(base + 3 * kBoxBytes, &tm_v, &bars->full[st], 64, g, row, seq);
                issued = li + 1;
            }
            // Do not leave while copies into this CTA's shared memory are in flight: wait
            // for the last phase issued on each stage (earlier ones completed before their
            // stage was refilled).
            for (int li = max(0, issued - kDStages); li < issued; ++li)
                mbar_drain_wait(&bars->full[li % kDStages], (li / kDStages) & 1);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int gq = lane >> 2;        // fragment row group
    const int qq = lane & 3;         // fragment column pair

    // q^T as B fragments (head dim = K, heads of the group = N), padded with zero heads.
    uint32_t qb[kD / 16][2];
    {
        const int n = gq;
        const bool valid = n < p.G;
        const __nv_bfloat16* qrow = p.q + (static_cast<size_t>(b) * p.Hq + g * p.G + (valid ? n : 0)) * kD;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            uint32_t lo = valid ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * qq) : 0u;
            uint32_t hi = valid ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * qq) : 0u;
            qb[ks][0] = lo;
            qb[ks][1] = hi;
        }
    }
    // Bias feature of the two heads this thread's accumulator columns belong to, and
    // the tables they read: per head (rank-1 form) or per sequence and head (curves of
    // a shared bank, coefficient 1).
    const float* wb = p.w + static_cast<size_t>(b) * p.w_bstride;
    float rs[2];
    int hcol[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int n = 2 * qq + e;
        hcol[e] = g * p.G + min(n, p.G - 1);
        // Columns n >= G are padding heads: their feature is never read (with G < 8
        // the address would belong to the next group, or lie past the end of r).
        const float coef =
            (p.r != nullptr && n < p.G) ? __ldg(p.r + static_cast<size_t>(b) * p.Hq + g * p.G + n) : 1.0f;
        rs[e] = (n < p.G) ? coef * p.inv_scale : 0.0f;
    }

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    float oacc[kD / 16][4];
#pragma unroll
    for (int dt = 0; dt < kD / 16; ++dt) oacc[dt][0] = oacc[dt][1] = oacc[dt][2] = oacc[dt][3] = 0.0f;

    const int last = N - 1;
    bool ok = true;
    for (int li = warp; li < nloc; li += kConsumers) {
        const int st = li % kDStages;
        const uint32_t ph = (li / kDStages) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->full[st], ph, abort_flag));
        if (!ok) break;
        const uint32_t kbase = smem_u32(sm->stages[st]);
        const uint32_t vbase = kbase + 2 * kBoxBytes;
        const int key0 = chunk0 + (c_begin + li) * kChunk;

        // S^T = K q^T for the chunk's groups of 16 keys.
        float sacc[kMT][4];
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
            sacc[mt][0] = sacc[mt][1] = sacc[mt][2] = sacc[mt][3] = 0.0f;
            const int mi = lane >> 3;
            const int key = mt * 16 + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                uint32_t a[4];
                ldsm_x4(kbase + swz(key, ks * 16 + ((mi >> 1) << 3)), a);
                mma_bf16(sacc[mt], a, qb[ks][0], qb[ks][1]);
            }
        }

        // Logits in log2 units, bias on the last R rows, mask rows past the cache end.
        const bool biased = key0 + kChunk - 1 >= N - p.R;
        float mc[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + mt * 16 + gq + ((e >> 1) << 3);
                const int col = e & 1;
                float x = sacc[mt][e];
                if (biased) {
                    const int dist = last - key;
                    if (dist >= 0 && dist < p.R)
                        x = fmaf(rs[col], __ldg(wb + static_cast<size_t>(hcol[col]) * p.R + dist), x);
                }
                bool visible = key <= last;
                if constexpr (PAGED) visible = visible && key >= key_lo;   // aligned chunks start early
                x = visible ? x * c1 : -INFINITY;
                sacc[mt][e] = x;
                mc[col] = fmaxf(mc[col], x);
            }
        }
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            mc[col] = fmaxf(mc[col], __shfl_xor_sync(0xffffffffu, mc[col], 4));
            mc[col] = fmaxf(mc[col], __shfl_xor_sync(0xffffffffu, mc[col], 8));
            mc[col] = fmaxf(mc[col], __shfl_xor_sync(0xffffffffu, mc[col], 16));
        }
        float base[2];
#pragma unroll
        for (int col = 0; col < 2; ++col) {
            const float m_new = fmaxf(m_run[col], mc[col]);
            const float alpha = (m_new == -INFINITY) ? 1.0f : ex2_approx(m_run[col] - m_new);
            l_run[col] *= alpha;
#pragma unroll
            for (int dt = 0; dt < kD / 16; ++dt) {
                oacc[dt][col] *= alpha;
                oacc[dt][col + 2] *= alpha;
            }
            m_run[col] = m_new;
            base[col] = (m_new == -INFINITY) ? 0.0f : m_new;
        }
        if constexpr (PAGED) {
            // Rows past the sequence's end in its last page hold whatever the pool had
            // there; their P is 0, but 0 * NaN is not, so zero those V rows first.  A row
            // of a 64-column box is 128 contiguous bytes (the swizzle permutes chunks
            // within it).
            const int first_dead = last - key0 + 1;
            if (first_dead < kChunk) {
                const int nb = (kChunk - first_dead) * 2 * 8;   // rows x boxes x 16-byte chunks
                for (int x = lane; x < nb; x += 32) {
                    const int rr = first_dead + x / 16, box = (x >> 3) & 1, ch = x & 7;
                    *reinterpret_cast<uint4*>(sm->stages[st] + 2 * kBoxBytes + box * kBoxBytes + rr * 128 + ch * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
            }
        }
        // P^T (keys x heads) -> bf16 -> transposed 8x8 blocks = B fragments.
        uint32_t pb[kMT][2];
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
            const float p0 = ex2_approx(sacc[mt][0] - base[0]);
            const float p1 = ex2_approx(sacc[mt][1] - base[1]);
            const float p2 = ex2_approx(sacc[mt][2] - base[0]);
            const float p3 = ex2_approx(sacc[mt][3] - base[1]);
            l_run[0] += p0 + p2;
            l_run[1] += p1 + p3;
            pb[mt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
            pb[mt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
        }
        // O^T += V^T P^T, head dim in 8 tiles of 16.
#pragma unroll
        for (int dt = 0; dt < kD / 16; ++dt) {
            const int mi = lane >> 3;
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                const int key = mt * 16 + (lane & 7) + ((mi >> 1) << 3);
                uint32_t a[4];
                ldsm_x4_trans(vbase + swz(key, dt * 16 + ((mi & 1) << 3)), a);
                mma_bf16(oacc[dt], a, pb[mt][0], pb[mt][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[st]);
    }

    // Per-warp partial -> shared memory.
#pragma unroll
    for (int col = 0; col < 2; ++col) {
        float lsum = l_run[col];
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        const int n = 2 * qq + col;
        if (gq == 0) {
            sm->warp_m[warp][n] = m_run[col];
            sm->warp_l[warp][n] = lsum;
        }
#pragma unroll
        for (int dt = 0; dt < kD / 16; ++dt) {
            sm->warp_o[warp][n][dt * 16 + gq] = oacc[dt][col];
            sm->warp_o[warp][n][dt * 16 + gq + 8] = oacc[dt][col + 2];
        }
    }
    named_bar_sync(1, kConsumers * 32);

    // Merge the four warps; one partial per (b, head) of the group.
    const int tid = threadIdx.x;            // 0..127
    const int n = tid >> 4;                 // head within group (8 x 16 threads)
    const int d0 = (tid & 15) * 8;
    if (n < p.G && ok) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sm->warp_m[w][n]);
        float sc[kConsumers];
        float Lsum = 0.0f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            sc[w] = (sm->warp_m[w][n] == -INFINITY) ? 0.0f : ex2_approx(sm->warp_m[w][n] - M);
            Lsum += sm->warp_l[w][n] * sc[w];
        }
        const int h = g * p.G + n;
        float* rec = p.part + ((static_cast<size_t>(b) * p.Hq + h) * p.nsplit + split) * kRec;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float acc = 0.0f;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) acc = fmaf(sm->warp_o[w][n][d0 + e], sc[w], acc);
            rec[d0 + e] = acc;
        }
        if ((tid & 15) == 0) {
            rec[kD] = M;
            rec[kD + 1] = Lsum;
        }
    }
}

// One warp per (b, h): merge nsplit partials by log-sum-exp.
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
    const int wid = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= p.B * p.Hq) return;
    const float* recs = p.part + static_cast<size_t>(wid) * p.nsplit * kRec;
    float M = -INFINITY;
    for (int s = lane; s < p.nsplit; s += 32) M = fmaxf(M, recs[s * kRec + kD]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.0f;
    for (int s = lane; s < p.nsplit; s += 32) {
        const float ms = recs[s * kRec + kD];
        if (ms != -INFINITY) L += recs[s * kRec + kD + 1] * ex2_approx(ms - M);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < p.nsplit; ++s) {
        const float ms = recs[s * kRec + kD];
        const float sc = (ms == -INFINITY) ? 0.0f : ex2_approx(ms - M);
        const float4 o4 = *reinterpret_cast<const float4*>(recs + s * kRec + lane * 4);
        acc.x = fmaf(o4.x, sc, acc.x);
        acc.y = fmaf(o4.y, sc, acc.y);
        acc.z = fmaf(o4.z, sc, acc.z);
        acc.w = fmaf(o4.w, sc, acc.w);
    }
    const float inv = 1.0f / L;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&lo);
    out.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p.o + static_cast<size_t>(wid) * kD + lane * 4) = out;
    if (p.lse != nullptr && lane == 0) p.lse[wid] = (M + __log2f(L)) * kLn2;
}

}  // namespace

namespace {
// One thread per (sequence and head, distance): the bank's curve for the one query
// row, sum_c rs[c] * proj[c, dist] ("Thinking Machines dropped RoPE", recipe step 2:
// the token's coefficients times the shared functions).
__global__ void __launch_bounds__(128) bank_curves_kernel(const float* __restrict__ rs,
                                                          const float* __restrict__ proj, float* __restrict__ curves,
                                                          int Hq, int C, int proj_heads, int R) {
    const int bh = blockIdx.y;
    const int dist = blockIdx.x * 128 + threadIdx.x;
    if (dist >= R) return;
    const float* coef = rs + static_cast<size_t>(bh) * C;
    const float* bank = proj + static_cast<size_t>(proj_heads == 1 ? 0 : bh % Hq) * C * R;
    float acc = 0.0f;
    for (int c = 0; c < C; ++c) acc = fmaf(__ldg(coef + c), __ldg(bank + static_cast<size_t>(c) * R + dist), acc);
    curves[static_cast<size_t>(bh) * R + dist] = acc;
}
}  // namespace

cudaError_t launch_bank_curves(const float* rs, const float* proj, float* curves, int BH, int Hq, int C,
                               int proj_heads, int R, cudaStream_t stream) {
    if (BH < 1 || R < 1) return cudaSuccess;
    dim3 grid((R + 127) / 128, BH);
    bank_curves_kernel<<<grid, 128, 0, stream>>>(rs, proj, curves, Hq, C, proj_heads, R);
    return cudaGetLastError();
}

int decode_num_splits(int B, int Hkv, int N, int window, int num_sms) {
    const int key_lo = window > 0 ? max(0, N - window) : 0;
    const int nchunks = (N - key_lo + kChunk - 1) / kChunk;
    const int target = num_sms * 8;   // eight full waves at one CTA per SM
    const int pairs = B * Hkv;
    int nsplit = (target + pairs - 1) / pairs;
    nsplit = max(1, min(nsplit, nchunks));
    const int cps = (nchunks + nsplit - 1) / nsplit;
    return (nchunks + cps - 1) / cps;
}

size_t decode_workspace_bytes(int B, int Hq, int nsplit, int d) {
    return static_cast<size_t>(B) * Hq * nsplit * (d + 4) * sizeof(float);
}

namespace {
template <bool PAGED>
cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream) {
    const int smem = static_cast<int>(sizeof(DecodeSmem)) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(decode_splitkv_kernel<PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.nsplit, p.Hkv, p.B);
    decode_splitkv_kernel<PAGED><<<grid, kDThreads, smem, stream>>>(tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<(p.B * p.Hq + 3) / 4, 128, 0, stream>>>(p);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_decode_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                               cudaStream_t stream) {
    return launch_decode<false>(tk, tv, p, stream);
}

cudaError_t launch_decode_paged_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                                     cudaStream_t stream) {
    return launch_decode<true>(tk, tv, p, stream);
}

}  // namespace relbias
