// prefill_sm100.cu -- bf16 prefill kernel for sm_100a: TMA-staged Q/K/V tiles,
// tcgen05 MMAs with accumulators in tensor memory, the relative-position bias
// added to the logits in registers, online softmax, causal / sliding-window tile
// skipping, and bias evaluation only on tiles that reach distances below R.
//
// The bias is produced "inside the tiled loop, block by block, as the scores
// form", as the essay "Thinking Machines dropped RoPE" says a fused kernel must
// (its closing section on kernel cost); logits are scale*q.k + r_i*w[h, i-j] for
// 0 <= i-j < R and scale*q.k beyond (recipe steps 3-5).
//
// Work item: (sequence b, key/value head g, a pair of query heads of that group,
// a 128-row query tile).  The two heads ("slots") share every K/V tile.
// Warp roles (384 threads, three warpgroups):
//   warps 0-3   softmax + epilogue of slot 0 (TMEM lanes 0-127, one row per thread)
//   warps 4-7   softmax + epilogue of slot 1
//   warp 8      TMA producer (Q per item, K and V per tile, 2-stage ring each)
//   warp 9      TMEM allocator and tcgen05.mma issuer
// The producer and MMA warps run their loops converged; one elected lane issues.
//   warps 10-11 idle; the third warpgroup hands its registers to the softmax
//               warpgroups (setmaxnreg), which hold a whole 128-wide row of S.
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D);
// the softmax writes P (bf16, packed in pairs) over the first 64 columns of its S.
// MMA issue order per KV tile j:  QK0(j)  PV1(j-1)  QK1(j)  PV0(j), so one slot's
// softmax overlaps the other slot's MMAs.  tcgen05.mma ops from one thread run in
// issue order, so QK_s(j+1) may overwrite P_s(j) once PV_s(j) has been issued, and
// when S_s(j) is complete, O_s holds everything up to PV_s(j-1) (softmax may
// rescale it before releasing P_s(j)).
//
// Bias lookup: thread t (query row i0+t) needs w[h, delta0 + t - c] for the 128
// key columns c of a tile -- a contiguous, descending run of the table.  The table
// is stored reversed (entry y holds w[h, Cmax - y], zero outside [0, R)), so the
// run is ascending, in NCOPY copies shifted by one entry each: every thread picks
// the copy that makes its run start on an NCOPY-float boundary and reads it with
// 64- or 128-bit loads.  Copy strides are chosen so that a warp's loads hit
// distinct banks.
//
// Instances: NCOPY in {1, 2, 4} is the rank-1 form with that many table copies;
// NCOPY = 0 is the shared-bank form, which reads each row's curve (written by
// bank_rows_kernel, below) from global memory in place of r_i * w.  PAGED reads K
// and V from a page pool through a block table, with per-sequence chunk offsets and
// lengths.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>

#include "kernels.h"
#include "ptx.cuh"

namespace relbias {

namespace {

constexpr int kBM = 128;            // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;            // keys per tile
constexpr int kStages = 2;          // K and V ring depth
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only if the max grows by > 2^8
// log2 units: a reference max may sit this far above a row's true running max (every
// weight then stays >= 2^-64, far inside the range of fp32 and bf16).
constexpr float kRefSlack = 64.0f;
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
constexpr int kMaxDynSmem = 232448;          // 227 KB per CTA on sm_100

// Reversed table: entry y <-> distance Cmax - y, Cmax = R + 255.  The largest
// distance a biased tile reaches is R + 254; the smallest a thread's run reaches is
// -254 (a chunk of queries that starts mid-tile puts the diagonal inside a tile), so
// the table runs down to distance -265 with zeros below 0 (those keys are masked).
__host__ __device__ constexpr int tab_cmax(int R) { return R + 255; }
__host__ __device__ constexpr int tab_len(int R) { return ((R + 520 + 31) / 32) * 32; }
__host__ __device__ constexpr int tab_stride(int R, int ncopy) {
    return tab_len(R) + (ncopy == 4 ? 8 : ncopy == 2 ? 18 : 0);
}
__host__ __device__ constexpr int tab_floats(int R, int ncopy) { return ncopy * tab_stride(R, ncopy); }

template <int D>
struct Layout {
    static constexpr int kTile = kBM * D * 2;     // bytes of one 128 x D bf16 tile
    static constexpr int kBox = kBM * 128;        // bytes of one 128-row x 64-col TMA box
    static constexpr int kQ = 0;                  // 2 slots
    static constexpr int kK = kQ + 2 * kTile;     // kStages
    static constexpr int kV = kK + kStages * kTile;
    static constexpr int kTab = kV + kStages * kTile;
};

struct Bars {
    uint64_t q_full[2], q_empty[2];   // per slot: each slot's query tile is reloaded on its own
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], o_final[2];
    uint64_t tab_sync[2];             // per slot: its four softmax warps meet around table staging
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

int smem_bytes_for(int d, int R, int ncopy) {
    const int lay = d == 64 ? Layout<64>::kTab : Layout<128>::kTab;
    return lay + 2 * tab_floats(R, ncopy) * 4 + static_cast<int>(sizeof(Bars)) + 1024;
}

struct Item {
    int qt, b, g, hp;
};

// Number of work items this CTA processes, and the k-th of them.
__device__ __forceinline__ int items_of_cta(const PrefillParams& p) {
    if (p.contiguous) {
        const int per = (p.total_items + gridDim.x - 1) / gridDim.x;
        return max(0, min(per, p.total_items - static_cast<int>(blockIdx.x) * per));
    }
    return (p.total_items - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
}

__device__ __forceinline__ Item item_at(const PrefillParams& p, int k) {
    Item it;
    if (p.contiguous) {
        // Runs of consecutive query tiles of the same (b, g, head pair).
        const int per = (p.total_items + gridDim.x - 1) / gridDim.x;
        const int u = static_cast<int>(blockIdx.x) * per + k;
        it.qt = u % p.n_qt;
        int rem = u / p.n_qt;
        it.hp = rem % p.HP;
        rem /= p.HP;
        it.g = rem % p.Hkv;
        it.b = rem / p.Hkv;
        return it;
    }
    const int u = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    const int per_qt = p.B * p.Hkv * p.HP;
    const int qr = u / per_qt;
    int rem = u - qr * per_qt;
    it.qt = p.n_qt - 1 - qr;   // heaviest query tiles first
    it.b = rem / (p.Hkv * p.HP);
    rem -= it.b * p.Hkv * p.HP;
    it.g = rem / p.HP;
    it.hp = rem - it.g * p.HP;
    return it;
}

// First key tile and number of key tiles the query tile with local first row i0
// visits.  Its rows sit at positions q_off + i0 ... q_off + i0 + 127 of the sequence
// (q_off > 0 for a chunk of queries after a cached prefix).
__device__ __forceinline__ void kv_range(const PrefillParams& p, int i0, int& j_first, int& ntiles) {
    const int a0 = p.q_off + i0;
    int lo = 0;
    if (p.window > 0) lo = max(0, a0 - p.window + 1);
    j_first = (lo / kBN) * kBN;
    const int j_last = ((a0 + kBM - 1) / kBN) * kBN;   // tile holding the last row's own key
    ntiles = (j_last - j_first) / kBN + 1;
}

// One 128-key tile of K or V from a page pool: two 64-row boxes, each inside one page
// (page_size is a multiple of 64).  Rows in a block past the table, or in a page index
// outside the pool, read zeros (TMA fills coordinates outside the tensor); the latter is
// reported when the row is one the chunk attends.
template <int D>
__device__ __forceinline__ void load_kv_paged(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                              const PrefillParams& p, const Item& it, int j0, int kv_end) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int row = j0 + 64 * half;
        const int blk = row / p.page_size;
        int page = -1, prow = 0;
        if (blk < p.max_pages) {
            page = __ldg(p.block_table + static_cast<size_t>(it.b) * p.max_pages + blk);
            prow = row - blk * p.page_size;
            if ((page < 0 || page >= p.num_pages) && row < kv_end) atomicOr(&g_status, kStatusBadLength);
        }
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
            tma_load_4d(dst + bx * kBM * 128 + half * 64 * 128, map, bar, bx * 64, it.g, prow, page);
    }
}

// Zero rows [first, 128) of a 128-row tile (D/64 boxes of 128-byte rows; the swizzle
// permutes chunks within a row, so whole rows are swizzle-free), by the 32 lanes of a
// warp, then order the writes before the tensor cores' reads of the tile.
template <int D>
__device__ __forceinline__ void zero_rows(uint8_t* tile, int first, int lane) {
    for (int x = lane; x < (kBM - first) * (D / 64) * 8; x += 32) {
        const int row = first + x / ((D / 64) * 8);
        const int rem = x % ((D / 64) * 8);
        *reinterpret_cast<uint4*>(tile + (rem >> 3) * kBM * 128 + row * 128 + (rem & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_shared();
    __syncwarp();
}

// Position of an item's first query row and its number of valid rows.  A chunk of
// a paged cache reads its sequence's offset and length from the device arrays
// (clamped into range and reported, when they are not).
template <bool PAGED>
__device__ __forceinline__ void item_rows(const PrefillParams& p, const Item& it, int& qo, int& nrows, int& kv_end) {
    const int i0 = it.qt * kBM;
    if constexpr (PAGED) {
        int off = __ldg(p.q_offs + it.b), len = __ldg(p.q_lens + it.b);
        const int cap = p.max_pages * p.page_size;
        if (off < 0 || len < 0 || len > p.T || static_cast<long long>(off) + len > cap) {
            atomicOr(&g_status, kStatusBadLength);
            off = min(max(off, 0), cap);
            len = min(max(len, 0), min(p.T, cap - off));
        }
        qo = off;
        nrows = min(kBM, len - i0);
        kv_end = off + len;
    } else {
        qo = p.q_off;
        nrows = min(kBM, p.T - i0);
        kv_end = p.q_off + p.T;
    }
}

// Key tiles of an item.  A paged item with no valid rows visits one tile (its outputs
// are not written), so every role walks the same tile stream.
template <bool PAGED>
__device__ __forceinline__ void item_kv_range(const PrefillParams& p, int i0, int qo, int nrows, int& j_first,
                                              int& ntiles) {
    if constexpr (PAGED) {
        if (nrows <= 0) {
            j_first = 0;
            ntiles = 1;
            return;
        }
        const int a0 = qo + i0;
        const int lo = p.window > 0 ? max(0, a0 - p.window + 1) : 0;
        j_first = (lo / kBN) * kBN;
        ntiles = (a0 + nrows - 1) / kBN - j_first / kBN + 1;
    } else {
        kv_range(p, i0, j_first, ntiles);
    }
}

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// The bias feature r[b, i, h] of this thread's row of an item (0 for rows past the
// item's valid rows).
template <bool PAGED>
__device__ __forceinline__ float load_feature(const PrefillParams& p, const Item& it, int slot, int t) {
    int qo, nrows, kv_end;
    item_rows<PAGED>(p, it, qo, nrows, kv_end);
    const int i = it.qt * kBM + t;
    const int h = it.g * p.G + it.hp * p.nslots + slot;
    return t < nrows ? __ldg(p.r + (static_cast<size_t>(it.b) * p.T + i) * p.Hq + h) : 0.0f;
}

// The four softmax warps of a slot meet: each arrives once (after its own shared-memory
// writes, which the arrival releases), then waits for the phase with a bounded wait.
__device__ __forceinline__ bool tab_meet(uint64_t* bar, uint32_t& phase, volatile int* abort_flag) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    const bool ok = warp_all(mbar_wait(bar, phase & 1, abort_flag));
    ++phase;
    return ok;
}

template <int D>
__device__ __forceinline__ void issue_qk(bool leader, uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr,
                                         uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk & 3) * 32 + (kk >> 2) * Layout<D>::kBox;
        const uint64_t a = smem_desc_sw128(q_addr + off, 16, 1024);
        const uint64_t b = smem_desc_sw128(k_addr + off, 16, 1024);
        if (leader) umma_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
    }
}

template <int D>
__device__ __forceinline__ void issue_pv(bool leader, uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         uint32_t idesc, bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
        // V tile: keys are the K dimension (8-row groups 1024 B apart), head dim
        // is the N dimension (64-column TMA boxes kBox apart): MN-major operand.
        const uint64_t b = smem_desc_sw128(v_addr + kk * 16 * 128, Layout<D>::kBox, 1024);
        if (leader) umma_ts(d_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// 2^x for a pair of fp32 values on the FMA pipe, relieving the MUFU unit (which
// computes 16 exponentials per SM per clock against 128 FMA lanes).  Cody-Waite
// style split x = n + f with n = round(x) (added to 1.5*2^23, whose low mantissa
// bits then hold n) and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose
// coefficients are a minimax fit of the relative error on that interval (7.5e-5);
// 2^n added into the exponent field.  x is clamped below at -126.5, so exponents
// stay in range and -inf (masked keys) gives ~5e-39 instead of 0: weights that
// small change no sum and no bf16 P.
constexpr float kExpC0 = 9.999280572e-01f, kExpC1 = 6.932609677e-01f, kExpC2 = 2.426111251e-01f,
                kExpC3 = 5.517166853e-02f;
constexpr int kEmuPer8 = 2;   // of every 8 exponential pairs, this many run on the FMA pipe

__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x2) {
    float a, b;
    f2_unpack(x2, a, b);
    const uint64_t xc = f2_pack(fmaxf(a, -126.5f), fmaxf(b, -126.5f));
    const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
    const uint64_t y = f2_add(xc, magic);
    const uint64_t n = f2_add(y, f2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), xc);
    uint64_t q = f2_fma(f, f2_pack(kExpC3, kExpC3), f2_pack(kExpC2, kExpC2));
    q = f2_fma(q, f, f2_pack(kExpC1, kExpC1));
    q = f2_fma(q, f, f2_pack(kExpC0, kExpC0));
    float qa, qb, ya, yb;
    f2_unpack(q, qa, qb);
    f2_unpack(y, ya, yb);
    return f2_pack(__uint_as_float(__float_as_uint(qa) + (__float_as_uint(ya) << 23)),
                   __uint_as_float(__float_as_uint(qb) + (__float_as_uint(yb) << 23)));
}

// s[c] += rs * w[h, delta0 + t - c] for the 128 columns, from this thread's run of
// the reversed table (`run` points at entry base_t, NCOPY-float aligned).
template <int NCOPY>
__device__ __forceinline__ void add_bias(float (&s)[kBN], const float* run, float rs) {
    const uint64_t rs2 = f2_pack(rs, rs);
#pragma unroll
    for (int c = 0; c < kBN; c += 4) {
        float w0, w1, w2, w3;
        if constexpr (NCOPY == 4) {
            const float4 v = *reinterpret_cast<const float4*>(run + c);
            w0 = v.x, w1 = v.y, w2 = v.z, w3 = v.w;
        } else if constexpr (NCOPY == 2) {
            const float2 a = *reinterpret_cast<const float2*>(run + c);
            const float2 b = *reinterpret_cast<const float2*>(run + c + 2);
            w0 = a.x, w1 = a.y, w2 = b.x, w3 = b.y;
        } else {
            w0 = run[c], w1 = run[c + 1], w2 = run[c + 2], w3 = run[c + 3];
        }
        const uint64_t lo = f2_fma(rs2, f2_pack(w0, w1), f2_pack(s[c], s[c + 1]));
        const uint64_t hi = f2_fma(rs2, f2_pack(w2, w3), f2_pack(s[c + 2], s[c + 3]));
        f2_unpack(lo, s[c], s[c + 1]);
        f2_unpack(hi, s[c + 2], s[c + 3]);
    }
}

// s[c] += rs * curve[delta0 + t - c] for the 128 columns, from this row's curve of
// the shared bank in global memory (the bank form: the row has its own curve).  `row`
// points at distance 0 of the row's padded curve and dlo = delta0 + t - 127 is the
// distance of column 127; the padding makes row + dlo a 32-byte boundary.  Eight
// distances per 32-byte load, columns descending; loads that reach no distance in
// [0, R) are skipped (zeros).
__device__ __forceinline__ void add_bias_curves(float (&s)[kBN], const float* row, int dlo, int R, float rs) {
    const uint64_t rs2 = f2_pack(rs, rs);
#pragma unroll
    for (int v = 0; v < kBN / 8; ++v) {
        const int d0 = dlo + 8 * v;   // distances d0 .. d0+7 <-> columns 127-8v .. 120-8v
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (d0 + 7 >= 0 && d0 < R) {
            a = __ldg(reinterpret_cast<const float4*>(row + d0));
            b = __ldg(reinterpret_cast<const float4*>(row + d0 + 4));
        }
        const float w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int c = kBN - 2 - 8 * v - 2 * m;   // columns c, c+1 <-> distances d0+1+2m, d0+2m
            const uint64_t r2 = f2_fma(rs2, f2_pack(w[2 * m + 1], w[2 * m]), f2_pack(s[c], s[c + 1]));
            f2_unpack(r2, s[c], s[c + 1]);
        }
    }
}

// NCOPY == 0: the shared-bank form, with each row's bias curve read from global
// memory (no staged table).  PAGED: K and V come from a page pool through a block
// table, each 128-key tile as two 64-row boxes (the pool's tensor maps have 64-row
// boxes), and every sequence has its own chunk offset and length.
template <int D, int NCOPY, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
    using L = Layout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base for the 128-byte-swizzled tiles; stays a shared-space
    // pointer, so table reads compile to shared-memory loads.
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tstride = tab_stride(p.R, NCOPY);
    const int tslot = NCOPY * tstride;
    float* tables = reinterpret_cast<float*>(smem + L::kTab);
    Bars* bars = reinterpret_cast<Bars*>(smem + L::kTab + 2 * tslot * 4);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full[0], 1);
        mbar_init(&bars->q_empty[0], 1);
        mbar_init(&bars->q_full[1], 1);
        mbar_init(&bars->q_empty[1], 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->p_full[s], kBM / 32);   // one arrival per softmax warp of the slot
            mbar_init(&bars->o_final[s], 1);
            mbar_init(&bars->tab_sync[s], kBM / 32);
        }
        mbar_init(&bars->mma_done, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;

    if (warp >= 8) {
        regs_decrease<kOtherRegs>();
        if (warp == 8) {
            // -------------------------------------------------------- TMA producer
            const bool leader = elect_one();
            int kv_it = 0;
            bool ok = true;
            // Loads issued so far (warp-uniform): each barrier has at most its last phase
            // in flight, which the drain below waits for.  K and V load number n go to
            // stage n % 2 and complete phase n / 2 of its barrier.
            int nq0 = 0, nq1 = 0, nk = 0, nv = 0;
            const int nitems = items_of_cta(p);
            for (int item_it = 0; ok && item_it < nitems; ++item_it) {
                const Item it = item_at(p, item_it);
                const int i0 = it.qt * kBM;
                int qo, nrows, kv_end, j_first, ntiles;
                item_rows<PAGED>(p, it, qo, nrows, kv_end);
                item_kv_range<PAGED>(p, i0, qo, nrows, j_first, ntiles);
                const int h0 = it.g * p.G + it.hp * p.nslots;
                for (int s = 0; ok && s < p.nslots; ++s) {
                    if (item_it > 0 && !(ok = warp_all(mbar_wait(&bars->q_empty[s], (item_it - 1) & 1, abort_flag))))
                        break;
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->q_full[s], L::kTile);
                        for (int bx = 0; bx < D / 64; ++bx)
                            tma_load_4d(smem + L::kQ + s * L::kTile + bx * L::kBox, &tm_q, &bars->q_full[s],
                                        bx * 64, h0 + s, i0, it.b);
                    }
                    if (s == 0) ++nq0; else ++nq1;
                }
                if (!ok) break;
                if (leader && item_it + 1 < nitems) {
                    // Warm L2 with the next item's query tiles while this item runs.
                    const Item nx = item_at(p, item_it + 1);
                    for (int s = 0; s < p.nslots; ++s)
                        for (int bx = 0; bx < D / 64; ++bx)
                            tma_prefetch_l2_4d(&tm_q, bx * 64, nx.g * p.G + nx.hp * p.nslots + s, nx.qt * kBM, nx.b);
                }
                for (int t = 0; t < ntiles; ++t, ++kv_it) {
                    const int st = kv_it & 1;
                    const uint32_t ph = (kv_it >> 1) & 1;
                    const int j0 = j_first + t * kBN;
                    if (!(ok = warp_all(mbar_wait(&bars->k_empty[st], ph ^ 1, abort_flag)))) break;
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->k_full[st], L::kTile);
                        if constexpr (PAGED) {
                            load_kv_paged<D>(smem + L::kK + st * L::kTile, &tm_k, &bars->k_full[st], p, it, j0, kv_end);
                        } else {
                            for (int bx = 0; bx < D / 64; ++bx)
                                tma_load_4d(smem + L::kK + st * L::kTile + bx * L::kBox, &tm_k, &bars->k_full[st],
                                            bx * 64, it.g, j0, it.b);
                        }
                    }
                    ++nk;
                    if (!(ok = warp_all(mbar_wait(&bars->v_empty[st], ph ^ 1, abort_flag)))) break;
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->v_full[st], L::kTile);
                        if constexpr (PAGED) {
                            load_kv_paged<D>(smem + L::kV + st * L::kTile, &tm_v, &bars->v_full[st], p, it, j0, kv_end);
                        } else {
                            for (int bx = 0; bx < D / 64; ++bx)
                                tma_load_4d(smem + L::kV + st * L::kTile + bx * L::kBox, &tm_v, &bars->v_full[st],
                                            bx * 64, it.g, j0, it.b);
                        }
                    }
                    ++nv;
                }
            }
            // Drain, also after an abort: the CTA must not exit (and hand its shared
            // memory to another CTA) while a copy into it is in flight.
            if (nq0 > 0) mbar_drain_wait(&bars->q_full[0], (nq0 - 1) & 1);
            if (nq1 > 0) mbar_drain_wait(&bars->q_full[1], (nq1 - 1) & 1);
            for (int n = max(0, nk - kStages); n < nk; ++n) mbar_drain_wait(&bars->k_full[n & 1], (n >> 1) & 1);
            for (int n = max(0, nv - kStages); n < nv; ++n) mbar_drain_wait(&bars->v_full[n & 1], (n >> 1) & 1);
        } else if (warp == 9) {
            // -------------------------------------------------------- MMA issuer
            // The key tiles of all this CTA's items form one stream g = 0, 1, ...; per tile
            // the issue order is QK0(g) PV1(g-1) QK1(g) PV0(g), across item boundaries too:
            // a slot's first QK of the next item follows its last PV directly, so the next
            // item's first logits are computed while the softmax warps write the output.
            const bool leader = elect_one();
            const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
            const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
            const uint32_t s_tm[2] = {tmem_base, tmem_base + 128};
            const uint32_t o_tm[2] = {tmem_base + 256, tmem_base + 384};
            const uint32_t q_addr[2] = {smem_u32(smem + L::kQ), smem_u32(smem + L::kQ + L::kTile)};
            int kv_it = 0;
            uint32_t pcnt[2] = {0, 0};
            // Slot 1's PV of the previous tile (issued after the next tile's QK0).
            bool prev = false, prev_first = false, prev_last = false;
            int prev_st = 0;
            bool ok = true;
            const int nitems = items_of_cta(p);
            for (int item_it = 0; ok && item_it < nitems; ++item_it) {
                const Item it = item_at(p, item_it);
                int qo, nrows, kv_end, j_first, ntiles;
                item_rows<PAGED>(p, it, qo, nrows, kv_end);
                item_kv_range<PAGED>(p, it.qt * kBM, qo, nrows, j_first, ntiles);
                for (int t = 0; t < ntiles; ++t, ++kv_it) {
                    const int st = kv_it & 1;
                    const uint32_t ph = (kv_it >> 1) & 1;
                    const bool first = t == 0, last = t == ntiles - 1;
                    const uint32_t k_addr = smem_u32(smem + L::kK + st * L::kTile);
                    const uint32_t v_addr = smem_u32(smem + L::kV + st * L::kTile);
                    if (!(ok = warp_all(mbar_wait(&bars->k_full[st], ph, abort_flag)))) break;
                    if (first && !(ok = warp_all(mbar_wait(&bars->q_full[0], item_it & 1, abort_flag)))) break;
                    tc_fence_after();
                    issue_qk<D>(leader, s_tm[0], q_addr[0], k_addr, idesc_qk);
                    if (leader) umma_commit(&bars->s_full[0]);
                    if (leader && last) umma_commit(&bars->q_empty[0]);
                    if (p.nslots == 2) {
                        if (prev) {
                            if (!(ok = warp_all(mbar_wait(&bars->p_full[1], pcnt[1] & 1, abort_flag)))) break;
                            ++pcnt[1];
                            tc_fence_after();
                            issue_pv<D>(leader, o_tm[1], s_tm[1], smem_u32(smem + L::kV + prev_st * L::kTile),
                                        idesc_pv, !prev_first);
                            if (leader) umma_commit(&bars->v_empty[prev_st]);
                            if (leader && prev_last) umma_commit(&bars->o_final[1]);
                        }
                        if (first && !(ok = warp_all(mbar_wait(&bars->q_full[1], item_it & 1, abort_flag)))) break;
                        tc_fence_after();
                        issue_qk<D>(leader, s_tm[1], q_addr[1], k_addr, idesc_qk);
                        if (leader) umma_commit(&bars->s_full[1]);
                        if (leader && last) umma_commit(&bars->q_empty[1]);
                    }
                    if (leader) umma_commit(&bars->k_empty[st]);
                    if (!(ok = warp_all(mbar_wait(&bars->v_full[st], ph, abort_flag)))) break;
                    if constexpr (PAGED) {
                        // Cache rows at or past the sequence's end may hold anything, and a
                        // NaN times a zero weight is NaN: zero those rows of the V tile before
                        // the first PV that reads it (both slots' PVs come after).
                        const int dead = kv_end - (j_first + t * kBN);
                        if (dead < kBN) zero_rows<D>(smem + L::kV + st * L::kTile, max(dead, 0), lane);
                    }
                    if (!(ok = warp_all(mbar_wait(&bars->p_full[0], pcnt[0] & 1, abort_flag)))) break;
                    ++pcnt[0];
                    tc_fence_after();
                    issue_pv<D>(leader, o_tm[0], s_tm[0], v_addr, idesc_pv, !first);
                    if (leader && p.nslots == 1) umma_commit(&bars->v_empty[st]);
                    if (leader && last) umma_commit(&bars->o_final[0]);
                    prev = true;
                    prev_st = st;
                    prev_first = first;
                    prev_last = last;
                }
            }
            if (ok && p.nslots == 2 && prev) {
                if ((ok = warp_all(mbar_wait(&bars->p_full[1], pcnt[1] & 1, abort_flag)))) {
                    tc_fence_after();
                    issue_pv<D>(leader, o_tm[1], s_tm[1], smem_u32(smem + L::kV + prev_st * L::kTile), idesc_pv,
                                !prev_first);
                    if (leader) umma_commit(&bars->v_empty[prev_st]);
                    if (leader && prev_last) umma_commit(&bars->o_final[1]);
                }
            }
            // Drain: wait (bounded, regardless of abort) until every MMA issued has finished,
            // before tensor memory is released and the CTA exits.
            if (leader) umma_commit(&bars->mma_done);
            mbar_drain_wait(&bars->mma_done, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        regs_increase<kSoftmaxRegs>();
        const int slot = threadIdx.x >> 7;
        const int t = threadIdx.x & 127;
        const uint32_t lane_off = static_cast<uint32_t>(t & ~31) << 16;
        const uint32_t s_tm = tmem_base + lane_off + slot * 128;
        const uint32_t o_tm = tmem_base + lane_off + 256 + slot * 128;
        float* wtab = tables + slot * tslot;
        const int cmax = tab_cmax(p.R);
        int tile_it = 0;
        int staged_head = -1;
        uint32_t tab_phase = 0;
        bool ok = slot < p.nslots;
        const int nitems = items_of_cta(p);
        // The row's bias feature (rank-1 form) is loaded one item ahead, off the path
        // between an item's last tile and the next item's first.
        float r_next = 0.0f;
        if (NCOPY > 0 && ok && nitems > 0) r_next = load_feature<PAGED>(p, item_at(p, 0), slot, t);
        // The reference max an item's rows start from: the previous item's final running
        // max of this thread's row (none for the first item).
        float m_hint = -INFINITY;
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const Item it = item_at(p, item_it);
            const int i0 = it.qt * kBM;
            const float r_cur = r_next;
            if (NCOPY > 0 && item_it + 1 < nitems) r_next = load_feature<PAGED>(p, item_at(p, item_it + 1), slot, t);
            int qo, nrows, kv_end, j_first, ntiles;
            item_rows<PAGED>(p, it, qo, nrows, kv_end);
            item_kv_range<PAGED>(p, i0, qo, nrows, j_first, ntiles);
            const int h = it.g * p.G + it.hp * p.nslots + slot;

            // This head's reversed distance table, NCOPY shifted copies, staged when the
            // head changes.  Loads are issued eight at a time so their L2 latencies overlap.
            if (NCOPY > 0 && h != staged_head) {
            // The slot's four warps meet before the table is rewritten (all done reading
            // the old one) and after (the new one complete).  The meeting is a bounded
            // mbarrier wait, so a warp that has wound down after an abort cannot leave
            // the others waiting for good.
            staged_head = h;
            if (!(ok = tab_meet(&bars->tab_sync[slot], tab_phase, abort_flag))) break;
            {
                const float* wrow = p.w + static_cast<size_t>(h) * p.R;
                for (int x0 = 0; x0 < tslot; x0 += 8 * kBM) {
                    float v[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int x = x0 + k * kBM + t;
                        const int cp = x / tstride;
                        const int dd = cmax - (x - cp * tstride + cp);
                        v[k] = (x < tslot && dd >= 0 && dd < p.R) ? __ldg(wrow + dd) : 0.0f;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int x = x0 + k * kBM + t;
                        if (x < tslot) wtab[x] = v[k];
                    }
                }
            }
            if (!(ok = tab_meet(&bars->tab_sync[slot], tab_phase, abort_flag))) break;
            }

            const int i = i0 + t;
            const bool row_ok = t < nrows;
            // Bias coefficient, in units of the unscaled logit: r_i / scale (rank-1 form), or
            // 1 / scale for the bank form, whose curve holds the whole bias.
            float rs = 0.0f;
            const float* curve_row = nullptr;
            if constexpr (NCOPY == 0) {
                rs = row_ok ? p.inv_scale : 0.0f;
                curve_row = p.curves +
                            (static_cast<size_t>(it.b) * p.T + (row_ok ? i : 0)) * p.Hq * p.curve_stride +
                            static_cast<size_t>(h) * p.curve_stride + (7 - ((qo + i) & 7));
            } else {
                rs = row_ok ? r_cur * p.inv_scale : 0.0f;
            }
            // Running reference max (log2 units) and the largest tile max seen.  Every
            // exponential is taken against m_used; m_used starts at the hint and is kept
            // within [m_seen - kRefSlack, m_seen + kRescaleThreshold] once m_seen is finite.
            float m_used = m_hint;
            float m_seen = -INFINITY;
            uint64_t l2 = 0;            // running sum, two partial lanes (0.0f, 0.0f)
            // Logit scale of this row, log2 units, with the context-length temperature:
            // a row that sees n > temp_n0 keys has its logits (content and bias) scaled
            // by ln n / ln temp_n0 (the essay, "The temperature scale is dependent on
            // context length").
            float c1 = p.scale_log2;
            if (p.temp_n0 > 1) {
                const int n = p.window > 0 ? min(qo + i + 1, p.window) : qo + i + 1;
                if (n > p.temp_n0) c1 *= __logf(static_cast<float>(n)) * p.inv_log_n0;
            }
            const uint64_t c1x2 = f2_pack(c1, c1);

            for (int tt = 0; tt < ntiles; ++tt, ++tile_it) {
                const int j0 = j_first + tt * kBN;
                const int delta0 = qo + i0 - j0;   // distance of (row t, key c) is delta0 + t - c
                ok = warp_all(mbar_wait(&bars->s_full[slot], tile_it & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t pk[kBN / 2];
                uint64_t acc[4];
                // One pass: logits from S (still in tensor memory), bias and mask, then the
                // exponentials against m_used with the tile's max found alongside.  A second
                // pass runs only when the tile shows m_used to be off: its max more than
                // 2^8 above it, or the first finite max of the item more than 2^64 below it
                // (a hint far too high).  The row is then re-referenced at its running max.
                for (int pass = 0;; ++pass) {
                    uint32_t sr[kBN];
#pragma unroll
                    for (int c = 0; c < kBN; c += 32) tmem_ld32(s_tm + c, sr + c);
                    tmem_ld_wait_regs(sr);
#pragma unroll
                    for (int c = 32; c < kBN; c += 32) tmem_regs_fence(sr + c);
                    float s[kBN];
#pragma unroll
                    for (int c = 0; c < kBN; ++c) s[c] = __uint_as_float(sr[c]);

                    if (delta0 - (kBN - 1) < p.R) {
                        // Some key of this tile is closer than R: add r_i * w[h, i-j] (in units
                        // of the unscaled logit; the table is zero outside [0, R)).
                        const int base = cmax - delta0 - t;
                        const int cp = base & (NCOPY - 1);
                        if constexpr (NCOPY == 0) {
                            if (row_ok) {
                                const int dlo = delta0 + t - (kBN - 1);
                                add_bias_curves(s, curve_row, dlo, p.R, rs);
                                // The next key tile's run (the 128 distances below this one's)
                                // into L2 meanwhile; addresses clamped into the row's curve.
                                if (pass == 0 && tt + 1 < ntiles && dlo > 0) {
#pragma unroll
                                    for (int k = 0; k < kBN; k += 32)
                                        prefetch_l2(curve_row + min(max(dlo - kBN + k, 0), p.R - 1));
                                }
                            }
                        } else {
                            add_bias<NCOPY>(s, wtab + cp * tstride + (base - cp), rs);
                        }
                    }
                    if (delta0 < kBN || (p.window > 0 && delta0 + kBM - 1 >= p.window)) {
                        // Key c is visible to row t iff lo <= c <= hi.  A 32-column chunk the
                        // whole warp sees entirely is skipped (a warp-uniform branch); other
                        // chunks pay per-element compares.
                        const int hi = delta0 + t;
                        const int lo = p.window > 0 ? delta0 + t - p.window + 1 : INT_MIN;
                        const int t0 = t & ~31;
                        const int hi_min = delta0 + t0;
                        const int lo_max = p.window > 0 ? hi_min + 31 - p.window + 1 : INT_MIN;
#pragma unroll
                        for (int cc = 0; cc < kBN; cc += 32) {
                            if (!(hi_min >= cc + 31 && lo_max <= cc)) {               // not all visible
#pragma unroll
                                for (int c = cc; c < cc + 32; ++c) s[c] = (c > hi || c < lo) ? -INFINITY : s[c];
                            }
                        }
                    }
                    if (__any_sync(0xffffffffu, m_used == -INFINITY)) {
                        // No reference yet (the first item's first tiles): the tile's max first.
                        float mc[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) mc[e] = fmaxf(s[2 * e], s[2 * e + 1]);
#pragma unroll
                        for (int c = 16; c < kBN; c += 16)
#pragma unroll
                            for (int e = 0; e < 8; ++e) mc[e] = fmax3f(mc[e], s[c + 2 * e], s[c + 2 * e + 1]);
                        const float mx = fmaxf(fmax3f(mc[0], mc[1], mc[2]), fmax3f(fmax3f(mc[3], mc[4], mc[5]), mc[6], mc[7]));
                        if (m_used == -INFINITY) m_used = mx * c1;
                    }
                    const float mb = (m_used == -INFINITY) ? 0.0f : m_used;
                    const uint64_t nm2 = f2_pack(-mb, -mb);
                    float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[e] = 0;
#pragma unroll
                    for (int c = 0; c < kBN; c += 2) {
                        mc[(c >> 1) & 3] = fmax3f(mc[(c >> 1) & 3], s[c], s[c + 1]);
                        const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c1x2, nm2);
                        float p0, p1;
                        if (((c >> 1) & 7) < kEmuPer8) {
                            f2_unpack(exp2_fma2(x2), p0, p1);
                        } else {
                            float x0, x1;
                            f2_unpack(x2, x0, x1);
                            p0 = ex2_approx(x0);
                            p1 = ex2_approx(x1);
                        }
                        acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2_pack(p0, p1));
                        pk[c / 2] = pack_bf16x2(p0, p1);
                    }
                    const float m_tile = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])) * c1;
                    m_seen = fmaxf(m_seen, m_tile);
                    const bool grow = m_tile > m_used + kRescaleThreshold;
                    const bool sink = m_tile > -INFINITY && m_seen < m_used - kRefSlack;
                    if (pass > 0 || !__any_sync(0xffffffffu, grow || sink)) break;
                    // Re-reference at the running max.  A growing max scales what the row has
                    // summed so far by 2^(m_used - m_seen); a sinking one is only possible on
                    // the first tile with a finite max, so what precedes it is masked keys
                    // and is dropped.
                    float alpha = 1.0f;
                    if (grow || sink) {
                        alpha = grow ? ex2_approx(m_used - m_seen) : 0.0f;
                        l2 = f2_mul(l2, f2_pack(alpha, alpha));
                        m_used = m_seen;
                    }
                    if (tt > 0) {
                        // O holds every PV up to the previous tile: rescale it in place.
                        uint32_t ob[32];
#pragma unroll
                        for (int c = 0; c < D; c += 32) {
                            tmem_ld32(o_tm + c, ob);
                            tmem_ld_wait_regs(ob);
#pragma unroll
                            for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * alpha);
                            tmem_st32(o_tm + c, ob);
                            tmem_st_wait();   // ob is refilled by the next chunk
                            tmem_regs_keep16(ob);
                            tmem_regs_keep16(ob + 16);
                        }
                        tmem_st_wait();
                    }
                }
                l2 = f2_add(l2, f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])));
                tmem_st32(s_tm, pk);
                tmem_st32(s_tm + 32, pk + 32);
                tmem_st_wait();
#pragma unroll
                for (int c = 0; c < kBN / 2; c += 16) tmem_regs_keep16(pk + c);
                tc_fence_before();
                // One arrival per warp, once every lane's P is in tensor memory.
                __syncwarp();
                if ((t & 31) == 0) mbar_arrive(&bars->p_full[slot]);
            }
            if (!ok) break;

            // Epilogue: O / l to bf16, and the row's log-sum-exp.
            ok = warp_all(mbar_wait(&bars->o_final[slot], item_it & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float la, lb;
            f2_unpack(l2, la, lb);
            const float l = la + lb;
            const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
            m_hint = m_used;
            __nv_bfloat16* orow = p.o + ((static_cast<size_t>(it.b) * p.T + i) * p.Hq + h) * D;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                uint32_t ob[32];
                tmem_ld32(o_tm + c, ob);
                tmem_ld_wait_regs(ob);
                uint32_t packed[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    packed[e] = pack_bf16x2(__uint_as_float(ob[2 * e]) * inv_l, __uint_as_float(ob[2 * e + 1]) * inv_l);
                if (row_ok) {
                    // Each thread writes its own row: 32-byte stores when O allows them
                    // (whole sectors, half the store instructions), else 16-byte ones.
                    if (p.o_v8) {
                        st_global_v8(orow + c, packed);
                        st_global_v8(orow + c + 16, packed + 8);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            st_global_v4(orow + c + 8 * e, packed[4 * e], packed[4 * e + 1], packed[4 * e + 2],
                                         packed[4 * e + 3]);
                    }
                }
            }
            if (p.lse != nullptr && row_ok)
                p.lse[(static_cast<size_t>(it.b) * p.Hq + h) * p.T + i] = (m_used + __log2f(l)) * kLn2;
            tc_fence_before();
        }
    }

    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int D, int NCOPY, bool PAGED = false>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const PrefillParams& p, int smem, int grid, cudaStream_t stream) {
    auto kern = prefill_bf16_sm100_kernel<D, NCOPY, PAGED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

// Curves of the shared bank for every (sequence, row, head) of a prefill, into the
// padded layout the kernel's curve variant reads ("Thinking Machines dropped RoPE",
// recipe step 2: the token's coefficients times the bank's functions):
//   out[row * S + pad + dist] = sum_c rs[row, c] * proj[hp, c, dist]   for dist in [0, R)
// and zeros elsewhere in the row, with row = (b * T + i) * Hq + h, hp = 0 or h, and
// pad = 7 - (position & 7): a prefill thread's run of 128 distances for one key tile
// then starts on a 32-byte boundary.
// A block covers the 32 rows of one (sequence, head) in a 256-row span whose positions
// agree mod 8 (so they share the pad), and its threads the padded positions x (two
// each, 128 apart): a thread loads the C function values at distance x - pad once and
// applies them to every row (C multiply-adds per value), and a warp writes 32
// consecutive floats of a row (whole 128-byte lines).
constexpr int kCurveRows = 32;   // rows per block, 8 apart (a 256-row span)
constexpr int kCurveThreads = 128;   // threads per block, 2 positions each (grid y: position blocks)

__global__ void __launch_bounds__(kCurveThreads, 8) bank_rows_kernel(const float* __restrict__ rs,
                                                                     const float* __restrict__ proj,
                                                                     float* __restrict__ out, int B, int T, int Hq,
                                                                     int q_off, int C, int proj_heads, int R, int S) {
    __shared__ __align__(16) float coef[kCurveRows][kMaxBankC];
    const int spans = (T + 8 * kCurveRows - 1) / (8 * kCurveRows);
    int blk = static_cast<int>(blockIdx.x);          // (b, h, span, residue)
    const int rho = blk & 7;
    blk >>= 3;
    const int span = blk % spans;
    blk /= spans;
    const int h = blk % Hq, b = blk / Hq;
    const int i0 = span * 8 * kCurveRows + rho;      // rows i0 + 8m, m < kCurveRows
    for (int x = threadIdx.x; x < kCurveRows * kMaxBankC; x += kCurveThreads) {
        const int m = x / kMaxBankC, c = x % kMaxBankC;
        const int i = i0 + 8 * m;
        coef[m][c] = (i < T && c < C) ? __ldg(rs + ((static_cast<size_t>(b) * T + i) * Hq + h) * C + c) : 0.0f;
    }
    __syncthreads();
    // Positions x0 and x0 + 128 of this thread (the second may lie past S).
    const int x0 = static_cast<int>(blockIdx.y) * 2 * kCurveThreads + static_cast<int>(threadIdx.x);
    if (i0 >= T || x0 >= S) return;
    const bool two = x0 + kCurveThreads < S;
    const int nrows = min(kCurveRows, (T - i0 + 7) / 8);
    const int pad = 7 - ((q_off + i0) & 7);
    const float* bank = proj + static_cast<size_t>(proj_heads == 1 ? 0 : h) * C * R;
    const size_t row_step = static_cast<size_t>(8) * Hq * S;      // floats between rows i and i + 8
    float* dst = out + ((static_cast<size_t>(b) * T + i0) * Hq + h) * S + x0;
    float pc[2][kMaxBankC];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int dist = x0 + q * kCurveThreads - pad;
        const bool inside = dist >= 0 && dist < R && (q == 0 || two);
#pragma unroll
        for (int c = 0; c < kMaxBankC; ++c)
            pc[q][c] = (c < C && inside) ? __ldg(bank + static_cast<size_t>(c) * R + dist) : 0.0f;
    }
    // Row by row: the row's C coefficients (broadcast shared-memory loads) serve both
    // positions; each sum is split in halves (4 independent chains per row).
    for (int m = 0; m < nrows; ++m, dst += row_step) {
        float lo[2] = {0.0f, 0.0f}, hi[2] = {0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < kMaxBankC / 2; c += 4) {
            const float4 u = *reinterpret_cast<const float4*>(&coef[m][c]);
            const float4 w = *reinterpret_cast<const float4*>(&coef[m][c + kMaxBankC / 2]);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                lo[q] = fmaf(u.x, pc[q][c], lo[q]), lo[q] = fmaf(u.y, pc[q][c + 1], lo[q]);
                lo[q] = fmaf(u.z, pc[q][c + 2], lo[q]), lo[q] = fmaf(u.w, pc[q][c + 3], lo[q]);
                hi[q] = fmaf(w.x, pc[q][c + 8], hi[q]), hi[q] = fmaf(w.y, pc[q][c + 9], hi[q]);
                hi[q] = fmaf(w.z, pc[q][c + 10], hi[q]), hi[q] = fmaf(w.w, pc[q][c + 11], hi[q]);
            }
        }
        dst[0] = lo[0] + hi[0];
        if (two) dst[kCurveThreads] = lo[1] + hi[1];
    }
}

int prefill_bf16_table_copies(int d, int R) {
    for (int nc = 4; nc >= 1; nc >>= 1)
        if (smem_bytes_for(d, R, nc) <= kMaxDynSmem) return nc;
    return 0;
}

int prefill_bf16_smem_bytes(int d, int R, int nc) {
    // Each CTA allocates all 512 TMEM columns: never let two CTAs share an SM
    // (228 KB of shared memory per SM, so more than 114 KB each).
    return std::max(smem_bytes_for(d, R, nc), 120 * 1024);
}

int prefill_bank_curve_stride(int R) { return ((R + 14) + 7) / 8 * 8; }

cudaError_t launch_bank_rows(const float* rs, const float* proj, float* curves, int B, int T, int Hq, int q_off, int C,
                             int proj_heads, int R, cudaStream_t stream) {
    if (B < 1 || T < 1 || R < 1) return cudaSuccess;
    const int S = prefill_bank_curve_stride(R);
    const long long blocks = static_cast<long long>(B) * Hq * ((T + 8 * kCurveRows - 1) / (8 * kCurveRows)) * 8;
    if (blocks > INT32_MAX) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(blocks), (S + 2 * kCurveThreads - 1) / (2 * kCurveThreads));
    bank_rows_kernel<<<grid, kCurveThreads, 0, stream>>>(rs, proj, curves, B, T, Hq, q_off, C, proj_heads, R, S);
    return cudaGetLastError();
}

cudaError_t launch_prefill_bf16_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                      const PrefillParams& p, int d, int grid, cudaStream_t stream) {
    if (p.curves != nullptr) {
        // The bank form: no staged table (shared memory as for R = 0).
        const int smem = prefill_bf16_smem_bytes(d, 0, 0);
        if (d == 128) return launch_variant<128, 0>(tq, tk, tv, p, smem, grid, stream);
        return launch_variant<64, 0>(tq, tk, tv, p, smem, grid, stream);
    }
    const int nc = prefill_bf16_table_copies(d, p.R);
    if (nc == 0) return cudaErrorInvalidValue;
    const int smem = prefill_bf16_smem_bytes(d, p.R, nc);
    if (p.paged) {
        if (d == 128) {
            if (nc == 4) return launch_variant<128, 4, true>(tq, tk, tv, p, smem, grid, stream);
            if (nc == 2) return launch_variant<128, 2, true>(tq, tk, tv, p, smem, grid, stream);
            return launch_variant<128, 1, true>(tq, tk, tv, p, smem, grid, stream);
        }
        if (nc == 4) return launch_variant<64, 4, true>(tq, tk, tv, p, smem, grid, stream);
        if (nc == 2) return launch_variant<64, 2, true>(tq, tk, tv, p, smem, grid, stream);
        return launch_variant<64, 1, true>(tq, tk, tv, p, smem, grid, stream);
    }
    if (d == 128) {
        if (nc == 4) return launch_variant<128, 4>(tq, tk, tv, p, smem, grid, stream);
        if (nc == 2) return launch_variant<128, 2>(tq, tk, tv, p, smem, grid, stream);
        return launch_variant<128, 1>(tq, tk, tv, p, smem, grid, stream);
    }
    if (nc == 4) return launch_variant<64, 4>(tq, tk, tv, p, smem, grid, stream);
    if (nc == 2) return launch_variant<64, 2>(tq, tk, tv, p, smem, grid, stream);
    return launch_variant<64, 1>(tq, tk, tv, p, smem, grid, stream);
}

}  // namespace relbias
