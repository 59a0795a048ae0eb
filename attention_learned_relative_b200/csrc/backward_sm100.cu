// backward_sm100.cu -- gradients of the biased attention forward pass on the tcgen05
// tensor cores (bf16 inputs, fp32 accumulation in tensor memory).
//
// For one row (b, h, i) with logits l_j = tau_i * (scale * q_i.k_j + r_i * w[h, i-j])
// over the attended keys, p_j = exp(l_j - LSE_i) and D_i = dO_i.O_i, the derivative
// of the loss with respect to l_j is dl_j = p_j (dO_i.v_j - D_i), and
//   dq_i = tau_i scale sum_j dl_j k_j        dk_j = sum_(h,i) tau_i scale dl_j q_i
//   dv_j = sum_(h,i) p_j dO_i                 dr_i = tau_i sum_j dl_j w[h, i-j]
//   dw[h, d] = sum_i tau_i dl_(i, i-d) r_i
// (the plain derivative of the forward definition: "Thinking Machines dropped RoPE",
// recipe steps 3-5, for the bias; the pages train the model but print no backward).
//
// Kernels (one row of a 128 x 128 tile per thread, 64 of its columns per warp: two
// warps share each TMEM lane quadrant):
//   bwd_dvec_kernel        D_i = dO_i . O_i for every row (and dr zeroed).
//   bwd_dq_sm100_kernel    per (sequence, query head, 128-row query tile): over the
//       visible key tiles, S = Q K^T and dP = dO V^T into tensor memory, dl in
//       registers (dr accumulated with the staged distance table, as the forward adds
//       the bias), dS = tau scale dl written back over S as bf16, dQ += dS K.
//   bwd_dkv_sm100_kernel   per (sequence, key/value head, 128-key tile): over the
//       group's query heads and the query tiles that see the keys, S^T = K Q^T and
//       dP^T = V dO^T, P^T and dS^T in registers (one key row per thread), then
//       dV += P^T dO and dK += dS^T Q with P^T and dS^T read from tensor memory; dw
//       summed along the tile's diagonals.
// The shared-bank form (NCOPY = 0 instances) reads each row's curve in place of
// r_i * w and writes dL/dcurve instead of dr and dw; bank_drs_kernel and
// bank_dproj_kernel turn it into the gradients of the coefficients and the bank.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

#include <type_traits>

namespace relbias {

namespace {

// ------------------------------------------------------------------------- dQ kernel

constexpr int kBqThreads = 320;   // warps 0-7 rows (two per TMEM lane quadrant), 8 TMA producer, 9 MMA issuer
constexpr int kBqRowWarps = 8;

template <int D>
struct BqLayout {
    static constexpr int kTile = kBM * D * 2;
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTile;
    static constexpr int kK = kDO + kTile;             // 2 stages
    static constexpr int kV = kK + 2 * kTile;          // 2 stages
    static constexpr int kTab = kV + 2 * kTile;
};

struct BqBars {
    uint64_t q_full, q_empty, do_full, do_empty;
    uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
    uint64_t sdp_full;     // S(g) and dP(g) complete
    uint64_t dp_free;      // the rows' warps hold dP(g) in registers
    uint64_t ds_ready;     // dS(g) is in tensor memory
    uint64_t dq_final;     // an item's last dQ MMA complete
    uint64_t dq_free;      // the rows' warps have read an item's dQ
    uint64_t tab_sync;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

int bq_smem_bytes(int d, int R, int ncopy) {
    const int lay = d == 64 ? BqLayout<64>::kTab : BqLayout<128>::kTab;
    return lay + tab_floats(R, ncopy) * 4 + static_cast<int>(sizeof(BqBars)) + 1024;
}

// The tile stream of a CTA: item by item, key tile by key tile.
struct TileCursor {
    int item_it, nitems, t, ntiles, j_first;
    Item it;
    __device__ __forceinline__ void load(const PrefillParams& p) {
        it = item_at(p, item_it);
        kv_range(p, it.qt * kBM, j_first, ntiles);
        t = 0;
    }
    __device__ __forceinline__ bool next(const PrefillParams& p) {
        if (++t < ntiles) return true;
        if (++item_it >= nitems) return false;
        load(p);
        return true;
    }
    __device__ __forceinline__ bool first() const { return t == 0; }
    __device__ __forceinline__ bool last() const { return t == ntiles - 1; }
    __device__ __forceinline__ int j0() const { return j_first + t * kBN; }
};

// D_i = dO_i . O_i for every row (b, i, h), into dvec [B, Hq, T], and dr zeroed.
template <int D>
__global__ void __launch_bounds__(256) bwd_dvec_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout, float* __restrict__ dvec,
                                                       float* __restrict__ dr, int B, int T, int Hq) {
    // D / 8 lanes per row, 16 bytes of o and of dout each (rows are 16-byte aligned).
    constexpr int kLanes = D / 8;
    const long long row = static_cast<long long>(blockIdx.x) * (256 / kLanes) + threadIdx.x / kLanes;   // (b * T + i) * Hq + h
    const int sub = threadIdx.x % kLanes;
    const bool ok = row < static_cast<long long>(B) * T * Hq;
    float acc = 0.0f;
    if (ok) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + sub);
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + sub);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[u]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[u]));
            acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
        }
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (ok && sub == 0) {
        const int h = static_cast<int>(row % Hq);
        const long long bi = row / Hq;
        const int i = static_cast<int>(bi % T), b = static_cast<int>(bi / T);
        dvec[(static_cast<size_t>(b) * Hq + h) * T + i] = acc;
        if (dr != nullptr) dr[row] = 0.0f;   // the dQ kernel's two column halves add into it
    }
}

// A dQ-kernel row's inputs: D_i, LSE_i (natural log) and r_i (zeros past T).
__device__ __forceinline__ float3 bq_row_inputs(const PrefillParams& p, const BwdTcParams& bp, const Item& it, int t) {
    const int i = it.qt * kBM + t;
    if (i >= p.T) return make_float3(0.f, 0.f, 0.f);
    const int h = it.g * p.G + it.hp;
    const size_t hrow = (static_cast<size_t>(it.b) * p.Hq + h) * p.T + i;
    return make_float3(__ldg(bp.dvec + hrow), __ldg(bp.lse + hrow),
                       __ldg(p.r + (static_cast<size_t>(it.b) * p.T + i) * p.Hq + h));
}

// An accumulating MMA (dQ += dS K, dV += P^T dO, dK += dS^T Q) whose A operand is bf16
// in tensor memory, written by two warps per lane quadrant: the warp of column half h
// packs its 64 values of a row at columns [64 h, 64 h + 32), over fp32 columns only it
// has read, so neither warp overwrites values the other has yet to load.
template <int D>
__device__ __forceinline__ void issue_acc_split(bool leader, uint32_t d_tmem, uint32_t p_tmem, uint32_t b_addr,
                                                uint32_t idesc, bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < kBM / 16; ++kk) {
        const uint64_t b = smem_desc_sw128(b_addr + kk * 16 * 128, Layout<D>::kBox, 1024);
        const uint32_t a = p_tmem + kk * 8 + (kk >= kBM / 32 ? 32 : 0);
        if (leader) umma_ts(d_tmem, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

template <int D, int NCOPY>
__global__ void __launch_bounds__(kBqThreads, 1)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const PrefillParams p, const BwdTcParams bp) {
    using L = BqLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tstride = tab_stride(p.R, NCOPY);
    const int tslot = NCOPY * tstride;
    float* wtab = reinterpret_cast<float*>(smem + L::kTab);
    BqBars* bars = reinterpret_cast<BqBars*>(smem + L::kTab + tslot * 4);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->do_full, 1);
        mbar_init(&bars->do_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], 1);
        }
        mbar_init(&bars->sdp_full, 1);
        mbar_init(&bars->dp_free, kBqRowWarps);
        mbar_init(&bars->ds_ready, kBqRowWarps);
        mbar_init(&bars->dq_final, 1);
        mbar_init(&bars->dq_free, kBqRowWarps);
        mbar_init(&bars->tab_sync, kBqRowWarps);
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
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    const int nitems = items_of_cta(p);
    // Tensor memory: S(g) in [128 * (g & 1), +128), dP [256, 384), dQ [384, 384 + D).

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        const bool leader = elect_one();
        bool ok = true;
        int nq = 0, nkv = 0;   // items and key tiles whose copies were issued
        int g = 0;
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const Item it = item_at(p, item_it);
            const int i0 = it.qt * kBM;
            int j_first, ntiles;
            kv_range(p, i0, j_first, ntiles);
            const int h = it.g * p.G + it.hp;
            if (item_it > 0 && !(ok = warp_all(mbar_wait(&bars->q_empty, (item_it - 1) & 1, abort_flag)))) break;
            if (leader) {
                mbar_arrive_expect_tx(&bars->q_full, L::kTile);
                for (int bx = 0; bx < D / 64; ++bx)
                    tma_load_4d(smem + L::kQ + bx * kBM * 128, &tm_q, &bars->q_full, bx * 64, h, i0, it.b);
            }
            if (item_it > 0 && !(ok = warp_all(mbar_wait(&bars->do_empty, (item_it - 1) & 1, abort_flag)))) break;
            if (leader) {
                mbar_arrive_expect_tx(&bars->do_full, L::kTile);
                for (int bx = 0; bx < D / 64; ++bx)
                    tma_load_4d(smem + L::kDO + bx * kBM * 128, &tm_do, &bars->do_full, bx * 64, h, i0, it.b);
            }
            ++nq;
            for (int t = 0; t < ntiles; ++t, ++g) {
                const int st = g & 1;
                const uint32_t ph = (g >> 1) & 1;
                const int j0 = j_first + t * kBN;
                if (!(ok = warp_all(mbar_wait(&bars->k_empty[st], ph ^ 1, abort_flag)))) break;
                if (!(ok = warp_all(mbar_wait(&bars->v_empty[st], ph ^ 1, abort_flag)))) break;
                if (leader) {
                    mbar_arrive_expect_tx(&bars->k_full[st], L::kTile);
                    mbar_arrive_expect_tx(&bars->v_full[st], L::kTile);
                    for (int bx = 0; bx < D / 64; ++bx) {
                        tma_load_4d(smem + L::kK + st * L::kTile + bx * kBM * 128, &tm_k, &bars->k_full[st],
                                    bx * 64, it.g, j0, it.b);
                        tma_load_4d(smem + L::kV + st * L::kTile + bx * kBM * 128, &tm_v, &bars->v_full[st],
                                    bx * 64, it.g, j0, it.b);
                    }
                    // Warm L2 with the tile two ahead within the item (its stage frees late).
                    if (t + 2 < ntiles)
                        for (int bx = 0; bx < D / 64; ++bx) {
                            tma_prefetch_l2_4d(&tm_k, bx * 64, it.g, j0 + 2 * kBN, it.b);
                            tma_prefetch_l2_4d(&tm_v, bx * 64, it.g, j0 + 2 * kBN, it.b);
                        }
                }
                ++nkv;
            }
        }
        // Drain, also after an abort: no copy into this CTA's shared memory may be in flight
        // when it exits.  Each barrier has at most its last phase outstanding.
        if (nq > 0) {
            mbar_drain_wait(&bars->q_full, (nq - 1) & 1);
            mbar_drain_wait(&bars->do_full, (nq - 1) & 1);
        }
        for (int n = max(0, nkv - 2); n < nkv; ++n) {
            mbar_drain_wait(&bars->k_full[n & 1], (n >> 1) & 1);
            mbar_drain_wait(&bars->v_full[n & 1], (n >> 1) & 1);
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        // Per tile g the issue order is QK(g+1), dP(g+1), dQ(g): the next tile's S and dP
        // are computed while the rows' warps work on tile g (S is double-buffered; dP is
        // rewritten once the warps hold dP(g) in registers).
        const bool leader = elect_one();
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
        const uint32_t idesc_dq = idesc_bf16_f32(kBM, D, false, true);
        const uint32_t dp_tm = tmem_base + 256, dq_tm = tmem_base + 384;
        const uint32_t q_addr = smem_u32(smem + L::kQ), do_addr = smem_u32(smem + L::kDO);
        bool ok = nitems > 0;
        TileCursor cur{0, nitems, 0, 0, 0, {}};
        if (ok) cur.load(p);
        // Issue QK and dP of tile g (its stage st); first tiles of an item wait for Q / dO.
        auto issue_s_dp = [&](const TileCursor& c, int g, bool wait_dp_free) -> bool {
            const int st = g & 1;
            const uint32_t ph = (g >> 1) & 1;
            if (!warp_all(mbar_wait(&bars->k_full[st], ph, abort_flag))) return false;
            if (c.first() && !warp_all(mbar_wait(&bars->q_full, c.item_it & 1, abort_flag))) return false;
            tc_fence_after();
            issue_qk<D>(leader, tmem_base + 128 * (g & 1), q_addr, smem_u32(smem + L::kK + st * L::kTile), idesc_qk);
            if (leader && c.last()) umma_commit(&bars->q_empty);
            if (wait_dp_free && !warp_all(mbar_wait(&bars->dp_free, (g - 1) & 1, abort_flag))) return false;
            if (!warp_all(mbar_wait(&bars->v_full[st], ph, abort_flag))) return false;
            if (c.first() && !warp_all(mbar_wait(&bars->do_full, c.item_it & 1, abort_flag))) return false;
            tc_fence_after();
            issue_qk<D>(leader, dp_tm, do_addr, smem_u32(smem + L::kV + st * L::kTile), idesc_qk);
            if (leader) umma_commit(&bars->v_empty[st]);
            if (leader && c.last()) umma_commit(&bars->do_empty);
            if (leader) umma_commit(&bars->sdp_full);
            return true;
        };
        if (ok) ok = issue_s_dp(cur, 0, false);
        for (int g = 0; ok; ++g) {
            TileCursor nxt = cur;
            const bool have_next = nxt.next(p);
            if (have_next && !(ok = issue_s_dp(nxt, g + 1, true))) break;
            if (!(ok = warp_all(mbar_wait(&bars->ds_ready, g & 1, abort_flag)))) break;
            if (cur.first() && cur.item_it > 0 &&
                !(ok = warp_all(mbar_wait(&bars->dq_free, (cur.item_it - 1) & 1, abort_flag))))
                break;
            tc_fence_after();
            // dQ += dS K: dS (bf16 pairs over the first 64 columns of S(g)) times the key tile,
            // keys on the K dimension (MN-major operand, as V in the forward's PV).
            issue_acc_split<D>(leader, dq_tm, tmem_base + 128 * (g & 1),
                               smem_u32(smem + L::kK + (g & 1) * L::kTile), idesc_dq, !cur.first());
            if (leader) umma_commit(&bars->k_empty[g & 1]);
            if (leader && cur.last()) umma_commit(&bars->dq_final);
            if (!have_next) break;
            cur = nxt;
        }
        if (leader) umma_commit(&bars->mma_done);
        mbar_drain_wait(&bars->mma_done, 0);
    } else {
        // ---------------------------------------------------------------- rows
        const int t = threadIdx.x & (kBM - 1);           // row t of the query tile (TMEM lane)
        const int half = threadIdx.x >> 7;               // key columns [64 half, 64 half + 64) of each tile
        const uint32_t lane_off = static_cast<uint32_t>(t & ~31) << 16;
        const uint32_t dp_tm = tmem_base + lane_off + 256, dq_tm = tmem_base + lane_off + 384;
        const int cmax = tab_cmax(p.R);
        int staged_head = -1;
        uint32_t tab_phase = 0;
        int g = 0;
        bool ok = true;
        // The row's D_i, LSE and bias feature are loaded one item ahead.
        float3 nxt = nitems > 0 ? bq_row_inputs(p, bp, item_at(p, 0), t) : make_float3(0.f, 0.f, 0.f);
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const Item it = item_at(p, item_it);
            const int i0 = it.qt * kBM;
            int j_first, ntiles;
            kv_range(p, i0, j_first, ntiles);
            const int h = it.g * p.G + it.hp;
            const float3 cur = nxt;
            if (item_it + 1 < nitems) nxt = bq_row_inputs(p, bp, item_at(p, item_it + 1), t);
            if (NCOPY > 0 && h != staged_head) {
                staged_head = h;
                if (!(ok = tab_meet(&bars->tab_sync, tab_phase, abort_flag))) break;
                const float* wrow = p.w + static_cast<size_t>(h) * p.R;
                for (int x = threadIdx.x; x < tslot; x += kBqRowWarps * 32) {
                    const int cp = x / tstride;
                    const int dd = cmax - (x - cp * tstride + cp);
                    wtab[x] = (dd >= 0 && dd < p.R) ? __ldg(wrow + dd) : 0.0f;
                }
                if (!(ok = tab_meet(&bars->tab_sync, tab_phase, abort_flag))) break;
            }
            const int i = i0 + t;
            const bool row_ok = i < p.T;
            const size_t row = (static_cast<size_t>(it.b) * p.T + (row_ok ? i : 0)) * p.Hq + h;   // [B, T, Hq]
            const size_t hrow = (static_cast<size_t>(it.b) * p.Hq + h) * p.T + (row_ok ? i : 0);  // [B, Hq, T]
            // D_i (from the D kernel), the row's log-sum-exp in log2 units, the logit scale
            // with the context-length temperature, and the bias coefficient (log2 units).
            const float Di = cur.x;
            const float lse2 = cur.y * 1.4426950408889634f;
            float tau = 1.0f;
            if (p.temp_n0 > 1) {
                const int n = p.window > 0 ? min(i + 1, p.window) : i + 1;
                if (n > p.temp_n0) tau = __logf(static_cast<float>(n)) * p.inv_log_n0;
            }
            const float c1 = p.scale_log2 * tau;
            // Bias coefficient, log2 units: r_i / scale (rank-1 form) or 1 / scale (the
            // bank form, whose curve holds the whole bias).
            const float rb = (NCOPY > 0 ? cur.z : 1.0f) * p.inv_scale * c1;
            // The bank form: the row's curve and its gradient, at distance 0 (padded rows).
            const size_t crow = row * static_cast<size_t>(bp.curve_stride) + (7 - (i & 7));
            const float* curve = NCOPY == 0 ? bp.curves + crow : nullptr;
            float* dcurve = NCOPY == 0 ? bp.dcv + crow : nullptr;
            const float ds_scale = tau * bp.scale;   // dS = tau * scale * dl, the dQ MMA's operand
            float dr_acc = 0.0f;                     // sum_j dl_j w[h, i-j]

            for (int tt = 0; tt < ntiles; ++tt, ++g) {
                const int j0 = j_first + tt * kBN;
                const int delta0 = i0 - j0;
                const uint32_t s_tm = tmem_base + lane_off + 128 * (g & 1);
                if (!(ok = warp_all(mbar_wait(&bars->sdp_full, g & 1, abort_flag)))) break;
                tc_fence_after();
                uint32_t dp[kBN / 2];   // this half's columns
#pragma unroll
                for (int c = 0; c < kBN / 2; c += 32) tmem_ld32(dp_tm + 64 * half + c, dp + c);
                tmem_ld_wait_regs(dp);
                tmem_regs_fence(dp + 32);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dp_free);
                const bool biased = delta0 - (kBN - 1) < p.R;
                const int base = cmax - delta0 - t;
                const int cp = base & (NCOPY - 1);
                const float* run = wtab + cp * tstride + (base - cp);
                const bool edge = delta0 < kBN || (p.window > 0 && delta0 + kBM - 1 >= p.window);
                const int hi = delta0 + t;
                const int lo = p.window > 0 ? delta0 + t - p.window + 1 : INT_MIN;
                uint32_t pk2[4][8];   // the chunks' dS: live until the stores are waited for
                // The chunk loop, compiled with the table bias (a biased tile of the rank-1 form)
                // and without it, so that no table load sits under a per-chunk branch.  Chunks of
                // 16 columns keep the bank form's prefetched curve values in registers.
                auto chunks = [&](auto bias_tag) {
                    constexpr bool kBiasTab = NCOPY > 0 && decltype(bias_tag)::value;
#pragma unroll
                    for (int lc = 0; lc < 4; ++lc) {
                        const int ch = 4 * half + lc;   // this half's chunks of 16 columns
                        uint32_t* pk = pk2[lc];
                        // The bank form: this chunk's curve values (four aligned groups of four
                        // distances), loaded ahead of the tensor-memory load.
                        float4 cv4[4];
                        if constexpr (NCOPY == 0) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int dlo4 = delta0 + t - (16 * ch + 4 * u) - 3;
                                cv4[u] = (biased && row_ok && dlo4 + 3 >= 0 && dlo4 < p.R)
                                             ? __ldg(reinterpret_cast<const float4*>(curve + dlo4))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                            }
                        }
                        uint32_t sv[16];
                        tmem_ld16(s_tm + 16 * ch, sv);
                        tmem_ld_wait_regs16(sv);
#pragma unroll
                        for (int e = 0; e < 16; e += 4) {
                            float w4[4] = {0.f, 0.f, 0.f, 0.f};
                            // Distances of columns c .. c+3 are dlo4+3 .. dlo4 (a 16-byte aligned
                            // group of the padded curve row).
                            const int dlo4 = delta0 + t - (16 * ch + e) - 3;
                            const bool in_curve = row_ok && dlo4 + 3 >= 0 && dlo4 < p.R;
                            if constexpr (NCOPY == 0) {
                                const float4 v = cv4[e / 4];
                                w4[0] = v.w, w4[1] = v.z, w4[2] = v.y, w4[3] = v.x;
                            } else if constexpr (kBiasTab) {
                                if constexpr (NCOPY == 4) {
                                    const float4 v = *reinterpret_cast<const float4*>(run + 16 * ch + e);
                                    w4[0] = v.x, w4[1] = v.y, w4[2] = v.z, w4[3] = v.w;
                                } else if constexpr (NCOPY == 2) {
                                    const float2 a = *reinterpret_cast<const float2*>(run + 16 * ch + e);
                                    const float2 b = *reinterpret_cast<const float2*>(run + 16 * ch + e + 2);
                                    w4[0] = a.x, w4[1] = a.y, w4[2] = b.x, w4[3] = b.y;
                                } else {
#pragma unroll
                                    for (int k = 0; k < 4; ++k) w4[k] = run[16 * ch + e + k];
                                }
                            }
                            float dl[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int c = 16 * ch + e + k;
                                const float x = fmaf(__uint_as_float(sv[e + k]), c1, fmaf(rb, w4[k], -lse2));
                                const bool vis = !edge | ((c <= hi) & (c >= lo));
                                const float pr = vis ? ex2_approx(x) : 0.0f;
                                dl[k] = pr * (__uint_as_float(dp[16 * lc + e + k]) - Di);
                                if constexpr (NCOPY > 0) dr_acc = fmaf(dl[k], w4[k], dr_acc);
                            }
                            if (NCOPY == 0 && biased && in_curve)
                                *reinterpret_cast<float4*>(dcurve + dlo4) =
                                    make_float4(tau * dl[3], tau * dl[2], tau * dl[1], tau * dl[0]);
                            pk[e / 2] = pack_bf16x2(dl[0] * ds_scale, dl[1] * ds_scale);
                            pk[e / 2 + 1] = pack_bf16x2(dl[2] * ds_scale, dl[3] * ds_scale);
                        }
                        tmem_st8(s_tm + 8 * ch + 32 * half, pk);
                    }
                };
                if constexpr (NCOPY > 0) {
                    if (biased)
                        chunks(std::true_type{});
                    else
                        chunks(std::false_type{});
                } else {
                    chunks(std::false_type{});
                }
                tmem_st_wait();
#pragma unroll
                for (int lc = 0; lc < 4; ++lc) tmem_regs_keep8(pk2[lc]);
                tc_fence_before();
                // S is double-buffered and dP(g+1) needs only dp_free(g), so a warp can
                // reach this arrival for tile g while another has yet to arrive for g-1.
                // Arrivals for two tiles must not mix in one phase: wait until phase g-1
                // (every warp's dS(g-1)) is complete before arriving for g.
                if (g > 0 && !(ok = warp_all(mbar_wait(&bars->ds_ready, (g - 1) & 1, abort_flag)))) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->ds_ready);
            }
            if (!ok) break;

            // Epilogue: dr (the two halves' partial sums added into the zeros the D kernel
            // wrote; a sum of two terms does not depend on their order) and the row of dq.
            if (NCOPY > 0 && row_ok) atomicAdd(bp.dr + row, dr_acc * tau);
            if (!(ok = warp_all(mbar_wait(&bars->dq_final, item_it & 1, abort_flag)))) break;
            tc_fence_after();
            float* dqrow = bp.dq + row * D;
#pragma unroll
            for (int c = half * D / 2; c < (half + 1) * D / 2; c += 32) {
                uint32_t v[32];
                tmem_ld32(dq_tm + c, v);
                tmem_ld_wait_regs(v);
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        st_global_v4(dqrow + c + e, v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dq_free);
        }
    }

    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}


// ------------------------------------------------------------------------- dK/dV kernel

constexpr int kBkThreads = 320;   // warps 0-7 key rows (two per TMEM lane quadrant), 8 TMA producer, 9 MMA issuer
constexpr int kBkRowWarps = 8;

template <int D>
struct BkLayout {
    static constexpr int kTile = kBM * D * 2;
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTile;
    static constexpr int kQ = kV + kTile;              // 2 stages
    static constexpr int kDO = kQ + 2 * kTile;         // 2 stages
    static constexpr int kCol = kDO + 2 * kTile;       // per-column constants, 2 buffers of [128] float4
    static constexpr int kEm = kCol + 2 * kBM * 16;    // per key-row warp: its diagonal sums by column [8][128]
    static constexpr int kDw = kEm + kBkRowWarps * kBN * 4;   // table gradient accumulator [R]
};

struct BkBars {
    uint64_t kv_full, kv_empty;
    uint64_t q_full[2], q_empty[2], do_full[2], do_empty[2];
    uint64_t sdp_full;     // S^T(s) and dP^T(s) complete
    uint64_t pd_ready;     // P^T(s) and dS^T(s) are in tensor memory
    uint64_t acc_final;    // an item's last dK / dV MMA complete
    uint64_t acc_free;     // the rows' warps have read an item's dK and dV
    uint64_t col_sync;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

// Non-reversed distance table: entry y <-> distance y - 265 (zeros outside [0, R)),
// NCOPY copies shifted by one entry; a key row's run over the 128 query columns of a
// tile is ascending.
constexpr int kBkDmin = -265;

int bk_smem_bytes(int d, int R, int ncopy) {
    const int lay = d == 64 ? BkLayout<64>::kDw : BkLayout<128>::kDw;
    return lay + ((R + 3) / 4) * 16 + tab_floats(R, ncopy) * 4 + static_cast<int>(sizeof(BkBars)) + 1024;
}

// Query tiles that see key tile kt: [qt_lo, qt_hi].
__device__ __forceinline__ void q_range(const PrefillParams& p, int kt, int& qt_lo, int& qt_hi) {
    const int k0 = kt * kBN;
    qt_lo = k0 / kBM;
    const int last_row = p.window > 0 ? min(p.T - 1, k0 + kBN - 1 + p.window - 1) : p.T - 1;
    qt_hi = last_row / kBM;
}

// Items: (b, key/value head g, key tile), heaviest (earliest) key tiles first for causal
// layers, runs of consecutive key tiles for windowed ones.
struct BkItem {
    int kt, b, g;
};
__device__ __forceinline__ int bk_items_of_cta(const PrefillParams& p) {
    if (p.contiguous) {
        const int per = (p.total_items + gridDim.x - 1) / gridDim.x;
        return max(0, min(per, p.total_items - static_cast<int>(blockIdx.x) * per));
    }
    return (p.total_items - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
}
__device__ __forceinline__ BkItem bk_item_at(const PrefillParams& p, int k) {
    BkItem it;
    if (p.contiguous) {
        const int per = (p.total_items + gridDim.x - 1) / gridDim.x;
        const int u = static_cast<int>(blockIdx.x) * per + k;
        it.kt = u % p.n_qt;
        const int rem = u / p.n_qt;
        it.g = rem % p.Hkv;
        it.b = rem / p.Hkv;
        return it;
    }
    const int u = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    const int per_kt = p.B * p.Hkv;
    it.kt = u / per_kt;
    const int rem = u - it.kt * per_kt;
    it.b = rem / p.Hkv;
    it.g = rem - it.b * p.Hkv;
    return it;
}

// Query row qt * 128 + t of head (g * G + hl): its (r, LSE, D) (zeros past T).
__device__ __forceinline__ float3 bk_col_inputs(const PrefillParams& p, const BwdTcParams& bp, const BkItem& it, int hl,
                                                int qt, int t) {
    const int i = qt * kBM + t;
    if (i >= p.T) return make_float3(0.f, 0.f, 0.f);
    const int h = it.g * p.G + hl;
    const size_t hrow = (static_cast<size_t>(it.b) * p.Hq + h) * p.T + i;
    return make_float3(__ldg(p.r + (static_cast<size_t>(it.b) * p.T + i) * p.Hq + h), __ldg(bp.lse + hrow),
                       __ldg(bp.dvec + hrow));
}

template <int D, int NCOPY>
__global__ void __launch_bounds__(kBkThreads, 1)
    bwd_dkv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const PrefillParams p, const BwdTcParams bp) {
    using L = BkLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tstride = tab_stride(p.R, NCOPY);
    const int tslot = NCOPY * tstride;
    float* dw_s = reinterpret_cast<float*>(smem + L::kDw);
    float* emit = reinterpret_cast<float*>(smem + L::kEm);
    const int dw_len = ((p.R + 3) / 4) * 4;
    float* wtab = dw_s + dw_len;
    BkBars* bars = reinterpret_cast<BkBars*>(reinterpret_cast<uint8_t*>(wtab) + tslot * 4);
    volatile int* abort_flag = &bars->abort_flag;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        mbar_init(&bars->kv_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 1);
            mbar_init(&bars->do_full[s], 1);
            mbar_init(&bars->do_empty[s], 1);
        }
        mbar_init(&bars->sdp_full, 1);
        mbar_init(&bars->pd_ready, kBkRowWarps);
        mbar_init(&bars->acc_final, 1);
        mbar_init(&bars->acc_free, kBkRowWarps);
        mbar_init(&bars->col_sync, kBkRowWarps);
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
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    const int nitems = bk_items_of_cta(p);
    // Tensor memory: S^T [0, 128) (P^T over it, packed bf16: queries 0-63 at [0, 32),
    // 64-127 at [64, 96)), dP^T [128, 256) (dS^T over it, likewise),
    // dV [256, 256 + D), dK [384, 384 + D).  Steps s run over (head of the group, query
    // tile) within an item, and across items.

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        const bool leader = elect_one();
        bool ok = true;
        int nkv = 0, ns = 0;
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const BkItem it = bk_item_at(p, item_it);
            const int k0 = it.kt * kBN;
            int qt_lo, qt_hi;
            q_range(p, it.kt, qt_lo, qt_hi);
            if (item_it > 0 && !(ok = warp_all(mbar_wait(&bars->kv_empty, (item_it - 1) & 1, abort_flag)))) break;
            if (leader) {
                mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kTile);
                for (int bx = 0; bx < D / 64; ++bx) {
                    tma_load_4d(smem + L::kK + bx * kBM * 128, &tm_k, &bars->kv_full, bx * 64, it.g, k0, it.b);
                    tma_load_4d(smem + L::kV + bx * kBM * 128, &tm_v, &bars->kv_full, bx * 64, it.g, k0, it.b);
                }
            }
            ++nkv;
            for (int hl = 0; ok && hl < p.G; ++hl) {
                const int h = it.g * p.G + hl;
                for (int qt = qt_lo; qt <= qt_hi; ++qt, ++ns) {
                    const int st = ns & 1;
                    const uint32_t ph = (ns >> 1) & 1;
                    if (!(ok = warp_all(mbar_wait(&bars->q_empty[st], ph ^ 1, abort_flag)))) break;
                    if (!(ok = warp_all(mbar_wait(&bars->do_empty[st], ph ^ 1, abort_flag)))) break;
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->q_full[st], L::kTile);
                        mbar_arrive_expect_tx(&bars->do_full[st], L::kTile);
                        for (int bx = 0; bx < D / 64; ++bx) {
                            tma_load_4d(smem + L::kQ + st * L::kTile + bx * kBM * 128, &tm_q, &bars->q_full[st],
                                        bx * 64, h, qt * kBM, it.b);
                            tma_load_4d(smem + L::kDO + st * L::kTile + bx * kBM * 128, &tm_do, &bars->do_full[st],
                                        bx * 64, h, qt * kBM, it.b);
                        }
                    }
                }
            }
        }
        if (nkv > 0) mbar_drain_wait(&bars->kv_full, (nkv - 1) & 1);
        for (int n = max(0, ns - 2); n < ns; ++n) {
            mbar_drain_wait(&bars->q_full[n & 1], (n >> 1) & 1);
            mbar_drain_wait(&bars->do_full[n & 1], (n >> 1) & 1);
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        const bool leader = elect_one();
        const uint32_t idesc_s = idesc_bf16_f32(kBM, kBM, false, false);
        const uint32_t idesc_acc = idesc_bf16_f32(kBN, D, false, true);
        const uint32_t st_tm = tmem_base, dpt_tm = tmem_base + 128, dv_tm = tmem_base + 256,
                       dk_tm = tmem_base + 384;
        const uint32_t k_addr = smem_u32(smem + L::kK), v_addr = smem_u32(smem + L::kV);
        bool ok = true;
        int ns = 0;
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const BkItem it = bk_item_at(p, item_it);
            int qt_lo, qt_hi;
            q_range(p, it.kt, qt_lo, qt_hi);
            const int nsteps = p.G * (qt_hi - qt_lo + 1);
            if (!(ok = warp_all(mbar_wait(&bars->kv_full, item_it & 1, abort_flag)))) break;
            if (item_it > 0 && !(ok = warp_all(mbar_wait(&bars->acc_free, (item_it - 1) & 1, abort_flag)))) break;
            for (int s = 0; s < nsteps; ++s, ++ns) {
                const int st = ns & 1;
                const uint32_t ph = (ns >> 1) & 1;
                const uint32_t q_addr = smem_u32(smem + L::kQ + st * L::kTile);
                const uint32_t do_addr = smem_u32(smem + L::kDO + st * L::kTile);
                if (!(ok = warp_all(mbar_wait(&bars->q_full[st], ph, abort_flag)))) break;
                if (!(ok = warp_all(mbar_wait(&bars->do_full[st], ph, abort_flag)))) break;
                tc_fence_after();
                // S^T = K Q^T and dP^T = V dO^T (keys on M, query rows on N).
                issue_qk<D>(leader, st_tm, k_addr, q_addr, idesc_s);
                issue_qk<D>(leader, dpt_tm, v_addr, do_addr, idesc_s);
                if (leader) umma_commit(&bars->sdp_full);
                if (!(ok = warp_all(mbar_wait(&bars->pd_ready, ns & 1, abort_flag)))) break;
                tc_fence_after();
                // dV += P^T dO and dK += dS^T Q: query rows on the K dimension.
                issue_acc_split<D>(leader, dv_tm, st_tm, do_addr, idesc_acc, s > 0);
                issue_acc_split<D>(leader, dk_tm, dpt_tm, q_addr, idesc_acc, s > 0);
                if (leader) {
                    umma_commit(&bars->q_empty[st]);
                    umma_commit(&bars->do_empty[st]);
                }
            }
            if (!ok) break;
            if (leader) {
                umma_commit(&bars->kv_empty);
                umma_commit(&bars->acc_final);
            }
        }
        if (leader) umma_commit(&bars->mma_done);
        mbar_drain_wait(&bars->mma_done, 0);
    } else {
        // ---------------------------------------------------------------- key rows
        const int t = threadIdx.x & (kBM - 1);   // key k0 + t of the tile (TMEM lane)
        const int half = threadIdx.x >> 7;        // columns [64 half, 64 half + 64) of each step
        const uint32_t lane_off = static_cast<uint32_t>(t & ~31) << 16;
        const uint32_t st_tm = tmem_base + lane_off, dpt_tm = tmem_base + lane_off + 128,
                       dv_tm = tmem_base + lane_off + 256, dk_tm = tmem_base + lane_off + 384;
        // Per query column {c1, rb, lse2, D}: one 16-byte load per cell, since these broadcast
        // loads bound the cell loop.  The cell's other two factors follow from them:
        // tau * scale = c1 ln 2 and tau * r = rb ln 2 (c1 = tau * scale * log2 e, rb = c1 r / scale).
        float4* col = reinterpret_cast<float4*>(smem + L::kCol);   // [2][128]
        uint32_t col_phase = 0;
        int ns = 0;
        bool ok = true;
        // Query row i0 + t's (r, LSE, D) for the next step, loaded one step ahead: steps
        // run over (item, head of the group, query tile).
        int s_item = 0, s_hl = 0, s_qt = 0;
        bool s_valid = nitems > 0;
        if (s_valid) {
            int lo, hi;
            q_range(p, bk_item_at(p, 0).kt, lo, hi);
            s_qt = lo;
        }
        float3 nxt = s_valid ? bk_col_inputs(p, bp, bk_item_at(p, 0), 0, s_qt, t) : make_float3(0.f, 0.f, 0.f);
        for (int item_it = 0; ok && item_it < nitems; ++item_it) {
            const BkItem it = bk_item_at(p, item_it);
            const int k0 = it.kt * kBN;
            const int j = k0 + t;
            const bool key_ok = j < p.T;
            int qt_lo, qt_hi;
            q_range(p, it.kt, qt_lo, qt_hi);
            for (int hl = 0; ok && hl < p.G; ++hl) {
                const int h = it.g * p.G + hl;
                // This head's table (ascending) and a zeroed dw accumulator.
                if (!(ok = tab_meet(&bars->col_sync, col_phase, abort_flag))) break;
                if (NCOPY > 0 && p.R > 0) {
                    const float* wrow = p.w + static_cast<size_t>(h) * p.R;
                    for (int x = threadIdx.x; x < tslot; x += kBkRowWarps * 32) {
                        const int cp = x / tstride;
                        const int dd = x - cp * tstride + cp + kBkDmin;
                        wtab[x] = (dd >= 0 && dd < p.R) ? __ldg(wrow + dd) : 0.0f;
                    }
                    for (int x = threadIdx.x; x < dw_len; x += kBkRowWarps * 32) dw_s[x] = 0.0f;
                }
                for (int qt = qt_lo; qt <= qt_hi; ++qt, ++ns) {
                    const int i0 = qt * kBM;
                    float4* cb = col + (ns & 1) * kBM;
                    const float3 cur = nxt;
                    {
                        // The step after this one, and its inputs in flight meanwhile.
                        if (++s_qt > qt_hi) {
                            if (++s_hl >= p.G) {
                                s_hl = 0;
                                if (++s_item >= nitems) s_valid = false;
                            }
                            if (s_valid) {
                                int lo, hi;
                                q_range(p, bk_item_at(p, s_item).kt, lo, hi);
                                s_qt = lo;
                            }
                        }
                        if (s_valid) nxt = bk_col_inputs(p, bp, bk_item_at(p, s_item), s_hl, s_qt, t);
                    }
                    {
                        // Column constants of query row i0 + t (this thread fills column t).
                        const int i = i0 + t;
                        float tau = 1.0f;
                        if (p.temp_n0 > 1) {
                            const int n = p.window > 0 ? min(i + 1, p.window) : i + 1;
                            if (n > p.temp_n0) tau = __logf(static_cast<float>(n)) * p.inv_log_n0;
                        }
                        const float c1 = p.scale_log2 * tau;
                        const float ri = cur.x;
                        // (the bank form's curve holds the whole bias: coefficient 1 / scale)
                        const float rcoef = NCOPY > 0 ? ri : 1.0f;
                        if (half == 0) cb[t] = make_float4(c1, rcoef * p.inv_scale * c1, cur.y * 1.4426950408889634f, cur.z);
                    }
                    if (!(ok = tab_meet(&bars->col_sync, col_phase, abort_flag))) break;
                    if (!(ok = warp_all(mbar_wait(&bars->sdp_full, ns & 1, abort_flag)))) break;
                    tc_fence_after();
                    const int delta0 = i0 - k0;                // distance of (key t, column c) is delta0 + c - t
                    const bool biased = delta0 - (kBN - 1) < p.R;
                    const int y0 = delta0 - t - kBkDmin;       // table entry of column 0
                    const int cp = y0 & (NCOPY - 1);
                    const float* run = wtab + cp * tstride + (y0 - cp);
                    // Query column c sees key row t iff lo <= c <= hi (dist >= 0, inside the
                    // window, query row inside the sequence, key row inside it).  Integer
                    // bounds per step, so that a cell's test is two compares and no branch.
                    int vis_lo = max(0, t - delta0);
                    int vis_hi = min(kBM - 1, p.T - 1 - i0);
                    if (p.window > 0) vis_hi = min(vis_hi, t - delta0 + p.window - 1);
                    if (!key_ok) vis_hi = -1;
                    // The bank form: query row i0 + c's curve at distance delta0 + c - t is
                    // cstep[c * cstride - (c & 7)] (rows (b, i, h) of curve_stride floats, the
                    // row of position i padded by 7 - (i & 7)).
                    const size_t cstride = static_cast<size_t>(p.Hq) * bp.curve_stride + 1;
                    const float* cstep =
                        NCOPY == 0 ? bp.curves + ((static_cast<size_t>(it.b) * p.T + i0) * p.Hq + h) * bp.curve_stride +
                                         delta0 + 7 - t
                                   : nullptr;
                    // dw: the cells of a distance lie on a diagonal (key t, column c) -> (t+1, c+1).
                    // A conveyor sums them: per column, zdw = g + (lane above's zdw), so lane 31
                    // holds a finished sum of its warp's part of one diagonal each column
                    // (stashed by column in `em`), and after the half's last column lanes 0-30
                    // hold the diagonals that leave there.  Each warp then adds 2 + 1
                    // distinct-address rows of sums to dw instead of one per cell.
                    float zdw = 0.0f;
                    float* em = emit + (threadIdx.x >> 5) * kBN;
                    // The chunk loop, compiled with the dw conveyor (a biased tile of the rank-1
                    // form) and without it, so that no warp shuffle sits under a per-cell branch.
                    // Chunks of 16 columns: with 32, the two tensor-memory loads, the packed
                    // results and the cells in flight spilled registers.
                    auto chunks = [&](auto conveyor) {
                        constexpr bool kConvey = NCOPY > 0 && decltype(conveyor)::value;
#pragma unroll 1
                        for (int ch = 4 * half; ch < 4 * half + 4; ++ch) {
                            // The bank form: this chunk's 16 curve values, loaded ahead of the
                            // tensor-memory loads so their latencies overlap (values of masked
                            // cells are not used).
                            float cw[16];
                            if constexpr (NCOPY == 0) {
#pragma unroll
                                for (int k = 0; k < 16; ++k) {
                                    const int c = 16 * ch + k, dist = delta0 + c - t;
                                    cw[k] = (biased && dist >= 0 && dist < p.R && i0 + c < p.T)
                                                ? __ldg(cstep + c * cstride - (c & 7))
                                                : 0.0f;
                                }
                            }
                            uint32_t sv[16], dv[16];
                            tmem_ld16(st_tm + 16 * ch, sv);
                            tmem_ld16(dpt_tm + 16 * ch, dv);
                            tmem_ld_wait_regs16(sv);
                            tmem_regs_fence16(dv);
                            uint32_t pp[8], pd[8];
                            // Lane 31's finished diagonal sums by column, kept in registers and
                            // stored when the chunk ends: a store per column sat between the
                            // next column's shared-memory loads and this column's sum, which
                            // chained the columns' latencies.
                            float emr[16];
#pragma unroll
                            for (int e = 0; e < 16; e += 2) {
                                float pr[2], dsv[2];
#pragma unroll
                                for (int k = 0; k < 2; ++k) {
                                    const int c = 16 * ch + e + k;
                                    const float4 a = cb[c];
                                    const bool vis = (c >= vis_lo) & (c <= vis_hi);
                                    float wv = 0.0f;
                                    if constexpr (NCOPY > 0) {
                                        if (kConvey) wv = run[c];
                                    } else {
                                        wv = cw[e + k];
                                    }
                                    const float x = fmaf(__uint_as_float(sv[e + k]), a.x, fmaf(a.y, wv, -a.z));
                                    const float pv = vis ? ex2_approx(x) : 0.0f;
                                    const float dl = pv * (__uint_as_float(dv[e + k]) - a.w);
                                    pr[k] = pv;
                                    dsv[k] = dl * (a.x * kLn2);
                                    if constexpr (kConvey) {
                                        // Every cell of a diagonal has one distance: the range
                                        // [0, R) is checked once, where the diagonal's sum is added.
                                        const float up = __shfl_up_sync(0xffffffffu, zdw, 1);
                                        zdw = fmaf(dl, a.y, lane > 0 ? up : 0.0f);   // x ln 2 at the flush
                                        emr[e + k] = zdw;
                                    }
                                }
                                pp[e / 2] = pack_bf16x2(pr[0], pr[1]);
                                pd[e / 2] = pack_bf16x2(dsv[0], dsv[1]);
                            }
                            if (kConvey && lane == 31) {
                                float4* e4 = reinterpret_cast<float4*>(em + 16 * ch);
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    e4[q] = make_float4(emr[4 * q], emr[4 * q + 1], emr[4 * q + 2], emr[4 * q + 3]);
                            }
                            tmem_st8(st_tm + 8 * ch + 32 * half, pp);
                            tmem_st8(dpt_tm + 8 * ch + 32 * half, pd);
                            // pp and pd are this loop iteration's registers: wait before reuse.
                            tmem_st_wait();
                            tmem_regs_keep8(pp);
                            tmem_regs_keep8(pd);
                        }
                    };
                    if constexpr (NCOPY > 0) {
                        if (biased)
                            chunks(std::true_type{});
                        else
                            chunks(std::false_type{});
                    } else {
                        chunks(std::false_type{});
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->pd_ready);
                    if (NCOPY > 0 && biased) {
                        // Lane 31's sums: distance delta0 + c - (32 w + 31) at column c.
                        const int dbase = delta0 - ((t & ~31) + 31);
#pragma unroll
                        for (int q = 2 * half; q < 2 * half + 2; ++q) {
                            const int d = dbase + lane + 32 * q;
                            if (d >= 0 && d < p.R) atomicAdd(dw_s + d, em[lane + 32 * q]);
                        }
                        // Diagonals leaving at the half's last column: distance delta0 + 64 half + 63 - t.
                        const int d = delta0 + 64 * half + 63 - t;
                        if (lane < 31 && d >= 0 && d < p.R) atomicAdd(dw_s + d, zdw);
                        __syncwarp();
                    }
                }
                if (!ok) break;
                // This head's table gradient from this key tile, into the output (dw_s holds
                // sums of dl rb; tau r = rb ln 2).
                if (!(ok = tab_meet(&bars->col_sync, col_phase, abort_flag))) break;
                for (int x = threadIdx.x; NCOPY > 0 && x < p.R; x += kBkRowWarps * 32)
                    if (dw_s[x] != 0.0f) atomicAdd(bp.dw + static_cast<size_t>(h) * p.R + x, dw_s[x] * kLn2);
            }
            if (!ok) break;
            // Epilogue: the key row's dk and dv (fp32).
            if (!(ok = warp_all(mbar_wait(&bars->acc_final, item_it & 1, abort_flag)))) break;
            tc_fence_after();
            const size_t krow = (static_cast<size_t>(it.b) * p.T + (key_ok ? j : 0)) * p.Hkv + it.g;
#pragma unroll 1
            for (int c = half * D / 2; c < (half + 1) * D / 2; c += 32) {
                uint32_t a[32], b[32];
                tmem_ld32(dk_tm + c, a);
                tmem_ld32(dv_tm + c, b);
                tmem_ld_wait_regs(a);
                tmem_regs_fence(b);
                if (key_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        st_global_v4(bp.dk + krow * D + c + e, a[e], a[e + 1], a[e + 2], a[e + 3]);
                        st_global_v4(bp.dv + krow * D + c + e, b[e], b[e + 1], b[e + 2], b[e + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_free);
        }
    }

    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

template <int D>
int bq_copies(int R) {
    for (int nc = 4; nc >= 1; nc >>= 1)
        if (bq_smem_bytes(D, R, nc) <= kMaxDynSmem) return nc;
    return 0;
}

template <int D, int NCOPY>
cudaError_t launch_bq(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk, const CUtensorMap& tv,
                      const PrefillParams& p, const BwdTcParams& bp, int grid, cudaStream_t stream) {
    auto kern = bwd_dq_sm100_kernel<D, NCOPY>;
    // More than half of an SM's shared memory: one CTA (and one 512-column TMEM allocation) per SM.
    const int smem = std::max(bq_smem_bytes(D, p.R, NCOPY), 120 * 1024);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kBqThreads, smem, stream>>>(tq, tdo, tk, tv, p, bp);
    return cudaGetLastError();
}

template <int D, int NCOPY>
cudaError_t launch_bk(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk, const CUtensorMap& tv,
                      const PrefillParams& p, const BwdTcParams& bp, int grid, cudaStream_t stream) {
    auto kern = bwd_dkv_sm100_kernel<D, NCOPY>;
    const int smem = std::max(bk_smem_bytes(D, p.R, NCOPY), 120 * 1024);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kBkThreads, smem, stream>>>(tq, tdo, tk, tv, p, bp);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_tc(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, const PrefillParams& p_dq, const PrefillParams& p_dkv,
                          const BwdTcParams& bp, int grid, cudaStream_t stream) {
    const long long rows = static_cast<long long>(p_dq.B) * p_dq.T * p_dq.Hq;
    constexpr int kRowsPerBlock = 256 / (D / 8);
    bwd_dvec_kernel<D><<<static_cast<unsigned>((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, stream>>>(
        bp.o, bp.dout, bp.dvec, bp.dr, p_dq.B, p_dq.T, p_dq.Hq);
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
    const int g_dq = std::min(grid, p_dq.total_items), g_dkv = std::min(grid, p_dkv.total_items);
    if (bp.curves != nullptr) {
        // The bank form: biases from the per-row curves, dL/dcurve in place of dr and dw.
        const cudaError_t e = launch_bq<D, 0>(tq, tdo, tk, tv, p_dq, bp, g_dq, stream);
        if (e != cudaSuccess) return e;
        return launch_bk<D, 0>(tq, tdo, tk, tv, p_dkv, bp, g_dkv, stream);
    }
    const int nc = bq_copies<D>(p_dq.R);
    cudaError_t e = nc == 4   ? launch_bq<D, 4>(tq, tdo, tk, tv, p_dq, bp, g_dq, stream)
                    : nc == 2 ? launch_bq<D, 2>(tq, tdo, tk, tv, p_dq, bp, g_dq, stream)
                              : launch_bq<D, 1>(tq, tdo, tk, tv, p_dq, bp, g_dq, stream);
    if (e != cudaSuccess) return e;
    return launch_bk<D, 1>(tq, tdo, tk, tv, p_dkv, bp, g_dkv, stream);
}

// ------------------------------------------------------------ bank-form gradients
// From dcv[row, d] = tau_i dl(i, i-d) (the dQ kernel's output, padded rows of S floats,
// row = (b * T + i) * Hq + h, distance d at 7 - (i & 7) + d):
//   drs[row, c]     = sum_d dcv[row, d] proj[hp, c, d]
//   dproj[hp, c, d] = sum over the rows of head group hp of rs[row, c] dcv[row, d]
// (the chain rule through curve = sum_c rs[c] proj[c, :], "Thinking Machines dropped
// RoPE", recipe step 2).
constexpr int kDrsRows = 128;    // rows of one (b, h) per block
constexpr int kDrsK = 32;        // distances per pass
constexpr int kDprojRows = 512;  // rows of one (b, h) per block
constexpr int kDprojThreads = 256;

// A GEMM tile: 128 rows x 16 functions per block, distances in passes of 32.  Each pass
// stages the rows' 32 gradient values (a warp reads whole 128-byte row segments) and
// the functions' 32 values in shared memory; each thread then owns 4 rows x 4
// functions: per distance, 4 + 1 shared-memory loads feed 16 multiply-adds.
__global__ void __launch_bounds__(128) bank_drs_kernel(const float* __restrict__ proj, const float* __restrict__ dcv,
                                                       float* __restrict__ drs, int T, int Hq, int C, int proj_heads,
                                                       int R, int S) {
    __shared__ float gs[kDrsK][kDrsRows + 1];                 // [d][row], padded rows
    __shared__ __align__(16) float ps[kDrsK][kMaxBankC];      // [d][c]
    const int iblocks = (T + kDrsRows - 1) / kDrsRows;
    const int ib = static_cast<int>(blockIdx.x) % iblocks;
    const int bh = static_cast<int>(blockIdx.x) / iblocks;
    const int h = bh % Hq, b = bh / Hq;
    const int i0 = ib * kDrsRows;
    const int tid = static_cast<int>(threadIdx.x), lane = tid & 31, warp = tid >> 5;
    const int rg = tid >> 2, cg = tid & 3;          // rows rg + 32u (u < 4), functions 4cg .. 4cg+3
    const float* pr = proj + static_cast<size_t>(proj_heads == 1 ? 0 : h) * C * R;
    const size_t row_step = static_cast<size_t>(Hq) * S;
    const float* base = dcv + ((static_cast<size_t>(b) * T + i0) * Hq + h) * S;
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.0f;
    for (int d0 = 0; d0 < R; d0 += kDrsK) {
        __syncthreads();
        // Gradient tile: warp w loads rows w, w+4, ..., lane = distance.
        for (int r = warp; r < kDrsRows; r += 4) {
            const int i = i0 + r, d = d0 + lane;
            gs[lane][r] = (i < T && d < R) ? __ldg(base + r * row_step + (7 - (i & 7)) + d) : 0.0f;
        }
        for (int x = tid; x < kDrsK * kMaxBankC; x += 128) {
            const int c = x / kDrsK, dd = x % kDrsK;
            ps[dd][c] = (c < C && d0 + dd < R) ? __ldg(pr + static_cast<size_t>(c) * R + d0 + dd) : 0.0f;
        }
        __syncthreads();
#pragma unroll 8
        for (int dd = 0; dd < kDrsK; ++dd) {
            const float4 q = *reinterpret_cast<const float4*>(&ps[dd][4 * cg]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float g = gs[dd][rg + 32 * u];
                acc[u][0] = fmaf(g, q.x, acc[u][0]), acc[u][1] = fmaf(g, q.y, acc[u][1]);
                acc[u][2] = fmaf(g, q.z, acc[u][2]), acc[u][3] = fmaf(g, q.w, acc[u][3]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + rg + 32 * u;
        if (i >= T) continue;
        float* out = drs + ((static_cast<size_t>(b) * T + i) * Hq + h) * C;
#pragma unroll
        for (int v = 0; v < 4; ++v)
            if (4 * cg + v < C) out[4 * cg + v] = acc[u][v];
    }
}

__global__ void __launch_bounds__(kDprojThreads) bank_dproj_kernel(const float* __restrict__ rs,
                                                                   const float* __restrict__ dcv,
                                                                   float* __restrict__ dproj, int T, int Hq, int C,
                                                                   int proj_heads, int R, int S) {
    __shared__ __align__(16) float rsm[kDprojRows][kMaxBankC];
    const int iblocks = (T + kDprojRows - 1) / kDprojRows;
    const int ib = static_cast<int>(blockIdx.x) % iblocks;
    const int bh = static_cast<int>(blockIdx.x) / iblocks;
    const int h = bh % Hq, b = bh / Hq;
    const int i0 = ib * kDprojRows;
    for (int x = threadIdx.x; x < kDprojRows * kMaxBankC; x += kDprojThreads) {
        const int r = x / kMaxBankC, c = x % kMaxBankC;
        const int i = i0 + r;
        rsm[r][c] = (i < T && c < C) ? __ldg(rs + ((static_cast<size_t>(b) * T + i) * Hq + h) * C + c) : 0.0f;
    }
    __syncthreads();
    const int nrows = min(kDprojRows, T - i0);
    const size_t row_step = static_cast<size_t>(Hq) * S;     // floats between rows i and i + 1
    const float* base = dcv + ((static_cast<size_t>(b) * T + i0) * Hq + h) * S;
    float* out = dproj + static_cast<size_t>(proj_heads == 1 ? 0 : h) * C * R;
    for (int d = threadIdx.x; d < R; d += kDprojThreads) {
        float acc[kMaxBankC];
#pragma unroll
        for (int c = 0; c < kMaxBankC; ++c) acc[c] = 0.0f;
#pragma unroll 4
        for (int r = 0; r < nrows; ++r) {
            const float v = __ldg(base + r * row_step + (7 - ((i0 + r) & 7)) + d);
#pragma unroll
            for (int c = 0; c < kMaxBankC; c += 4) {
                const float4 q = *reinterpret_cast<const float4*>(&rsm[r][c]);
                acc[c] = fmaf(v, q.x, acc[c]), acc[c + 1] = fmaf(v, q.y, acc[c + 1]);
                acc[c + 2] = fmaf(v, q.z, acc[c + 2]), acc[c + 3] = fmaf(v, q.w, acc[c + 3]);
            }
        }
        for (int c = 0; c < C; ++c) atomicAdd(out + static_cast<size_t>(c) * R + d, acc[c]);
    }
}

}  // namespace

bool backward_bank_tc_supported(int d) { return d == 128 || d == 64; }

cudaError_t launch_bank_grads(const float* rs, const float* proj, const float* dcv, float* drs, float* dproj, int B,
                              int T, int Hq, int C, int proj_heads, int R, int S, cudaStream_t stream) {
    if (B < 1 || T < 1 || R < 1) return cudaSuccess;
    const long long bh = static_cast<long long>(B) * Hq;
    const long long n1 = bh * ((T + kDrsRows - 1) / kDrsRows), n2 = bh * ((T + kDprojRows - 1) / kDprojRows);
    if (n1 > INT32_MAX || n2 > INT32_MAX) return cudaErrorInvalidValue;
    bank_drs_kernel<<<static_cast<unsigned>(n1), 128, 0, stream>>>(proj, dcv, drs, T, Hq, C, proj_heads, R, S);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bank_dproj_kernel<<<static_cast<unsigned>(n2), kDprojThreads, 0, stream>>>(rs, dcv, dproj, T, Hq, C, proj_heads, R,
                                                                               S);
    return cudaGetLastError();
}

bool backward_tc_supported(int d, int R) {
    if (d == 128) return bq_copies<128>(R) > 0 && bk_smem_bytes(128, R, 1) <= kMaxDynSmem;
    if (d == 64) return bq_copies<64>(R) > 0 && bk_smem_bytes(64, R, 1) <= kMaxDynSmem;
    return false;
}

cudaError_t launch_backward_sm100(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const PrefillParams& p_dq, const PrefillParams& p_dkv,
                                  const BwdTcParams& bp, int d, int grid, cudaStream_t stream) {
    if (d == 128) return launch_bwd_tc<128>(tq, tdo, tk, tv, p_dq, p_dkv, bp, grid, stream);
    if (d == 64) return launch_bwd_tc<64>(tq, tdo, tk, tv, p_dq, p_dkv, bp, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace relbias
