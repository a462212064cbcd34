// attn_bwd.cu -- flash-style attention backward for sm_100a (TMA + tcgen05/TMEM).
//
// The gradient of the attention of attn_fwd.cu (the pages obtain it by automatic
// differentiation of the same graph).  With P_ij = exp(s'_ij - LSE_i) recomputed from the
// forward's log-sum-exp, dP_ij = dO_i . v_j and delta_i = sum_d dO_id O_id:
//     dV_j  += sum_i P_ij dO_i
//     dS_ij  = P_ij (dP_ij - delta_i) * (1 - tanh^2(s_ij / c))      (last factor: cap only)
//     dQ'_i += scale sum_j dS_ij k'_j        dK'_j += scale sum_i dS_ij q'_i
// followed by the transposed RoPE and RMSNorm on dK' and dQ' (k_grad_finalize).
//
// One CTA owns a 128-key tile of one (b, kv head) and loops over the G query heads of the
// group and every 128-row query tile that sees those keys, so dK and dV of the group sum in
// TMEM without atomics.  dQ' tiles are added into an fp32 accumulator with vector reductions.
// Warp roles (512 threads):
//   warp 0      TMA producer: K', V once; Q', dO tiles into a 2- or 3-stage ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 4-11  P / dS computation, two warpgroups on the same key rows (thread = key row =
//               TMEM lane), queries [0,64) and [64,128); then the dV / dK' epilogue
//   warps 12-15 dQ' drain: TMEM -> fp32 reductions into the global accumulator (unscaled;
//               k_grad_finalize applies the score scale)
// TMEM (512 columns): dV [0,D), dK [128,128+D), S^T [256,384), dP^T [384,512).  P^T is
// written as packed bf16 over S^T columns (A operand of the dV MMA), dS^T likewise over
// dP^T columns (A operand of the dK' MMA); dQ' then reuses the dP^T columns.  MMA order per
// tile: dV(i) and S^T(i+1) as soon as P^T(i) is in TMEM (while the P/dS warps still form
// dS(i)), then dK'(i), dQ'(i) once dS(i) is complete, then dP^T(i+1) once the drain has read
// dQ' out of TMEM.  The P/dS warps go from dS(i) straight to P(i+1) (S^T(i+1) is ready by
// then) while dK', dQ', the drain and dP^T(i+1) run, then dS(i+1) once dP^T arrives.  dS^T also goes to shared memory (128x128 bf16, 128-byte
// swizzle), where read MN-major it is the A operand of dQ'.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "csa_internal.h"
#include "ptx.cuh"
#include "rowops.cuh"

namespace csa {

template <int D>
struct BwdCfg {
    static constexpr int SW = (D % 64 == 0) ? 128 : 64;
    static constexpr int AE = SW / 2;
    static constexpr int NA = D / AE;
    static constexpr uint32_t LAYOUT = (SW == 128) ? kLayoutSw128 : kLayoutSw64;
    static constexpr int TILE = kBM * D * 2;
    // Q'/dO ring depth: a stage is refilled only after the dQ' drain has reduced out of it, so
    // a third stage (when it fits) keeps the next tiles' loads off the critical path
    static constexpr int STAGES = (D <= 96) ? 3 : 2;
    // With two stages the Q' tile is released as soon as dK' has read it and the drain stages
    // dQ' through the dO tile alone (two rounds of D/2 columns)
    static constexpr bool SPLIT = STAGES == 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = TILE;
    static constexpr int OFF_Q = 2 * TILE;
    static constexpr int OFF_DO = OFF_Q + STAGES * TILE;
    static constexpr int OFF_DS = OFF_DO + STAGES * TILE;    // 128 x 128 bf16, SW128
    static constexpr int OFF_LSE = OFF_DS + 128 * 128 * 2;   // 2 x 128 fp32 (log2 units)
    static constexpr int OFF_DELTA = OFF_LSE + 2 * 128 * 4;  // 2 x 128 fp32
    static constexpr int OFF_BAR = OFF_DELTA + 2 * 128 * 4;
    // kv_full, q_full[STAGES], do_full[STAGES], q_empty[STAGES], do_empty[STAGES], s_full,
    // dp_full, ds_full, ds_free, dq_full, dq_empty, acc_full, wg_sync, drain_sync, epi_sync[2],
    // p_full
    static constexpr int NBAR = 1 + 4 * STAGES + 12;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);  // S^T, dP^T
    static constexpr uint32_t IDESC_KV = idesc_bf16(128, D, false, true);    // dV, dK
    static constexpr uint32_t IDESC_Q = idesc_bf16(128, D, true, true);      // dQ'
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct BwdArgs {
    Problem P;
    const float* lse;      // [B, Hq, T] natural log
    const float* delta;    // [B, Hq, T]
    float* dq_acc;         // [B, T, Hq, D] fp32, zeroed
    int nkt;  // key tiles per (b, kv head)
};

// TMEM column (relative to S^T) of P^T's packed bf16 pairs for the 16-query MMA K-step ks.
// Each softmax half writes its P^T over its own first 32 S^T columns, so neither half can
// overwrite scores the other has not read: queries [0,64) -> [0,32), [64,128) -> [64,96).
__device__ __forceinline__ uint32_t pt_col(int ks) { return 8 * ks + (ks >= 4 ? 32 : 0); }

// Queries that see key j: [lo, hi] (empty when lo > hi).
__device__ __forceinline__ void col_bounds(const Problem& P, int b, int j, int& lo, int& hi) {
    if (j >= P.T || j < 0) {
        lo = P.T;
        hi = -1;
        return;
    }
    int l = P.causal ? j : 0, h = P.T - 1;
    if (P.seg_start) {
        l = max(l, (int)P.seg_start[(size_t)b * P.T + j]);
        h = min(h, P.seg_end[(size_t)b * P.T + j] - 1);
    }
    if (P.window > 0) {
        h = min(h, j + P.window - 1);
        if (!P.causal) l = max(l, j - P.window + 1);
    }
    lo = l;
    hi = h;
}

// CM: soft-cap mode, 0 off, 1 hardware tanh (MUFU), 2 tanh series on the FMA pipe (scores
// bounded by QK-norm, see cap_series).
template <int D, int CM>
__global__ void __launch_bounds__(512, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dv,
               const __grid_constant__ CUtensorMap tm_dk, const BwdArgs A) {
    using C = BwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const Problem& P = A.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    constexpr int NS = C::STAGES;
    uint64_t* kv_full = bars + 0;
    uint64_t* q_full = bars + 1;                // [NS]
    uint64_t* do_full = bars + 1 + NS;          // [NS]
    uint64_t* q_empty = bars + 1 + 2 * NS;   // [NS]
    uint64_t* do_empty = bars + 1 + 3 * NS;  // [NS]
    uint64_t* s_full = bars + 1 + 4 * NS;
    uint64_t* dp_full = s_full + 1;
    uint64_t* ds_full = s_full + 2;
    uint64_t* ds_free = s_full + 3;
    uint64_t* dq_full = s_full + 4;
    uint64_t* dq_empty = s_full + 5;
    uint64_t* acc_full = s_full + 6;
    uint64_t* wg_sync = s_full + 7;     // the P/dS warpgroup's own barrier (bounded, unlike bar.sync)
    uint64_t* drain_sync = s_full + 8;  // the dQ drain warpgroup's own barrier
    uint64_t* epi_sync = s_full + 9;    // [2] each P/dS half's epilogue staging is complete
    uint64_t* p_full = s_full + 11;     // P^T of the current tile is in TMEM (the dV MMA's A)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* lse_s = reinterpret_cast<float*>(smem + C::OFF_LSE);
    float* delta_s = reinterpret_cast<float*>(smem + C::OFF_DELTA);

    // ---- work item: key tile n of (b, kvh); heavy (small n, causal) first
    const int n = blockIdx.x / (P.B * P.Hkv);
    const int b = (blockIdx.x % (P.B * P.Hkv)) / P.Hkv;
    const int kvh = blockIdx.x % P.Hkv;
    int m_lo, m_hi;
    {
        int lo0, hi0, lo1, hi1;
        col_bounds(P, b, n * kBN, lo0, hi0);
        col_bounds(P, b, min(n * kBN + kBN - 1, P.T - 1), lo1, hi1);
        m_lo = lo0 / kBM;
        m_hi = hi1 / kBM;
    }
    const int nm = m_hi - m_lo + 1;
    const int nit = nm > 0 ? P.G * nm : 0;

    // the swizzled tiles need a 1024-byte aligned base; the condition is uniform over the CTA
    if ((smem_u32(smem) & 1023u) != 0) {
        if (tid == 0) atomicCAS(P.status, 0, CSA_ERR_LAUNCH);
        return;
    }
    if (tid == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&do_full[s], 1);
            // MMA commit + drain (staging read by the reduce); the Q' tile holds no staging in
            // the split scheme
            mbar_init(&q_empty[s], C::SPLIT ? 1 : 2);
            mbar_init(&do_empty[s], 2);
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_full, 8);       // one arrival per P/dS warp
        mbar_init(ds_full, 8);      // one arrival per P/dS warp
        mbar_init(ds_free, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_empty, 4);     // one arrival per drain warp
        mbar_init(acc_full, 1);
        mbar_init(wg_sync, 8);
        mbar_init(drain_sync, 4);
        mbar_init(&epi_sync[0], 4);
        mbar_init(&epi_sync[1], 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0 && nit > 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
            for (int a = 0; a < C::NA; ++a) {
                tma_load_4d(&tm_k, kv_full, smem + C::OFF_K + a * kBM * C::SW, a * C::AE, kvh, n * kBN, b);
                tma_load_4d(&tm_v, kv_full, smem + C::OFF_V + a * kBM * C::SW, a * C::AE, kvh, n * kBN, b);
            }
            // iteration it is query head h of the group and query tile m (h = it / nm, m = m_lo +
            // it % nm, kept as counters: no division per iteration)
            int h = kvh * P.G, m = m_lo;
            for (int it = 0; it < nit; ++it, (++m > m_lo + nm - 1) ? (m = m_lo, ++h) : 0) {
                const int s = it % NS;
                const uint32_t ph = ((it / NS) - 1) & 1;
                if (it >= NS && !mbar_wait(&q_empty[s], ph, abort_flag, P.status)) break;
                mbar_arrive_expect_tx(&q_full[s], C::TILE);
                for (int a = 0; a < C::NA; ++a)
                    tma_load_4d(&tm_q, &q_full[s], smem + C::OFF_Q + s * C::TILE + a * kBM * C::SW, a * C::AE, h,
                                m * kBM, b);
                if (it >= NS && !mbar_wait(&do_empty[s], ph, abort_flag, P.status)) break;
                mbar_arrive_expect_tx(&do_full[s], C::TILE);
                for (int a = 0; a < C::NA; ++a)
                    tma_load_4d(&tm_do, &do_full[s], smem + C::OFF_DO + s * C::TILE + a * kBM * C::SW, a * C::AE, h,
                                m * kBM, b);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0 && nit > 0) {
            // operand descriptors, built once; each MMA adds a compile-time K-step offset
            constexpr uint32_t kTileU = C::TILE >> 4;
            const uint64_t dk_k = sdesc(smem_u32(smem + C::OFF_K), 16, 8 * C::SW, C::LAYOUT);   // K' as A (K-major)
            const uint64_t dk_mn = sdesc(smem_u32(smem + C::OFF_K), kBM * C::SW, 8 * C::SW, C::LAYOUT);  // K' as B of dQ
            const uint64_t dv_k = sdesc(smem_u32(smem + C::OFF_V), 16, 8 * C::SW, C::LAYOUT);
            const uint64_t dq_k = sdesc(smem_u32(smem + C::OFF_Q), 16, 8 * C::SW, C::LAYOUT);
            const uint64_t dq_mn = sdesc(smem_u32(smem + C::OFF_Q), kBM * C::SW, 8 * C::SW, C::LAYOUT);
            const uint64_t ddo_k = sdesc(smem_u32(smem + C::OFF_DO), 16, 8 * C::SW, C::LAYOUT);
            const uint64_t ddo_mn = sdesc(smem_u32(smem + C::OFF_DO), kBM * C::SW, 8 * C::SW, C::LAYOUT);
            const uint64_t dds_mn = sdesc(smem_u32(smem + C::OFF_DS), 128 * 128, 1024, kLayoutSw128);  // dS, A of dQ'
            auto kk = [](int ks) { return koff_kmajor<C::SW, kBM>(ks); };
            auto kmn = [](int ks) { return koff_mnmajor<C::SW>(ks); };
            const uint32_t t_dv = tmem, t_dk = tmem + 128, t_s = tmem + 256, t_dp = tmem + 384;
            // S^T = K' Q'^T and dP^T = V dO^T (M = 128 keys, N = 128 queries, K = D)
            auto issue_s = [&](int st) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_ss(t_s, dk_k + kk(ks), dq_k + st * kTileU + kk(ks), C::IDESC_S, ks > 0);
                umma_commit(s_full);
            };
            auto issue_dp = [&](int st) {
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_ss(t_dp, dv_k + kk(ks), ddo_k + st * kTileU + kk(ks), C::IDESC_S, ks > 0);
                umma_commit(dp_full);
            };
            bool ok = mbar_wait(kv_full, 0, abort_flag, P.status) && mbar_wait(&q_full[0], 0, abort_flag, P.status);
            if (ok) {
                tc_fence_after();
                issue_s(0);
                ok = mbar_wait(&do_full[0], 0, abort_flag, P.status);
                if (ok) {
                    tc_fence_after();
                    issue_dp(0);
                }
            }
            for (int it = 0; ok && it < nit; ++it) {
                const int s = it % NS;
                const bool next = it + 1 < nit;
                const int s1 = (it + 1) % NS, ph1 = ((it + 1) / NS) & 1;
                // dV needs only P^T: it (and the next S^T behind it) runs while the P/dS warps
                // are still forming dS of this tile
                if (!(ok = mbar_wait(p_full, it & 1, abort_flag, P.status))) break;
                tc_fence_after();
                // dV += P^T dO   (A = P^T from TMEM; B = dO, MN-major)
#pragma unroll
                for (int ks = 0; ks < kBM / 16; ++ks)
                    umma_ts(t_dv, t_s + pt_col(ks), ddo_mn + s * kTileU + kmn(ks), C::IDESC_KV,
                            (it > 0 || ks > 0) ? 1u : 0u);
                // S^T of the next tile right behind dV (which consumed P^T from these columns;
                // MMAs of one thread run in issue order): its P phase overlaps dK', dQ' below
                if (next) {
                    if (!(ok = mbar_wait(&q_full[s1], ph1, abort_flag, P.status))) break;
                    tc_fence_after();
                    issue_s(s1);
                }
                if (!(ok = mbar_wait(ds_full, it & 1, abort_flag, P.status))) break;
                tc_fence_after();
                // dK' += dS^T Q'  (A = dS^T from TMEM, packed over dP^T columns; B = Q', MN-major)
#pragma unroll
                for (int ks = 0; ks < kBM / 16; ++ks)
                    umma_ts(t_dk, t_dp + pt_col(ks), dq_mn + s * kTileU + kmn(ks), C::IDESC_KV,
                            (it > 0 || ks > 0) ? 1u : 0u);
                if constexpr (C::SPLIT) umma_commit(&q_empty[s]);  // last reader of this Q' tile
                // dQ' = dS K' into the dP^T columns (read by the P/dS warps before ds_full; the
                // packed dS^T there is consumed by dK', issued before).  Issued last, so dq_full
                // also means dV and dK' are done: the drain may stage into this stage's dO and
                // Q' tiles as soon as it sees dq_full.
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks)
                    umma_ss(t_dp, dds_mn + koff_mnmajor<128>(ks), dk_mn + kmn(ks), C::IDESC_Q, ks > 0);
                umma_commit(dq_full);
                umma_commit(&do_empty[s]);
                if constexpr (!C::SPLIT) umma_commit(&q_empty[s]);
                umma_commit(ds_free);  // dS read by dQ'
                if (next) {
                    // dP^T of the next tile once the drain has read dQ' out of those columns
                    if (!(ok = mbar_wait(&do_full[s1], ph1, abort_flag, P.status) &&
                               mbar_wait(dq_empty, it & 1, abort_flag, P.status)))
                        break;
                    tc_fence_after();
                    issue_dp(s1);
                }
            }
            if (ok) umma_commit(acc_full);
        }
    } else if (warp >= 4 && warp < 12) {
        // ================= P / dS, then the dK / dV epilogue.  Two warpgroups on the same key
        // rows (TMEM lanes): `half` 0 takes queries [0, 64), half 1 queries [64, 128).
        const int half = (warp >= 8) ? 1 : 0;
        const int kr = tid - 128 - 128 * half;
        const int key = n * kBN + kr;
        int lo, hi;
        col_bounds(P, b, key, lo, hi);
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + 256, t_dp = tmem + lane_base + 384;
        uint8_t* ds_row = smem + C::OFF_DS + kr * 128;
        const float kLog2e = 1.4426950408889634f;
        bool ok = nit > 0;
        // this thread's LSE (log2 units) and delta for query row kr of iteration `it`, loaded
        // from global one iteration ahead so the load latency hides behind the compute
        // (head, query tile) of an iteration advance as counters: no division per iteration
        const int m_last = m_lo + nm - 1;
        int fh = kvh * P.G, fm = m_lo;  // the iteration fetched next
        auto fetch = [&](float& l2, float& d) {
            const int q = fm * kBM + kr;
            const size_t o = ((size_t)b * P.Hq + fh) * P.T + (q < P.T ? q : 0);
            l2 = (q < P.T) ? A.lse[o] * kLog2e : INFINITY;
            d = (q < P.T) ? A.delta[o] : 0.f;
            if (++fm > m_last) {
                fm = m_lo;
                ++fh;
            }
        };
        float nl2 = INFINITY, nd = 0.f;
        if (nit > 0) fetch(nl2, nd);
        int cur_m = m_lo;
        for (int it = 0; ok && it < nit; ++it) {
            const int m = cur_m;
            cur_m = (cur_m == m_last) ? m_lo : cur_m + 1;
            const int q0 = m * kBM;
            const int buf = it & 1;
            if (half == 0) lse_s[buf * 128 + kr] = nl2;
            else delta_s[buf * 128 + kr] = nd;
            if (it + 1 < nit) fetch(nl2, nd);
            warp_arrive(wg_sync);
            ok = mbar_wait(wg_sync, it & 1, abort_flag, P.status);
            ok = ok && mbar_wait(s_full, it & 1, abort_flag, P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            // masked tile (warp-uniform): query column k is visible when k - (lo - q0) lies in
            // [0, span], one unsigned compare per entry; an empty row (lo > hi) masks them all
            const bool full = __all_sync(0xffffffffu, (q0 >= lo) && (q0 + kBM - 1 <= hi));
            const int vis0 = (lo <= hi) ? lo - q0 : (1 << 20);
            const unsigned span = (lo <= hi) ? (unsigned)(hi - lo) : 0u;
            const float* ls = lse_s + buf * 128;
            const float* dl = delta_s + buf * 128;
            // P phase (needs S^T only): P^T goes to TMEM for dV; P times the cap factor stays in
            // registers as bf16 pairs (the value dS is built from once dP^T arrives)
            uint32_t pd[2][16];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
                uint32_t sv[32];
                tmem_ld32(t_s + 32 * c, sv);
                tmem_ld_wait();
                tmem_ld_fence(sv);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(ls + 32 * c + e);
                    const float2 r01 = make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
                    const float2 r23 = make_float2(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
                    const float2 nl01 = make_float2(-l4.x, -l4.y), nl23 = make_float2(-l4.z, -l4.w);
                    float2 x01, x23, t01, t23;
                    if constexpr (CM == 0) {
                        const float2 sl2 = make_float2(P.scale_log2, P.scale_log2);
                        x01 = ffma2(r01, sl2, nl01);
                        x23 = ffma2(r23, sl2, nl23);
                    } else {
                        const float2 cin = make_float2(P.cap_in, P.cap_in), cl2 = make_float2(P.cap_log2, P.cap_log2);
                        if constexpr (CM == 1) {
                            t01 = make_float2(tanh_approx(r01.x * P.cap_in), tanh_approx(r01.y * P.cap_in));
                            t23 = make_float2(tanh_approx(r23.x * P.cap_in), tanh_approx(r23.y * P.cap_in));
                        } else {
                            t01 = tanh_series2(fmul2(r01, cin));
                            t23 = tanh_series2(fmul2(r23, cin));
                        }
                        x01 = ffma2(t01, cl2, nl01);
                        x23 = ffma2(t23, cl2, nl23);
                    }
                    float pp[4] = {ex2(x01.x), ex2(x01.y), ex2(x23.x), ex2(x23.y)};
                    if (!full) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if ((unsigned)(32 * c + e + u - vis0) > span) pp[u] = 0.f;
                    }
                    pk[e / 2] = pack_bf16x2(pp[0], pp[1]);
                    pk[e / 2 + 1] = pack_bf16x2(pp[2], pp[3]);
                    if constexpr (CM != 0) {
                        // P times the cap's derivative factor 1 - tanh^2
                        const float2 one = make_float2(1.f, 1.f);
                        const float2 f01 = fmul2(make_float2(pp[0], pp[1]), ffma2(t01, make_float2(-t01.x, -t01.y), one));
                        const float2 f23 = fmul2(make_float2(pp[2], pp[3]), ffma2(t23, make_float2(-t23.x, -t23.y), one));
                        pd[cc][e / 2] = pack_bf16x2(f01.x, f01.y);
                        pd[cc][e / 2 + 1] = pack_bf16x2(f23.x, f23.y);
                    } else {
                        pd[cc][e / 2] = pk[e / 2];
                        pd[cc][e / 2 + 1] = pk[e / 2 + 1];
                    }
                }
                tmem_st16(t_s + pt_col(2 * c), pk);  // P^T (bf16) over this half's S^T columns already read
            }
            // P^T is complete in TMEM: the dV MMA (and the next S^T behind it) may start
            tmem_st_wait();
            tc_fence_before();
            warp_arrive(p_full);
            // dS phase: dP^T of this tile, and the dS buffer free (dQ' of the last tile done)
            ok = mbar_wait(dp_full, it & 1, abort_flag, P.status);
            if (ok && it > 0) ok = mbar_wait(ds_free, (it - 1) & 1, abort_flag, P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                tmem_st_wait();
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
                uint32_t dpv[32];
                tmem_ld32(t_dp + 32 * c, dpv);
                tmem_ld_wait();
                tmem_ld_fence(dpv);
                uint32_t dk16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(dl + 32 * c + e);
                    const uint32_t w0 = pd[cc][e / 2], w1 = pd[cc][e / 2 + 1];
                    const float2 p01 = make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xffff0000u));
                    const float2 p23 = make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xffff0000u));
                    const float2 g01 = fadd2(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                             make_float2(-d4.x, -d4.y));
                    const float2 g23 = fadd2(make_float2(__uint_as_float(dpv[e + 2]), __uint_as_float(dpv[e + 3])),
                                             make_float2(-d4.z, -d4.w));
                    const float2 s01 = fmul2(p01, g01), s23 = fmul2(p23, g23);
                    dk16[e / 2] = pack_bf16x2(s01.x, s01.y);
                    dk16[e / 2 + 1] = pack_bf16x2(s23.x, s23.y);
                }
                // dS^T (bf16) over this half's dP^T columns already read: A operand of dK'
                tmem_st16(t_dp + pt_col(2 * c), dk16);
                // dS^T row kr, queries [32c, 32c+32): 4 chunks of 16 bytes, 128-byte swizzle
                // (read MN-major as the A operand of dQ')
                uint8_t* atom_row = ds_row + (c >> 1) * (128 * 128);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    const int chunk = ((c & 1) * 4 + v4) ^ (kr & 7);
                    *reinterpret_cast<uint4*>(atom_row + chunk * 16) =
                        make_uint4(dk16[4 * v4], dk16[4 * v4 + 1], dk16[4 * v4 + 2], dk16[4 * v4 + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(ds_full);
        }
        // ---- epilogue: dV, dK of this key tile (sums over the group's query heads).  Each half
        // stages its tile in shared memory that no MMA reads any more (V tile for dV; K tile,
        // then the dS buffer, for dK) in the layout of a TMA box, and one thread stores it with
        // tiled TMA stores (rows past T are not written).
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, P.status));
        if (ok) {
            tc_fence_after();
            const bool transform = P.rope || P.qk_norm;
            // 32 bf16 values (16 words) of row kr at element d0 of a bf16 tile (TMA box layout)
            auto stage_bf16 = [&](uint8_t* tile, int d0, const uint32_t* w) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int de = d0 + 8 * q;
                    const int a = de / C::AE, j = (de % C::AE) / 8;
                    const int swz = (C::SW == 128) ? (kr & 7) : ((kr >> 1) & 3);
                    *reinterpret_cast<uint4*>(tile + a * (kBM * C::SW) + kr * C::SW + ((j ^ swz) * 16)) =
                        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                }
            };
            // fp32 atoms of 16 columns x 128 rows (64-byte swizzle): the K tile holds D/32 of
            // them, the dS buffer the rest
            auto f32_atom = [&](int t) -> uint8_t* {
                return (t < D / 32) ? smem + C::OFF_K + t * 8192 : smem + C::OFF_DS + (t - D / 32) * 8192;
            };
            const uint32_t t_acc = tmem + lane_base + (half == 0 ? 0 : 128);
            const float sc = (half == 1 && !transform) ? P.scale : 1.0f;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(t_acc + 32 * c, v);
                tmem_ld_wait();
                tmem_ld_fence(v);
                if (half == 1 && transform) {  // raw fp32 dK' for the finalize kernel
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint8_t* row = f32_atom(2 * c + h2) + kr * 64;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4*>(row + ((j ^ ((kr >> 1) & 3)) * 16)) =
                                make_uint4(v[16 * h2 + 4 * j], v[16 * h2 + 4 * j + 1], v[16 * h2 + 4 * j + 2],
                                           v[16 * h2 + 4 * j + 3]);
                    }
                } else {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
                    stage_bf16(smem + (half == 0 ? C::OFF_V : C::OFF_K), 32 * c, w);
                }
            }
            fence_proxy_async_smem();
            warp_arrive(&epi_sync[half]);
            ok = __all_sync(0xffffffffu, mbar_wait(&epi_sync[half], 0, abort_flag, P.status));
            if (ok && kr == 0) {
                if (half == 0) {
                    for (int a = 0; a < C::NA; ++a)
                        tma_store_4d(&tm_dv, smem + C::OFF_V + a * kBM * C::SW, a * C::AE, kvh, n * kBN, b);
                } else if (transform) {
                    for (int t = 0; t < D / 16; ++t) tma_store_4d(&tm_dk, f32_atom(t), t * 16, kvh, n * kBN, b);
                } else {
                    for (int a = 0; a < C::NA; ++a)
                        tma_store_4d(&tm_dk, smem + C::OFF_K + a * kBM * C::SW, a * C::AE, kvh, n * kBN, b);
                }
                bulk_commit_group();
                bulk_wait_group_read0();  // the global writes complete with the grid
            }
        }
    } else if (warp >= 12) {
        // ================= dQ' drain (thread = query row of the current tile)
        // TMEM -> registers -> fp32 tile in shared memory -> TMA reduce-add into the global
        // accumulator, as boxes of 16 floats x 128 rows (8 KB) in the 64-byte swizzle.  The
        // staging space is the finished stage's dO tile (its MMAs are complete once dQ' is),
        // which holds D/2 fp32 columns, plus its Q' tile for the other half; in the split
        // scheme the Q' tile is already back with the producer and the two halves go through
        // the dO tile one after the other.  The dQ' columns are released as soon as they are
        // read; the stage once the reduce has read the staging.
        const int r = tid - 384;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_dq = tmem + lane_base + 384;  // dQ' shares the dP^T columns
        constexpr int kAtoms = D / 16;                   // 8 KB each
        constexpr int kHalf = kAtoms / 2;
        bool ok = nit > 0;
        uint32_t dph = 0;  // drain_sync phase
        auto drain_bar = [&]() -> bool {
            warp_arrive(drain_sync);
            const bool w = __all_sync(0xffffffffu, mbar_wait(drain_sync, dph, abort_flag, P.status));
            dph ^= 1u;
            return w;
        };
        // (head, query tile) of an iteration as counters: no division per iteration
        int h = kvh * P.G, m = m_lo;
        for (int it = 0; ok && it < nit; ++it, (++m > m_lo + nm - 1) ? (m = m_lo, ++h) : 0) {
            const int s = it % NS;
            const int q0 = m * kBM;
            ok = __all_sync(0xffffffffu, mbar_wait(dq_full, it & 1, abort_flag, P.status));
            if (!ok) break;
            tc_fence_after();
            // atom a < kHalf: this stage's dO tile; a >= kHalf: its Q' tile (dV and dK', their
            // readers, finished before dQ' did)
            auto atom_base = [&](int a) -> uint8_t* {
                return (a < kHalf) ? smem + C::OFF_DO + s * C::TILE + a * 8192
                                   : smem + C::OFF_Q + s * C::TILE + (a - kHalf) * 8192;
            };
            auto stage_atom = [&](int a, const uint32_t* v) {  // 16 floats of row r, 64-byte swizzle
                uint8_t* row = atom_base(a) + r * 64;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4*>(row + ((j ^ ((r >> 1) & 3)) * 16)) =
                        make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            };
            auto reduce = [&](int a0, int a1, int col0) {  // atoms [a0, a1) -> columns col0 + 16 (a - a0)
                for (int a = a0; a < a1; ++a) tma_reduce_add_4d(&tm_dq, atom_base(a), col0 + (a - a0) * 16, h, q0, b);
                bulk_commit_group();
                bulk_wait_group_read0();
            };
            if constexpr (C::SPLIT) {
                // first half straight into the dO tile, second half held in registers
#pragma unroll 1
                for (int a = 0; a < kHalf; ++a) {
                    uint32_t v[16];
                    tmem_ld16(t_dq + 16 * a, v);
                    tmem_ld_wait();
                    tmem_ld_fence(v);
                    stage_atom(a, v);
                }
                uint32_t hold[D / 2];
#pragma unroll
                for (int a = 0; a < kHalf; ++a)
                    tmem_ld16(t_dq + 16 * (kHalf + a), reinterpret_cast<uint32_t(&)[16]>(hold[16 * a]));
                tmem_ld_wait();
                tmem_ld_fence(hold);
                tc_fence_before();
                warp_arrive(dq_empty);  // every dQ' column has been read: the dP^T columns are free
                fence_proxy_async_smem();
                if (!(ok = drain_bar())) break;
                if (r == 0) reduce(0, kHalf, 0);
                if (!(ok = drain_bar())) break;  // first half read out of the dO tile
#pragma unroll
                for (int a = 0; a < kHalf; ++a) stage_atom(a, hold + 16 * a);
                fence_proxy_async_smem();
                if (!(ok = drain_bar())) break;
                if (r == 0) {
                    reduce(0, kHalf, D / 2);
                    mbar_arrive(&do_empty[s]);  // second arrival: staging read, dO tile reusable
                }
            } else {
                // the whole row in registers first: the dQ' columns (which the next dP^T MMA
                // waits for) are released after one TMEM read, before any staging
                uint32_t hold[D];
#pragma unroll
                for (int a = 0; a < kAtoms; ++a)
                    tmem_ld16(t_dq + 16 * a, reinterpret_cast<uint32_t(&)[16]>(hold[16 * a]));
                tmem_ld_wait();
                tmem_ld_fence(hold);
                tc_fence_before();
                warp_arrive(dq_empty);  // every dQ' column has been read: the dP^T columns are free
#pragma unroll
                for (int a = 0; a < kAtoms; ++a) stage_atom(a, hold + 16 * a);
                fence_proxy_async_smem();
                if (!(ok = drain_bar())) break;
                if (r == 0) {
                    reduce(0, kAtoms, 0);
                    mbar_arrive(&do_empty[s]);  // second arrivals: staging read, stage reusable
                    mbar_arrive(&q_empty[s]);
                }
            }
        }
        if (r == 0) bulk_wait_group_read0();  // the global writes complete with the grid
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int CM>
static cudaError_t launch_bwd_cap(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdv, const CUtensorMap& tdk,
                                const float* lse, const float* delta, float* dq_acc, cudaStream_t st) {
    using C = BwdCfg<D>;
    const cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(k_attn_bwd<D, CM>), C::SMEM);
    if (e != cudaSuccess) return e;
    BwdArgs A;
    A.P = P;
    A.lse = lse;
    A.delta = delta;
    A.dq_acc = dq_acc;
    A.nkt = (P.T + kBN - 1) / kBN;
    const int grid = A.nkt * P.B * P.Hkv;
    k_attn_bwd<D, CM><<<grid, 512, C::SMEM, st>>>(tq, tk, tv, tdo, tdq, tdv, tdk, A);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_bwd_d(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdv, const CUtensorMap& tdk,
                                const float* lse, const float* delta, float* dq_acc, cudaStream_t st) {
    if (P.softcap <= 0.f) return launch_bwd_cap<D, 0>(P, tq, tk, tv, tdo, tdq, tdv, tdk, lse, delta, dq_acc, st);
    return P.cap_series ? launch_bwd_cap<D, 2>(P, tq, tk, tv, tdo, tdq, tdv, tdk, lse, delta, dq_acc, st)
                        : launch_bwd_cap<D, 1>(P, tq, tk, tv, tdo, tdq, tdv, tdk, lse, delta, dq_acc, st);
}

cudaError_t launch_bwd(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdv, const CUtensorMap& tdk,
                       const float* lse, const float* delta, float* dq_acc, cudaStream_t st) {
#define CSA_BWD(d) launch_bwd_d<d>(P, tq, tk, tv, tdo, tdq, tdv, tdk, lse, delta, dq_acc, st)
    switch (P.D) {
        case 32: return CSA_BWD(32);
        case 64: return CSA_BWD(64);
        case 96: return CSA_BWD(96);
        case 128: return CSA_BWD(128);
        default: return cudaErrorInvalidValue;
    }
#undef CSA_BWD
}

}  // namespace csa
