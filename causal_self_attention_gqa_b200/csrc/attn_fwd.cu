// attn_fwd.cu -- flash-style attention forward for sm_100a (TMA + tcgen05/TMEM), persistent.
//
// Computes, per (b, h) and query row i, O_i = sum_j softmax_j(s'_ij) v_j over the keys j
// visible to i, and LSE_i = log sum_j exp(s'_ij) (natural log), where s'_ij is the scaled
// (and optionally soft-capped) score of q'_i and k'_j: the scaled dot-product attention of
// the GPT-pretraining page ("Multihead Attention"), with the grouped-query heads and
// score soft-capping of the nanogpt-jax-181m model card ("Architecture").  The softmax is
// evaluated online over key tiles (running max and sum, rescaling the partial output),
// which reaches the same result as the row softmax up to rounding.
//
// A work item is up to two 128-row query tiles that read the same key/value head:
//   * G = Hq/Hkv >= 2: two query heads of one group at the same 128 positions, so both
//     tiles see exactly the same keys and share every K/V tile;
//   * G == 1: two consecutive 128-position tiles of one head.
// Items are numbered heaviest first.  The grid has one CTA per SM; each CTA takes items
// from an atomic counter until they run out, so the loads and first MMAs of the next item
// overlap the epilogue of the current one and no CTA setup is repeated.
// Warp roles (384 threads):
//   warp 0      producer: claims items, publishes them through a 2-slot ring, TMA-loads the
//               two Q tiles of each item and its K/V tiles into a STAGES ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 4-7   softmax and epilogue of query tile 0 (thread = row = TMEM lane)
//   warps 8-11  softmax and epilogue of query tile 1
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [384,384+D).  P_i is
// written as packed bf16 over the first 64 columns of S_i and fed to the PV MMA from TMEM.
// MMA order per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while one softmax group
// works on its scores the tensor core serves the other one.
// Epilogue: O (normalised, bf16) goes through one shared staging tile in the TMA box layout
// and leaves with tiled TMA stores; the two softmax warpgroups take turns on it.
// Over a key/value cache (chunked prefill) the Tq query rows sit at absolute positions
// qoff + i, qoff = T - Tq, against the T cached keys; the plain forward has Tq = T, qoff = 0.
// All mbarrier waits are bounded (see mbar_wait); a wait that runs out records
// CSA_ERR_DEVICE_TIMEOUT and every role unwinds, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>


#include "csa_internal.h"
#include "ptx.cuh"

namespace csa {

constexpr int kItemWords = 10;  // item ring slot: index, then the fields of FwdItem

template <int D>
struct FwdCfg {
    static constexpr int SW = (D % 64 == 0) ? 128 : 64;  // swizzle span (bytes) of a tile row
    static constexpr int AE = SW / 2;                     // bf16 elements per swizzle row
    static constexpr int NA = D / AE;                     // swizzle-atom columns per tile
    static constexpr uint32_t LAYOUT = (SW == 128) ? kLayoutSw128 : kLayoutSw64;
    static constexpr int TILE = kBM * D * 2;              // bytes of one 128 x D bf16 tile
    static constexpr int STAGES = (D == 128) ? 2 : ((D == 96) ? 3 : 4);
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + STAGES * TILE;
    static constexpr int OFF_O = OFF_V + STAGES * TILE;  // O staging for the TMA store
    static constexpr int OFF_BAR = OFF_O + TILE;
    // barriers: q_full, q_empty, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2],
    // o_full[2], o_empty[2], item_full[2], item_empty[2]
    // o_turn[2] (staging hand-off between the two warpgroups), ep_sync[2]
    static constexpr int NBAR = 2 + 3 * STAGES + 16;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    static constexpr int OFF_RING = OFF_MISC + 16;       // item ring [2][kItemWords]
    static constexpr int SMEM = OFF_RING + 2 * kItemWords * 4;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(D % AE == 0 && D % 32 == 0, "head dim");
};

struct FwdArgs {
    Problem P;
    float* lse;
    int* counter;  // work-item counter (zeroed by the call)
    int nqt;       // query tiles per (b, h)
    int pairs;     // G >= 2: head pairs per group; G == 1: tile pairs per head
    int items;     // number of work items
};

// Keys visible to query row q (absolute position qoff + q): [lo, hi] (empty when lo > hi).
__device__ __forceinline__ void row_bounds(const Problem& P, int b, int q, int& lo, int& hi) {
    if (q >= P.Tq || q < 0) {
        lo = P.T;
        hi = -1;
        return;
    }
    const int pos = q + P.qoff;
    int l = 0, h = P.causal ? min(pos, P.T - 1) : P.T - 1;
    if (P.seg_start) {  // segments only without a cache (Tq = T, qoff = 0)
        l = P.seg_start[(size_t)b * P.T + q];
        h = min(h, P.seg_end[(size_t)b * P.T + q] - 1);
    }
    if (P.window > 0) {
        l = max(l, pos - P.window + 1);
        if (!P.causal) h = min(h, pos + P.window - 1);
    }
    lo = l;
    hi = h;
}

__device__ __forceinline__ float capped_log2(float raw, const Problem& P) {
    // s' * log2(e) with s' = c * tanh(s / c), s = scale * raw
    return P.cap_log2 * tanh_approx(raw * P.cap_in);
}

// One work item.  The producer decodes it once and publishes the fields in the item ring
// (the code runs once per item, so in the consumers it would run cold, out of the
// instruction cache).
struct FwdItem {
    int b, kvh, hh[2], mm[2];
    bool two;
    int kt_begin, nkt;
};


__device__ __forceinline__ FwdItem decode_item(const FwdArgs& A, int idx) {
    const Problem& P = A.P;
    FwdItem w;
    if (P.G >= 2) {
        const int per = P.B * P.Hkv * A.pairs;
        const int m = A.nqt - 1 - idx / per;
        int rem = idx % per;
        w.b = rem / (P.Hkv * A.pairs);
        rem %= P.Hkv * A.pairs;
        w.kvh = rem / A.pairs;
        const int pg = rem % A.pairs;
        w.hh[0] = w.kvh * P.G + 2 * pg;
        w.hh[1] = (2 * pg + 1 < P.G) ? w.hh[0] + 1 : -1;
        w.mm[0] = w.mm[1] = m;
    } else {
        const int per = P.B * P.Hq;
        const int pp = A.pairs - 1 - idx / per;
        const int rem = idx % per;
        w.b = rem / P.Hq;
        w.kvh = rem % P.Hq;
        w.hh[0] = w.hh[1] = w.kvh;
        w.mm[0] = 2 * pp;
        w.mm[1] = 2 * pp + 1;
        if (w.mm[1] >= A.nqt) w.hh[1] = -1;
    }
    w.two = w.hh[1] >= 0;
    // key-tile range: union over the (one or two) query tiles; bounds are monotone in q
    int lo0, hi0, lo1, hi1;
    row_bounds(P, w.b, w.mm[0] * kBM, lo0, hi0);
    const int last = w.two ? w.mm[1] : w.mm[0];
    row_bounds(P, w.b, min(last * kBM + kBM - 1, P.Tq - 1), lo1, hi1);
    w.kt_begin = lo0 / kBN;
    w.nkt = hi1 / kBN - w.kt_begin + 1;
    return w;
}

// CM: soft-cap mode, 0 off, 1 hardware tanh (MUFU), 2 tanh series on the FMA pipe (scores
// bounded by QK-norm, see cap_series).
template <int D, int CM>
__global__ void __launch_bounds__(384, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const FwdArgs A) {
    using C = FwdCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const Problem& P = A.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;
    uint64_t* k_full = bars + 2;
    uint64_t* v_full = bars + 2 + C::STAGES;
    uint64_t* kv_empty = bars + 2 + 2 * C::STAGES;
    uint64_t* s_full = bars + 2 + 3 * C::STAGES;  // [2]
    uint64_t* p_full = s_full + 2;                 // [2]
    uint64_t* o_full = s_full + 4;                 // [2]
    uint64_t* o_empty = s_full + 6;                // [2]
    uint64_t* item_full = s_full + 8;              // [2]
    uint64_t* item_empty = s_full + 10;            // [2]
    uint64_t* o_turn = s_full + 12;                // [2] warpgroup i is done with the O staging
    uint64_t* ep_sync = s_full + 14;               // [2] warpgroup i has staged its O tile
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    volatile int* item_ring = reinterpret_cast<volatile int*>(smem + C::OFF_RING);  // [2][kItemWords]

    // the swizzled tiles need a 1024-byte aligned base; the condition is uniform over the CTA
    if ((smem_u32(smem) & 1023u) != 0) {
        if (tid == 0) atomicCAS(P.status, 0, CSA_ERR_LAUNCH);
        return;
    }
    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);   // one arrival per softmax warp
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);  // one arrival per softmax warp, O read out
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], 9);  // MMA thread + 8 softmax warps
            mbar_init(&o_turn[i], 1);
            mbar_init(&ep_sync[i], 4);
        }
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

    // next item from the ring (slot n & 1); index -1 ends the loop
    auto take_item = [&](int n, int& idx, FwdItem& w) -> bool {
        if (!mbar_wait(&item_full[n & 1], (n >> 1) & 1, abort_flag, P.status)) return false;
        const volatile int* r = item_ring + (n & 1) * kItemWords;
        idx = r[0];
        w.b = r[1];
        w.kvh = r[2];
        w.hh[0] = r[3];
        w.hh[1] = r[4];
        w.mm[0] = r[5];
        w.mm[1] = r[6];
        w.two = r[7] != 0;
        w.kt_begin = r[8];
        w.nkt = r[9];
        return true;
    };

    if (warp == 0) {
        // ================= producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int g = 0;  // key/value tiles loaded so far by this CTA
            for (int n = 0;; ++n) {
                const int idx = atomicAdd(A.counter, 1);
                const int slot = n & 1;
                if (n >= 2 && !mbar_wait(&item_empty[slot], ((n >> 1) - 1) & 1, abort_flag, P.status)) break;
                volatile int* r = item_ring + slot * kItemWords;
                FwdItem w{};
                if (idx < A.items) {
                    w = decode_item(A, idx);
                    r[0] = idx;
                    r[1] = w.b;
                    r[2] = w.kvh;
                    r[3] = w.hh[0];
                    r[4] = w.hh[1];
                    r[5] = w.mm[0];
                    r[6] = w.mm[1];
                    r[7] = w.two ? 1 : 0;
                    r[8] = w.kt_begin;
                    r[9] = w.nkt;
                } else {
                    r[0] = -1;
                }
                mbar_arrive(&item_full[slot]);
                if (idx >= A.items) break;
                // Q tiles of this item once the previous item's last S MMA has read the old ones
                if (n >= 1 && !mbar_wait(q_empty, (n - 1) & 1, abort_flag, P.status)) break;
                mbar_arrive_expect_tx(q_full, (w.two ? 2 : 1) * C::TILE);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i == 1 && !w.two) break;
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_4d(&tm_q, q_full, smem + C::OFF_Q + i * C::TILE + a * kBM * C::SW, a * C::AE,
                                    w.hh[i], w.mm[i] * kBM, w.b);
                }
                bool ok = true;
                for (int jj = 0; jj < w.nkt; ++jj, ++g) {
                    const int s = g % C::STAGES;
                    if (g >= C::STAGES && !(ok = mbar_wait(&kv_empty[s], ((g / C::STAGES) - 1) & 1, abort_flag, P.status)))
                        break;
                    const int t0 = (w.kt_begin + jj) * kBN;
                    mbar_arrive_expect_tx(&k_full[s], C::TILE);
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_4d(&tm_k, &k_full[s], smem + C::OFF_K + s * C::TILE + a * kBM * C::SW, a * C::AE,
                                    w.kvh, t0, w.b);
                    mbar_arrive_expect_tx(&v_full[s], C::TILE);
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_4d(&tm_v, &v_full[s], smem + C::OFF_V + s * C::TILE + a * kBM * C::SW, a * C::AE,
                                    w.kvh, t0, w.b);
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            // operand descriptors of the first Q tile and first K/V stage; others are offsets
            const uint64_t dq0 = sdesc(smem_u32(smem + C::OFF_Q), 16, 8 * C::SW, C::LAYOUT);
            const uint64_t dk0 = sdesc(smem_u32(smem + C::OFF_K), 16, 8 * C::SW, C::LAYOUT);
            const uint64_t dv0 = sdesc(smem_u32(smem + C::OFF_V), kBM * C::SW, 8 * C::SW, C::LAYOUT);
            constexpr uint32_t kTileU = C::TILE >> 4;
            auto issue_s = [&](int i, int s) {
                const uint32_t d = tmem + i * 128;
                const uint64_t qd = dq0 + i * kTileU, kd = dk0 + s * kTileU;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    umma_ss(d, qd + koff_kmajor<C::SW, kBM>(ks), kd + koff_kmajor<C::SW, kBM>(ks), C::IDESC_S, ks > 0);
                umma_commit(&s_full[i]);
            };
            auto issue_pv = [&](int i, int s, bool acc) {
                const uint32_t d = tmem + 256 + i * 128;
                const uint64_t vd = dv0 + s * kTileU;
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks)
                    umma_ts(d, tmem + i * 128 + ks * 8, vd + koff_mnmajor<C::SW>(ks), C::IDESC_PV,
                            (acc || ks > 0) ? 1u : 0u);
            };
            int g = 0;                // key/value tiles consumed
            int ps[2] = {0, 0};       // steps completed per tile (p_full parity)
            int no[2] = {0, 0};       // items completed per tile (o_full / o_empty parity)
            bool ok = true;
            for (int n = 0; ok; ++n) {
                int idx;
                FwdItem w;
                if (!(ok = take_item(n, idx, w))) break;
                mbar_arrive(&item_empty[n & 1]);
                if (idx < 0) break;
                if (!(ok = mbar_wait(q_full, n & 1, abort_flag, P.status) &&
                           mbar_wait(&k_full[g % C::STAGES], (g / C::STAGES) & 1, abort_flag, P.status)))
                    break;
                tc_fence_after();
                issue_s(0, g % C::STAGES);
                if (w.two) issue_s(1, g % C::STAGES);
                if (w.nkt == 1) umma_commit(q_empty);
                for (int jj = 0; ok && jj < w.nkt; ++jj, ++g) {
                    const int s = g % C::STAGES, ph = (g / C::STAGES) & 1;
                    const bool next = jj + 1 < w.nkt;
                    const int s2 = (g + 1) % C::STAGES, ph2 = ((g + 1) / C::STAGES) & 1;
                    // i is a compile-time index (unrolled), so ps[] and no[] stay in registers
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (i == 1 && !w.two) break;
                        ok = mbar_wait(&v_full[s], ph, abort_flag, P.status) &&
                             mbar_wait(&p_full[i], ps[i] & 1, abort_flag, P.status);
                        // the first PV of an item overwrites O_i: the previous epilogue must have read it
                        if (ok && jj == 0 && no[i] > 0) ok = mbar_wait(&o_empty[i], (no[i] - 1) & 1, abort_flag, P.status);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(i, s, jj > 0);
                        ++ps[i];
                        if (next) {
                            if (i == 0 && !(ok = mbar_wait(&k_full[s2], ph2, abort_flag, P.status))) break;
                            tc_fence_after();
                            issue_s(i, s2);
                        } else {
                            // tile i's output is complete with this PV: its epilogue need not
                            // wait for the other tile's last softmax
                            umma_commit(&o_full[i]);
                            ++no[i];
                        }
                    }
                    if (!ok) break;
                    if (jj + 2 == w.nkt) umma_commit(q_empty);  // the item's last S MMAs are issued
                    umma_commit(&kv_empty[s]);
                }
            }
        }
    } else if (warp >= 4) {
        // ================= softmax + epilogue, one query tile per warpgroup
        const int i = (warp >= 8) ? 1 : 0;
        const int r = tid - 128 * (i + 1);  // row in tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + i * 128;
        const uint32_t tO = tmem + lane_base + 256 + i * 128;
        int ps = 0;  // steps processed by this tile (s_full parity)
        int no = 0;  // items finished by this tile (o_full parity)
        int nt = 0;  // O-staging turns taken (warpgroup 0 goes first in every item)
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int idx = -1;
            FwdItem w;
            ok = __all_sync(0xffffffffu, take_item(n, idx, w));
            warp_arrive(&item_empty[n & 1]);
            if (!ok || idx < 0) break;
            if (i == 1 && !w.two) {
                // no second tile in this item: pass the staging turn straight back
                if (r == 0) {
                    ok = mbar_wait(&o_turn[0], nt & 1, abort_flag, P.status);
                    if (ok) mbar_arrive(&o_turn[1]);
                }
                ok = __all_sync(0xffffffffu, ok);
                ++nt;
                continue;
            }
            // selects, not w.hh[i]: a runtime index would put the item in local memory
            const int h = i ? w.hh[1] : w.hh[0];
            const int m0 = i ? w.mm[1] : w.mm[0];
            const int q = m0 * kBM + r;
            int lo, hi;
            row_bounds(P, w.b, q, lo, hi);
            float m_used = -INFINITY, l = 0.f;
            for (int jj = 0; ok && jj < w.nkt; ++jj, ++ps) {
                ok = mbar_wait(&s_full[i], ps & 1, abort_flag, P.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const int k0 = (w.kt_begin + jj) * kBN;
                uint32_t raw[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, reinterpret_cast<uint32_t(&)[32]>(raw[32 * c]));
                tmem_ld_wait();
                tmem_ld_fence(raw);
                // logits in log2 units: with the cap x = c log2(e) tanh(s / c) (computed here);
                // without it x = raw * scale_log2, so the max and the mask work on the raw
                // scores and the scale folds into the exponent's FFMA (scale > 0)
                if constexpr (CM == 1) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) raw[c] = __float_as_uint(capped_log2(__uint_as_float(raw[c]), P));
                } else if constexpr (CM == 2) {
                    const float2 cin = make_float2(P.cap_in, P.cap_in), cl2 = make_float2(P.cap_log2, P.cap_log2);
#pragma unroll
                    for (int c = 0; c < 128; c += 2) {
                        const float2 x = fmul2(
                            tanh_series2(fmul2(make_float2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), cin)),
                            cl2);
                        raw[c] = __float_as_uint(x.x);
                        raw[c + 1] = __float_as_uint(x.y);
                    }
                }
                const bool full = (k0 >= lo) && (k0 + kBN - 1 <= hi);
                const bool masked = !__all_sync(0xffffffffu, full);
                if (masked) {
                    // visible columns [a, a + span] of this tile, one unsigned compare per key (an
                    // empty row, lo > hi, masks every key)
                    const int a = (lo <= hi) ? lo - k0 : (1 << 20);
                    const unsigned span = (lo <= hi) ? (unsigned)(hi - lo) : 0u;
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if ((unsigned)(c - a) > span) raw[c] = 0xff800000u;  // -inf
                }
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < 128; c += 8) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        mx4[u] = fmax3(mx4[u], __uint_as_float(raw[c + 2 * u]), __uint_as_float(raw[c + 2 * u + 1]));
                }
                const float xmul = CM ? 1.0f : P.scale_log2;
                const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * xmul;
                // rescale only when the running max grows by more than 2^8 (exact either way:
                // O and l always share the same reference max)
                const float m_new = fmaxf(m_used, mx);
                const bool need = m_new > m_used + 8.0f;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2(m_used - m_new);  // 0 when m_used = -inf
                    m_used = m_new;
                }
                const float nbase = (m_used == -INFINITY) ? 0.f : -m_used;
                const float2 xm2 = make_float2(xmul, xmul), nb2 = make_float2(nbase, nbase);
                float2 rsa = make_float2(0.f, 0.f), rsb = make_float2(0.f, 0.f);
                // p = 2^(x - m): MUFU for most pairs; one pair in four goes to the FMA pipe so
                // both units share the work (one in two when tanh takes a MUFU slot too; none
                // when the series tanh already loads the FMA pipe).  The FMA-pipe result of a
                // masked key (x = -inf, clamped to -126) is set back to exactly 0.  One code
                // path serves full and masked tiles alike: a second, select-free copy for full
                // tiles measured 1% faster on causal rows but 12% slower where masked tiles are
                // common (windows, packed documents), through instruction-cache misses.
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 xv = ffma2(make_float2(__uint_as_float(raw[32 * c + 2 * e]),
                                                            __uint_as_float(raw[32 * c + 2 * e + 1])),
                                                xm2, nb2);
                        float2 pv;
                        if (CM == 1 ? (e & 1) == 1 : (CM == 0 && (e & 3) == 3)) {
                            pv = exp2_fma2(make_float2(fmaxf(xv.x, -126.f), fmaxf(xv.y, -126.f)));
                            if (xv.x == -INFINITY) pv.x = 0.f;
                            if (xv.y == -INFINITY) pv.y = 0.f;
                        } else {
                            pv = make_float2(ex2(xv.x), ex2(xv.y));
                        }
                        if (e & 1) rsb = fadd2(rsb, pv);
                        else rsa = fadd2(rsa, pv);
                        pk[e] = pack_bf16x2(pv.x, pv.y);
                    }
                    tmem_st16(tS + 16 * c, pk);
                }
                const float rs = (rsa.x + rsa.y) + (rsb.x + rsb.y);
                l = l * alpha + rs;
                if (jj > 0 && __any_sync(0xffffffffu, need)) {
                    // the previous PV has completed (it was issued before this S MMA)
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(tO + 32 * c, ov);
                        tmem_ld_wait();
                        tmem_ld_fence(ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st32(tO + 32 * c, ov);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                warp_arrive(&p_full[i]);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_full[i], no & 1, abort_flag, P.status));
            if (!ok) break;
            ++no;
            tc_fence_after();
            // O leaves TMEM first, then the next item's PV may overwrite it
            const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
            uint32_t pk[D / 2];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(tO + 32 * c, ov);
                tmem_ld_wait();
                tmem_ld_fence(ov);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[16 * c + e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
            }
            tc_fence_before();
            warp_arrive(&o_empty[i]);
            if (q < P.Tq)
                A.lse[((size_t)w.b * P.Hq + h) * P.Tq + q] =
                    (l > 0.f) ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
            // O goes out through one shared staging tile (TMA box layout) and tiled TMA stores;
            // the two warpgroups take turns, warpgroup 0 first
            if (i == 0) {
                if (nt > 0) ok = mbar_wait(&o_turn[1], (nt - 1) & 1, abort_flag, P.status);
            } else {
                ok = mbar_wait(&o_turn[0], nt & 1, abort_flag, P.status);
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ++nt;
#pragma unroll
            for (int v4 = 0; v4 < D / 8; ++v4) {
                const int a = (8 * v4) / C::AE, j = ((8 * v4) % C::AE) / 8;
                const int swz = (C::SW == 128) ? (r & 7) : ((r >> 1) & 3);
                *reinterpret_cast<uint4*>(smem + C::OFF_O + a * (kBM * C::SW) + r * C::SW + ((j ^ swz) * 16)) =
                    make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            }
            fence_proxy_async_smem();
            warp_arrive(&ep_sync[i]);
            ok = __all_sync(0xffffffffu, mbar_wait(&ep_sync[i], (no - 1) & 1, abort_flag, P.status));
            if (!ok) break;
            if (r == 0) {
                for (int a = 0; a < C::NA; ++a)
                    tma_store_4d(&tm_o, smem + C::OFF_O + a * kBM * C::SW, a * C::AE, h, m0 * kBM, w.b);
                bulk_commit_group();
                bulk_wait_group_read0();
                mbar_arrive(&o_turn[i]);  // staging read: the other warpgroup's turn
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
static cudaError_t launch_fwd_cap(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, float* lse, cudaStream_t st) {
    using C = FwdCfg<D>;
    const cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(k_attn_fwd<D, CM>), C::SMEM);
    if (e != cudaSuccess) return e;
    FwdArgs A;
    A.P = P;
    A.lse = lse;
    A.counter = P.counters;  // cleared together with the status word by the call
    A.nqt = (P.Tq + kBM - 1) / kBM;
    if (P.G >= 2) {
        A.pairs = (P.G + 1) / 2;
        A.items = P.B * P.Hkv * A.pairs * A.nqt;
    } else {
        A.pairs = (A.nqt + 1) / 2;
        A.items = P.B * P.Hq * A.pairs;
    }
    const int grid = A.items < num_sms() ? A.items : num_sms();
    k_attn_fwd<D, CM><<<grid, 384, C::SMEM, st>>>(tq, tk, tv, to, A);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_fwd_d(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, float* lse, cudaStream_t st) {
    if (P.softcap <= 0.f) return launch_fwd_cap<D, 0>(P, tq, tk, tv, to, lse, st);
    return P.cap_series ? launch_fwd_cap<D, 2>(P, tq, tk, tv, to, lse, st)
                        : launch_fwd_cap<D, 1>(P, tq, tk, tv, to, lse, st);
}

cudaError_t launch_fwd(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, float* lse, cudaStream_t st) {
    switch (P.D) {
        case 32: return launch_fwd_d<32>(P, tq, tk, tv, to, lse, st);
        case 64: return launch_fwd_d<64>(P, tq, tk, tv, to, lse, st);
        case 96: return launch_fwd_d<96>(P, tq, tk, tv, to, lse, st);
        case 128: return launch_fwd_d<128>(P, tq, tk, tv, to, lse, st);
        default: return cudaErrorInvalidValue;
    }
}

int fwd_swizzle_bytes(int D) { return (D % 64 == 0) ? 128 : 64; }

}  // namespace csa
