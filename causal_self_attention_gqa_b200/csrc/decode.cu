// decode.cu -- attention of a few new queries over a key/value cache (KV-cache decoding).
//
// GPT-pretraining post (dekermanjian.github.io, llm_gpt_pretrain), section "Bonus: KV Caching":
// generation feeds only the new token(s); their queries attend over the cached keys and
// values of the whole history.
// With Tk cached entries and Tq new queries, offset = Tk - Tq and query i sits at absolute
// position offset + i: it sees key j only when j <= offset + i (and, with a window W, when
// offset + i - j < W).  The cache holds keys as stored after their own QK-norm and RoPE; the
// raw queries get the norm and RoPE here, at their absolute positions (181M model card,
// "Architecture").
//
// Decoding reads the whole cache for a handful of queries, so it is bound by HBM bandwidth,
// not by the tensor cores: the arithmetic runs on the CUDA cores and the kernel is built
// around keeping the memory system busy.  One launch, k_decode, one CTA per (key range,
// kv head, b):
//   * the CTA first forms q' = RoPE(RMSNorm(q)) * scale for the R = G * Tq query rows of its
//     (b, kv head) in shared memory (fp32; the rotation angle in fp64, positions reach 2^20);
//   * a producer warp streams the range in 128-key chunks with TMA tile loads (the same
//     swizzled 128-row boxes as the attention kernels) into a ring of K/V stages, so several
//     chunks are in flight per CTA at any time;
//   * four compute warps take 32 keys of each chunk: lane = key for the scores (rows of the
//     swizzled tile read without bank conflicts, the q' rows 16 bytes at a time, packed
//     f32x2 FMAs), lane = 4 dimensions for P V (the probabilities of four keys at a time
//     read back from shared memory), online softmax in log2 units;
//   * the CTA's partial (m, l, o) goes to the workspace, and the last CTA of each
//     (b, kv head) to count itself done merges every range: o = sum 2^(m_s - m) o_s / l.
//     It also resets that counter, so the next call needs no clearing pass.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "csa_internal.h"
#include "ptx.cuh"
#include "rowops.cuh"

namespace csa {

constexpr int kDecWarps = 4;                    // compute warps; warp 4 is the TMA producer
constexpr int kDecThreads = 32 * (kDecWarps + 1);
constexpr int kDecChunk = 32 * kDecWarps;       // keys per chunk (one 128-row TMA box)

template <int D, int RMAX>
struct DecCfg {
    static constexpr int SW = (D % 64 == 0) ? 128 : 64;  // swizzle span of a tile row (bytes)
    static constexpr int AE = SW / 2;                     // bf16 elements per swizzle row
    static constexpr int NA = D / AE;                     // swizzle-atom columns per tile
    static constexpr int TILE = kDecChunk * D * 2;        // one K (or V) chunk
    // stages: enough bytes in flight per SM with two CTAs resident where they fit
    static constexpr int STAGES = (D <= 32) ? 4 : ((D <= 64) ? 3 : 2);
    static constexpr int OFF_KV = 0;                                   // [STAGES][K tile, V tile]
    static constexpr int OFF_Q = OFF_KV + STAGES * 2 * TILE;           // q' [RMAX][D] fp32
    static constexpr int OFF_WO = OFF_Q + RMAX * D * 4;                // [4][RMAX][D] fp32
    static constexpr int OFF_WML = OFF_WO + kDecWarps * RMAX * D * 4;  // m, l [4][RMAX] each
    static constexpr int OFF_PS = OFF_WML + 2 * kDecWarps * RMAX * 4;  // p of a warp's keys [4][RMAX][32]
    static constexpr int OFF_BAR = OFF_PS + kDecWarps * RMAX * 32 * 4;
    static constexpr int NBAR = 2 * STAGES;                            // full[S], empty[S]
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;                // abort flag, last flag
    static constexpr int SMEM = OFF_MISC + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(OFF_BAR % 8 == 0, "barrier alignment");
};

struct DecArgs {
    Problem P;
    int Tq, R, splits, keys_per_split;  // keys_per_split: a multiple of kDecChunk
    const __nv_bfloat16* q;             // [B, Tq, Hq, D] raw
    float* part;                        // [B, Hkv, splits, R, D + 2]: o (unnormalised), m, l
    int* done;                          // [B, Hkv] key ranges finished (zero between calls)
    __nv_bfloat16* o;                   // [B, Tq, Hq, D]
    float* lse;                         // [B, Hq, Tq]
};

// o and LSE of one (b, kv head) from the partials of all its key ranges:
// m = max_s m_s, l = sum_s 2^(m_s - m) l_s, o = sum_s 2^(m_s - m) o_s / l.  The partials come
// from other CTAs: read through L2 (ld.global.cg), never from this SM's L1, eight ranges'
// values at a time with every load issued before the first use (a range's loads do not wait
// for the previous range's).
template <int D>
__device__ void merge_partials(const DecArgs& A, int b, int kvh) {
    const Problem& P = A.P;
    const float* src = A.part + (((size_t)b * P.Hkv + kvh) * A.splits) * A.R * (D + 2);
    constexpr int kBatch = 8;
    for (int e = threadIdx.x; e < A.R * D; e += blockDim.x) {
        const int r = e / D, d = e % D;
        float mm = -INFINITY, acc = 0.f, ll = 0.f;
        for (int s0 = 0; s0 < A.splits; s0 += kBatch) {
            float ms[kBatch], os[kBatch], ls[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const float* ps = src + ((size_t)(s0 + u) * A.R + r) * (D + 2);
                const bool in = s0 + u < A.splits;
                ms[u] = in ? __ldcg(ps + D) : -INFINITY;
                os[u] = in ? __ldcg(ps + d) : 0.f;
                ls[u] = in ? __ldcg(ps + D + 1) : 0.f;
            }
            float bm = mm;
#pragma unroll
            for (int u = 0; u < kBatch; ++u) bm = fmaxf(bm, ms[u]);
            // rescale what is summed so far to the new reference max, then add this batch
            const float f0 = (mm == -INFINITY) ? 0.f : ex2(mm - bm);
            acc *= f0;
            ll *= f0;
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const float f = (ms[u] == -INFINITY) ? 0.f : ex2(ms[u] - bm);
                acc += f * os[u];
                ll += f * ls[u];
            }
            mm = bm;
        }
        const int i = r % A.Tq, h = kvh * P.G + r / A.Tq;
        A.o[((size_t)(b * A.Tq + i) * P.Hq + h) * D + d] = __float2bfloat16_rn(ll > 0.f ? acc / ll : 0.f);
        if (d == 0)
            A.lse[((size_t)b * P.Hq + h) * A.Tq + i] =
                (ll > 0.f) ? (mm + __log2f(ll)) * 0.6931471805599453f : -INFINITY;
    }
}

// Visible keys of row r (query i = r % Tq): [lo, hi].
__device__ __forceinline__ void dec_bounds(const Problem& P, int Tq, int r, int& lo, int& hi) {
    const int pos = P.T - Tq + r % Tq;
    hi = P.causal ? pos : P.T - 1;
    lo = 0;
    if (P.window > 0) {
        lo = max(0, pos - P.window + 1);
        if (!P.causal) hi = min(hi, pos + P.window - 1);
    }
}

// Byte offset of element d of row r in a swizzled 128-row tile (atoms of 128 rows x SW bytes,
// 16-byte chunk j of row r stored at chunk j ^ x(r), the pattern the TMA box writes).
template <int SW>
__device__ __forceinline__ uint32_t swz_off(int r, int d) {
    constexpr int AE = SW / 2;
    const int a = d / AE, j = (d % AE) / 8, w = d % 8;
    const int x = (SW == 128) ? (r & 7) : ((r >> 1) & 3);
    return (uint32_t)(a * (kDecChunk * SW) + r * SW + ((j ^ x) * 16) + w * 2);
}

template <int D, int RMAX, bool CAP>
__global__ void __launch_bounds__(kDecThreads) k_decode(const __grid_constant__ CUtensorMap tm_k,
                                                       const __grid_constant__ CUtensorMap tm_v, const DecArgs A,
                                                       const RopeFreq F) {
    using C = DecCfg<D, RMAX>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const Problem& P = A.P;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = A.R;
    float(*qsh)[D] = reinterpret_cast<float(*)[D]>(smem + C::OFF_Q);
    float(*wo)[RMAX][D] = reinterpret_cast<float(*)[RMAX][D]>(smem + C::OFF_WO);
    float(*wm)[RMAX] = reinterpret_cast<float(*)[RMAX]>(smem + C::OFF_WML);
    float(*wl)[RMAX] = reinterpret_cast<float(*)[RMAX]>(smem + C::OFF_WML + kDecWarps * RMAX * 4);
    float(*psh)[RMAX][32] = reinterpret_cast<float(*)[RMAX][32]>(smem + C::OFF_PS);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
    int* last = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);

    // the swizzled tiles need a 1024-byte aligned base; the condition is uniform over the CTA
    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0) atomicCAS(P.status, 0, CSA_ERR_LAUNCH);
        return;
    }
    const int k_begin = split * A.keys_per_split;
    const int k_end = min(P.T, k_begin + A.keys_per_split);
    const int nchunks = k_end > k_begin ? (k_end - k_begin + kDecChunk - 1) / kDecChunk : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecWarps);  // one arrival per compute warp
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kDecWarps) {
        // ================= producer: K and V chunks of the range into the stage ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % C::STAGES;
                if (c >= C::STAGES && !mbar_wait(&empty[s], ((c / C::STAGES) - 1) & 1, abort_flag, P.status)) break;
                const int k0 = k_begin + c * kDecChunk;
                uint8_t* kt = smem + C::OFF_KV + s * 2 * C::TILE;
                mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
                for (int a = 0; a < C::NA; ++a)
                    tma_load_4d(&tm_k, &full[s], kt + a * kDecChunk * C::SW, a * C::AE, kvh, k0, b);
                for (int a = 0; a < C::NA; ++a)
                    tma_load_4d(&tm_v, &full[s], kt + C::TILE + a * kDecChunk * C::SW, a * C::AE, kvh, k0, b);
            }
        }
    } else {
        // ================= q' of the R rows: one warp per row (rows w, w + 4, ...)
        constexpr int kPer = D / 32;  // elements per lane: d = lane + 32 t
        for (int r = warp; r < RMAX; r += kDecWarps) {
            if (r >= R) {
#pragma unroll
                for (int t = 0; t < kPer; ++t) qsh[r][lane + 32 * t] = 0.f;
                continue;
            }
            const int i = r % A.Tq, h = kvh * P.G + r / A.Tq;
            const __nv_bfloat16* x = A.q + ((size_t)(b * A.Tq + i) * P.Hq + h) * D;
            float v[kPer];
            float ss = 0.f;
#pragma unroll
            for (int t = 0; t < kPer; ++t) {
                v[t] = __bfloat162float(x[lane + 32 * t]);
                ss += v[t] * v[t];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float rn = P.qk_norm ? rsqrtf(ss * (1.0f / D) + P.eps) : 1.0f;
#pragma unroll
            for (int t = 0; t < kPer; ++t) qsh[r][lane + 32 * t] = v[t] * rn;
            __syncwarp();
            float out[kPer];
#pragma unroll
            for (int t = 0; t < kPer; ++t) {
                const int d = lane + 32 * t, d2 = d % (D / 2);
                float y = qsh[r][d];
                if (P.rope) {
                    const float2 ang = rope_angle(P.T - A.Tq + i, F.theta[d2]);
                    const float a = qsh[r][d2], bb = qsh[r][d2 + D / 2];
                    y = (d < D / 2) ? a * ang.x - bb * ang.y : bb * ang.x + a * ang.y;
                }
                out[t] = y * P.scale;
            }
            __syncwarp();
#pragma unroll
            for (int t = 0; t < kPer; ++t) qsh[r][lane + 32 * t] = out[t];
        }
        // the four compute warps share the q' rows
        named_bar_sync(1, 32 * kDecWarps);

        const float kLog2e = 1.4426950408889634f;
        float m[RMAX], l[RMAX];
        float2 acc[RMAX][2];  // dimensions 4 lane + {0, 1}, 4 lane + {2, 3}
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            m[r] = -INFINITY;
            l[r] = 0.f;
            acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
        }
        const bool pv_lane = 4 * lane < D;  // lane owns dimensions [4 lane, 4 lane + 4) in P V
        const int row = 32 * warp + lane;    // this lane's key row in every chunk (scores)
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % C::STAGES;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (c / C::STAGES) & 1, abort_flag, P.status))) break;
            const uint8_t* kt = smem + C::OFF_KV + s * 2 * C::TILE;
            const uint8_t* vt = kt + C::TILE;
            const int k0 = k_begin + c * kDecChunk + 32 * warp;  // this warp's first key
            const int key = k0 + lane;
            const bool kin = key < k_end;
            // scores of this lane's key against every row (q' rows broadcast from shared memory,
            // 16 bytes at a time; products of element pairs with packed f32x2 FMAs)
            float2 sc2[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) sc2[r] = make_float2(0.f, 0.f);
#pragma unroll 4
            for (int d8 = 0; d8 < D; d8 += 8) {
                const uint4 u = *reinterpret_cast<const uint4*>(kt + swz_off<C::SW>(row, d8));
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
                float2 kf[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    kf[e] = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xffff0000u));
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    const float4 qa = *reinterpret_cast<const float4*>(&qsh[r][d8]);
                    const float4 qb = *reinterpret_cast<const float4*>(&qsh[r][d8 + 4]);
                    sc2[r] = ffma2(make_float2(qa.x, qa.y), kf[0], sc2[r]);
                    sc2[r] = ffma2(make_float2(qa.z, qa.w), kf[1], sc2[r]);
                    sc2[r] = ffma2(make_float2(qb.x, qb.y), kf[2], sc2[r]);
                    sc2[r] = ffma2(make_float2(qb.z, qb.w), kf[3], sc2[r]);
                }
            }
            float sc[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) sc[r] = sc2[r].x + sc2[r].y;
            // logits in log2 units, masked to -inf
            float x[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                int lo, hi;
                dec_bounds(P, A.Tq, r, lo, hi);
                const float v = CAP ? P.cap_log2 * tanh_approx(sc[r] * (1.0f / P.softcap)) : sc[r] * kLog2e;
                x[r] = (r < R && kin && key >= lo && key <= hi) ? v : -INFINITY;
            }
            // online softmax per row over this warp's 32 keys
            float p[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) {
                float cm = x[r];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
                const float mn = fmaxf(m[r], cm);
                const float alpha = (m[r] == -INFINITY) ? 0.f : ex2(m[r] - mn);
                p[r] = (x[r] == -INFINITY) ? 0.f : ex2(x[r] - mn);
                float ps = p[r];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                if (mn != -INFINITY) {
                    l[r] = l[r] * alpha + ps;
                    const float2 a2 = make_float2(alpha, alpha);
                    acc[r][0] = fmul2(acc[r][0], a2);
                    acc[r][1] = fmul2(acc[r][1], a2);
                    m[r] = mn;
                }
                psh[warp][r][lane] = p[r];
            }
            __syncwarp();
            // P V: lane owns 4 consecutive dims; the probabilities of four keys at a time are
            // read back from shared memory (keys past the range have p = 0 and finite rows)
            const int nk4 = (max(0, min(32, k_end - k0)) + 3) & ~3;
            if (pv_lane) {
#pragma unroll 2
                for (int k4 = 0; k4 < nk4; k4 += 4) {
                    float4 p4[RMAX];
#pragma unroll
                    for (int r = 0; r < RMAX; ++r) p4[r] = *reinterpret_cast<const float4*>(&psh[warp][r][k4]);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint2 vu = *reinterpret_cast<const uint2*>(vt + swz_off<C::SW>(32 * warp + k4 + u, 4 * lane));
                        const float2 v01 = make_float2(__uint_as_float(vu.x << 16), __uint_as_float(vu.x & 0xffff0000u));
                        const float2 v23 = make_float2(__uint_as_float(vu.y << 16), __uint_as_float(vu.y & 0xffff0000u));
#pragma unroll
                        for (int r = 0; r < RMAX; ++r) {
                            const float pk = (u == 0) ? p4[r].x : (u == 1) ? p4[r].y : (u == 2) ? p4[r].z : p4[r].w;
                            const float2 pk2 = make_float2(pk, pk);
                            acc[r][0] = ffma2(pk2, v01, acc[r][0]);
                            acc[r][1] = ffma2(pk2, v23, acc[r][1]);
                        }
                    }
                }
            }
            __syncwarp();            // psh is rewritten by the next chunk
            warp_arrive(&empty[s]);  // this warp is done with the stage
        }
        // this warp's partial to shared memory
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            if (lane == 0) {
                wm[warp][r] = m[r];
                wl[warp][r] = l[r];
            }
            if (pv_lane)
                *reinterpret_cast<float4*>(&wo[warp][r][4 * lane]) =
                    make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
        }
    }
    __syncthreads();
    if (*abort_flag) return;  // a bounded wait ran out: the status word says so, nothing merges
    // merge the four warps; the CTA's partial goes to the workspace
    float* dst = A.part + ((((size_t)b * P.Hkv + kvh) * A.splits + split) * R) * (D + 2);
    for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
        const int r = e / D, d = e % D;
        float mm = -INFINITY;
        for (int w = 0; w < kDecWarps; ++w) mm = fmaxf(mm, wm[w][r]);
        float o = 0.f, ll = 0.f;
        for (int w = 0; w < kDecWarps; ++w) {
            const float f = (wm[w][r] == -INFINITY) ? 0.f : ex2(wm[w][r] - mm);
            o += f * wo[w][r][d];
            ll += f * wl[w][r];
        }
        dst[(size_t)r * (D + 2) + d] = o;
        if (d == 0) {
            dst[(size_t)r * (D + 2) + D] = mm;
            dst[(size_t)r * (D + 2) + D + 1] = ll;
        }
    }
    // the last CTA of this (b, kv head) to finish merges every key range (no waiting: the
    // others have published their partials before counting themselves done), then resets
    // the counter for the next call
    __threadfence();
    __syncthreads();
    int* cnt = &A.done[b * P.Hkv + kvh];
    if (threadIdx.x == 0) *last = (atomicAdd(cnt, 1) == A.splits - 1) ? 1 : 0;
    __syncthreads();
    if (!*last) return;
    __threadfence();
    merge_partials<D>(A, b, kvh);
    if (threadIdx.x == 0) *cnt = 0;
}

// ------------------------------------------------------------------ host side
// Key ranges (multiples of the 128-key chunk) for `resident` CTAs per SM: one wave of the
// grid.  The workspace is sized for resident = 8, more than any launch uses.
static void split_keys(const Problem& P, int resident, int& splits, int& keys_per_split) {
    const int ctas = P.B * P.Hkv;
    int s = ctas > 0 ? resident * num_sms() / ctas : 1;
    const int max_s = (P.T + kDecChunk - 1) / kDecChunk;
    s = s < 1 ? 1 : (s > max_s ? max_s : s);
    const int kps = (P.T + s - 1) / s;
    keys_per_split = (kps + kDecChunk - 1) / kDecChunk * kDecChunk;
    splits = (P.T + keys_per_split - 1) / keys_per_split;
}

DecodePlan decode_plan(const Problem& P, int Tq) {
    DecodePlan d;
    d.Tq = Tq;
    d.R = P.G * Tq;
    split_keys(P, 8, d.splits, d.keys_per_split);
    d.part_bytes = (size_t)P.B * P.Hkv * d.splits * d.R * (P.D + 2) * sizeof(float);
    d.done_bytes = (size_t)P.B * P.Hkv * sizeof(int);
    return d;
}

template <int D, int RMAX, bool CAP>
static cudaError_t launch_dec(DecArgs A, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
    using C = DecCfg<D, RMAX>;
    const void* fn = reinterpret_cast<const void*>(k_decode<D, RMAX, CAP>);
    cudaError_t e = ensure_dyn_smem(fn, C::SMEM);
    if (e != cudaSuccess) return e;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_decode<D, RMAX, CAP>, kDecThreads, C::SMEM) !=
            cudaSuccess ||
        n < 1) {
        cudaGetLastError();
        n = 1;
    }
    split_keys(A.P, n < 8 ? n : 8, A.splits, A.keys_per_split);
    const RopeFreq F = rope_freq(D, A.P.rope_log_base);
    dim3 grid(A.splits, A.P.Hkv, A.P.B);
    k_decode<D, RMAX, CAP><<<grid, kDecThreads, C::SMEM, st>>>(tk, tv, A, F);
    return cudaGetLastError();
}

template <int D, bool CAP>
static cudaError_t launch_dec_r(const DecArgs& A, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
    if (A.R <= 2) return launch_dec<D, 2, CAP>(A, tk, tv, st);
    if (A.R <= 4) return launch_dec<D, 4, CAP>(A, tk, tv, st);
    if (A.R <= 8) return launch_dec<D, 8, CAP>(A, tk, tv, st);
    return launch_dec<D, 16, CAP>(A, tk, tv, st);
}

cudaError_t launch_decode(const Problem& P, const DecodePlan& d, const void* q, const CUtensorMap& tk,
                          const CUtensorMap& tv, float* part, int* done, void* o, float* lse, cudaStream_t st) {
    DecArgs A;
    A.P = P;
    A.Tq = d.Tq;
    A.R = d.R;
    A.splits = d.splits;
    A.keys_per_split = d.keys_per_split;
    A.q = static_cast<const __nv_bfloat16*>(q);
    A.part = part;
    A.done = done;
    A.o = static_cast<__nv_bfloat16*>(o);
    A.lse = lse;
#define CALL(D_) ((P.softcap > 0.f) ? launch_dec_r<D_, true>(A, tk, tv, st) : launch_dec_r<D_, false>(A, tk, tv, st))
    switch (P.D) {
        case 32: return CALL(32);
        case 64: return CALL(64);
        case 96: return CALL(96);
        case 128: return CALL(128);
        default: return cudaErrorInvalidValue;
    }
#undef CALL
}

}  // namespace csa
