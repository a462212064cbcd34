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
// not by the tensor cores: the work runs on the CUDA cores, split over the cache.
//   k_decode_q       q' = RoPE(RMSNorm(q)) * scale for the G * Tq rows of every (b, kv head),
//                    fp32; the rotation phase is formed and reduced in fp64 (positions reach
//                    2^20)
//   k_decode_split   one CTA per (key range, kv head, b): each warp streams 32 keys at a time
//                    (lane = key for the scores, lane = 4 dimensions for P V), online softmax
//                    in log2 units; the CTA's partial (m, l, o) goes to the workspace, and the
//                    last CTA of each (b, kv head) merges them: o = sum 2^(m_s - m) o_s / l
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "csa_internal.h"
#include "ptx.cuh"

namespace csa {

constexpr int kDecThreads = 128;  // 4 warps per CTA
constexpr int kDecKeysPerCta = 128;  // smallest key range per CTA

// ------------------------------------------------------------------ q prologue
// RoPE frequencies base^(-2d/D), d < D/2, computed on the host in fp64.
struct RopeFreq {
    double theta[64];
};

// One warp per query row (b, i, h); writes qs[b][kvh][r][d], r = (h % G) * Tq + i.
template <int D>
__global__ void __launch_bounds__(128) k_decode_q(const __nv_bfloat16* __restrict__ q, float* __restrict__ qs,
                                                  Problem P, int Tq, const RopeFreq F) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int rows = P.B * Tq * P.Hq;
    if (warp >= rows) return;  // whole warps leave together
    const int h = warp % P.Hq, i = (warp / P.Hq) % Tq, b = warp / (P.Hq * Tq);
    const __nv_bfloat16* x = q + ((size_t)(b * Tq + i) * P.Hq + h) * D;
    constexpr int kPer = D / 32;  // elements per lane: d = lane + 32 t
    float v[kPer];
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
        v[t] = __bfloat162float(x[lane + 32 * t]);
        ss += v[t] * v[t];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = P.qk_norm ? rsqrtf(ss * (1.0f / D) + P.eps) : 1.0f;
    __shared__ float row[4][D];
    float* y = row[threadIdx.x >> 5];
#pragma unroll
    for (int t = 0; t < kPer; ++t) y[lane + 32 * t] = v[t] * r;
    __syncwarp();
    if (P.rope) {
        const int pos = P.T - Tq + i;
        float out[kPer];
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
            const int d = lane + 32 * t, d2 = d % (D / 2);
            // phase pos * theta in fp64 (it reaches ~1e6 rad), reduced to [-pi, pi] with a
            // two-part 2 pi (Cody-Waite), then the fp32 sine / cosine of the remainder
            const double phi = (double)pos * F.theta[d2];
            const double k = rint(phi * 0.15915494309189535);  // 1 / (2 pi)
            const double red = fma(-k, 2.4492935982947064e-16, fma(-k, 6.283185307179586, phi));
            float sn, cs;
            sincosf((float)red, &sn, &cs);
            const float a = y[d2], bb = y[d2 + D / 2];
            out[t] = (d < D / 2) ? a * cs - bb * sn : bb * cs + a * sn;
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < kPer; ++t) y[lane + 32 * t] = out[t];
        __syncwarp();
    }
    const int G = P.G, kvh = h / G, rr = (h % G) * Tq + i, R = G * Tq;
    float* dst = qs + (((size_t)b * P.Hkv + kvh) * R + rr) * D;
#pragma unroll
    for (int t = 0; t < kPer; ++t) dst[lane + 32 * t] = y[lane + 32 * t] * P.scale;
}

// ------------------------------------------------------------------ split over the cache
struct DecArgs {
    Problem P;
    int Tq, R, splits, keys_per_split;
    const float* qs;               // [B, Hkv, R, D] q' * scale
    const __nv_bfloat16* kc;       // [B, Tk, Hkv, D]
    const __nv_bfloat16* vc;       // [B, Tk, Hkv, D]
    float* part;                   // [B, Hkv, splits, R, D + 2]: o (unnormalised), m, l
    int* done;                     // [B, Hkv] key ranges finished (zeroed by the call)
    __nv_bfloat16* o;              // [B, Tq, Hq, D]
    float* lse;                    // [B, Hq, Tq]
};

// o and LSE of one (b, kv head) from the partials of all its key ranges:
// m = max_s m_s, l = sum_s 2^(m_s - m) l_s, o = sum_s 2^(m_s - m) o_s / l.  The partials come
// from other CTAs: read through L2 (ld.global.cg), never from this SM's L1.
template <int D>
__device__ void merge_partials(const DecArgs& A, int b, int kvh) {
    const Problem& P = A.P;
    const float* src = A.part + (((size_t)b * P.Hkv + kvh) * A.splits) * A.R * (D + 2);
    for (int e = threadIdx.x; e < A.R * D; e += blockDim.x) {
        const int r = e / D, d = e % D;
        float mm = -INFINITY;
        for (int s = 0; s < A.splits; ++s) mm = fmaxf(mm, __ldcg(src + ((size_t)s * A.R + r) * (D + 2) + D));
        float acc = 0.f, ll = 0.f;
        for (int s = 0; s < A.splits; ++s) {
            const float* ps = src + ((size_t)s * A.R + r) * (D + 2);
            const float ms = __ldcg(ps + D);
            const float f = (ms == -INFINITY) ? 0.f : ex2(ms - mm);
            acc += f * __ldcg(ps + d);
            ll += f * __ldcg(ps + D + 1);
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

template <int D, int RMAX, bool CAP>
__global__ void __launch_bounds__(kDecThreads, RMAX >= 16 ? 2 : 4) k_decode_split(const DecArgs A) {
    const Problem& P = A.P;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = A.R;
    __shared__ float qsh[RMAX][D];
    __shared__ float wm[4][RMAX], wl[4][RMAX];
    __shared__ float wo[4][RMAX][D];
    const float* qsrc = A.qs + ((size_t)b * P.Hkv + kvh) * R * D;
    for (int e = threadIdx.x; e < RMAX * D; e += kDecThreads) qsh[e / D][e % D] = (e / D < R) ? qsrc[e] : 0.f;
    __syncthreads();

    const float kLog2e = 1.4426950408889634f;
    float m[RMAX], l[RMAX], acc[RMAX][4];
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[r][t] = 0.f;
    }
    const int k_begin = split * A.keys_per_split;
    const int k_end = min(P.T, k_begin + A.keys_per_split);
    const size_t row_stride = (size_t)P.Hkv * D;  // elements between consecutive cache rows
    const __nv_bfloat16* kbase = A.kc + ((size_t)b * P.T * P.Hkv + kvh) * D;
    const __nv_bfloat16* vbase = A.vc + ((size_t)b * P.T * P.Hkv + kvh) * D;
    const bool pv_lane = 4 * lane < D;  // lane owns dimensions [4 lane, 4 lane + 4) in P V

    // warps take interleaved chunks of 32 keys
    for (int k0 = k_begin + 32 * warp; k0 < k_end; k0 += 32 * 4) {
        const int key = k0 + lane;
        const bool kin = key < k_end;
        // scores of this lane's key against every row (q' rows broadcast from shared memory)
        float s[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) s[r] = 0.f;
        if (kin) {
            const uint4* kr = reinterpret_cast<const uint4*>(kbase + (size_t)key * row_stride);
#pragma unroll 4
            for (int c = 0; c < D / 8; ++c) {
                const uint4 u = kr[c];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                float kf[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = __uint_as_float(w[e] << 16);
                    kf[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
#pragma unroll
                for (int r = 0; r < RMAX; ++r)
#pragma unroll
                    for (int e = 0; e < 8; ++e) s[r] = fmaf(qsh[r][8 * c + e], kf[e], s[r]);
            }
        }
        // logits in log2 units, masked to -inf
        float x[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            int lo, hi;
            dec_bounds(P, A.Tq, r, lo, hi);
            const float v = CAP ? P.cap_log2 * tanh_approx(s[r] * (1.0f / P.softcap)) : s[r] * kLog2e;
            x[r] = (r < R && kin && key >= lo && key <= hi) ? v : -INFINITY;
        }
        // online softmax per row over this chunk
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
#pragma unroll
                for (int t = 0; t < 4; ++t) acc[r][t] *= alpha;
                m[r] = mn;
            }
        }
        // P V: key kk's probabilities broadcast from lane kk; lane owns 4 consecutive dims.
        // Value rows are fetched 8 keys at a time, so their loads are in flight together.
        const int nk = min(32, k_end - k0);
        for (int k8 = 0; k8 < nk; k8 += 8) {
            uint2 vu[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                vu[u] = make_uint2(0u, 0u);
                if (pv_lane && k8 + u < nk)
                    vu[u] = *reinterpret_cast<const uint2*>(vbase + (size_t)(k0 + k8 + u) * row_stride + 4 * lane);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float vf[4] = {__uint_as_float(vu[u].x << 16), __uint_as_float(vu[u].x & 0xffff0000u),
                                     __uint_as_float(vu[u].y << 16), __uint_as_float(vu[u].y & 0xffff0000u)};
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    const float pk = __shfl_sync(0xffffffffu, p[r], (k8 + u) & 31);
#pragma unroll
                    for (int t = 0; t < 4; ++t) acc[r][t] = fmaf(pk, vf[t], acc[r][t]);
                }
            }
        }
    }
    // merge the four warps, then the CTA's partial goes to the workspace
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (lane == 0) {
            wm[warp][r] = m[r];
            wl[warp][r] = l[r];
        }
        if (pv_lane)
#pragma unroll
            for (int t = 0; t < 4; ++t) wo[warp][r][4 * lane + t] = acc[r][t];
    }
    __syncthreads();
    float* dst = A.part + ((((size_t)b * P.Hkv + kvh) * A.splits + split) * R) * (D + 2);
    for (int e = threadIdx.x; e < R * D; e += kDecThreads) {
        const int r = e / D, d = e % D;
        float mm = -INFINITY;
        for (int w = 0; w < 4; ++w) mm = fmaxf(mm, wm[w][r]);
        float o = 0.f, ll = 0.f;
        for (int w = 0; w < 4; ++w) {
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
    // others have published their partials before counting themselves done)
    __threadfence();
    __syncthreads();
    __shared__ int last;
    if (threadIdx.x == 0) last = (atomicAdd(&A.done[b * P.Hkv + kvh], 1) == A.splits - 1) ? 1 : 0;
    __syncthreads();
    if (!last) return;
    __threadfence();
    merge_partials<D>(A, b, kvh);
}

// ------------------------------------------------------------------ host side
// Key ranges for `resident` CTAs per SM: one wave of the grid, at least 128 keys per range.
// The workspace is sized for resident = 8, the most any launch uses.
static void split_keys(const Problem& P, int resident, int& splits, int& keys_per_split) {
    const int ctas = P.B * P.Hkv;
    int s = ctas > 0 ? resident * num_sms() / ctas : 1;
    const int max_s = (P.T + kDecKeysPerCta - 1) / kDecKeysPerCta;
    s = s < 1 ? 1 : (s > max_s ? max_s : s);
    const int kps = (P.T + s - 1) / s;
    keys_per_split = (kps + 31) / 32 * 32;
    splits = (P.T + keys_per_split - 1) / keys_per_split;
}

DecodePlan decode_plan(const Problem& P, int Tq) {
    DecodePlan d;
    d.Tq = Tq;
    d.R = P.G * Tq;
    split_keys(P, 8, d.splits, d.keys_per_split);
    d.qs_bytes = (size_t)P.B * P.Hkv * d.R * P.D * sizeof(float);
    d.part_bytes = (size_t)P.B * P.Hkv * d.splits * d.R * (P.D + 2) * sizeof(float);
    d.done_bytes = (size_t)P.B * P.Hkv * sizeof(int);
    return d;
}

static DecArgs dec_args(const Problem& P, const DecodePlan& d, const float* qs, const void* kc, const void* vc,
                        float* part, int* done, void* o, float* lse) {
    DecArgs A;
    A.P = P;
    A.Tq = d.Tq;
    A.R = d.R;
    A.splits = d.splits;
    A.keys_per_split = d.keys_per_split;
    A.qs = qs;
    A.kc = static_cast<const __nv_bfloat16*>(kc);
    A.vc = static_cast<const __nv_bfloat16*>(vc);
    A.part = part;
    A.done = done;
    A.o = static_cast<__nv_bfloat16*>(o);
    A.lse = lse;
    return A;
}

// The grid is one wave: as many key ranges as the SMs hold CTAs of this instance at once
// (never more than the workspace was sized for).
template <int D, int RMAX, bool CAP>
static cudaError_t launch_split(DecArgs A, cudaStream_t st) {
    static int resident = 0;
    if (!resident) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_decode_split<D, RMAX, CAP>, kDecThreads, 0) !=
                cudaSuccess ||
            n < 1) {
            cudaGetLastError();
            n = 4;
        }
        resident = n < 8 ? n : 8;
    }
    split_keys(A.P, resident, A.splits, A.keys_per_split);
    dim3 grid(A.splits, A.P.Hkv, A.P.B);
    k_decode_split<D, RMAX, CAP><<<grid, kDecThreads, 0, st>>>(A);
    return cudaGetLastError();
}

template <int D, bool CAP>
static cudaError_t launch_split_r(const DecArgs& A, cudaStream_t st) {
    if (A.R <= 2) return launch_split<D, 2, CAP>(A, st);
    if (A.R <= 4) return launch_split<D, 4, CAP>(A, st);
    if (A.R <= 8) return launch_split<D, 8, CAP>(A, st);
    return launch_split<D, 16, CAP>(A, st);
}

#define CSA_DEC_DISPATCH(CALL)                  \
    switch (P.D) {                              \
        case 32: return CALL(32);               \
        case 64: return CALL(64);               \
        case 96: return CALL(96);               \
        case 128: return CALL(128);             \
        default: return cudaErrorInvalidValue;  \
    }

cudaError_t launch_decode_q(const Problem& P, const DecodePlan& d, const void* q, float* qs, cudaStream_t st) {
    const int rows = P.B * d.Tq * P.Hq;
    const int blocks = (rows + 3) / 4;
    RopeFreq F;
    for (int i = 0; i < P.D / 2; ++i) F.theta[i] = P.rope ? exp((-2.0 * i / P.D) * P.rope_log_base) : 0.0;
#define CALL(D_)                                                                                              \
    (k_decode_q<D_><<<blocks, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q), qs, P, d.Tq, F), cudaGetLastError())
    CSA_DEC_DISPATCH(CALL)
#undef CALL
}

cudaError_t launch_decode_split(const Problem& P, const DecodePlan& d, const float* qs, const void* kc,
                                const void* vc, float* part, int* done, void* o, float* lse, cudaStream_t st) {
    const DecArgs A = dec_args(P, d, qs, kc, vc, part, done, o, lse);
#define CALL(D_) ((P.softcap > 0.f) ? launch_split_r<D_, true>(A, st) : launch_split_r<D_, false>(A, st))
    CSA_DEC_DISPATCH(CALL)
#undef CALL
}

}  // namespace csa
