// rows.cu -- the HBM-bound row kernels around the two attention kernels:
//   k_prep         segment bounds of every token (maximal runs of equal segment_ids); only
//                  launched when segment_ids are given
//   k_qk_prologue  q' = RoPE(RMSNorm(q)), k' = RoPE(RMSNorm(k)) -> bf16 copies in the workspace
//   k_bwd_pre      delta_i = sum_d dO_id O_id per (b, h, i) and a zeroed fp32 dQ accumulator
//   k_grad_finalize dq (and dk when QK-norm or RoPE is on) = RMSNorm^T(RoPE^T(scale * acc))
//                  -> bf16, from the fp32 dQ' accumulator and the raw dK' sums
// The RoPE angle of position p and frequency theta_d = base^(-2d/D) is formed in the kernels
// (fp64 phase, reduced, fp32 sine / cosine: rope_angle), once per token and frequency.
//
// The norm is the parameter-free RMSNorm and the rotation the rotate-half RoPE of the
// nanogpt-jax-181m model card ("Architecture"); positions restart at each packed segment
// (same section, "RoPE frequencies are computed from packed segment positions").
//
// The prologue and the finalize give each token an aligned group of lanes that walks over
// the token's heads; a lane owns whole rotation pairs (d, d + D/2), so a rotation never
// crosses lanes.
#include <cuda_bf16.h>
#include <stdint.h>

#include "csa_internal.h"
#include "rowops.cuh"

namespace csa {

// ------------------------------------------------------------------ segment bounds
template <bool kMax>
__device__ __forceinline__ int block_scan_1024(int v, int* sh) {
    // inclusive scan (max or min) across the 1024 threads of the block, in thread order
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v = kMax ? max(v, n) : min(v, n);
    }
    if (lane == 31) sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w = kMax ? max(w, n) : min(w, n);
        }
        sh[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v = kMax ? max(v, sh[warp - 1]) : min(v, sh[warp - 1]);
    __syncthreads();
    return v;
}

// One block per batch row: seg_start[t] = first index of t's maximal run of equal ids (a
// running max of run-start indices), seg_end[t] = one past its last index (a running min,
// from the right, of run ends).
__global__ void __launch_bounds__(1024) k_prep(int T, const int32_t* __restrict__ ids, int32_t* __restrict__ seg_start,
                                               int32_t* __restrict__ seg_end) {
    __shared__ int sh[32];
    const int b = blockIdx.x;
    const int32_t* id = ids + (size_t)b * T;
    int carry = 0;
    for (int base = 0; base < T; base += 1024) {
        const int t = base + threadIdx.x;
        int v = -1;
        if (t < T) v = (t == 0 || id[t] != id[t - 1]) ? t : -1;
        v = block_scan_1024<true>(v, sh);
        v = max(v, carry);
        if (t < T) seg_start[(size_t)b * T + t] = v;
        if (threadIdx.x == 1023) sh[0] = v;
        __syncthreads();
        carry = sh[0];
        __syncthreads();
    }
    carry = T;
    for (int top = T - 1; top >= 0; top -= 1024) {
        const int t = top - (int)threadIdx.x;
        int v = T;
        if (t >= 0) v = (t == T - 1 || id[t] != id[t + 1]) ? t + 1 : T;
        v = block_scan_1024<false>(v, sh);
        v = min(v, carry);
        if (t >= 0) seg_end[(size_t)b * T + t] = v;
        if (threadIdx.x == 1023) sh[0] = v;
        __syncthreads();
        carry = sh[0];
        __syncthreads();
    }
}

// ------------------------------------------------------------------ q/k prologue
// A group of GS lanes owns one token (b, t) and walks over all of its query heads, then its
// key heads (4 head rows in flight per lane).  A lane owns the 8 rotation pairs
// (d, d + D/2) for d in [8g, 8g + 8): its loads and stores are 16 bytes wide, and it forms the
// RoPE angle of those 8 frequencies once for the token, whatever the number of heads.  The
// D/16 active lanes of a token form an aligned group of GS lanes (a power of two; D = 96
// leaves 2 of 8 idle).
template <int D>
struct TokGeom {
    static constexpr int LPR = D / 16;
    static constexpr int GS = (LPR <= 2) ? 2 : (LPR <= 4 ? 4 : 8);
    static constexpr int TOK = 128 / GS;  // tokens per 128-thread block
};

// Normalises and rotates H head rows of one token: x, y point at the token's first head.
template <int D>
__device__ __forceinline__ void prologue_heads(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                               int H, bool active, int d0, const float (&cs)[8], const float (&sn)[8],
                                               const Problem& P) {
    using G = TokGeom<D>;
    constexpr int kHalf = D / 2;
    constexpr int kIn = 4;  // head rows in flight
    for (int h0 = 0; h0 < H; h0 += kIn) {  // H is the same for every lane of the warp
        float lo[kIn][8], hi[kIn][8];
#pragma unroll
        for (int j = 0; j < kIn; ++j) {
            if (active && h0 + j < H) {
                load_bf16x8(x + (size_t)(h0 + j) * D + d0, lo[j]);
                load_bf16x8(x + (size_t)(h0 + j) * D + kHalf + d0, hi[j]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) lo[j][i] = hi[j][i] = 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < kIn; ++j) {
            float rs = 1.0f;
            if (P.qk_norm) {
                float ss = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) ss += lo[j][i] * lo[j][i] + hi[j][i] * hi[j][i];
                ss = group_sum<G::GS>(ss);
                rs = rsqrtf(ss * (1.0f / D) + P.eps);
            }
            if (!active || h0 + j >= H) continue;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a = lo[j][i] * rs, bb = hi[j][i] * rs;
                lo[j][i] = a * cs[i] - bb * sn[i];
                hi[j][i] = bb * cs[i] + a * sn[i];
            }
            store_bf16x8(y + (size_t)(h0 + j) * D + d0, lo[j]);
            store_bf16x8(y + (size_t)(h0 + j) * D + kHalf + d0, hi[j]);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(128, 7) k_qk_prologue(const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ k,
                                                     __nv_bfloat16* __restrict__ qo, __nv_bfloat16* __restrict__ ko,
                                                     Problem P, const RopeFreq F, uint32_t tokens) {
    using G = TokGeom<D>;
    const int g = threadIdx.x & (G::GS - 1);
    const uint32_t tok_raw = blockIdx.x * (uint32_t)G::TOK + threadIdx.x / G::GS;  // b * Tq + t
    // no early return: every lane of the warp takes part in the group shuffles
    const bool valid = tok_raw < tokens;
    const uint32_t tok = valid ? tok_raw : 0;
    const bool active = valid && g < G::LPR;
    const int d0 = 8 * (active ? g : 0);
    float cs[8], sn[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        cs[i] = 1.f;
        sn[i] = 0.f;
    }
    if (P.rope && active) {
        const uint32_t b = fastdiv(tok, P.div_tq);
        const int t = (int)(tok - b * (uint32_t)P.Tq);
        // queries over a cache sit at qoff + t; segments only come without a cache (Tq = T)
        const int pos = P.seg_start ? t - P.seg_start[tok] : t + P.qoff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 a = rope_angle(pos, F.theta[d0 + i]);
            cs[i] = a.x;
            sn[i] = a.y;
        }
    }
    prologue_heads<D>(q + (size_t)tok * P.Hq * D, qo + (size_t)tok * P.Hq * D, P.Hq, active, d0, cs, sn, P);
    // keys: same tokens (a key tensor is only passed without a cache, where Tq = T and qoff = 0)
    if (k) prologue_heads<D>(k + (size_t)tok * P.Hkv * D, ko + (size_t)tok * P.Hkv * D, P.Hkv, active, d0, cs, sn, P);
}

// ------------------------------------------------------------------ backward preprocess
template <int D>
__global__ void __launch_bounds__(256) k_bwd_pre(const __nv_bfloat16* __restrict__ o,
                                                 const __nv_bfloat16* __restrict__ dout, float* __restrict__ delta,
                                                 float* __restrict__ dq_acc, Problem P, uint32_t rows) {
    const int lane16 = threadIdx.x & 15;
    const uint32_t row_raw = blockIdx.x * 16u + (threadIdx.x >> 4);
    const bool valid = row_raw < rows;  // no early return: the group shuffles need every lane
    const uint32_t row = valid ? row_raw : 0;
    const bool active = valid && lane16 < D / 8;
    float acc = 0.f;
    if (active) {
        float a[8], g[8];
        load_bf16x8(o + (size_t)row * D + 8 * lane16, a);
        load_bf16x8(dout + (size_t)row * D + 8 * lane16, g);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += a[i] * g[i];
        float4* z = reinterpret_cast<float4*>(dq_acc + (size_t)row * D + 8 * lane16);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    acc = group_sum<16>(acc);
    if (valid && lane16 == 0) {
        const uint32_t tok = fastdiv(row, P.div_hq);
        const uint32_t h = row - tok * (uint32_t)P.Hq;
        const uint32_t b = fastdiv(tok, P.div_t);
        const uint32_t t = tok - b * (uint32_t)P.T;
        delta[((size_t)b * P.Hq + h) * P.T + t] = acc;
    }
}

// ------------------------------------------------------------------ gradient finalize
// dq = RMSNorm^T(RoPE^T(scale * dQ')) from the fp32 accumulator and raw q, for every query
// head of a token; then the same for dk from raw dK' and raw k (only when QK-norm or RoPE is
// on; otherwise the attention kernel already wrote dk).  A group of GS lanes owns one token;
// a lane owns 4 rotation pairs (16-byte fp32 loads of each half) and forms their RoPE angles
// once for the token.
template <int D>
struct FinGeom {
    static constexpr int LPR = D / 8;
    static constexpr int GS = (LPR <= 4) ? 4 : (LPR <= 8 ? 8 : 16);
    static constexpr int TOK = 256 / GS;
};

// Two head rows in flight per lane (64 registers, four 256-thread blocks per SM).
template <int D>
__device__ __forceinline__ void finalize_heads(const float* __restrict__ acc, const __nv_bfloat16* __restrict__ x,
                                               __nv_bfloat16* __restrict__ out, int H, bool active, int d0,
                                               const float (&cs)[4], const float (&sn)[4], const Problem& P) {
    using G = FinGeom<D>;
    constexpr int kHalf = D / 2;
    constexpr int kIn = 2;
    for (int h0 = 0; h0 < H; h0 += kIn) {
        float u_lo[kIn][4], u_hi[kIn][4], x_lo[kIn][4], x_hi[kIn][4];
#pragma unroll
        for (int j = 0; j < kIn; ++j) {
#pragma unroll
            for (int i = 0; i < 4; ++i) u_lo[j][i] = u_hi[j][i] = x_lo[j][i] = x_hi[j][i] = 0.f;
            if (active && h0 + j < H) {
                const float* a = acc + (size_t)(h0 + j) * D;
                const float4 l4 = *reinterpret_cast<const float4*>(a + d0);
                const float4 h4 = *reinterpret_cast<const float4*>(a + kHalf + d0);
                u_lo[j][0] = l4.x; u_lo[j][1] = l4.y; u_lo[j][2] = l4.z; u_lo[j][3] = l4.w;
                u_hi[j][0] = h4.x; u_hi[j][1] = h4.y; u_hi[j][2] = h4.z; u_hi[j][3] = h4.w;
                if (P.qk_norm) {
                    load_bf16x4(x + (size_t)(h0 + j) * D + d0, x_lo[j]);
                    load_bf16x4(x + (size_t)(h0 + j) * D + kHalf + d0, x_hi[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kIn; ++j) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                u_lo[j][i] *= P.scale;
                u_hi[j][i] *= P.scale;
                rope_transpose(u_lo[j][i], u_hi[j][i], make_float2(cs[i], sn[i]));
            }
            if (P.qk_norm) {
                float ss = 0.f, dot = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    ss += x_lo[j][i] * x_lo[j][i] + x_hi[j][i] * x_hi[j][i];
                    dot += u_lo[j][i] * x_lo[j][i] + u_hi[j][i] * x_hi[j][i];
                }
                ss = group_sum<G::GS>(ss);
                dot = group_sum<G::GS>(dot);
                const float rs = rsqrtf(ss * (1.0f / D) + P.eps);
                const float k3 = rs * rs * rs * dot * (1.0f / D);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    u_lo[j][i] = rs * u_lo[j][i] - k3 * x_lo[j][i];
                    u_hi[j][i] = rs * u_hi[j][i] - k3 * x_hi[j][i];
                }
            }
            if (!active || h0 + j >= H) continue;
            store_bf16x4(out + (size_t)(h0 + j) * D + d0, u_lo[j]);
            store_bf16x4(out + (size_t)(h0 + j) * D + kHalf + d0, u_hi[j]);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(256, 4) k_grad_finalize(const float* __restrict__ dq_acc,
                                                       const float* __restrict__ dk_acc,
                                                       const __nv_bfloat16* __restrict__ q,
                                                       const __nv_bfloat16* __restrict__ k,
                                                       __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                                                       Problem P, const RopeFreq F, uint32_t tokens) {
    using G = FinGeom<D>;
    const int g = threadIdx.x & (G::GS - 1);
    const uint32_t tok_raw = blockIdx.x * (uint32_t)G::TOK + threadIdx.x / G::GS;  // b * T + t
    const bool valid = tok_raw < tokens;  // no early return: the group shuffles need every lane
    const uint32_t tok = valid ? tok_raw : 0;
    const bool active = valid && g < G::LPR;
    const int d0 = 4 * (active ? g : 0);
    float cs[4], sn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        cs[i] = 1.f;
        sn[i] = 0.f;
    }
    if (P.rope && active) {
        const int t = (int)(tok - fastdiv(tok, P.div_t) * (uint32_t)P.T);
        const int pos = P.seg_start ? t - P.seg_start[tok] : t;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = rope_angle(pos, F.theta[d0 + i]);
            cs[i] = a.x;
            sn[i] = a.y;
        }
    }
    const size_t oq = (size_t)tok * P.Hq * D;
    finalize_heads<D>(dq_acc + oq, q + oq, dq + oq, P.Hq, active, d0, cs, sn, P);
    if (dk_acc) {
        const size_t ok = (size_t)tok * P.Hkv * D;
        finalize_heads<D>(dk_acc + ok, k + ok, dk + ok, P.Hkv, active, d0, cs, sn, P);
    }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_prep(const Problem& P, const int32_t* ids, int32_t* seg_start, int32_t* seg_end, cudaStream_t st) {
    if (!ids || P.B == 0) return cudaSuccess;
    k_prep<<<P.B, 1024, 0, st>>>(P.T, ids, seg_start, seg_end);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_prologue_d(const Problem& P, const void* q, const void* k, void* qo, void* ko,
                                     cudaStream_t st) {
    const long long tokens = (long long)P.B * P.Tq;  // k == null: queries only (over a cache)
    const long long blocks = (tokens + TokGeom<D>::TOK - 1) / TokGeom<D>::TOK;
    const RopeFreq F = rope_freq(D, P.rope_log_base);
    // 128-thread blocks, seven per SM: the last wave of a large launch is less ragged than
    // with three 256-thread blocks (2048 blocks are 1.98 waves at 148 SMs instead of 2.3)
    k_qk_prologue<D><<<(unsigned)blocks, 128, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                      (__nv_bfloat16*)qo, (__nv_bfloat16*)ko, P, F, (uint32_t)tokens);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_bwd_pre_d(const Problem& P, const void* o, const void* dout, float* delta,
                                    float* dq_acc, cudaStream_t st) {
    const long long rows = (long long)P.B * P.T * P.Hq;
    k_bwd_pre<D><<<(unsigned)((rows + 15) / 16), 256, 0, st>>>((const __nv_bfloat16*)o,
                                                             (const __nv_bfloat16*)dout, delta, dq_acc, P, (uint32_t)rows);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_grad_finalize_d(const Problem& P, const float* dq_acc, const float* dk_acc, const void* q,
                                          const void* k, void* dq, void* dk, cudaStream_t st) {
    const long long tokens = (long long)P.B * P.T;
    const long long blocks = (tokens + FinGeom<D>::TOK - 1) / FinGeom<D>::TOK;
    const RopeFreq F = rope_freq(D, P.rope_log_base);
    k_grad_finalize<D><<<(unsigned)blocks, 256, 0, st>>>(
        dq_acc, (P.rope || P.qk_norm) ? dk_acc : nullptr, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
        (__nv_bfloat16*)dq, (__nv_bfloat16*)dk, P, F, (uint32_t)tokens);
    return cudaGetLastError();
}

#define CSA_DISPATCH_D(D_, CALL) \
    switch (D_) {                 \
        case 32: return CALL(32); \
        case 64: return CALL(64); \
        case 96: return CALL(96); \
        case 128: return CALL(128); \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t launch_prologue(const Problem& P, const void* q, const void* k, void* qo, void* ko, cudaStream_t st) {
#define CALL(d) launch_prologue_d<d>(P, q, k, qo, ko, st)
    CSA_DISPATCH_D(P.D, CALL)
#undef CALL
}
cudaError_t launch_bwd_pre(const Problem& P, const void* o, const void* dout, float* delta, float* dq_acc,
                           cudaStream_t st) {
#define CALL(d) launch_bwd_pre_d<d>(P, o, dout, delta, dq_acc, st)
    CSA_DISPATCH_D(P.D, CALL)
#undef CALL
}
cudaError_t launch_grad_finalize(const Problem& P, const float* dq_acc, const float* dk_acc, const void* q,
                                 const void* k, void* dq, void* dk, cudaStream_t st) {
#define CALL(d) launch_grad_finalize_d<d>(P, dq_acc, dk_acc, q, k, dq, dk, st)
    CSA_DISPATCH_D(P.D, CALL)
#undef CALL
}

}  // namespace csa
