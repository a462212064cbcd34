// rows.cu -- the HBM-bound row kernels around the two attention kernels:
//   k_prep         segment bounds of every token (maximal runs of equal segment_ids) and the
//                  RoPE (cos, sin) table for positions 0..T-1, computed in fp64
//   k_qk_prologue  q' = RoPE(RMSNorm(q)), k' = RoPE(RMSNorm(k)) -> bf16 copies in the workspace
//   k_bwd_pre      delta_i = sum_d dO_id O_id per (b, h, i) and a zeroed fp32 dQ accumulator
//   k_grad_finalize dq (and dk when QK-norm or RoPE is on) = RMSNorm^T(RoPE^T(scale * acc))
//                  -> bf16, from the fp32 dQ' accumulator and the raw dK' sums
//
// The norm is the parameter-free RMSNorm and the rotation the rotate-half RoPE of the
// nanogpt-jax-181m model card ("Architecture"); positions restart at each packed segment
// (same section, "RoPE frequencies are computed from packed segment positions").
//
// Row kernels give each [.., D] row an aligned group of lanes; a lane owns whole rotation
// pairs (d, d + D/2), so a rotation never crosses lanes.  The finalize uses 16-lane groups
// with 4 pairs per lane (it holds twice the data per pair, and 16-byte lanes cost it occupancy).
#include <cuda_bf16.h>
#include <stdint.h>

#include "csa_internal.h"
#include "rowops.cuh"

namespace csa {

// ------------------------------------------------------------------ segments + RoPE table
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

__global__ void __launch_bounds__(1024) k_prep(int B, int T, const int32_t* __restrict__ ids,
                                               int32_t* __restrict__ seg_start, int32_t* __restrict__ seg_end,
                                               float2* __restrict__ rope_cs, int half, double log_base) {
    __shared__ int sh[32];
    const int seg_blocks = ids ? B : 0;
    if ((int)blockIdx.x < seg_blocks) {
        const int b = blockIdx.x;
        const int32_t* id = ids + (size_t)b * T;
        int carry = 0;
        for (int base = 0; base < T; base += 1024) {  // start: running max of run-start indices
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
        for (int top = T - 1; top >= 0; top -= 1024) {  // end: running min (from the right) of run ends
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
        return;
    }
    if (!rope_cs) return;
    const uint32_t idx = (blockIdx.x - seg_blocks) * blockDim.x + threadIdx.x;  // T * half < 2^27
    if (idx >= (uint32_t)T * half) return;
    const int t = (int)(idx / half), d = (int)(idx - (uint32_t)t * half);
    const double theta = exp((-2.0 * d / (2.0 * half)) * log_base);  // base^(-2d/D)
    double s, c;
    sincos((double)t * theta, &s, &c);
    rope_cs[idx] = make_float2((float)c, (float)s);
}

// ------------------------------------------------------------------ q/k prologue
// Row geometry of the prologue: a lane owns the 8 rotation pairs
// (d, d + D/2) for d in [8g, 8g + 8), so its loads and stores are 16 bytes wide; the D/16
// lanes of a row form an aligned group of GS lanes (a power of two; D = 96 leaves 2 of 8 idle).
template <int D>
struct RowGeom {
    static constexpr int LPR = D / 16;
    static constexpr int GS = (LPR <= 2) ? 2 : (LPR <= 4 ? 4 : 8);
    static constexpr int ROWS = 256 / GS;  // rows per 256-thread block
};

template <int D>
__global__ void __launch_bounds__(256) k_qk_prologue(const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ k,
                                                     __nv_bfloat16* __restrict__ qo, __nv_bfloat16* __restrict__ ko,
                                                     Problem P, uint32_t rows_q, uint32_t rows_total) {
    using G = RowGeom<D>;
    constexpr int kHalf = D / 2;
    const int g = threadIdx.x & (G::GS - 1);
    const uint32_t row_raw = blockIdx.x * (uint32_t)G::ROWS + threadIdx.x / G::GS;
    // no early return: every lane of the warp takes part in the group shuffles below
    const bool valid = row_raw < rows_total;
    const uint32_t row = valid ? row_raw : 0;
    const bool is_q = row < rows_q;
    const uint32_t r = is_q ? row : row - rows_q;
    const uint32_t tok = fastdiv(r, is_q ? P.div_hq : P.div_hkv);  // b * T + t (queries: b * Tq + t)
    const uint32_t b = fastdiv(tok, is_q ? P.div_tq : P.div_t);
    const int t = (int)(tok - b * (uint32_t)(is_q ? P.Tq : P.T));
    const __nv_bfloat16* x = (is_q ? q : k) + (size_t)r * D;
    __nv_bfloat16* y = (is_q ? qo : ko) + (size_t)r * D;
    const bool active = valid && g < G::LPR;
    const int d0 = 8 * g;
    float lo[8], hi[8];
    float4 cs[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) lo[i] = hi[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) cs[i] = make_float4(1.f, 0.f, 1.f, 0.f);
    if (active) {
        load_bf16x8(x + d0, lo);
        load_bf16x8(x + kHalf + d0, hi);
        if (P.rope) {  // issued together with the row loads: its latency overlaps theirs
            // queries over a cache sit at qoff + t; segments only come without a cache
            const int pos = P.seg_start ? t - P.seg_start[tok] : t + (is_q ? P.qoff : 0);
            const float4* c = reinterpret_cast<const float4*>(P.rope_cs + (size_t)pos * kHalf + d0);
#pragma unroll
            for (int i = 0; i < 4; ++i) cs[i] = c[i];
        }
    }
    float rs = 1.0f;
    if (P.qk_norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += lo[i] * lo[i] + hi[i] * hi[i];
        ss = group_sum<G::GS>(ss);
        rs = rsqrtf(ss * (1.0f / D) + P.eps);
    }
    if (!active) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        lo[i] *= rs;
        hi[i] *= rs;
    }
    if (P.rope) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float c = (i & 1) ? cs[i / 2].z : cs[i / 2].x;
            const float sn = (i & 1) ? cs[i / 2].w : cs[i / 2].y;
            const float a = lo[i], bb = hi[i];
            lo[i] = a * c - bb * sn;
            hi[i] = bb * c + a * sn;
        }
    }
    store_bf16x8(y + d0, lo);
    store_bf16x8(y + kHalf + d0, hi);
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
// Rows [0, rows_q): dq = RMSNorm^T(RoPE^T(scale * dQ')) from the fp32 accumulator and raw q.
// Rows [rows_q, rows_q + rows_k): the same for dk from raw dK' and raw k (only when QK-norm
// or RoPE is on; otherwise the attention kernel already wrote dk).
template <int D>
__global__ void __launch_bounds__(256) k_grad_finalize(const float* __restrict__ dq_acc,
                                                       const float* __restrict__ dk_acc,
                                                       const __nv_bfloat16* __restrict__ q,
                                                       const __nv_bfloat16* __restrict__ k,
                                                       __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                                                       Problem P, uint32_t rows_q, uint32_t rows_total) {
    constexpr int kHalf = D / 2;
    const int lane16 = threadIdx.x & 15;
    const uint32_t row_raw = blockIdx.x * 16u + (threadIdx.x >> 4);
    const bool valid = row_raw < rows_total;  // no early return: the group shuffles need every lane
    const uint32_t row0 = valid ? row_raw : 0;
    const bool is_q = row0 < rows_q;
    const size_t row = is_q ? row0 : row0 - rows_q;
    const float* acc = is_q ? dq_acc : dk_acc;
    const __nv_bfloat16* x = is_q ? q : k;
    __nv_bfloat16* out = is_q ? dq : dk;
    const bool active = valid && lane16 < D / 8;
    const int d0 = 4 * lane16;
    float u_lo[4] = {0.f, 0.f, 0.f, 0.f}, u_hi[4] = {0.f, 0.f, 0.f, 0.f};
    float x_lo[4] = {0.f, 0.f, 0.f, 0.f}, x_hi[4] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
        const float4 a = *reinterpret_cast<const float4*>(acc + row * D + d0);
        const float4 c = *reinterpret_cast<const float4*>(acc + row * D + kHalf + d0);
        u_lo[0] = a.x * P.scale; u_lo[1] = a.y * P.scale; u_lo[2] = a.z * P.scale; u_lo[3] = a.w * P.scale;
        u_hi[0] = c.x * P.scale; u_hi[1] = c.y * P.scale; u_hi[2] = c.z * P.scale; u_hi[3] = c.w * P.scale;
        if (P.qk_norm) {
            load_bf16x4(x + row * D + d0, x_lo);
            load_bf16x4(x + row * D + kHalf + d0, x_hi);
        }
        if (P.rope) {
            const uint32_t tok = fastdiv((uint32_t)row, is_q ? P.div_hq : P.div_hkv);  // b * T + t
            const int t = (int)(tok - fastdiv(tok, P.div_t) * (uint32_t)P.T);
            const int pos = P.seg_start ? t - P.seg_start[tok] : t;
            const float4* cs = reinterpret_cast<const float4*>(P.rope_cs + (size_t)pos * kHalf + d0);
            const float4 c01 = cs[0], c23 = cs[1];
            rope_transpose(u_lo[0], u_hi[0], make_float2(c01.x, c01.y));
            rope_transpose(u_lo[1], u_hi[1], make_float2(c01.z, c01.w));
            rope_transpose(u_lo[2], u_hi[2], make_float2(c23.x, c23.y));
            rope_transpose(u_lo[3], u_hi[3], make_float2(c23.z, c23.w));
        }
    }
    if (P.qk_norm) {
        float ss = 0.f, dot = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ss += x_lo[i] * x_lo[i] + x_hi[i] * x_hi[i];
            dot += u_lo[i] * x_lo[i] + u_hi[i] * x_hi[i];
        }
        ss = group_sum<16>(ss);
        dot = group_sum<16>(dot);
        const float rs = rsqrtf(ss * (1.0f / D) + P.eps);
        const float k3 = rs * rs * rs * dot * (1.0f / D);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            u_lo[i] = rs * u_lo[i] - k3 * x_lo[i];
            u_hi[i] = rs * u_hi[i] - k3 * x_hi[i];
        }
    }
    if (!active) return;
    store_bf16x4(out + row * D + d0, u_lo);
    store_bf16x4(out + row * D + kHalf + d0, u_hi);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_prep(const Problem& P, const int32_t* ids, int32_t* seg_start, int32_t* seg_end,
                        float2* rope_cs, double rope_base, cudaStream_t st) {
    const int half = P.D / 2;
    const int seg_blocks = ids ? P.B : 0;
    const long long rope_n = rope_cs ? (long long)P.T * half : 0;
    const int rope_blocks = (int)((rope_n + 1023) / 1024);
    if (seg_blocks + rope_blocks == 0) return cudaSuccess;
    k_prep<<<seg_blocks + rope_blocks, 1024, 0, st>>>(P.B, P.T, ids, seg_start, seg_end, rope_cs, half,
                                                       rope_base > 0 ? log(rope_base) : 0.0);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_prologue_d(const Problem& P, const void* q, const void* k, void* qo, void* ko,
                                     cudaStream_t st) {
    const long long rows_q = (long long)P.B * P.Tq * P.Hq;
    const long long rows = rows_q + (k ? (long long)P.B * P.T * P.Hkv : 0);  // k == null: queries only
    const long long blocks = (rows + RowGeom<D>::ROWS - 1) / RowGeom<D>::ROWS;
    k_qk_prologue<D><<<(unsigned)blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (__nv_bfloat16*)qo, (__nv_bfloat16*)ko, P, (uint32_t)rows_q, (uint32_t)rows);
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
    const long long rows_q = (long long)P.B * P.T * P.Hq;
    const long long rows_k = (P.rope || P.qk_norm) ? (long long)P.B * P.T * P.Hkv : 0;
    const long long rows = rows_q + rows_k;
    k_grad_finalize<D><<<(unsigned)((rows + 15) / 16), 256, 0, st>>>(
        dq_acc, dk_acc, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (__nv_bfloat16*)dq, (__nv_bfloat16*)dk, P,
        (uint32_t)rows_q, (uint32_t)rows);
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
