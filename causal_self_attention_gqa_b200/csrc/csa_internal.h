// csa_internal.h -- definitions shared by the host code and the kernels of libcsa.
#pragma once
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include <cuda.h>
#include <cuda_runtime.h>

#include "csa.h"

namespace csa {

// A bounded wait inside a kernel gives up after this many SM clocks (about a second).
constexpr long long kWaitLimitCycles = 2000000000LL;

constexpr int kBM = 128;  // query rows per tile (the MMA M)
constexpr int kBN = 128;  // keys per tile

// n / d for 0 <= n < 2^31 without a division instruction: with l = ceil(log2 d) and
// m = ceil(2^(31+l) / d) (< 2^32), floor(n m / 2^(31+l)) = floor(n / d), because the excess
// n (m - 2^(31+l)/d) / 2^(31+l) < 2^-l <= 1/d never reaches the next multiple of 1/d.
struct FastDiv {
    uint32_t d, m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    FastDiv f;
    f.d = d;
    f.m = (uint32_t)(((1ull << (31 + l)) + d - 1) / d);
    f.s = 31 + l;
    return f;
}
#ifdef __CUDACC__
__host__ __device__
#endif
inline uint32_t fastdiv(uint32_t n, FastDiv f) {
    return (uint32_t)(((uint64_t)n * f.m) >> f.s);
}

// Everything a kernel needs to know about the problem.
struct Problem {
    int B, T, Hq, Hkv, D, G;
    // Query rows and the absolute position of query row 0.  Tq = T and qoff = 0 everywhere
    // except the forward over a key/value cache, where T is the cache length and the Tq
    // queries are its last positions (qoff = T - Tq).
    int Tq, qoff;
    int causal, window;
    float softcap;          // 0 = off
    float cap_in;           // scale / softcap: tanh argument per raw score (cap on)
    float cap_log2;         // softcap * log2(e): capped logit in log2 units per unit of tanh
    int cap_series;         // 1: every |scale * q'.k' / softcap| <= 1/4 is guaranteed (QK-norm on
                            // our own prologue's output), so tanh may use its short series
    float scale;            // effective score scale
    float scale_log2;       // scale * log2(e)
    int rope, qk_norm;
    float eps;
    const int32_t* seg_start;  // [B, T] first index of each token's segment, or null
    const int32_t* seg_end;    // [B, T] one past its last index, or null
    double rope_log_base;      // ln(base) when RoPE is on
    FastDiv div_hq, div_hkv, div_t, div_tq;  // row -> (token, head), token -> (batch row, position)
    int* status;               // device status word (workspace, or the caller's)
    int* counters;             // [2] work-item counters of the persistent kernels (workspace,
                               // zeroed by every call): forward, backward
};

// RoPE frequencies theta_d = base^(-2d/D), d < D/2, computed on the host in fp64 and passed
// to the kernels that rotate (by value, as a kernel parameter).
struct RopeFreq {
    double theta[64];
};
inline RopeFreq rope_freq(int D, double log_base) {
    RopeFreq F;
    for (int i = 0; i < 64; ++i) F.theta[i] = (i < D / 2) ? exp((-2.0 * i / D) * log_base) : 0.0;
    return F;
}

// Work split of the KV-cache decode (decode.cu): Tq new queries, R = G * Tq rows per
// (b, kv head), the cache cut into `splits` ranges of keys_per_split keys.
struct DecodePlan {
    int Tq, R, splits, keys_per_split;
    size_t part_bytes, done_bytes;
};

// One projection GEMM (gemm.cu): C[M, N] = sum_k A[m, k] B[k, n] over row-major bf16
// matrices, fp32 accumulation; C is bf16 (stored) or fp32 (added to what C holds).  A is read
// K-major ([M, K] in memory) or M-major ([K, M]); B K-major ([N, K]) or N-major ([K, N]).
// An operand may come in up to three pieces (separate tensors, one tensor map each): pieces
// of C, and of B when b_by_k is 0, split N at n_bound; pieces of A, and of B when b_by_k is
// 1, split K at k_bound.  Unused bounds equal N (resp. K).
struct GemmArgs {
    int M, N, K;
    int bn;                 // N per tile: 64, 128, 192 or 256 (divides every inner N bound)
    int a_mn, b_mn, f32_out;
    int b_by_k;
    int n_bound[4], k_bound[4];  // [0] = 0, [3] = N (resp. K); inner bounds multiples of bn (64)
    int mt, nt, splits, kb_total, kb_per_split, units;
    int pair;               // 1: CTA pairs (cta_group::2), 256-row x 256-column tiles, mt counts 256-row tiles
    int* status;
};
struct GemmMaps {
    CUtensorMap a[3], b[3], c[3];
};

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the CURRENT device, once per
// (kernel, device): the attribute is per device, so a process that drives several GPUs sets
// it on each.  Thread-safe.
cudaError_t ensure_dyn_smem(const void* kernel, int bytes);

// Kernel ids for the timing interface (order = csa_kernel_name()).
enum KernelId {
    kPrep = 0, kPrologue, kFwd, kBwdPre, kBwd, kGradFinalize, kDecode,
    kGemmQkv, kGemmOut, kGemmDout, kGemmDwo, kGemmDx, kGemmDw, kNumKernels
};

}  // namespace csa
