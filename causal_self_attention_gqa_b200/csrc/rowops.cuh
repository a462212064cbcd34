// rowops.cuh -- small per-row helpers shared by the row kernels and the attention
// kernels' epilogues: bf16 vector loads/stores, lane-group sums, the RoPE rotation angle,
// transposed RoPE.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "csa_internal.h"

namespace csa {

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        f[2 * i] = __low2float(h);
        f[2 * i + 1] = __high2float(h);
    }
}
__device__ __forceinline__ void load_bf16x4(const __nv_bfloat16* p, float (&f)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    f[0] = __low2float(a); f[1] = __high2float(a);
    f[2] = __low2float(b); f[3] = __high2float(b);
}
__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* p, const float (&f)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* p, const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
// Sum over aligned groups of GS lanes (GS a power of two <= 32).
template <int GS>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = GS / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, GS);
    return v;
}
// (cos phi, sin phi) of the RoPE angle phi = pos * theta (theta = base^(-2d/D) from the
// host, fp64).  phi reaches ~1e6 rad at the longest sequences, so it is formed and reduced
// to [-pi, pi] in fp64 (Cody-Waite, 2 pi split into its nearest double and the remainder),
// and only the remainder goes to the hardware sine and cosine (__sincosf: absolute error
// below 2^-21.4 on [-pi, pi], far inside the bf16 rounding of the rotated values).
__device__ __forceinline__ float2 rope_angle(int pos, double theta) {
    const double phi = (double)pos * theta;
    const double k = rint(phi * 0.15915494309189535);  // 1 / (2 pi)
    const double red = fma(-k, 2.4492935982947064e-16, fma(-k, 6.283185307179586, phi));
    float sn, cs;
    __sincosf((float)red, &sn, &cs);
    return make_float2(cs, sn);
}
// Transpose of the rotate-half rotation by phi (i.e. rotation by -phi) applied to a
// gradient pair (g_a at d, g_b at d + D/2); cs = (cos phi, sin phi).
__device__ __forceinline__ void rope_transpose(float& ga, float& gb, float2 cs) {
    const float a = ga, b = gb;
    ga = a * cs.x + b * cs.y;
    gb = b * cs.x - a * cs.y;
}

}  // namespace csa
