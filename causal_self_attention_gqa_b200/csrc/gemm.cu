// gemm.cu -- the projections around attention: the Q/K/V projection of the block input with
// 3-D weights (one launch for all three), the output projection, and their backward products
// (input gradients, and weight gradients accumulated in fp32).
//
// Source: the nanogpt-jax-181m model card, section "Architecture", keeps the attention weights
// 3-D -- wq, wk, wv of shape (d_emb, heads, head_dim) and wo of shape (heads, head_dim, d_emb)
// -- and the GPT-pretraining page (dekermanjian.github.io, llm_gpt_pretrain), section
// "Multihead Attention", projects the block input to q, k, v, attends, and projects the
// concatenated heads back to the model width.  Row-major, a (C, H, D) weight is the matrix
// [C, H*D] and an activation [B, T, H, D] is [B*T, H*D], so every product is a plain GEMM:
//
//   forward   q|k|v = x [wq|wk|wv]          A = x K-major,   B = w N-major,  C pieced by N
//             y     = o wo                  A = o K-major,   B = wo N-major
//   backward  dO    = dy wo^T               A = dy K-major,  B = wo K-major
//             dx    = [dq|dk|dv] [wq|wk|wv]^T   A, B pieced by K, both K-major
//             dwo  += o^T dy                A = o M-major,   B = dy N-major, fp32 out
//             dwq|dwk|dwv += x^T [dq|dk|dv] A = x M-major,   B, C pieced by N, fp32 out
//
// Two kernels, both persistent (one CTA per SM, 192 threads) with the same roles: k_gemm_pair
// (below) runs large products on CTA pairs with 256 x 256 tiles; k_gemm runs the rest on
// single CTAs.  k_gemm: tiles of 128 x bn (bn up to 256), K in blocks of 64 through a
// STAGES-deep shared-memory ring:
//   warp 0, one lane   TMA producer: the A tile (one 64 x 128 box K-major, or two 64 x 64
//                      boxes M-major) and the B tile of the next K block, 128-byte swizzle;
//   warp 1, one lane   tcgen05.mma issuer (M = 128, N = bn, K = 16 per instruction) into one
//                      of two TMEM accumulators, so a tile's epilogue overlaps the next tile's
//                      MMAs; a committed barrier frees each ring slot;
//   warps 2-5          epilogue: each warp owns 32 accumulator rows (its TMEM lane quarter),
//                      reads 32 / 64 columns at a time, converts (bf16) or not (fp32), writes
//                      them into one of two swizzled staging boxes and issues a TMA store
//                      (bf16) or TMA reduce-add (fp32).
// Weight gradients reduce over B*T, so their few tiles are split along K and every split adds
// its partial product into the fp32 output (which therefore accumulates).  No multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "csa_internal.h"
#include "ptx.cuh"

namespace csa {
namespace {

constexpr int kGM = 128;  // tile rows (the MMA M)
constexpr int kGK = 64;   // K per ring slot: one 128-byte swizzle row of bf16

template <int BN, bool F32>
struct GemmCfg {
    static constexpr int A_BYTES = kGM * kGK * 2;
    static constexpr int B_BYTES = BN * kGK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STG_WARP = 2 * 32 * 128;  // two staging boxes of 32 rows x 128 bytes
    static constexpr int RING_BUDGET = 232448 - 4 * STG_WARP - 2048;
    static constexpr int STAGES = (RING_BUDGET / STAGE) > 8 ? 8 : (RING_BUDGET / STAGE);
    static constexpr int OFF_STG = STAGES * STAGE;
    static constexpr int OFF_BAR = OFF_STG + 4 * STG_WARP;
    static constexpr int NBAR = 2 * STAGES + 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    static constexpr int SMEM = OFF_MISC + 16 + 1024;    // + slack to align the base to 1024
    static constexpr int ACC = BN <= 64 ? 64 : (BN <= 128 ? 128 : 256);  // TMEM columns per accumulator
    static constexpr int TMEM_COLS = 2 * ACC;
    static constexpr int CHUNK = F32 ? 32 : 64;  // output columns per staging box (128 bytes a row)
    static_assert(STAGES >= 2, "ring too shallow");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(BN % CHUNK == 0 && BN % 64 == 0, "tile width");
};

// Piece of a bound table that holds `x` (bounds ascending; unused bounds equal the extent).
__device__ __forceinline__ int piece(const int (&bound)[4], int x) {
    return (x >= bound[1]) + (x >= bound[2]);
}

// One epilogue chunk of one warp: 32 accumulator rows (this warp's TMEM lane quarter, from
// column address `tcol`) x 32 fp32 or 64 bf16 columns -> one 32 x 128-byte staging box in
// the TMA box layout (128-byte swizzle: 16-byte chunk j of row r at j ^ (r & 7)) -> a TMA
// reduce-add (fp32) or store (bf16) at (column, row) of `map`.  `nst` counts this warp's
// chunks so far; the two boxes alternate, and a box is rewritten only once the store that
// last read it has finished reading.  Every lane of the warp calls it.
template <bool F32>
__device__ __forceinline__ void epilogue_chunk(uint32_t tcol, uint8_t* stg, int nst, const CUtensorMap* map,
                                               int column, int row) {
    const int lane = threadIdx.x & 31, sw = lane & 7;
    uint8_t* box = stg + (nst & 1) * 4096;
    if (lane == 0 && nst >= 2) bulk_wait_group_read1();
    __syncwarp();
    if (F32) {
        uint32_t v[32];
        tmem_ld32(tcol, v);
        tmem_ld_wait();
        tmem_ld_fence(v);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ sw) * 16)) =
                make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
        uint32_t v0[32], v1[32];
        tmem_ld32(tcol, v0);
        tmem_ld32(tcol + 32, v1);
        tmem_ld_wait();
        tmem_ld_fence(v0);
        tmem_ld_fence(v1);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ sw) * 16)) = make_uint4(
                pack_bf16x2(__uint_as_float(v0[8 * j]), __uint_as_float(v0[8 * j + 1])),
                pack_bf16x2(__uint_as_float(v0[8 * j + 2]), __uint_as_float(v0[8 * j + 3])),
                pack_bf16x2(__uint_as_float(v0[8 * j + 4]), __uint_as_float(v0[8 * j + 5])),
                pack_bf16x2(__uint_as_float(v0[8 * j + 6]), __uint_as_float(v0[8 * j + 7])));
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(box + lane * 128 + (((j + 4) ^ sw) * 16)) = make_uint4(
                pack_bf16x2(__uint_as_float(v1[8 * j]), __uint_as_float(v1[8 * j + 1])),
                pack_bf16x2(__uint_as_float(v1[8 * j + 2]), __uint_as_float(v1[8 * j + 3])),
                pack_bf16x2(__uint_as_float(v1[8 * j + 4]), __uint_as_float(v1[8 * j + 5])),
                pack_bf16x2(__uint_as_float(v1[8 * j + 6]), __uint_as_float(v1[8 * j + 7])));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        if (F32)
            tma_reduce_add_2d(map, box, column, row);
        else
            tma_store_2d(map, box, column, row);
        bulk_commit_group();
    }
}

template <int BN, bool A_MN, bool B_MN, bool F32>
__global__ void __launch_bounds__(192, 1) k_gemm(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs g) {
    using C = GemmCfg<BN, F32>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;                    // [STAGES] ring slot loaded
    uint64_t* empty = bars + C::STAGES;       // [STAGES] ring slot consumed by the MMAs
    uint64_t* acc_full = bars + 2 * C::STAGES;  // [2] accumulator complete
    uint64_t* acc_empty = acc_full + 2;         // [2] accumulator read out (4 epilogue warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // unit -> (first row, first column, K blocks [kb0, kb1)); the column tile runs fastest, so
    // the CTAs that run at the same time share A rows (and all of B) through L2
    auto coords = [&](int u, int& m0, int& n0, int& kb0, int& kb1) {
        const int s = u % g.splits, t = u / g.splits;
        n0 = (t % g.nt) * BN;
        m0 = (t / g.nt) * kGM;
        kb0 = s * g.kb_per_split;
        kb1 = min(g.kb_total, kb0 + g.kb_per_split);
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < 3; ++i) {
                tma_prefetch_desc(&maps.a[i]);
                tma_prefetch_desc(&maps.b[i]);
            }
            bool ok = true;
            int it = 0;  // ring slots filled so far
            for (int u = blockIdx.x; u < g.units && ok; u += gridDim.x) {
                int m0, n0, kb0, kb1;
                coords(u, m0, n0, kb0, kb1);
                const int np = piece(g.n_bound, n0);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (it >= C::STAGES && !(ok = mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, abort_flag, g.status)))
                        break;
                    const int k0 = kb * kGK;
                    const int kp = piece(g.k_bound, k0);
                    const int kl = k0 - g.k_bound[kp];
                    uint8_t* sa = smem + s * C::STAGE;
                    uint8_t* sb = sa + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    const CUtensorMap* ma = &maps.a[kp];
                    if (A_MN) {
                        tma_load_2d(ma, &full[s], sa, m0, kl);
                        tma_load_2d(ma, &full[s], sa + 8192, m0 + 64, kl);
                    } else {
                        tma_load_2d(ma, &full[s], sa, kl, m0);
                    }
                    const CUtensorMap* mb = &maps.b[g.b_by_k ? kp : np];
                    const int bk = g.b_by_k ? kl : k0;
                    const int bn0 = g.b_by_k ? n0 : n0 - g.n_bound[np];
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j) tma_load_2d(mb, &full[s], sb + j * 8192, bn0 + 64 * j, bk);
                    } else {
                        tma_load_2d(mb, &full[s], sb, bk, bn0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16(kGM, BN, A_MN, B_MN);
            // MN-major: 64-element atom columns of 64 K rows (8 KB apart), 8-row groups 1 KB apart;
            // K-major: 128-byte rows, 8-row groups 1 KB apart
            constexpr uint32_t A_LBO = A_MN ? 8192 : 16, B_LBO = B_MN ? 8192 : 16;
            bool ok = true;
            int it = 0, t = 0;
            for (int u = blockIdx.x; u < g.units && ok; u += gridDim.x, ++t) {
                int m0, n0, kb0, kb1;
                coords(u, m0, n0, kb0, kb1);
                const int buf = t & 1, use = t >> 1;
                if (use >= 1 && !(ok = mbar_wait(&acc_empty[buf], (use - 1) & 1, abort_flag, g.status))) break;
                tc_fence_after();
                const uint32_t d = tmem + buf * C::ACC;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (!(ok = mbar_wait(&full[s], (it / C::STAGES) & 1, abort_flag, g.status))) break;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE), sb = sa + C::A_BYTES;
                    const uint64_t ad = sdesc(sa, A_LBO, 1024, kLayoutSw128);
                    const uint64_t bd = sdesc(sb, B_LBO, 1024, kLayoutSw128);
#pragma unroll
                    for (int ks = 0; ks < kGK / 16; ++ks) {
                        const uint32_t ao = A_MN ? koff_mnmajor<128>(ks) : koff_kmajor<128, kGM>(ks);
                        const uint32_t bo = B_MN ? koff_mnmajor<128>(ks) : koff_kmajor<128, BN>(ks);
                        umma_ss(d, ad + ao, bd + bo, IDESC, (kb > kb0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&acc_full[buf]);
            }
        }
    } else {
        const int quarter = warp & 3;  // the TMEM lanes (tile rows) this warp may read
        uint8_t* stg = smem + C::OFF_STG + (warp - 2) * C::STG_WARP;
        int t = 0, nst = 0;
        for (int u = blockIdx.x; u < g.units; u += gridDim.x, ++t) {
            int m0, n0, kb0, kb1;
            coords(u, m0, n0, kb0, kb1);
            const int buf = t & 1, use = t >> 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1, abort_flag, g.status))) break;
            tc_fence_after();
            const int np = piece(g.n_bound, n0);
            const int nl = n0 - g.n_bound[np];
            const CUtensorMap* mc = &maps.c[np];
            const uint32_t ta = tmem + ((uint32_t)(32 * quarter) << 16) + buf * C::ACC;
            const int row0 = m0 + 32 * quarter;
#pragma unroll 1
            for (int c = 0; c < BN / C::CHUNK; ++c, ++nst)
                epilogue_chunk<F32>(ta + C::CHUNK * c, stg, nst, mc, nl + C::CHUNK * c, row0);
            // every column of this accumulator is in registers or staged: the MMAs may reuse it
            tc_fence_before();
            warp_arrive(&acc_empty[buf]);
        }
        if (lane == 0) bulk_wait_group_read0();  // the global writes complete with the grid
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int BN, bool A_MN, bool B_MN, bool F32>
cudaError_t launch_t(const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
    using C = GemmCfg<BN, F32>;
    const void* fn = reinterpret_cast<const void*>(k_gemm<BN, A_MN, B_MN, F32>);
    const cudaError_t e = ensure_dyn_smem(fn, C::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = g.units < num_sms() ? g.units : num_sms();
    k_gemm<BN, A_MN, B_MN, F32><<<grid, 192, C::SMEM, st>>>(maps, g);
    return cudaGetLastError();
}

template <bool A_MN, bool B_MN, bool F32>
cudaError_t by_bn(const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
    switch (g.bn) {
        case 64: return launch_t<64, A_MN, B_MN, F32>(maps, g, st);
        case 128: return launch_t<128, A_MN, B_MN, F32>(maps, g, st);
        case 192: return launch_t<192, A_MN, B_MN, F32>(maps, g, st);
        case 256: return launch_t<256, A_MN, B_MN, F32>(maps, g, st);
        default: return cudaErrorInvalidValue;
    }
}


// ------------------------------------------------------------------ CTA pairs
// The same roles on a cluster of two CTAs that computes a 256 x 256 tile with M = 256 MMAs
// (cta_group::2) issued by the leader (rank 0).  Each CTA stages its own 128 rows of A and its
// own 128 columns of B -- 32 KB a ring slot instead of 48, so six slots fit and the loads in
// flight cover their latency -- and keeps its 128 x 256 half of the accumulator in its own
// TMEM.  Both CTAs' loads complete on the leader's ring barriers; the leader's commits arrive
// on the barriers of both.  B and C pieces are looked up per 64 columns, so a tile may
// straddle pieces (their bounds are multiples of 64).  No multicast load.
constexpr int kPairBN = 256;

template <bool F32>
struct PairCfg {
    static constexpr int A_BYTES = 128 * kGK * 2;
    static constexpr int B_BYTES = (kPairBN / 2) * kGK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STG_WARP = 2 * 32 * 128;
    static constexpr int RING_BUDGET = 232448 - 4 * STG_WARP - 2048;
    static constexpr int STAGES = (RING_BUDGET / STAGE) > 8 ? 8 : (RING_BUDGET / STAGE);
    static constexpr int OFF_STG = STAGES * STAGE;
    static constexpr int OFF_BAR = OFF_STG + 4 * STG_WARP;
    static constexpr int NBAR = 2 * STAGES + 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int ACC = 256;
    static constexpr int TMEM_COLS = 512;
    static constexpr int CHUNK = F32 ? 32 : 64;
    static_assert(STAGES >= 4, "ring too shallow");
    static_assert(SMEM <= 232448, "shared memory");
};

template <bool A_MN, bool B_MN, bool F32>
__global__ void __launch_bounds__(192, 1)
    k_gemm_pair(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs g) {
    using C = PairCfg<F32>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the same offset in both CTAs (same kernel, same static layout): the leader's MMA
    // descriptors address the peer's tiles at the offsets of its own
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;                      // [STAGES] both CTAs' halves loaded (leader's used)
    uint64_t* empty = bars + C::STAGES;         // [STAGES] slot consumed (arrives in both CTAs)
    uint64_t* acc_full = bars + 2 * C::STAGES;  // [2] accumulator complete (both CTAs)
    uint64_t* acc_empty = acc_full + 2;         // [2] both halves read out (leader's: 8 warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated before any use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto coords = [&](int u, int& m0, int& n0, int& kb0, int& kb1) {
        const int s = u % g.splits, t = u / g.splits;
        n0 = (t % g.nt) * kPairBN;
        m0 = (t / g.nt) * 256 + (int)rank * 128;  // this CTA's rows
        kb0 = s * g.kb_per_split;
        kb1 = min(g.kb_total, kb0 + g.kb_per_split);
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < 3; ++i) {
                tma_prefetch_desc(&maps.a[i]);
                tma_prefetch_desc(&maps.b[i]);
            }
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);  // the leader's full[0]
            bool ok = true;
            int it = 0;
            for (int u = pair_id; u < g.units && ok; u += npairs) {
                int m0, n0, kb0, kb1;
                coords(u, m0, n0, kb0, kb1);
                const int nh = n0 + (int)rank * (kPairBN / 2);  // this CTA's B columns
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (it >= C::STAGES && !(ok = mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, abort_flag, g.status)))
                        break;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
                    const uint32_t fb = full0 + 8u * (uint32_t)s;
                    const int k0 = kb * kGK;
                    const int kp = piece(g.k_bound, k0);
                    const int kl = k0 - g.k_bound[kp];
                    uint8_t* sa = smem + s * C::STAGE;
                    uint8_t* sb = sa + C::A_BYTES;
                    const CUtensorMap* ma = &maps.a[kp];
                    if (A_MN) {
                        tma_load_2d_pair(ma, fb, sa, m0, kl);
                        tma_load_2d_pair(ma, fb, sa + 8192, m0 + 64, kl);
                    } else {
                        tma_load_2d_pair(ma, fb, sa, kl, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int n = nh + 64 * j;
                            const int np = piece(g.n_bound, n);
                            tma_load_2d_pair(&maps.b[np], fb, sb + j * 8192, n - g.n_bound[np], k0);
                        }
                    } else {
                        // K-major B: one N piece (checked on the host); pieces, if any, split K
                        tma_load_2d_pair(&maps.b[g.b_by_k ? kp : 0], fb, sb, g.b_by_k ? kl : k0, nh);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16(256, kPairBN, A_MN, B_MN);
            constexpr uint32_t A_LBO = A_MN ? 8192 : 16, B_LBO = B_MN ? 8192 : 16;
            bool ok = true;
            int it = 0, t = 0;
            for (int u = pair_id; u < g.units && ok; u += npairs, ++t) {
                int m0, n0, kb0, kb1;
                coords(u, m0, n0, kb0, kb1);
                const int buf = t & 1, use = t >> 1;
                if (use >= 1 && !(ok = mbar_wait(&acc_empty[buf], (use - 1) & 1, abort_flag, g.status))) break;
                tc_fence_after();
                const uint32_t d = tmem + buf * C::ACC;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    if (!(ok = mbar_wait(&full[s], (it / C::STAGES) & 1, abort_flag, g.status))) break;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE), sb = sa + C::A_BYTES;
                    const uint64_t ad = sdesc(sa, A_LBO, 1024, kLayoutSw128);
                    const uint64_t bd = sdesc(sb, B_LBO, 1024, kLayoutSw128);
#pragma unroll
                    for (int ks = 0; ks < kGK / 16; ++ks) {
                        const uint32_t ao = A_MN ? koff_mnmajor<128>(ks) : koff_kmajor<128, 128>(ks);
                        const uint32_t bo = B_MN ? koff_mnmajor<128>(ks) : koff_kmajor<128, 128>(ks);
                        umma_ss_pair(d, ad + ao, bd + bo, IDESC, (kb > kb0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit_pair(&empty[s], 0x3);
                }
                if (!ok) break;
                umma_commit_pair(&acc_full[buf], 0x3);
            }
        }
    } else {
        const int quarter = warp & 3;
        uint8_t* stg = smem + C::OFF_STG + (warp - 2) * C::STG_WARP;
        const uint32_t acc_empty0 = mapa_shared(smem_u32(&acc_empty[0]), 0);  // the leader's
        int t = 0, nst = 0;
        for (int u = pair_id; u < g.units; u += npairs, ++t) {
            int m0, n0, kb0, kb1;
            coords(u, m0, n0, kb0, kb1);
            const int buf = t & 1, use = t >> 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1, abort_flag, g.status))) break;
            tc_fence_after();
            const uint32_t ta = tmem + ((uint32_t)(32 * quarter) << 16) + buf * C::ACC;
            const int row0 = m0 + 32 * quarter;
#pragma unroll 1
            for (int c = 0; c < kPairBN / C::CHUNK; ++c) {
                const int n = n0 + C::CHUNK * c;
                if (n >= g.N) break;  // warp-uniform; columns past N are never stored
                const int np = piece(g.n_bound, n);
                epilogue_chunk<F32>(ta + C::CHUNK * c, stg, nst++, &maps.c[np], n - g.n_bound[np], row0);
            }
            // this CTA's half is out of TMEM: tell the leader's MMA thread
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(&acc_empty[buf]);
                else
                    mbar_arrive_cluster(acc_empty0 + 8u * (uint32_t)buf);
            }
        }
        if (lane == 0) bulk_wait_group_read0();
    }

    // no CTA leaves while its peer may still address its shared memory or TMEM (the lanes of
    // warps 0 and 1 meet again first: the cluster barrier is warp-aligned)
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

template <bool A_MN, bool B_MN, bool F32>
cudaError_t launch_pair_t(const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
    using C = PairCfg<F32>;
    auto fn = k_gemm_pair<A_MN, B_MN, F32>;
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(fn), C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(192, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // as many pairs as can be resident at once (clusters are placed within a GPC); asked of
    // the runtime once per device for each of the three kernels
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        dev = -1;
    }
    static std::atomic<int> resident[64];  // 0: not asked yet (zero-initialised, static storage)
    int clusters = dev >= 0 ? resident[dev].load(std::memory_order_relaxed) : 0;
    if (clusters < 1) {
        cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
        e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg);
        if (e != cudaSuccess || clusters < 1) {
            cudaGetLastError();
            clusters = num_sms() / 2;
        }
        if (dev >= 0) resident[dev].store(clusters, std::memory_order_relaxed);
    }
    const int npairs = g.units < clusters ? g.units : clusters;
    cfg.gridDim = dim3(2 * npairs, 1, 1);
    e = cudaLaunchKernelEx(&cfg, fn, maps, g);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}
}  // namespace

// The three operand forms the projections use: forward (K-major A, N-major B, bf16 out),
// input gradients (both K-major, bf16 out), weight gradients (M-major A, N-major B, fp32 out).
cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
    if (g.pair) {
        if (!g.a_mn && g.b_mn && !g.f32_out) return launch_pair_t<false, true, false>(maps, g, st);
        if (!g.a_mn && !g.b_mn && !g.f32_out) return launch_pair_t<false, false, false>(maps, g, st);
        if (g.a_mn && g.b_mn && g.f32_out) return launch_pair_t<true, true, true>(maps, g, st);
        return cudaErrorInvalidValue;
    }
    if (!g.a_mn && g.b_mn && !g.f32_out) return by_bn<false, true, false>(maps, g, st);
    if (!g.a_mn && !g.b_mn && !g.f32_out) return by_bn<false, false, false>(maps, g, st);
    if (g.a_mn && g.b_mn && g.f32_out) return by_bn<true, true, true>(maps, g, st);
    return cudaErrorInvalidValue;
}

}  // namespace csa
