// api.cu -- the C ABI of libcsa.so (declared in include/csa.h): argument validation,
// workspace layout, TMA tensor maps, kernel launches and optional per-kernel timing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <initializer_list>
#include <mutex>
#include <utility>
#include <vector>

#include "csa_internal.h"

namespace csa {
int run_selftest_wait(int* status, void* out, cudaStream_t st);
size_t selftest_out_bytes();
cudaError_t launch_prep(const Problem& P, const int32_t* ids, int32_t* seg_start, int32_t* seg_end, cudaStream_t st);
cudaError_t launch_prologue(const Problem& P, const void* q, const void* k, void* qo, void* ko, cudaStream_t st);
cudaError_t launch_bwd_pre(const Problem& P, const void* o, const void* dout, float* delta, float* dq_acc,
                           cudaStream_t st);
cudaError_t launch_grad_finalize(const Problem& P, const float* dq_acc, const float* dk_acc, const void* q,
                                 const void* k, void* dq, void* dk, cudaStream_t st);
cudaError_t launch_fwd(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, float* lse, cudaStream_t st);
cudaError_t launch_bwd(const Problem& P, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdv, const CUtensorMap& tdk,
                       const float* lse, const float* delta, float* dq_acc, cudaStream_t st);
DecodePlan decode_plan(const Problem& P, int Tq);
cudaError_t launch_decode(const Problem& P, const DecodePlan& d, const void* q, const CUtensorMap& tk,
                          const CUtensorMap& tv, float* part, int* done, void* o, float* lse, cudaStream_t st);

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;
    }
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev] = n;
    }
    return cache[dev];
}

cudaError_t ensure_dyn_smem(const void* kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::vector<std::pair<const void*, int>> done;  // (kernel, device) pairs already set
    std::lock_guard<std::mutex> lock(mu);
    for (const auto& d : done)
        if (d.first == kernel && d.second == dev) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.emplace_back(kernel, dev);
    return e;
}

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ------------------------------------------------------------------ workspace layout
struct Layout {
    size_t status = 0, seg_start = 0, seg_end = 0, qp = 0, kp = 0, delta = 0, dq_acc = 0, dk_acc = 0, total = 0;
};

bool needs_prologue(const csa_params& p) { return p.qk_norm != 0 || p.rope_base > 0.f; }

Layout layout(const csa_params& p, bool backward, bool has_seg) {
    Layout L;
    const size_t BT = (size_t)p.B * p.T;
    size_t off = 0;
    L.status = off;
    off += kAlign;
    if (has_seg) {
        L.seg_start = off;
        off += up(BT * 4);
        L.seg_end = off;
        off += up(BT * 4);
    }
    if (needs_prologue(p)) {
        L.qp = off;
        off += up(BT * p.Hq * p.D * 2);
        L.kp = off;
        off += up(BT * p.Hkv * p.D * 2);
    }
    if (backward) {
        L.delta = off;
        off += up(BT * p.Hq * 4);
        L.dq_acc = off;
        off += up(BT * p.Hq * p.D * 4);
        if (needs_prologue(p)) {
            L.dk_acc = off;
            off += up(BT * p.Hkv * p.D * 4);
        }
    }
    L.total = off;
    return L;
}

int check_params(const csa_params* p) {
    if (!p) return CSA_ERR_INVALID_ARG;
    if (p->B < 0 || p->T < 0 || p->T > (1 << 20)) return CSA_ERR_INVALID_ARG;
    if (p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv != 0) return CSA_ERR_INVALID_ARG;
    if (p->D != 32 && p->D != 64 && p->D != 96 && p->D != 128) return CSA_ERR_INVALID_ARG;
    if (p->causal != 0 && p->causal != 1) return CSA_ERR_INVALID_ARG;
    if (!isfinite(p->softcap) || !isfinite(p->rope_base) || !isfinite(p->scale)) return CSA_ERR_INVALID_ARG;
    if (p->qk_norm != 0 && p->qk_norm != 1) return CSA_ERR_INVALID_ARG;
    if (p->qk_norm && !(p->qk_norm_eps > 0.f && isfinite(p->qk_norm_eps))) return CSA_ERR_INVALID_ARG;
    // row indices of the row kernels are 31-bit (multiply-shift division)
    if ((double)p->B * p->T * (p->Hq + p->Hkv) >= 2147483648.0) return CSA_ERR_INVALID_ARG;
    return CSA_OK;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// ------------------------------------------------------------------ device checks
int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    static int known[64] = {0};  // 0 unknown, 1 ok, 2 wrong arch
    if (dev < 64 && known[dev]) return known[dev] == 1 ? CSA_OK : CSA_ERR_ARCH;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    const bool ok = (major == 10 && minor == 0);
    if (dev < 64) known[dev] = ok ? 1 : 2;
    return ok ? CSA_OK : CSA_ERR_ARCH;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
        else
            cudaGetLastError();
    }
    return fn;
}

// [B, T, H, D] bf16 tensor, boxes of (swizzle-atom width) x 1 head x 128 rows x 1 batch.
// promote: L2 fills of 256 bytes around each box row -- right when the other heads of the same
// tokens are read at about the same time (the attention kernels), wasted bytes when they are
// not (the decode kernel streams one head of a token long before or after its neighbours).
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int D, bool promote = true) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int sw = (D % 64 == 0) ? 128 : 64;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)(sw / 2), 1, (cuuint32_t)kBM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          sw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          promote ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [B, T, H, D] fp32 accumulator for TMA reduce-adds: boxes of 16 floats x 1 head x 128 rows x
// 1 batch, 64-byte swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4, (cuuint64_t)T * H * D * 4};
    cuuint32_t box[4] = {16, 1, (cuuint32_t)kBM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ timing
struct TimingRec {
    int kernel;
    cudaEvent_t a, b;
};
bool g_timing = false;
std::vector<TimingRec> g_records;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

template <class F>
int timed(int kernel, cudaStream_t st, F&& launch) {
    cudaEvent_t a = nullptr, b = nullptr;
    if (g_timing) {
        a = take_event();
        b = take_event();
        if (a) cudaEventRecord(a, st);
    }
    const cudaError_t e = launch();
    if (g_timing && a && b) {
        cudaEventRecord(b, st);
        g_records.push_back({kernel, a, b});
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_LAUNCH;
    }
    return CSA_OK;
}

Problem make_problem(const csa_params& p, int* status) {
    Problem P;
    P.B = p.B;
    P.T = p.T;
    P.Hq = p.Hq;
    P.Hkv = p.Hkv;
    P.D = p.D;
    P.G = p.Hq / p.Hkv;
    P.causal = p.causal;
    P.window = p.window > 0 ? p.window : 0;
    P.softcap = p.softcap > 0.f ? p.softcap : 0.f;
    P.scale = p.scale > 0.f ? p.scale : (float)(1.0 / sqrt((double)p.D));
    P.scale_log2 = (float)((double)P.scale * 1.4426950408889634);
    P.cap_in = P.softcap > 0.f ? (float)((double)P.scale / (double)P.softcap) : 0.f;
    P.cap_log2 = (float)((double)P.softcap * 1.4426950408889634);
    // With QK-norm on the prologue's own output, |q'| and |k'| are at most sqrt(D) (RMS at
    // most 1; bf16 rounding adds below 2^-9 each), so |scale q'.k' / softcap| is at most
    // D scale / softcap times 1.004; the series tanh serves while that stays under 1/4
    // (2% margin).  Callers whose keys do not come from the prologue clear the flag.
    P.cap_series = (P.softcap > 0.f && p.qk_norm &&
                    (double)p.D * (double)P.scale / (double)P.softcap * 1.02 <= 0.25) ? 1 : 0;
    P.rope = p.rope_base > 0.f ? 1 : 0;
    P.rope_log_base = p.rope_base > 0.f ? log((double)p.rope_base) : 0.0;
    P.qk_norm = p.qk_norm;
    P.eps = p.qk_norm_eps;
    P.seg_start = nullptr;
    P.seg_end = nullptr;
    P.div_hq = make_fastdiv((uint32_t)p.Hq);
    P.div_hkv = make_fastdiv((uint32_t)p.Hkv);
    P.div_t = make_fastdiv((uint32_t)(p.T > 0 ? p.T : 1));
    P.Tq = p.T;
    P.qoff = 0;
    P.div_tq = P.div_t;
    P.status = status;
    P.counters = status ? status + 1 : nullptr;
    return P;
}

// Shared front half of both calls: checks, status reset, segment bounds, prologue.
struct Prepared {
    Problem P;
    Layout L;
    const void* qk_q;  // tensors the attention kernels read as Q and K (raw or prologue output)
    const void* qk_k;
};

// reuse: the forward already left the segment bounds and q', k' in the same workspace (same
// layout: the backward only appends); nothing is launched but the reset.
int prepare(const csa_params* p, bool backward, const void* q, const void* k, const int32_t* seg, void* ws,
            size_t ws_bytes, cudaStream_t st, Prepared& out, bool reuse = false) {
    const bool has_seg = seg != nullptr;
    out.L = layout(*p, backward, has_seg);
    if (ws_bytes < out.L.total) return CSA_ERR_WORKSPACE;
    uint8_t* w = static_cast<uint8_t*>(ws);
    out.P = make_problem(*p, reinterpret_cast<int*>(w + out.L.status));
    // status word and the persistent kernels' work counters start at zero
    if (cudaMemsetAsync(w + out.L.status, 0, 4 * sizeof(int), st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    int32_t* ss = has_seg ? reinterpret_cast<int32_t*>(w + out.L.seg_start) : nullptr;
    int32_t* se = has_seg ? reinterpret_cast<int32_t*>(w + out.L.seg_end) : nullptr;
    out.P.seg_start = ss;
    out.P.seg_end = se;
    if (reuse) {
        out.qk_q = needs_prologue(*p) ? static_cast<const void*>(w + out.L.qp) : q;
        out.qk_k = needs_prologue(*p) ? static_cast<const void*>(w + out.L.kp) : k;
        return CSA_OK;
    }
    if (has_seg) {
        const int rc = timed(kPrep, st, [&] { return launch_prep(out.P, seg, ss, se, st); });
        if (rc) return rc;
    }
    out.qk_q = q;
    out.qk_k = k;
    if (needs_prologue(*p)) {
        void* qp = w + out.L.qp;
        void* kp = w + out.L.kp;
        const int rc = timed(kPrologue, st, [&] { return launch_prologue(out.P, q, k, qp, kp, st); });
        if (rc) return rc;
        out.qk_q = qp;
        out.qk_k = kp;
    }
    return CSA_OK;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" {

size_t csa_workspace_size(const csa_params* p, int for_backward) {
    if (check_params(p) != CSA_OK) return 0;
    // segment_ids may or may not be passed: size for the larger case
    return layout(*p, for_backward != 0, true).total;
}

int csa_attn_fwd(const csa_params* p, const void* q, const void* k, const void* v, const int32_t* segment_ids, void* o,
                 float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_params(p);
    if (rc) return rc;
    if (p->B == 0 || p->T == 0) return CSA_OK;
    if (!q || !k || !v || !o || !lse || !workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(workspace, 256) || (segment_ids && !aligned(segment_ids, 4)))
        return CSA_ERR_ALIGNMENT;
    if (workspace_bytes < layout(*p, false, segment_ids != nullptr).total) return CSA_ERR_WORKSPACE;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Prepared pr;
    if ((rc = prepare(p, false, q, k, segment_ids, workspace, workspace_bytes, st, pr))) return rc;
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, pr.qk_q, p->B, p->T, p->Hq, p->D) || !make_map(&tk, pr.qk_k, p->B, p->T, p->Hkv, p->D) ||
        !make_map(&tv, v, p->B, p->T, p->Hkv, p->D) || !make_map(&to, o, p->B, p->T, p->Hq, p->D))
        return CSA_ERR_CUDA;
    return timed(kFwd, st, [&] { return launch_fwd(pr.P, tq, tk, tv, to, lse, st); });
}

}  // extern "C"

namespace csa {
namespace {
int attn_bwd(const csa_params* p, const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const int32_t* segment_ids, void* dq, void* dk, void* dv, void* workspace,
             size_t workspace_bytes, void* stream, bool reuse) {
    int rc = check_params(p);
    if (rc) return rc;
    if (p->B == 0 || p->T == 0) return CSA_OK;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256) ||
        (segment_ids && !aligned(segment_ids, 4)))
        return CSA_ERR_ALIGNMENT;
    if (workspace_bytes < layout(*p, true, segment_ids != nullptr).total) return CSA_ERR_WORKSPACE;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Prepared pr;
    if ((rc = prepare(p, true, q, k, segment_ids, workspace, workspace_bytes, st, pr, reuse))) return rc;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    float* delta = reinterpret_cast<float*>(w + pr.L.delta);
    float* dq_acc = reinterpret_cast<float*>(w + pr.L.dq_acc);
    float* dk_acc = needs_prologue(*p) ? reinterpret_cast<float*>(w + pr.L.dk_acc) : nullptr;
    if ((rc = timed(kBwdPre, st, [&] { return launch_bwd_pre(pr.P, o, dout, delta, dq_acc, st); }))) return rc;
    // dK leaves the kernel as raw fp32 sums (finalize applies scale, RoPE^T and the norm
    // backward) when QK-norm or RoPE is on, else as bf16 scale * dK'
    CUtensorMap tq, tk, tv, tdo, tdq, tdv, tdk;
    if (!make_map(&tq, pr.qk_q, p->B, p->T, p->Hq, p->D) || !make_map(&tk, pr.qk_k, p->B, p->T, p->Hkv, p->D) ||
        !make_map(&tv, v, p->B, p->T, p->Hkv, p->D) || !make_map(&tdo, dout, p->B, p->T, p->Hq, p->D) ||
        !make_map_f32(&tdq, dq_acc, p->B, p->T, p->Hq, p->D) || !make_map(&tdv, dv, p->B, p->T, p->Hkv, p->D) ||
        !(dk_acc ? make_map_f32(&tdk, dk_acc, p->B, p->T, p->Hkv, p->D) : make_map(&tdk, dk, p->B, p->T, p->Hkv, p->D)))
        return CSA_ERR_CUDA;
    if ((rc = timed(kBwd, st, [&] {
             return launch_bwd(pr.P, tq, tk, tv, tdo, tdq, tdv, tdk, lse, delta, dq_acc, st);
         })))
        return rc;
    return timed(kGradFinalize, st,
                 [&] { return launch_grad_finalize(pr.P, dq_acc, dk_acc, q, k, dq, dk, st); });
}
}  // namespace
}  // namespace csa

extern "C" {

int csa_attn_bwd(const csa_params* p, const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, const int32_t* segment_ids, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, void* stream) {
    return attn_bwd(p, q, k, v, o, dout, lse, segment_ids, dq, dk, dv, workspace, workspace_bytes, stream, false);
}

int csa_attn_bwd_after_fwd(const csa_params* p, const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, const int32_t* segment_ids, void* dq, void* dk,
                           void* dv, void* workspace, size_t workspace_bytes, void* stream) {
    return attn_bwd(p, q, k, v, o, dout, lse, segment_ids, dq, dk, dv, workspace, workspace_bytes, stream, true);
}

// ------------------------------------------------------------------ forward over a KV cache
// Tq queries at absolute positions T - Tq + i over a cache of p->T entries (chunked prefill);
// the tensor-core forward with its own query length and offset.  Workspace: status slot,
// q' (queries only: the cache holds processed keys).
static int check_prefill(const csa_params* p, int Tq) {
    int rc = check_params(p);
    if (rc) return rc;
    if (Tq < 1 || Tq > p->T) return CSA_ERR_INVALID_ARG;
    return CSA_OK;
}

static size_t prefill_ws_bytes(const csa_params* p, int Tq, size_t* qp_off) {
    size_t off = kAlign;
    *qp_off = off;
    if (needs_prologue(*p)) off += up((size_t)p->B * Tq * p->Hq * p->D * 2);
    return off;
}

size_t csa_prefill_workspace_size(const csa_params* p, int Tq) {
    if (check_prefill(p, Tq) != CSA_OK) return 0;
    size_t a;
    return prefill_ws_bytes(p, Tq, &a);
}

int csa_attn_prefill(const csa_params* p, int Tq, const void* q, const void* k_cache, const void* v_cache, void* o,
                     float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_prefill(p, Tq);
    if (rc) return rc;
    if (p->B == 0) return CSA_OK;
    if (!q || !k_cache || !v_cache || !o || !lse || !workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(workspace, 256))
        return CSA_ERR_ALIGNMENT;
    size_t qp_off;
    if (workspace_bytes < prefill_ws_bytes(p, Tq, &qp_off)) return CSA_ERR_WORKSPACE;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    if (cudaMemsetAsync(w, 0, 4 * sizeof(int), st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    Problem P = make_problem(*p, reinterpret_cast<int*>(w));
    P.Tq = Tq;
    P.qoff = p->T - Tq;
    P.div_tq = make_fastdiv((uint32_t)Tq);
    P.cap_series = 0;  // the cached keys come from the caller: no bound on the scores
    const void* qq = q;
    if (needs_prologue(*p)) {
        void* qp = w + qp_off;
        if ((rc = timed(kPrologue, st, [&] { return launch_prologue(P, q, nullptr, qp, nullptr, st); }))) return rc;
        qq = qp;
    }
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, qq, p->B, Tq, p->Hq, p->D) || !make_map(&tk, k_cache, p->B, p->T, p->Hkv, p->D) ||
        !make_map(&tv, v_cache, p->B, p->T, p->Hkv, p->D) || !make_map(&to, o, p->B, Tq, p->Hq, p->D))
        return CSA_ERR_CUDA;
    return timed(kFwd, st, [&] { return launch_fwd(P, tq, tk, tv, to, lse, st); });
}

// ------------------------------------------------------------------ KV-cache decode
// Tq new queries over a cache of p->T entries; the rows of one (b, kv head), G * Tq, are at
// most 16 (the decode kernel keeps them in registers).
static int check_decode(const csa_params* p, int Tq) {
    int rc = check_params(p);
    if (rc) return rc;
    if (Tq < 1 || Tq > 16 || Tq > p->T) return CSA_ERR_INVALID_ARG;
    if ((p->Hq / p->Hkv) * Tq > 16) return CSA_ERR_NOT_IMPLEMENTED;
    return CSA_OK;
}

// Workspace: status slot, the per-(b, kv head) range counters right behind it (one clearing
// memset covers both), then the partials of every key range.
static size_t decode_ws_bytes(const csa_params* p, int Tq) {
    const Problem P = make_problem(*p, nullptr);
    const DecodePlan d = decode_plan(P, Tq);
    return kAlign + up(d.done_bytes) + up(d.part_bytes);
}

size_t csa_decode_workspace_size(const csa_params* p, int Tq) {
    if (check_decode(p, Tq) != CSA_OK) return 0;
    return decode_ws_bytes(p, Tq);
}

int csa_attn_decode(const csa_params* p, int Tq, const void* q, const void* k_cache, const void* v_cache, void* o,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_decode(p, Tq);
    if (rc) return rc;
    if (p->B == 0) return CSA_OK;
    if (!q || !k_cache || !v_cache || !o || !lse || !workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(workspace, 256))
        return CSA_ERR_ALIGNMENT;
    if (workspace_bytes < decode_ws_bytes(p, Tq)) return CSA_ERR_WORKSPACE;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    const Problem P = make_problem(*p, reinterpret_cast<int*>(w));
    const DecodePlan d = decode_plan(P, Tq);
    int* done = reinterpret_cast<int*>(w + kAlign);
    float* part = reinterpret_cast<float*>(w + kAlign + up(d.done_bytes));
    CUtensorMap tk, tv;
    if (!make_map(&tk, k_cache, p->B, p->T, p->Hkv, p->D, false) ||
        !make_map(&tv, v_cache, p->B, p->T, p->Hkv, p->D, false))
        return CSA_ERR_CUDA;
    // status word and range counters start at zero
    if (cudaMemsetAsync(w, 0, kAlign + d.done_bytes, st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    return timed(kDecode, st, [&] { return launch_decode(P, d, q, tk, tv, part, done, o, lse, st); });
}

}  // extern "C"

// ------------------------------------------------------------------ projections around attention
// x [B*T, C] -> q, k, v through the 3-D weights, o -> y through wo, and the backward products
// (gemm.cu).  Every matrix is row-major; the status word sits at the start of the workspace.
namespace csa {
cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& g, cudaStream_t st);
namespace {

// Row-major [rows, cols] matrix (bf16, or fp32 when f32), boxes of box_cols x box_rows
// elements with 128-byte swizzle (box_cols x element size = 128 bytes).
bool make_map_2d(CUtensorMap* m, const void* base, long long rows, int cols, bool f32, int box_cols,
                 int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * es};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tile width: one of 256, 192, 128, 64 that divides every piece of N (all four when N is one
// piece).  The persistent grid gives each SM ceil(tiles / SMs) tiles, so the launch takes
// about that many tile times.  A tile's time is its width plus a fixed share worth 256
// columns -- the 128-row A operand streams through the SM whatever the width (fitted to the
// 181M layer: 256-wide tiles in 6 waves beat 192-wide ones in 7).  The weight gradients
// (split over K to fill the SMs) take the widest width instead.
int pick_bn(const int* widths, int npieces, int M, bool split_k) {
    static const int cand[4] = {256, 192, 128, 64};
    int N = 0;
    for (int i = 0; i < npieces; ++i) N += widths[i];
    const long long mt = (M + 127) / 128;
    const long long sms = num_sms();
    int best = 0;
    long long best_cost = 0;
    for (int c : cand) {
        bool ok = true;
        for (int i = 0; i < npieces && npieces > 1; ++i) ok = ok && (widths[i] % c == 0);
        if (!ok) continue;
        if (split_k) return c;
        const long long tiles = mt * ((N + c - 1) / c);
        const long long cost = (tiles + sms - 1) / sms * (c + 256);
        if (best == 0 || cost < best_cost) {
            best = c;
            best_cost = cost;
        }
    }
    return best;
}

// Fills the piece bounds (from the piece widths) and the tile / split plan.  Weight gradients
// (split_k) cut K so that about one unit runs per SM (per CTA pair), keeping at least 4 K
// blocks a split.  Large products run on CTA pairs (256 x 256 tiles, cta_group::2) when
// allow_pair: at least one unit for every pair of SMs.  A K-major B with several N pieces
// never does (its 128-column half-box would straddle them).  The operand forms (a_mn, b_mn,
// b_by_k) must be set in g before the call.
void plan_gemm(GemmArgs& g, int M, int N, int K, const int* nw, int nn, const int* kw, int nk, bool split_k,
               bool allow_pair, int* status) {
    g.M = M;
    g.N = N;
    g.K = K;
    g.n_bound[0] = g.k_bound[0] = 0;
    for (int i = 1; i < 4; ++i) {
        g.n_bound[i] = (i <= nn - 1) ? g.n_bound[i - 1] + nw[i - 1] : N;
        g.k_bound[i] = (i <= nk - 1) ? g.k_bound[i - 1] + kw[i - 1] : K;
    }
    g.kb_total = (K + 63) / 64;
    g.status = status;
    const int pairs = num_sms() / 2;
    // a K-major B is loaded as one 128-column half-box per CTA, which must not straddle N pieces
    if (!g.b_mn && !g.b_by_k && nn > 1) allow_pair = false;
    if (allow_pair) {
        const int mt2 = (M + 255) / 256, nt2 = (N + 255) / 256;
        int splits = 1;
        if (split_k) {
            splits = pairs / (mt2 * nt2);
            if (splits > g.kb_total / 4) splits = g.kb_total / 4;
            if (splits < 1) splits = 1;
        }
        if (mt2 * nt2 * splits >= (split_k ? pairs / 2 : pairs)) {
            g.pair = 1;
            g.bn = 256;
            g.mt = mt2;
            g.nt = nt2;
            g.kb_per_split = (g.kb_total + splits - 1) / splits;
            g.splits = (g.kb_total + g.kb_per_split - 1) / g.kb_per_split;
            g.units = g.mt * g.nt * g.splits;
            return;
        }
    }
    g.pair = 0;
    g.bn = pick_bn(nw, nn, M, split_k);
    g.mt = (M + 127) / 128;
    g.nt = (N + g.bn - 1) / g.bn;
    int splits = 1;
    if (split_k) {
        const int tiles = g.mt * g.nt;
        splits = num_sms() / tiles;
        if (splits > g.kb_total / 4) splits = g.kb_total / 4;
        if (splits < 1) splits = 1;
    }
    g.kb_per_split = (g.kb_total + splits - 1) / splits;
    g.splits = (g.kb_total + g.kb_per_split - 1) / g.kb_per_split;
    g.units = g.mt * g.nt * g.splits;
}

// Host-side checks shared by the projection calls: the attention parameters (for Hq, Hkv,
// D), the model width, the piece alignment, the workspace (status word only).
int check_proj(const csa_params* p, int d_model, const void* workspace, size_t workspace_bytes) {
    int rc = check_params(p);
    if (rc) return rc;
    if (d_model < 64 || d_model % 64 != 0 || d_model > (1 << 16)) return CSA_ERR_INVALID_ARG;
    if ((p->Hkv * p->D) % 64 != 0) return CSA_ERR_INVALID_ARG;
    if (!workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGNMENT;
    if (workspace_bytes < kAlign) return CSA_ERR_WORKSPACE;
    return CSA_OK;
}

int check_ptrs(std::initializer_list<const void*> ptrs) {
    for (const void* q : ptrs)
        if (!q) return CSA_ERR_INVALID_ARG;
    for (const void* q : ptrs)
        if (!aligned(q, 16)) return CSA_ERR_ALIGNMENT;
    return CSA_OK;
}

int run_gemm(int kernel, const GemmMaps& maps, const GemmArgs& g, cudaStream_t st) {
    if (g.units == 0) return CSA_OK;
    return timed(kernel, st, [&] { return launch_gemm(maps, g, st); });
}

}  // namespace
}  // namespace csa

extern "C" {

size_t csa_proj_workspace_size(void) { return kAlign; }

int csa_qkv_proj(const csa_params* p, int d_model, const void* x, const void* wq, const void* wk, const void* wv,
                 void* q, void* k, void* v, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_proj(p, d_model, workspace, workspace_bytes);
    if (rc) return rc;
    if ((rc = check_ptrs({x, wq, wk, wv, q, k, v}))) return rc;
    if ((rc = check_device())) return rc;
    const long long M = (long long)p->B * p->T;
    if (M == 0) return CSA_OK;
    const int hq = p->Hq * p->D, hk = p->Hkv * p->D;
    const int nw[3] = {hq, hk, hk};
    GemmArgs g{};
    g.a_mn = 0;
    g.b_mn = 1;
    g.f32_out = 0;
    g.b_by_k = 0;
    plan_gemm(g, (int)M, hq + 2 * hk, d_model, nw, 3, nullptr, 1, false, true, static_cast<int*>(workspace));
    GemmMaps maps;
    const void* w3[3] = {wq, wk, wv};
    void* o3[3] = {q, k, v};
    bool ok = make_map_2d(&maps.a[0], x, M, d_model, false, 64, 128);
    maps.a[1] = maps.a[2] = maps.a[0];
    for (int i = 0; i < 3; ++i) {
        ok = ok && make_map_2d(&maps.b[i], w3[i], d_model, nw[i], false, 64, 64);
        ok = ok && make_map_2d(&maps.c[i], o3[i], M, nw[i], false, 64, 32);
    }
    if (!ok) return CSA_ERR_CUDA;
    return run_gemm(kGemmQkv, maps, g, static_cast<cudaStream_t>(stream));
}

int csa_out_proj(const csa_params* p, int d_model, const void* o, const void* wo, void* y, void* workspace,
                 size_t workspace_bytes, void* stream) {
    int rc = check_proj(p, d_model, workspace, workspace_bytes);
    if (rc) return rc;
    if ((rc = check_ptrs({o, wo, y}))) return rc;
    if ((rc = check_device())) return rc;
    const long long M = (long long)p->B * p->T;
    if (M == 0) return CSA_OK;
    const int hq = p->Hq * p->D;
    GemmArgs g{};
    g.a_mn = 0;
    g.b_mn = 1;
    g.f32_out = 0;
    g.b_by_k = 0;
    plan_gemm(g, (int)M, d_model, hq, &d_model, 1, nullptr, 1, false, true, static_cast<int*>(workspace));
    GemmMaps maps;
    bool ok = make_map_2d(&maps.a[0], o, M, hq, false, 64, 128) && make_map_2d(&maps.b[0], wo, hq, d_model, false, 64, 64) &&
              make_map_2d(&maps.c[0], y, M, d_model, false, 64, 32);
    if (!ok) return CSA_ERR_CUDA;
    maps.a[1] = maps.a[2] = maps.a[0];
    maps.b[1] = maps.b[2] = maps.b[0];
    maps.c[1] = maps.c[2] = maps.c[0];
    return run_gemm(kGemmOut, maps, g, static_cast<cudaStream_t>(stream));
}

int csa_out_proj_bwd(const csa_params* p, int d_model, const void* o, const void* wo, const void* dy, void* dout,
                     float* dwo, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_proj(p, d_model, workspace, workspace_bytes);
    if (rc) return rc;
    if ((rc = check_ptrs({o, wo, dy, dout}))) return rc;
    if (dwo && !aligned(dwo, 16)) return CSA_ERR_ALIGNMENT;
    if ((rc = check_device())) return rc;
    const long long M = (long long)p->B * p->T;
    if (M == 0) return CSA_OK;
    const int hq = p->Hq * p->D;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(workspace);
    {  // dout = dy wo^T: A = dy [M, C] K-major, B = wo [hq, C] K-major
        GemmArgs g{};
        g.a_mn = 0;
        g.b_mn = 0;
        g.f32_out = 0;
        g.b_by_k = 0;
        plan_gemm(g, (int)M, hq, d_model, &hq, 1, nullptr, 1, false, true, status);
        GemmMaps maps;
        bool ok = make_map_2d(&maps.a[0], dy, M, d_model, false, 64, 128) &&
                  make_map_2d(&maps.b[0], wo, hq, d_model, false, 64, g.pair ? 128 : g.bn) &&
                  make_map_2d(&maps.c[0], dout, M, hq, false, 64, 32);
        if (!ok) return CSA_ERR_CUDA;
        maps.a[1] = maps.a[2] = maps.a[0];
        maps.b[1] = maps.b[2] = maps.b[0];
        maps.c[1] = maps.c[2] = maps.c[0];
        if ((rc = run_gemm(kGemmDout, maps, g, st))) return rc;
    }
    if (!dwo) return CSA_OK;
    // dwo += o^T dy: A = o [M, hq] read M-major, B = dy [M, C] N-major, fp32 reduce-adds
    GemmArgs g{};
    g.a_mn = 1;
    g.b_mn = 1;
    g.f32_out = 1;
    g.b_by_k = 0;
    plan_gemm(g, hq, d_model, (int)M, &d_model, 1, nullptr, 1, true, true, status);
    GemmMaps maps;
    bool ok = make_map_2d(&maps.a[0], o, M, hq, false, 64, 64) && make_map_2d(&maps.b[0], dy, M, d_model, false, 64, 64) &&
              make_map_2d(&maps.c[0], dwo, hq, d_model, true, 32, 32);
    if (!ok) return CSA_ERR_CUDA;
    maps.a[1] = maps.a[2] = maps.a[0];
    maps.b[1] = maps.b[2] = maps.b[0];
    maps.c[1] = maps.c[2] = maps.c[0];
    return run_gemm(kGemmDwo, maps, g, st);
}

int csa_qkv_proj_bwd(const csa_params* p, int d_model, const void* x, const void* wq, const void* wk, const void* wv,
                     const void* dq, const void* dk, const void* dv, void* dx, float* dwq, float* dwk, float* dwv,
                     void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_proj(p, d_model, workspace, workspace_bytes);
    if (rc) return rc;
    if ((rc = check_ptrs({x, wq, wk, wv, dq, dk, dv, dx}))) return rc;
    const bool wgrad = dwq || dwk || dwv;
    if (wgrad && (rc = check_ptrs({dwq, dwk, dwv}))) return rc;
    if ((rc = check_device())) return rc;
    const long long M = (long long)p->B * p->T;
    if (M == 0) return CSA_OK;
    const int hq = p->Hq * p->D, hk = p->Hkv * p->D;
    const int w3[3] = {hq, hk, hk};
    const void* wt[3] = {wq, wk, wv};
    const void* gt[3] = {dq, dk, dv};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(workspace);
    {  // dx = dq wq^T + dk wk^T + dv wv^T: K pieced; A = dq|dk|dv K-major, B = wq|wk|wv [C, h] K-major
        GemmArgs g{};
        g.a_mn = 0;
        g.b_mn = 0;
        g.f32_out = 0;
        g.b_by_k = 1;
        plan_gemm(g, (int)M, d_model, hq + 2 * hk, &d_model, 1, w3, 3, false, true, status);
        GemmMaps maps;
        bool ok = make_map_2d(&maps.c[0], dx, M, d_model, false, 64, 32);
        for (int i = 0; i < 3; ++i) {
            ok = ok && make_map_2d(&maps.a[i], gt[i], M, w3[i], false, 64, 128);
            ok = ok && make_map_2d(&maps.b[i], wt[i], d_model, w3[i], false, 64, g.pair ? 128 : g.bn);
        }
        if (!ok) return CSA_ERR_CUDA;
        maps.c[1] = maps.c[2] = maps.c[0];
        if ((rc = run_gemm(kGemmDx, maps, g, st))) return rc;
    }
    if (!wgrad) return CSA_OK;
    // dwq|dwk|dwv += x^T [dq|dk|dv]: A = x [M, C] read M-major, B and C pieced by N, fp32
    GemmArgs g{};
    g.a_mn = 1;
    g.b_mn = 1;
    g.f32_out = 1;
    g.b_by_k = 0;
    plan_gemm(g, d_model, hq + 2 * hk, (int)M, w3, 3, nullptr, 1, true, true, status);
    GemmMaps maps;
    float* dw3[3] = {dwq, dwk, dwv};
    bool ok = make_map_2d(&maps.a[0], x, M, d_model, false, 64, 64);
    maps.a[1] = maps.a[2] = maps.a[0];
    for (int i = 0; i < 3; ++i) {
        ok = ok && make_map_2d(&maps.b[i], gt[i], M, w3[i], false, 64, 64);
        ok = ok && make_map_2d(&maps.c[i], dw3[i], d_model, w3[i], true, 32, 32);
    }
    if (!ok) return CSA_ERR_CUDA;
    return run_gemm(kGemmDw, maps, g, st);
}

int csa_selftest_bounded_wait(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace) return CSA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return CSA_ERR_ALIGNMENT;
    if (workspace_bytes < 256 + selftest_out_bytes()) return CSA_ERR_WORKSPACE;
    int rc = check_device();
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = static_cast<int*>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    if ((rc = run_selftest_wait(status, static_cast<uint8_t*>(workspace) + 256, st))) return rc;
    return csa_device_status(workspace, stream);
}

int csa_device_status(void* workspace, void* stream) {
    if (!workspace) return CSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    int code = 0;
    if (cudaMemcpy(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    if (code != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    return code;
}

const char* csa_status_string(int code) {
    switch (code) {
        case CSA_OK: return "ok";
        case CSA_ERR_INVALID_ARG: return "invalid argument (shape, head ratio, head dim, option or null pointer)";
        case CSA_ERR_ALIGNMENT: return "misaligned pointer (tensors need 16 bytes, workspace 256 bytes)";
        case CSA_ERR_WORKSPACE: return "workspace smaller than csa_workspace_size()";
        case CSA_ERR_ARCH: return "device is not a compute capability 10.0 (B200) GPU";
        case CSA_ERR_LAUNCH: return "kernel launch failed";
        case CSA_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel ran out";
        case CSA_ERR_CUDA: return "CUDA runtime or driver call failed";
        case CSA_ERR_NOT_IMPLEMENTED: return "not implemented";
        default: return "unknown status code";
    }
}

int csa_timing_enable(int enable) {
    g_timing = enable != 0;
    return CSA_OK;
}

int csa_timing_collect(double* total_ms, int* launches, int n) {
    int rc = CSA_OK;
    for (const TimingRec& r : g_records) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            cudaGetLastError();
            rc = CSA_ERR_CUDA;
        } else if (r.kernel < n) {
            if (total_ms) total_ms[r.kernel] += ms;
            if (launches) launches[r.kernel] += 1;
        }
        g_event_pool.push_back(r.a);
        g_event_pool.push_back(r.b);
    }
    g_records.clear();
    return rc;
}

int csa_num_kernels(void) { return kNumKernels; }

const char* csa_kernel_name(int k) {
    static const char* names[kNumKernels] = {"k_prep",          "k_qk_prologue", "k_attn_fwd",
                                             "k_bwd_pre",       "k_attn_bwd",    "k_grad_finalize",
                                             "k_decode",        "k_gemm_qkv",    "k_gemm_out",
                                             "k_gemm_dout",     "k_gemm_dwo",    "k_gemm_dx",
                                             "k_gemm_dw"};
    return (k >= 0 && k < kNumKernels) ? names[k] : "";
}

}  // extern "C"

// ------------------------------------------------------------------ forward with library-owned scratch
// For callers that cannot allocate device memory themselves (see csa_attn_fwd_static_scratch
// in csa.h).  The scratch is one file-scope device array, loaded with the library and held
// by every GPU that loads it until the process exits.
namespace csa {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)CSA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  In host code the array's name
// is only a host-side stand-in; the real address comes from cudaGetSymbolAddress with that
// device current.  It is looked up on every call (a cheap table lookup once the module is
// loaded, and it allocates nothing), so a context torn down and re-created by
// cudaDeviceReset never leaves a stale address behind.
int static_scratch_address(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return CSA_ERR_CUDA;
    }
    *out = p;
    return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" int csa_attn_fwd_static_scratch(const csa_params* p, const void* q, const void* k, const void* v,
                                           const int32_t* segment_ids, void* o, float* lse, int* device_status,
                                           void* stream) {
    int rc = check_params(p);
    if (rc) return rc;
    if (p->B == 0 || p->T == 0) return CSA_OK;
    if (!q || !k || !v || !o || !lse) return CSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        (segment_ids && !aligned(segment_ids, 4)) || (device_status && !aligned(device_status, 4)))
        return CSA_ERR_ALIGNMENT;
    // the problem's scratch must fit in the fixed array; nothing is allocated to make room
    if (layout(*p, false, segment_ids != nullptr).total > kStaticScratchBytes) return CSA_ERR_WORKSPACE;
    if ((rc = check_device())) return rc;
    void* scratch = nullptr;
    if ((rc = static_scratch_address(&scratch))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word is the only part that must start at zero: cleared by prepare();
    // everything else the kernels read is rewritten by this call before it is read
    Prepared pr;
    if ((rc = prepare(p, false, q, k, segment_ids, scratch, kStaticScratchBytes, st, pr))) return rc;
    if (device_status) {
        if (cudaMemsetAsync(device_status, 0, sizeof(int), st) != cudaSuccess) {
            cudaGetLastError();
            return CSA_ERR_CUDA;
        }
        pr.P.status = device_status;
    }
    CUtensorMap tq, tk, tv, to;
    if (!make_map(&tq, pr.qk_q, p->B, p->T, p->Hq, p->D) || !make_map(&tk, pr.qk_k, p->B, p->T, p->Hkv, p->D) ||
        !make_map(&tv, v, p->B, p->T, p->Hkv, p->D) || !make_map(&to, o, p->B, p->T, p->Hq, p->D))
        return CSA_ERR_CUDA;
    return timed(kFwd, st, [&] { return launch_fwd(pr.P, tq, tk, tv, to, lse, st); });
}
