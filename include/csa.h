/*
 * csa.h -- C ABI of libcsa.so: causal (or bidirectional) multi-head / grouped-query
 * self-attention, forward and backward, for NVIDIA B200 (sm_100a).
 *
 * The operation (per batch row b and query head h, with key/value head kv = h / (Hq/Hkv)):
 *
 *   q' = RoPE(RMSNorm(q)), k' = RoPE(RMSNorm(k))           (each step optional)
 *   s_ij = scale * q'_i . k'_j,  s'_ij = c * tanh(s_ij / c)   (cap optional)
 *   P_i  = softmax over the keys j visible to query i,  O_i = sum_j P_ij v_j
 *   LSE_i = log sum_j exp(s'_ij)   (natural log, over the visible keys)
 *
 * Sources: the scaled dot-product attention equation and the causal (upper-triangular -inf)
 * mask are those of the GPT-pretraining page (dekermanjian.github.io, llm_gpt_pretrain),
 * section "Multihead Attention"; grouped-query heads, RoPE, QK-norm (parameter-free
 * RMSNorm), logits soft-capping and RoPE from packed segment positions come from the
 * nanogpt-jax-181m model card, section "Architecture", and packed rows with segment_ids
 * from its section "SFT"; the sliding window from the flaxchat README, "Core Features";
 * attention of new queries over a key/value cache from the GPT-pretraining page, section
 * "Bonus: KV Caching".
 * The pages give no formulas for RoPE, the norm, the cap or the window; the readings used
 * here are stated at each field of csa_params.
 *
 * Conventions shared by every entry point
 *  - Tensors are row-major and contiguous (the KV-cache calls state their own query length):
 *    q, o, dout, dq are [B, T, Hq, D] bf16;
 *    k, v, dk, dv are [B, T, Hkv, D] bf16; lse is [B, Hq, T] fp32; segment_ids is [B, T] int32.
 *    bf16 pointers are passed as void* and hold IEEE bfloat16 bit patterns.
 *  - Every tensor pointer is a DEVICE pointer, allocated and owned by the caller, aligned to
 *    16 bytes.  The workspace is caller-owned device memory of at least
 *    csa_workspace_size() bytes, aligned to 256 bytes.  No call allocates device memory.
 *    The one piece of device memory the library owns is the fixed scratch array of
 *    csa_attn_fwd_static_scratch (CSA_STATIC_SCRATCH_BYTES), a module-scope array that every
 *    GPU holds once the library is loaded on it.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued on it and
 *    the call returns without synchronising.  The only call that synchronises is
 *    csa_device_status().
 *  - Errors found on the host (bad shapes, pointers, workspace, device) are returned before
 *    anything is enqueued; outputs are then untouched.  No call prints, aborts or throws.
 *  - Errors found on the device (a bounded wait inside a kernel that ran out) are written
 *    to a status word inside the workspace and read back with csa_device_status().
 *  - Calls on the same workspace must not overlap on the device.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,     /* shape, head ratio, head dim, option value or NULL pointer   */
    CSA_ERR_ALIGNMENT = 2,       /* a tensor pointer is not 16-byte (workspace: 256-byte) aligned */
    CSA_ERR_WORKSPACE = 3,       /* workspace smaller than csa_workspace_size()                  */
    CSA_ERR_ARCH = 4,            /* current device is not a compute-capability 10.0 GPU          */
    CSA_ERR_LAUNCH = 5,          /* a kernel launch failed (cudaGetLastError after enqueue)      */
    CSA_ERR_DEVICE_TIMEOUT = 6,  /* a bounded wait inside a kernel ran out (device-side)         */
    CSA_ERR_CUDA = 7,            /* another CUDA runtime / driver call failed                    */
    CSA_ERR_NOT_IMPLEMENTED = 8
};

/* Problem description.  B, T >= 0 (0 is an empty problem: nothing is enqueued, CSA_OK);
 * Hq, Hkv >= 1 with Hq % Hkv == 0 (query head h uses key/value head h / (Hq / Hkv),
 * contiguous groups); D in {32, 64, 96, 128}; T <= 1 << 20; B * T * (Hq + Hkv) < 2^31. */
typedef struct csa_params {
    int B, T, Hq, Hkv, D;
    int causal;        /* 1: key j visible to query i only if j <= i (decoder self-attention);
                          0: bidirectional                                                     */
    int window;        /* <= 0: off; else causal: visible only if i - j < window (window keys
                          including i); bidirectional: only if |i - j| < window              */
    float softcap;     /* <= 0: off; else s' = softcap * tanh(s / softcap) on the scaled score,
                          before the mask                                                      */
    float rope_base;   /* <= 0: off; else rotate-half RoPE: for d < D/2, phi = pos * base^(-2d/D),
                          (x_d, x_{d+D/2}) -> (x_d cos phi - x_{d+D/2} sin phi,
                                               x_{d+D/2} cos phi + x_d sin phi);
                          pos = index within the token's segment (= t without segment_ids)     */
    int qk_norm;       /* 1: x -> x * (mean_d x^2 + qk_norm_eps)^(-1/2) on every q and k head
                          vector, before RoPE; no learnable scale                              */
    float qk_norm_eps; /* > 0 when qk_norm is on (1e-6 in the pages' models)                  */
    float scale;       /* <= 0: 1 / sqrt(D); else the score scale                              */
} csa_params;

/* Bytes of workspace csa_attn_fwd (for_backward = 0) or csa_attn_bwd (for_backward = 1)
 * needs for *p; 0 if *p is invalid.  A workspace sized for the backward also serves the
 * forward. */
size_t csa_workspace_size(const csa_params* p, int for_backward);

/* Forward.  Reads the RAW q, k (before norm and RoPE) and v; writes o and lse.
 * segment_ids may be NULL (one segment per row); otherwise tokens attend only within their
 * maximal run of equal ids, and RoPE positions restart at 0 at each run's first token.
 * Returns a status code (host-side checks); device-side problems: csa_device_status(). */
int csa_attn_fwd(const csa_params* p, const void* q, const void* k, const void* v,
                 const int32_t* segment_ids, void* o, float* lse, void* workspace,
                 size_t workspace_bytes, void* stream);

/* Backward.  Given the forward's inputs, its outputs o and lse, and dout = dL/do, writes
 * dq, dk, dv = dL/d(raw q, k, v).  dk and dv of a key/value head sum the contributions of
 * all query heads of its group.  Stateless: the norm / RoPE prologue is recomputed, so the
 * workspace need not be the forward's. */
int csa_attn_bwd(const csa_params* p, const void* q, const void* k, const void* v, const void* o,
                 const void* dout, const float* lse, const int32_t* segment_ids, void* dq, void* dk,
                 void* dv, void* workspace, size_t workspace_bytes, void* stream);

/* Backward that reuses what the forward left in the workspace: the normalised and rotated
 * q', k' (QK-norm / RoPE on) and the segment bounds, so no prologue runs (a training step
 * computes q', k' once, in its forward).  Same arguments and results as csa_attn_bwd.
 * Contract: the workspace (sized with for_backward = 1) was passed to csa_attn_fwd with the
 * same *p, q, k and segment_ids, on the same stream, and nothing has written to it since.
 * The library cannot check this; a broken contract gives wrong gradients (every access
 * stays inside the workspace), never a fault. */
int csa_attn_bwd_after_fwd(const csa_params* p, const void* q, const void* k, const void* v,
                           const void* o, const void* dout, const float* lse,
                           const int32_t* segment_ids, void* dq, void* dk, void* dv,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Forward over a key/value cache (prefill of a chunk of Tq new tokens; the GPT-pretraining
 * page (dekermanjian.github.io, llm_gpt_pretrain), section "Bonus: KV Caching"): the same masking and arguments as
 * csa_attn_decode below, for any 1 <= Tq <= p->T, on the tensor-core forward.  The cache's
 * last Tq entries are the new tokens' own keys and values.  Workspace 256-byte aligned and at
 * least csa_prefill_workspace_size(p, Tq) bytes (0 when the arguments are invalid). */
size_t csa_prefill_workspace_size(const csa_params* p, int Tq);
int csa_attn_prefill(const csa_params* p, int Tq, const void* q, const void* k_cache,
                     const void* v_cache, void* o, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/* KV-cache decoding (the GPT-pretraining page, dekermanjian.github.io, llm_gpt_pretrain,
 * section "Bonus: KV Caching"):
 * Tq new queries attend over a cache of p->T entries.  With offset = p->T - Tq, query i sits
 * at absolute position offset + i and sees cache entry j when j <= offset + i (p->causal = 1;
 * 0: every entry) and, with a window W > 0, when |offset + i - j| < W.
 *   q        [B, Tq, Hq, D] bf16, raw: QK-norm and RoPE (at the absolute positions) are applied
 *            here when p->qk_norm / p->rope_base ask for them;
 *   k_cache  [B, p->T, Hkv, D] bf16, keys as stored after their own QK-norm and RoPE (the
 *            forward's prologue output for the same positions);
 *   v_cache  [B, p->T, Hkv, D] bf16;
 *   o        [B, Tq, Hq, D] bf16;  lse [B, Hq, Tq] fp32 (natural log).
 * 1 <= Tq <= min(16, p->T) (CSA_ERR_INVALID_ARG otherwise) and (Hq / Hkv) * Tq <= 16
 * (CSA_ERR_NOT_IMPLEMENTED otherwise); segment_ids do not apply.  Tensors 16-byte aligned,
 * workspace 256-byte aligned and at least csa_decode_workspace_size(p, Tq) bytes (0 when the
 * arguments are invalid).  The pages give no kernel for this; it is memory-bound and runs on
 * the CUDA cores, split over the cache, then merged. */
size_t csa_decode_workspace_size(const csa_params* p, int Tq);
int csa_attn_decode(const csa_params* p, int Tq, const void* q, const void* k_cache,
                    const void* v_cache, void* o, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Projections around attention (the nanogpt-jax-181m model card, section "Architecture":
 * 3-D attention weights wq, wk, wv of shape (d_emb, heads, head_dim) and wo of shape
 * (heads, head_dim, d_emb); the GPT-pretraining page, section "Multihead Attention": q, k, v
 * are linear maps of the block input x, and the attention output goes through an output
 * projection).  No bias: the 3-D weights of the model card carry none.  With C = d_model:
 *   x, y, dx, dy   [B, T, C] bf16
 *   wq             [C, Hq, D] bf16;   wk, wv [C, Hkv, D] bf16;   wo [Hq, D, C] bf16
 *   q = x wq, k = x wk, v = x wv      (sum over C; q [B,T,Hq,D], k, v [B,T,Hkv,D] bf16)
 *   y = o wo                           (sum over heads and D; o [B,T,Hq,D])
 * Backward, for a loss L with dy = dL/dy (and dq, dk, dv = dL/dq, ...):
 *   csa_out_proj_bwd:  dout = dy wo^T (bf16 [B,T,Hq,D]);  dwo += o^T dy
 *   csa_qkv_proj_bwd:  dx = dq wq^T + dk wk^T + dv wv^T (bf16);
 *                      dwq += x^T dq, dwk += x^T dk, dwv += x^T dv
 * Weight gradients are fp32 tensors of the weights' shapes, ADDED to what they hold (zero
 * them for a plain gradient; leave them for accumulation over micro-batches).  Pass NULL for
 * dwo, or for all three of dwq, dwk, dwv, to skip them.  Products accumulate in fp32; bf16
 * outputs are rounded once, to nearest even.
 * Requirements (CSA_ERR_INVALID_ARG otherwise): *p valid as for csa_attn_fwd (only B, T, Hq,
 * Hkv, D are used), C a multiple of 64 (at most 65536), Hkv * D a multiple of 64.  Device
 * pointers 16-byte aligned, caller-owned.  The workspace holds only the status word: at least
 * csa_proj_workspace_size() bytes, 256-byte aligned (an attention workspace serves).  A
 * bounded wait that runs out records CSA_ERR_DEVICE_TIMEOUT there, read back with
 * csa_device_status(); these calls do not clear the word.  One launch per product: two for
 * each backward call with weight gradients. */
size_t csa_proj_workspace_size(void);
int csa_qkv_proj(const csa_params* p, int d_model, const void* x, const void* wq, const void* wk,
                 const void* wv, void* q, void* k, void* v, void* workspace, size_t workspace_bytes,
                 void* stream);
int csa_out_proj(const csa_params* p, int d_model, const void* o, const void* wo, void* y,
                 void* workspace, size_t workspace_bytes, void* stream);
int csa_out_proj_bwd(const csa_params* p, int d_model, const void* o, const void* wo,
                     const void* dy, void* dout, float* dwo, void* workspace,
                     size_t workspace_bytes, void* stream);
int csa_qkv_proj_bwd(const csa_params* p, int d_model, const void* x, const void* wq,
                     const void* wk, const void* wv, const void* dq, const void* dk,
                     const void* dv, void* dx, float* dwq, float* dwk, float* dwv,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream` and returns the device-side status recorded in `workspace` by the
 * last call that used it (CSA_OK, CSA_ERR_DEVICE_TIMEOUT, or CSA_ERR_CUDA when the
 * synchronisation itself failed).  Resets the recorded status to CSA_OK. */
int csa_device_status(void* workspace, void* stream);

/* Self-test of the bounded waits every kernel relies on (failure detection without a GPU
 * fault): launches one 128-thread CTA whose threads wait on mbarrier phases that never
 * complete.  Each wait gives up after about a second of SM clocks, or as soon as another
 * thread of the CTA has given up, records CSA_ERR_DEVICE_TIMEOUT in the workspace status
 * word and returns; the CTA then exits normally.  The workspace (>= 2048 bytes, 256-byte
 * aligned) receives the status word at offset 0 and, at offset 256, int gave_up[128]
 * followed by long long cycles[128] (1 = that thread's wait gave up; clocks it waited).
 * Synchronises the stream and returns the device status read back: CSA_ERR_DEVICE_TIMEOUT
 * when the mechanism works, a host-side error code otherwise. */
int csa_selftest_bounded_wait(void* workspace, size_t workspace_bytes, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* csa_status_string(int code);

/* Size of the library-owned scratch array used by csa_attn_fwd_static_scratch (16 MiB). */
#define CSA_STATIC_SCRATCH_BYTES (16u << 20)

/* Forward without a workspace argument, for callers that cannot allocate device memory:
 * code that runs inside a host framework which owns every device allocation through its
 * own allocator (and gives this caller none), or a latency-critical loop where a
 * cudaMalloc, which may synchronise the device, is not acceptable.  The pages describe no
 * such entry point; it has no counterpart there.
 *
 * Same arguments and results as csa_attn_fwd, minus the workspace.  Its scratch (status
 * word, segment bounds, normalised q/k copies) lives in one file-scope device
 * array of CSA_STATIC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine.
 *  - A problem whose scratch would exceed CSA_STATIC_SCRATCH_BYTES (roughly
 *    B*T*(Hq+Hkv)*D*2 bytes with QK-norm or RoPE, plus 8*B*T with segment_ids) is rejected
 *    with CSA_ERR_WORKSPACE before anything is enqueued.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress) with the
 *    caller's device current; the first call on a device also loads the library's module
 *    there, so make that first call before any stream capture.
 *  - Every call shares the one array, which keeps the last call's contents.  The call
 *    clears the status word it needs at zero and rewrites everything else before reading
 *    it.  Calls that overlap on the GPU (different streams, or threads) race on the array
 *    and give wrong results: serialise them.
 *  - device_status: optional device pointer to one int; when non-NULL it is cleared and
 *    receives the device-side status (CSA_ERR_DEVICE_TIMEOUT if a bounded wait ran out).
 *    When NULL that status is only recorded inside the library's array. */
int csa_attn_fwd_static_scratch(const csa_params* p, const void* q, const void* k, const void* v,
                                const int32_t* segment_ids, void* o, float* lse, int* device_status,
                                void* stream);

/* Kernel timing (for measurement).  While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the launch stream.  csa_timing_collect()
 * synchronises those events, adds each kernel's elapsed times into `total_ms[k]` and its
 * launch count into `launches[k]` for k < n (k indexes csa_kernel_name()), and forgets them.
 * Not thread-safe. */
int csa_timing_enable(int enable);
int csa_timing_collect(double* total_ms, int* launches, int n);
int csa_num_kernels(void);
const char* csa_kernel_name(int k);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
