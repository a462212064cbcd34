/*
 * oracle.c -- plain, slow fp64 CPU reference for causal self-attention (MHA / GQA),
 * forward and backward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * CPU-baseline leg of the benchmark are the only callers.  It shares no code, header,
 * table or constant with the CUDA path.
 *
 * What it computes, step by step, and where each step is stated:
 *
 *  - Scaled dot-product attention, softmax(Q K^T / sqrt(d_k)) V, applied per head:
 *    "GPT pretraining" page (dekermanjian.github.io, llm_gpt_pretrain), section
 *    "Multihead Attention", the attention equation and the MultiHeadAttention listing
 *    (logits = q k^T / sqrt(head_dim), future logits set to -inf, softmax over keys,
 *    weights times v).
 *  - Causal mask (token i sees keys j <= i): same section; also "Build and Train a MiniGPT
 *    with JAX", section "Model Architecture" (lower-triangular mask).
 *  - Grouped-query heads (8 query / 4 key-value heads): "nanogpt-jax-181m" model card,
 *    section "Architecture".  Head h reads key/value head floor(h / G), G = Hq / Hkv
 *    (contiguous groups; the pages do not spell the mapping out).
 *  - Parameter-free RMSNorm on Q and K ("QK-norm", "parameter-free RMSNorm (no learnable
 *    scale)"): model card, "Architecture", design choices; flaxchat README, "Core Features".
 *    Read as x * (mean_d x^2 + eps)^(-1/2) over the head dimension, eps = 1e-6.
 *  - RoPE, rotate-half form with base 10000, applied after the norm; positions restart
 *    at 0 in every packed segment ("RoPE frequencies are computed from packed segment
 *    positions"): model card, "Architecture"; flaxchat README, "Core Features".
 *    Pair (d, d + D/2) rotated by phi = pos * base^(-2d/D).
 *  - Soft-capping of scores, s' = c * tanh(s / c), after the 1/sqrt(D) scaling and before
 *    the mask: model card, "Architecture" ("logits soft-capping"); flaxchat README.
 *  - Sliding window: key j visible to query i only if i - j < W (W keys including i);
 *    flaxchat README, "Core Features" ("Sliding Window").
 *  - Packed rows with segment_ids: attention stays inside a maximal run of equal ids;
 *    model card, section "SFT" (BestFit-packed rows with segment_ids).
 *  - Backward: the gradient of the same composite function by the chain rule (the pages
 *    obtain it by automatic differentiation, value_and_grad in their train steps).
 *
 * Inputs are fp64 arrays in [B, T, H, D] row-major order (the projection's natural
 * layout); LSE is [B, Hq, T] (natural log).  Nothing here is blocked, fused or reordered:
 * every (b, h) pair builds its full T x T score matrix.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, T, Hq, Hkv, D;
    int causal;        /* 1: key j visible to query i only if j <= i; 0: bidirectional        */
    int window;        /* <= 0: off; else causal: 0 <= i-j < window, bidirectional: |i-j| < window */
    double softcap;    /* <= 0: off; else s' = softcap * tanh(s / softcap)                    */
    double rope_base;  /* <= 0: off; else rotate-half RoPE with this base                     */
    int qk_norm;       /* 1: parameter-free RMSNorm of every Q and K head vector              */
    double qk_norm_eps;
    double scale;      /* <= 0: 1 / sqrt(D)                                                   */
} oracle_params;

static double eff_scale(const oracle_params* p) {
    return p->scale > 0.0 ? p->scale : 1.0 / sqrt((double)p->D);
}

/* Segment of every token: start[t] is the first index of the maximal run of equal ids
 * that contains t, end[t] is one past its last index.  Without ids the whole row is one
 * segment. */
void oracle_segments(int B, int T, const int32_t* seg_ids, int32_t* start, int32_t* end) {
    for (int b = 0; b < B; ++b) {
        const int32_t* id = seg_ids ? seg_ids + (size_t)b * T : NULL;
        int s = 0;
        for (int t = 0; t < T; ++t) {
            if (id && t > 0 && id[t] != id[t - 1]) s = t;
            start[(size_t)b * T + t] = s;
        }
        int e = T;
        for (int t = T - 1; t >= 0; --t) {
            if (id && t < T - 1 && id[t] != id[t + 1]) e = t + 1;
            end[(size_t)b * T + t] = e;
        }
    }
}

/* Is key j visible to query i?  (causal / window / segment rules above) */
static int visible(const oracle_params* p, int i, int j, const int32_t* st, const int32_t* en) {
    if (p->causal && j > i) return 0;
    if (p->window > 0) {
        int d = i - j;
        if (p->causal) { if (d >= p->window) return 0; }
        else if (d >= p->window || -d >= p->window) return 0;
    }
    if (j < st[i] || j >= en[i]) return 0;
    return 1;
}

/* One head vector of length D at position pos: optional RMSNorm, then optional RoPE. */
static void norm_rope_vec(const oracle_params* p, const double* x, int pos, double* y) {
    const int D = p->D;
    double r = 1.0;
    if (p->qk_norm) {
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += x[d] * x[d];
        r = 1.0 / sqrt(ss / D + p->qk_norm_eps);
    }
    for (int d = 0; d < D; ++d) y[d] = x[d] * r;
    if (p->rope_base > 0.0) {
        const int h = D / 2;
        for (int d = 0; d < h; ++d) {
            double theta = pow(p->rope_base, -2.0 * d / D);
            double phi = pos * theta;
            double c = cos(phi), s = sin(phi);
            double a = y[d], bb = y[d + h];
            y[d] = a * c - bb * s;
            y[d + h] = bb * c + a * s;
        }
    }
}

/* Transposed chain of norm_rope_vec: given g = dL/dy, return dL/dx. */
static void norm_rope_vec_bwd(const oracle_params* p, const double* x, int pos,
                              const double* g, double* dx) {
    const int D = p->D;
    double* u = (double*)malloc(sizeof(double) * D);
    memcpy(u, g, sizeof(double) * D);
    if (p->rope_base > 0.0) {  /* rotation by -phi is the transpose of rotation by phi */
        const int h = D / 2;
        for (int d = 0; d < h; ++d) {
            double theta = pow(p->rope_base, -2.0 * d / D);
            double phi = pos * theta;
            double c = cos(phi), s = sin(phi);
            double ga = g[d], gb = g[d + h];
            u[d] = ga * c + gb * s;
            u[d + h] = -ga * s + gb * c;
        }
    }
    if (p->qk_norm) {
        /* xhat = r x, r = (mean x^2 + eps)^(-1/2):  dx = r (u - xhat * mean(u * xhat)) */
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += x[d] * x[d];
        double r = 1.0 / sqrt(ss / D + p->qk_norm_eps);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += u[d] * x[d] * r;
        for (int d = 0; d < D; ++d) dx[d] = r * (u[d] - x[d] * r * dot / D);
    } else {
        memcpy(dx, u, sizeof(double) * D);
    }
    free(u);
}

static size_t idx4(int b, int t, int h, int d, int T, int H, int D) {
    return (((size_t)b * T + t) * H + h) * D + d;
}

/* Normalised + rotated copy of a [B,T,H,D] tensor (the intermediate Q' or K'). */
void oracle_qk_prologue(const oracle_params* p, int H, const double* x, const int32_t* seg_ids,
                        double* y) {
    const int B = p->B, T = p->T, D = p->D;
    int32_t* st = (int32_t*)malloc(sizeof(int32_t) * (size_t)B * T);
    int32_t* en = (int32_t*)malloc(sizeof(int32_t) * (size_t)B * T);
    oracle_segments(B, T, seg_ids, st, en);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                int pos = t - st[(size_t)b * T + t];
                norm_rope_vec(p, x + idx4(b, t, h, 0, T, H, D), pos, y + idx4(b, t, h, 0, T, H, D));
            }
    free(st);
    free(en);
}

/* Scores, masked softmax and the probability matrix of one (b, h):
 * S[i][j] = scale * q'_i . k'_j, capped if asked; P[i][j] = softmax_j over visible keys.
 * S keeps the capped score; Sraw (optional) the uncapped one.  Masked entries of P are 0. */
static void probs_one(const oracle_params* p, const double* q, const double* k, int b, int h,
                      const int32_t* st, const int32_t* en, double* S, double* Sraw, double* P,
                      double* lse) {
    const int T = p->T, D = p->D, G = p->Hq / p->Hkv, kvh = h / G;
    const double sc = eff_scale(p);
    double* qp = (double*)malloc(sizeof(double) * (size_t)T * D);
    double* kp = (double*)malloc(sizeof(double) * (size_t)T * D);
    for (int t = 0; t < T; ++t) {
        int pos = t - st[t];
        norm_rope_vec(p, q + idx4(b, t, h, 0, T, p->Hq, D), pos, qp + (size_t)t * D);
        norm_rope_vec(p, k + idx4(b, t, kvh, 0, T, p->Hkv, D), pos, kp + (size_t)t * D);
    }
    for (int i = 0; i < T; ++i) {
        double m = -INFINITY;
        for (int j = 0; j < T; ++j) {
            double s = 0.0;
            for (int d = 0; d < D; ++d) s += qp[(size_t)i * D + d] * kp[(size_t)j * D + d];
            s *= sc;
            if (Sraw) Sraw[(size_t)i * T + j] = s;
            if (p->softcap > 0.0) s = p->softcap * tanh(s / p->softcap);
            S[(size_t)i * T + j] = s;
            if (visible(p, i, j, st, en) && s > m) m = s;
        }
        double l = 0.0;
        for (int j = 0; j < T; ++j) {
            double e = visible(p, i, j, st, en) ? exp(S[(size_t)i * T + j] - m) : 0.0;
            P[(size_t)i * T + j] = e;
            l += e;
        }
        for (int j = 0; j < T; ++j) P[(size_t)i * T + j] /= l;
        if (lse) lse[i] = m + log(l);
    }
    free(qp);
    free(kp);
}

/* The T x T probability matrix of one (b, h) (for invariant tests). */
void oracle_attn_probs(const oracle_params* p, const double* q, const double* k,
                       const int32_t* seg_ids, int b, int h, double* P) {
    const int T = p->T;
    int32_t* st = (int32_t*)malloc(sizeof(int32_t) * (size_t)p->B * T);
    int32_t* en = (int32_t*)malloc(sizeof(int32_t) * (size_t)p->B * T);
    oracle_segments(p->B, T, seg_ids, st, en);
    double* S = (double*)malloc(sizeof(double) * (size_t)T * T);
    probs_one(p, q, k, b, h, st + (size_t)b * T, en + (size_t)b * T, S, NULL, P, NULL);
    free(S);
    free(st);
    free(en);
}

static int check(const oracle_params* p) {
    if (p->B < 0 || p->T < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0) return 1;
    if (p->Hq % p->Hkv) return 1;
    if (p->rope_base > 0.0 && (p->D % 2)) return 1;
    return 0;
}

/* Forward: O [B,T,Hq,D], LSE [B,Hq,T]. */
int oracle_attn_fwd(const oracle_params* p, const double* q, const double* k, const double* v,
                    const int32_t* seg_ids, double* o, double* lse) {
    if (check(p)) return 1;
    const int B = p->B, T = p->T, Hq = p->Hq, D = p->D, G = p->Hq / p->Hkv;
    int32_t* st = (int32_t*)malloc(sizeof(int32_t) * ((size_t)B * T + 1));
    int32_t* en = (int32_t*)malloc(sizeof(int32_t) * ((size_t)B * T + 1));
    oracle_segments(B, T, seg_ids, st, en);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int kvh = h / G;
            double* S = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            double* P = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            probs_one(p, q, k, b, h, st + (size_t)b * T, en + (size_t)b * T, S, NULL, P,
                      lse + ((size_t)b * Hq + h) * T);
            for (int i = 0; i < T; ++i)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j < T; ++j)
                        acc += P[(size_t)i * T + j] * v[idx4(b, j, kvh, d, T, p->Hkv, D)];
                    o[idx4(b, i, h, d, T, Hq, D)] = acc;
                }
            free(S);
            free(P);
        }
    free(st);
    free(en);
    return 0;
}

/* Backward: given dO, the gradients of L = sum(O * dO) with respect to the raw inputs
 * q, k, v (before norm and RoPE).  The forward is recomputed here in fp64. */
int oracle_attn_bwd(const oracle_params* p, const double* q, const double* k, const double* v,
                    const double* dout, const int32_t* seg_ids, double* dq, double* dk,
                    double* dv) {
    if (check(p)) return 1;
    const int B = p->B, T = p->T, Hq = p->Hq, Hkv = p->Hkv, D = p->D, G = Hq / Hkv;
    const double sc = eff_scale(p);
    int32_t* st = (int32_t*)malloc(sizeof(int32_t) * ((size_t)B * T + 1));
    int32_t* en = (int32_t*)malloc(sizeof(int32_t) * ((size_t)B * T + 1));
    oracle_segments(B, T, seg_ids, st, en);
    memset(dk, 0, sizeof(double) * (size_t)B * T * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)B * T * Hkv * D);
    /* one unit per (b, kv head): the query heads of a group add into the same dK, dV */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            const int32_t* sb = st + (size_t)b * T;
            const int32_t* eb = en + (size_t)b * T;
            double* S = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            double* Sraw = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            double* P = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            double* dS = (double*)malloc(sizeof(double) * ((size_t)T * T + 1));
            double* qp = (double*)malloc(sizeof(double) * ((size_t)T * D + 1));
            double* kp = (double*)malloc(sizeof(double) * ((size_t)T * D + 1));
            double* gq = (double*)malloc(sizeof(double) * ((size_t)T * D + 1));
            double* gk = (double*)calloc((size_t)T * D + 1, sizeof(double));
            for (int t = 0; t < T; ++t)
                norm_rope_vec(p, k + idx4(b, t, kvh, 0, T, Hkv, D), t - sb[t], kp + (size_t)t * D);
            for (int h = kvh * G; h < (kvh + 1) * G; ++h) {
                for (int t = 0; t < T; ++t)
                    norm_rope_vec(p, q + idx4(b, t, h, 0, T, Hq, D), t - sb[t], qp + (size_t)t * D);
                probs_one(p, q, k, b, h, sb, eb, S, Sraw, P, NULL);
                for (int i = 0; i < T; ++i) {
                    /* dP_ij = dO_i . v_j; softmax Jacobian: dS'_ij = P_ij (dP_ij - sum_k P_ik dP_ik) */
                    double* dP = dS + (size_t)i * T;
                    double rowdot = 0.0;
                    for (int j = 0; j < T; ++j) {
                        double acc = 0.0;
                        for (int d = 0; d < D; ++d)
                            acc += dout[idx4(b, i, h, d, T, Hq, D)] * v[idx4(b, j, kvh, d, T, Hkv, D)];
                        dP[j] = acc;
                        rowdot += P[(size_t)i * T + j] * acc;
                    }
                    for (int j = 0; j < T; ++j) {
                        double g = P[(size_t)i * T + j] * (dP[j] - rowdot);
                        if (p->softcap > 0.0) { /* d/ds of c tanh(s/c) = 1 - tanh^2(s/c) */
                            double th = tanh(Sraw[(size_t)i * T + j] / p->softcap);
                            g *= 1.0 - th * th;
                        }
                        dP[j] = g; /* now dS_ij, gradient w.r.t. the scaled score */
                    }
                }
                /* dV_j += sum_i P_ij dO_i */
                for (int j = 0; j < T; ++j)
                    for (int d = 0; d < D; ++d) {
                        double acc = 0.0;
                        for (int i = 0; i < T; ++i)
                            acc += P[(size_t)i * T + j] * dout[idx4(b, i, h, d, T, Hq, D)];
                        dv[idx4(b, j, kvh, d, T, Hkv, D)] += acc;
                    }
                /* dq'_i = scale sum_j dS_ij k'_j ; dk'_j += scale sum_i dS_ij q'_i */
                for (int i = 0; i < T; ++i)
                    for (int d = 0; d < D; ++d) {
                        double acc = 0.0;
                        for (int j = 0; j < T; ++j) acc += dS[(size_t)i * T + j] * kp[(size_t)j * D + d];
                        gq[(size_t)i * D + d] = sc * acc;
                    }
                for (int j = 0; j < T; ++j)
                    for (int d = 0; d < D; ++d) {
                        double acc = 0.0;
                        for (int i = 0; i < T; ++i) acc += dS[(size_t)i * T + j] * qp[(size_t)i * D + d];
                        gk[(size_t)j * D + d] += sc * acc;
                    }
                for (int t = 0; t < T; ++t)
                    norm_rope_vec_bwd(p, q + idx4(b, t, h, 0, T, Hq, D), t - sb[t], gq + (size_t)t * D,
                                      dq + idx4(b, t, h, 0, T, Hq, D));
            }
            for (int t = 0; t < T; ++t)
                norm_rope_vec_bwd(p, k + idx4(b, t, kvh, 0, T, Hkv, D), t - sb[t], gk + (size_t)t * D,
                                  dk + idx4(b, t, kvh, 0, T, Hkv, D));
            free(S); free(Sraw); free(P); free(dS); free(qp); free(kp); free(gq); free(gk);
        }
    free(st);
    free(en);
    return 0;
}

/* Attention of Tq new queries over a key/value cache of p->T entries (KV-cache decoding):
 * the GPT-pretraining post (dekermanjian.github.io, llm_gpt_pretrain), section "Bonus: KV
 * Caching".  The new queries are
 * the last Tq positions of the sequence: offset = T - Tq, and query i sits at absolute
 * position offset + i, so it may see key j only when j <= offset + i (causal); with a
 * window also offset + i - j < W.  The cache holds keys as they were stored after their own
 * norm and RoPE (k'), and the values; the raw queries get the norm and RoPE here, at their
 * absolute positions.  q, o [B,Tq,Hq,D]; kc, vc [B,T,Hkv,D]; lse [B,Hq,Tq]. */
int oracle_attn_fwd_cached(const oracle_params* p, int Tq, const double* q, const double* kc,
                           const double* vc, double* o, double* lse) {
    if (check(p) || Tq < 0 || Tq > p->T) return 1;
    const int B = p->B, T = p->T, Hq = p->Hq, Hkv = p->Hkv, D = p->D, G = p->Hq / p->Hkv;
    const int offset = T - Tq;
    const double sc = eff_scale(p);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const int kvh = h / G;
            double* qp = (double*)malloc(sizeof(double) * (size_t)D);
            double* s = (double*)malloc(sizeof(double) * ((size_t)T + 1));
            for (int i = 0; i < Tq; ++i) {
                const int pos = offset + i;
                norm_rope_vec(p, q + idx4(b, i, h, 0, Tq, Hq, D), pos, qp);
                double m = -INFINITY;
                for (int j = 0; j < T; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += qp[d] * kc[idx4(b, j, kvh, d, T, Hkv, D)];
                    acc *= sc;
                    if (p->softcap > 0.0) acc = p->softcap * tanh(acc / p->softcap);
                    int vis = 1;
                    if (p->causal && j > pos) vis = 0;
                    if (p->window > 0) {
                        const int dd = pos - j;
                        if (dd >= p->window || (!p->causal && -dd >= p->window)) vis = 0;
                    }
                    s[j] = vis ? acc : -INFINITY;
                    if (s[j] > m) m = s[j];
                }
                double l = 0.0;
                for (int j = 0; j < T; ++j) {
                    s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
                    l += s[j];
                }
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j < T; ++j) acc += s[j] * vc[idx4(b, j, kvh, d, T, Hkv, D)];
                    o[idx4(b, i, h, d, Tq, Hq, D)] = acc / l;
                }
                lse[((size_t)b * Hq + h) * Tq + i] = m + log(l);
            }
            free(qp);
            free(s);
        }
    return 0;
}

/* Thread control for the CPU-baseline timing (OpenMP over (b, h) units). */
#ifdef _OPENMP
#include <omp.h>
void oracle_set_threads(int n) { if (n > 0) omp_set_num_threads(n); }
int oracle_max_threads(void) { return omp_get_max_threads(); }
#else
void oracle_set_threads(int n) { (void)n; }
int oracle_max_threads(void) { return 1; }
#endif
