"""fp64 oracle of the projections around attention, and of the whole attention layer.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` are its only callers.  It shares no code with the
CUDA path.

Definitions followed:
- the nanogpt-jax-181m model card, section "Architecture": the attention weights are 3-D,
  wq, wk, wv of shape (d_emb, heads, head_dim) and wo of shape (heads, head_dim, d_emb);
  a projection contracts the model axis of x (B, T, d_emb) with the weight's first axis,
  and the output projection contracts the (heads, head_dim) axes of o with wo's first two;
- the GPT-pretraining page (dekermanjian.github.io, llm_gpt_pretrain), section "Multihead
  Attention": the block input is projected to q, k and v, attention runs per head, and the
  heads' outputs, side by side, go through the output projection.  The model card's weights
  carry no bias, so there is none here.

Each product is one numpy einsum in fp64 (a library contraction used as one step, with the
index string spelling the definition); the backward is the calculus of those linear maps.
The attention itself is the C oracle (``oracle.attn_fwd`` / ``oracle.attn_bwd``).
"""
from __future__ import annotations

import numpy as np

from . import attn_bwd, attn_fwd


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def qkv_proj(x, wq, wk, wv):
    """q[b,t,h,d] = sum_c x[b,t,c] wq[c,h,d]; likewise k and v with wk, wv."""
    x = _f64(x)
    return tuple(np.einsum("btc,chd->bthd", x, _f64(w), optimize=True) for w in (wq, wk, wv))


def out_proj(o, wo):
    """y[b,t,c] = sum_{h,d} o[b,t,h,d] wo[h,d,c]."""
    return np.einsum("bthd,hdc->btc", _f64(o), _f64(wo), optimize=True)


def out_proj_bwd(o, wo, dy):
    """Adjoints of y = o wo: dout[b,t,h,d] = sum_c dy[b,t,c] wo[h,d,c] and
    dwo[h,d,c] = sum_{b,t} o[b,t,h,d] dy[b,t,c]."""
    o, wo, dy = _f64(o), _f64(wo), _f64(dy)
    dout = np.einsum("btc,hdc->bthd", dy, wo, optimize=True)
    dwo = np.einsum("bthd,btc->hdc", o, dy, optimize=True)
    return dout, dwo


def qkv_proj_bwd(x, wq, wk, wv, dq, dk, dv):
    """Adjoints of q = x wq, k = x wk, v = x wv: dx[b,t,c] = sum over the three of
    sum_{h,d} g[b,t,h,d] w[c,h,d], and dw[c,h,d] = sum_{b,t} x[b,t,c] g[b,t,h,d]."""
    x = _f64(x)
    dx = np.zeros(x.shape, dtype=np.float64)
    dws = []
    for w, g in ((wq, dq), (wk, dk), (wv, dv)):
        w, g = _f64(w), _f64(g)
        dx += np.einsum("bthd,chd->btc", g, w, optimize=True)
        dws.append(np.einsum("btc,bthd->chd", x, g, optimize=True))
    return (dx, *dws)


def attn_layer_fwd(x, wq, wk, wv, wo, segment_ids=None, **opts):
    """y = out_proj(attention(qkv_proj(x))): returns y and the intermediates
    (q, k, v, o, lse) of the attention in the middle."""
    q, k, v = qkv_proj(x, wq, wk, wv)
    o, lse = attn_fwd(q, k, v, segment_ids=segment_ids, **opts)
    return out_proj(o, wo), (q, k, v, o, lse)


def attn_layer_bwd(x, wq, wk, wv, wo, dy, segment_ids=None, **opts):
    """Gradients of <y, dy> with respect to x, wq, wk, wv and wo, through the chain
    out_proj -> attention -> qkv_proj."""
    q, k, v = qkv_proj(x, wq, wk, wv)
    o, _ = attn_fwd(q, k, v, segment_ids=segment_ids, **opts)
    dout, dwo = out_proj_bwd(o, wo, dy)
    dq, dk, dv = attn_bwd(q, k, v, dout, segment_ids=segment_ids, **opts)
    dx, dwq, dwk, dwv = qkv_proj_bwd(x, wq, wk, wv, dq, dk, dv)
    return dx, dwq, dwk, dwv, dwo
