"""Pins of the projection oracle (``oracle/proj.py``) against things other than itself (CPU).

* Closed forms: identity weights return the input with its axes regrouped into heads (and
  back); a permutation matrix moves each model channel to its image, which fixes the
  weight's orientation (a transposed weight would apply the inverse permutation).
* The adjoint identities of linear maps: <x wq, g> = <x, g wq^T> = <wq, x^T g>, for every
  piece, and the same for the output projection.  They pin each backward to its forward.
* A library composition: torch fp64 matmuls of the reshaped weights, scaled_dot_product_attention
  with is_causal and repeated K/V heads, and torch autograd for every gradient.
* Finite differences of L = <y, dy> through the whole layer with every attention option on.
* Planted mistakes (mutants of the oracle's source) that the pins above must reject.
"""
import math
import re

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import oracle.proj as proj

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")

B, T, C, HQ, HKV, D = 2, 12, 48, 4, 2, 8  # Hq * D = 32 != C on purpose


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _inputs(seed=0):
    x = _rand((B, T, C), seed)
    wq = _rand((C, HQ, D), seed + 1, 1 / math.sqrt(C))
    wk = _rand((C, HKV, D), seed + 2, 1 / math.sqrt(C))
    wv = _rand((C, HKV, D), seed + 3, 1 / math.sqrt(C))
    wo = _rand((HQ, D, C), seed + 4, 1 / math.sqrt(HQ * D))
    dy = _rand((B, T, C), seed + 5)
    return x, wq, wk, wv, wo, dy


# ---------------------------------------------------------------- the pins, as functions of a module
def pin_identity(m):
    Cm = HQ * D
    x = _rand((B, T, Cm), 11)
    eye = np.eye(Cm)
    q, _, _ = m.qkv_proj(x, eye.reshape(Cm, HQ, D), eye.reshape(Cm, HQ, D)[:, :HKV], eye.reshape(Cm, HQ, D)[:, :HKV])
    y = m.out_proj(q, eye.reshape(HQ, D, Cm))
    return np.array_equal(q, x.reshape(B, T, HQ, D)) and np.array_equal(y, x)


def pin_permutation(m):
    Cm = HQ * D
    rng = np.random.default_rng(12)
    perm = rng.permutation(Cm)
    W = np.zeros((Cm, Cm))
    W[np.arange(Cm), perm] = 1.0  # channel c goes to output column perm[c]
    x = _rand((B, T, Cm), 13)
    q, _, _ = m.qkv_proj(x, W.reshape(Cm, HQ, D), W.reshape(Cm, HQ, D)[:, :HKV], W.reshape(Cm, HQ, D)[:, :HKV])
    want = np.empty_like(x)
    want[..., perm] = x
    y = m.out_proj(want.reshape(B, T, HQ, D), W.T.reshape(HQ, D, Cm))  # the inverse map returns x
    return np.array_equal(q.reshape(B, T, Cm), want) and np.allclose(y, x, rtol=0, atol=0)


def pin_adjoint(m):
    x, wq, wk, wv, wo, dy = _inputs(20)
    gq, gk, gv = _rand((B, T, HQ, D), 21), _rand((B, T, HKV, D), 22), _rand((B, T, HKV, D), 23)
    q, k, v = m.qkv_proj(x, wq, wk, wv)
    dx, dwq, dwk, dwv = m.qkv_proj_bwd(x, wq, wk, wv, gq, gk, gv)
    lhs = np.sum(q * gq) + np.sum(k * gk) + np.sum(v * gv)
    ok = math.isclose(lhs, np.sum(x * dx), rel_tol=1e-12)
    ok &= math.isclose(lhs, np.sum(wq * dwq) + np.sum(wk * dwk) + np.sum(wv * dwv), rel_tol=1e-12)
    for w, g, dw in ((wq, gq, dwq), (wk, gk, dwk), (wv, gv, dwv)):  # piece by piece
        zero = [np.zeros_like(gq), np.zeros_like(gk), np.zeros_like(gv)]
        idx = [gq is g, gk is g, gv is g].index(True)
        zero[idx] = g
        dxp = m.qkv_proj_bwd(x, wq, wk, wv, *zero)[0]
        piece = m.qkv_proj(x, wq, wk, wv)[idx]
        ok &= math.isclose(np.sum(piece * g), np.sum(x * dxp), rel_tol=1e-12)
        ok &= math.isclose(np.sum(piece * g), np.sum(w * dw), rel_tol=1e-12)
    o = _rand((B, T, HQ, D), 24)
    y = m.out_proj(o, wo)
    dout, dwo = m.out_proj_bwd(o, wo, dy)
    ok &= math.isclose(np.sum(y * dy), np.sum(o * dout), rel_tol=1e-12)
    ok &= math.isclose(np.sum(y * dy), np.sum(wo * dwo), rel_tol=1e-12)
    return bool(ok)


def _torch_layer(x, wq, wk, wv, wo):
    """Library composition: plain matmuls of the reshaped weights, SDPA (causal, GQA by
    repeating K/V heads), and the output matmul."""
    Bx, Tx, Cx = x.shape
    q = (x.reshape(Bx * Tx, Cx) @ wq.reshape(Cx, -1)).reshape(Bx, Tx, HQ, D)
    k = (x.reshape(Bx * Tx, Cx) @ wk.reshape(Cx, -1)).reshape(Bx, Tx, HKV, D)
    v = (x.reshape(Bx * Tx, Cx) @ wv.reshape(Cx, -1)).reshape(Bx, Tx, HKV, D)
    G = HQ // HKV
    o = F.scaled_dot_product_attention(q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2),
                                       v.repeat_interleave(G, 2).transpose(1, 2), is_causal=True)
    o = o.transpose(1, 2).reshape(Bx * Tx, HQ * D)
    return (o @ wo.reshape(HQ * D, Cx)).reshape(Bx, Tx, Cx)


def pin_torch(m):
    arrs = _inputs(30)
    x, wq, wk, wv, wo, dy = arrs
    y, _ = m.attn_layer_fwd(x, wq, wk, wv, wo)
    grads = m.attn_layer_bwd(x, wq, wk, wv, wo, dy)
    tx = [torch.tensor(a, requires_grad=True) for a in (x, wq, wk, wv, wo)]
    ty = _torch_layer(*tx)
    (ty * torch.tensor(dy)).sum().backward()
    ok = np.allclose(y, ty.detach().numpy(), rtol=1e-10, atol=1e-12)
    for g, t in zip(grads, tx):
        ok &= np.allclose(g, t.grad.numpy(), rtol=1e-9, atol=1e-11)
    return bool(ok)


def pin_finite_differences(m):
    opts = dict(rope_base=10000.0, qk_norm=True, softcap=5.0, window=7)
    x, wq, wk, wv, wo, dy = _inputs(40)
    args = [x, wq, wk, wv, wo]
    grads = m.attn_layer_bwd(*args, dy, **opts)
    rng = np.random.default_rng(41)
    eps = 1e-5
    ok = True
    for i, a in enumerate(args):
        for _ in range(4):
            idx = tuple(rng.integers(0, s) for s in a.shape)
            plus = [b.copy() for b in args]
            minus = [b.copy() for b in args]
            plus[i][idx] += eps
            minus[i][idx] -= eps
            lp = np.sum(m.attn_layer_fwd(*plus, **opts)[0] * dy)
            lm = np.sum(m.attn_layer_fwd(*minus, **opts)[0] * dy)
            fd = (lp - lm) / (2 * eps)
            ok &= abs(fd - grads[i][idx]) <= 1e-6 * max(1.0, abs(fd))
    return bool(ok)


PINS = [pin_identity, pin_permutation, pin_adjoint, pin_torch, pin_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_proj_pin(pin):
    assert pin(proj)


def test_layer_intermediates_match_attention_oracle():
    x, wq, wk, wv, wo, _ = _inputs(50)
    y, (q, k, v, o, lse) = proj.attn_layer_fwd(x, wq, wk, wv, wo, qk_norm=True, rope_base=100.0)
    o2, lse2 = oracle.attn_fwd(q, k, v, qk_norm=True, rope_base=100.0)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    assert np.array_equal(y, proj.out_proj(o, wo))


# ---------------------------------------------------------------- planted mistakes
_SRC = open(proj.__file__).read()

MUTANTS = {
    # the k and v gradients paired with the wrong weights
    "swapped_kv_pairs": ("for w, g in ((wq, dq), (wk, dk), (wv, dv)):", "for w, g in ((wq, dq), (wk, dv), (wv, dk)):"),
    # dx keeps only the last piece
    "dx_overwritten": ("dx += np.einsum", "dx = np.einsum"),
    # the value projection reuses the key weight
    "v_from_wk": ("for w in (wq, wk, wv))", "for w in (wq, wk, wk))"),
    # weight gradient of wo taken against the wrong operand order (transposed result reshaped)
    "dwo_transposed": ('dwo = np.einsum("bthd,btc->hdc", o, dy, optimize=True)',
                       'dwo = np.einsum("bthd,btc->chd", o, dy, optimize=True).reshape(wo.shape)'),
    # the output projection contracts head_dim against the wrong weight axis order
    "wo_axes_swapped": ('np.einsum("bthd,hdc->btc", _f64(o), _f64(wo), optimize=True)',
                        'np.einsum("bthd,hdc->btc", _f64(o), _f64(wo).reshape(wo.shape[1], wo.shape[0], -1)'
                        '.transpose(1, 0, 2), optimize=True)'),
    # the layer backward forgets to go through the output projection's adjoint
    "skips_out_adjoint": ("dq, dk, dv = attn_bwd(q, k, v, dout,", "dq, dk, dv = attn_bwd(q, k, v, dout * 0.5,"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    assert _SRC.count(old) == 1, name
    src = _SRC.replace(old, new).replace("from . import attn_bwd, attn_fwd", "")
    ns = {"__name__": "proj_mutant_" + name, "attn_fwd": oracle.attn_fwd, "attn_bwd": oracle.attn_bwd}
    exec(compile(src, "proj_mutant_" + name, "exec"), ns)

    class M:
        pass

    for f in ("qkv_proj", "out_proj", "out_proj_bwd", "qkv_proj_bwd", "attn_layer_fwd", "attn_layer_bwd"):
        setattr(M, f, staticmethod(ns[f]))
    return M


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name):
    m = _mutant(name)
    failed = []
    for pin in PINS:
        try:
            ok = pin(m)
        except Exception:  # a mutant that breaks a shape is rejected as well
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


def test_mutant_sources_differ():
    for name, (old, new) in MUTANTS.items():
        assert old != new and re.sub(r"\s", "", old) != re.sub(r"\s", "", new), name
