"""The projections around attention (csa_qkv_proj, csa_out_proj, csa_out_proj_bwd,
csa_qkv_proj_bwd) against the fp64 projection oracle, on the same seeded bf16 inputs.

Tolerances, from the arithmetic:
- bf16 products: the kernel accumulates in fp32 and rounds once to bf16 (round to nearest
  even, relative error <= 2^-9), so each element is checked to |gpu - ref| <= 2^-8 |ref| +
  1e-3 rms(ref) (twice the rounding bound plus an accumulation allowance) and the whole
  tensor to relative L2 <= 4e-3;
- fp32 weight gradients: fp32 accumulation over B*T terms with split-K partial sums added
  in any order: relative L2 <= 1e-3 and |gpu - ref| <= 1e-3 (|ref| + rms(ref));
- the whole layer (projection -> attention -> projection, intermediates rounded to bf16 like
  any training step): the attention bounds, y relative L2 <= 1e-2 with max-abs <= 2e-2, every
  gradient relative L2 <= 2e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.proj as proj
from causal_self_attention_gqa_b200.workloads import (LAYER_WORKLOADS, LayerWorkload, Workload,
                                                      make_layer_inputs, packed_segment_ids)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding
    oracle.build()
    return _binding


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_bf16(got, ref, what):
    got = _np(got) if torch.is_tensor(got) else got
    assert np.all(np.isfinite(got)), what
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-3 * rms
    worst = float(np.max(err - bound))
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert worst <= 0 and rel <= 4e-3, (what, rel, worst)


def _check_f32(got, ref, what):
    got = got.cpu().numpy().astype(np.float64) if torch.is_tensor(got) else got
    rms = float(np.sqrt(np.mean(ref * ref)))
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    worst = float(np.max(np.abs(got - ref) - 1e-3 * (np.abs(ref) + rms)))
    assert rel <= 1e-3 and worst <= 0, (what, rel, worst)


def _rand_bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


SHAPES = [
    # (B, T, C, Hq, Hkv, D): ragged row tails, all head dims, and between them every tile
    # width of every operand form (the width follows the piece sizes and the wave count)
    (2, 300, 256, 4, 2, 64),    # small: 64-wide bf16 tiles; dw 128-wide
    (1, 200, 768, 8, 4, 96),    # 768 / 384 / 384 pieces; dw 192-wide
    (1, 130, 768, 6, 3, 128),   # D = 128
    (2, 128, 192, 6, 6, 32),    # 192 / 192 / 192
    (1, 77, 320, 2, 1, 64),     # 128 / 64 / 64 pieces; fewer rows than one tile; dw 64-wide
    (3, 700, 512, 8, 8, 64),    # Q/K/V 256-wide, dw 256-wide
    (1, 18944, 512, 8, 4, 64),  # 148 row tiles: every product 256-wide
    (1, 18944, 640, 5, 5, 128),  # Q/K/V and dw 128-wide
    (1, 2048, 768, 8, 4, 96),    # y, dO, dx 128-wide
    (2, 4096, 640, 5, 5, 128),   # y, dO, dx 192-wide
    # CTA pairs with a ragged last 256-row tile, an N tail (C = 320) and a 256-column tile that
    # straddles all three Q/K/V pieces (320 / 64 / 64)
    (1, 19044, 320, 5, 1, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dT%dC%dH%dx%dD%d" % s)
def test_products_match_oracle(csa, shape):
    B, T, C, Hq, Hkv, D = shape
    w = LayerWorkload("t", Workload("t", B=B, T=T, Hq=Hq, Hkv=Hkv, D=D), C=C, seed=sum(shape))
    inp = make_layer_inputs(w)
    x, wq, wk, wv, wo, dy = (inp[n].to(DEV) for n in ("x", "wq", "wk", "wv", "wo", "dy"))
    o = _rand_bf16((B, T, Hq, D), 7).to(DEV)
    gq, gk, gv = (_rand_bf16((B, T, H, D), 8 + i).to(DEV) for i, H in enumerate((Hq, Hkv, Hkv)))
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    q, k, v = csa.qkv_proj(x, wq, wk, wv, workspace=ws)
    y = csa.out_proj(o, wo, workspace=ws)
    dout, dwo = csa.out_proj_bwd(o, wo, dy, workspace=ws)
    # weight gradients ADD to what the buffers hold
    base = [torch.randn((C, H, D), generator=torch.Generator().manual_seed(20 + i)) for i, H in
            enumerate((Hq, Hkv, Hkv))]
    dws = [b.to(DEV) for b in base]
    dx, dwq, dwk, dwv = csa.qkv_proj_bwd(x, wq, wk, wv, gq, gk, gv, dwq=dws[0], dwk=dws[1], dwv=dws[2], workspace=ws)
    assert csa.device_status(ws) == 0
    rq, rk, rv = proj.qkv_proj(inp["x"].double().numpy(), inp["wq"].double().numpy(), inp["wk"].double().numpy(),
                               inp["wv"].double().numpy())
    for got, ref, n in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        _check_bf16(got, ref, n)
    _check_bf16(y, proj.out_proj(_np(o), _np(wo)), "y")
    rdout, rdwo = proj.out_proj_bwd(_np(o), _np(wo), _np(dy))
    _check_bf16(dout, rdout, "dout")
    _check_f32(dwo, rdwo, "dwo")
    rdx, rdwq, rdwk, rdwv = proj.qkv_proj_bwd(_np(x), _np(wq), _np(wk), _np(wv), _np(gq), _np(gk), _np(gv))
    _check_bf16(dx, rdx, "dx")
    for got, ref, b, n in ((dwq, rdwq, base[0], "dwq"), (dwk, rdwk, base[1], "dwk"), (dwv, rdwv, base[2], "dwv")):
        _check_f32(got.cpu().double() - b.double(), ref, n)


def test_weight_grad_skip_and_accumulate(csa):
    B, T, C, Hq, Hkv, D = 2, 256, 256, 4, 2, 64
    x = _rand_bf16((B, T, C), 1).to(DEV)
    wq, wk, wv = (_rand_bf16((C, H, D), 2 + i, C ** -0.5).to(DEV) for i, H in enumerate((Hq, Hkv, Hkv)))
    gq, gk, gv = (_rand_bf16((B, T, H, D), 5 + i).to(DEV) for i, H in enumerate((Hq, Hkv, Hkv)))
    dx0, n1, n2, n3 = csa.qkv_proj_bwd(x, wq, wk, wv, gq, gk, gv, weight_grad=False)
    assert n1 is None and n2 is None and n3 is None
    dx1, dwq, dwk, dwv = csa.qkv_proj_bwd(x, wq, wk, wv, gq, gk, gv)
    assert torch.equal(dx0, dx1)
    once = [t.clone() for t in (dwq, dwk, dwv)]
    csa.qkv_proj_bwd(x, wq, wk, wv, gq, gk, gv, dwq=dwq, dwk=dwk, dwv=dwv)
    for a, b in zip(once, (dwq, dwk, dwv)):
        assert torch.allclose(b, 2 * a, rtol=1e-5, atol=1e-5)
    o = _rand_bf16((B, T, Hq, D), 9).to(DEV)
    wo = _rand_bf16((Hq, D, C), 10, (Hq * D) ** -0.5).to(DEV)
    dy = _rand_bf16((B, T, C), 11).to(DEV)
    d0, none = csa.out_proj_bwd(o, wo, dy, weight_grad=False)
    d1, dwo = csa.out_proj_bwd(o, wo, dy)
    assert none is None and torch.equal(d0, d1)


def test_host_checks(csa):
    """Shapes the projections do not take come back as CSA_ERR_INVALID_ARG before any launch."""
    x = torch.zeros((1, 8, 96), dtype=torch.bfloat16, device=DEV)  # C = 96 is not a multiple of 64
    w = torch.zeros((96, 2, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(csa.CsaError) as e:
        csa.qkv_proj(x, w, w, w)
    assert e.value.code == csa.CSA_ERR_INVALID_ARG
    x = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((128, 1, 32), dtype=torch.bfloat16, device=DEV)  # Hkv * D = 32
    with pytest.raises(csa.CsaError) as e:
        csa.qkv_proj(x, w, w, w)
    assert e.value.code == csa.CSA_ERR_INVALID_ARG


def _layer_gpu(csa, inp, a, seg=None):
    """The training step of the layer through the C ABI: the sequence bench.py times."""
    x, wq, wk, wv, wo, dy = (inp[n].to(DEV) for n in ("x", "wq", "wk", "wv", "wo", "dy"))
    opts = a.options()
    q, k, v = csa.qkv_proj(x, wq, wk, wv)
    ws = csa.workspace_for(q, k, True, **opts)
    o, lse = csa.attn_fwd(q, k, v, segment_ids=seg, workspace=ws, **opts)
    y = csa.out_proj(o, wo, workspace=ws)
    dout, dwo = csa.out_proj_bwd(o, wo, dy, workspace=ws)
    dq, dk, dv = csa.attn_bwd(q, k, v, o, dout, lse, segment_ids=seg, workspace=ws, after_fwd=True, **opts)
    dx, dwq, dwk, dwv = csa.qkv_proj_bwd(x, wq, wk, wv, dq, dk, dv, workspace=ws)
    assert csa.device_status(ws) == 0
    return y, (dx, dwq, dwk, dwv, dwo)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


LAYER_SMALL = [
    (2, 300, 256, 4, 2, 64, dict(rope_base=10000.0, qk_norm=True, softcap=30.0)),
    (1, 257, 768, 8, 4, 96, dict(rope_base=10000.0, qk_norm=True)),
    (2, 200, 192, 6, 6, 32, dict(window=50)),
]


@pytest.mark.parametrize("case", LAYER_SMALL, ids=lambda c: "B%dT%dC%dH%dx%dD%d" % c[:6])
def test_layer_matches_oracle(csa, case):
    B, T, C, Hq, Hkv, D, opts = case
    a = Workload("t", B=B, T=T, Hq=Hq, Hkv=Hkv, D=D, **opts)
    inp = make_layer_inputs(LayerWorkload("t", a, C=C, seed=B * T + C))
    _check_layer(csa, a, inp, None)


def test_layer_packed_segments(csa):
    """The layer over packed rows: segment_ids restrict attention to each document and restart
    the RoPE positions, inside the same projection -> attention -> projection step."""
    a = Workload("t", B=2, T=400, Hq=4, Hkv=2, D=64, rope_base=10000.0, qk_norm=True, window=96)
    inp = make_layer_inputs(LayerWorkload("t", a, C=256, seed=77))
    seg = torch.from_numpy(packed_segment_ids(a.B, a.T, 20, 160, 77))
    _check_layer(csa, a, inp, seg)


def _check_layer(csa, a, inp, seg):
    y, grads = _layer_gpu(csa, inp, a, None if seg is None else seg.to(DEV))
    ref_in = [inp[n].double().numpy() for n in ("x", "wq", "wk", "wv", "wo")]
    ref_y, _ = proj.attn_layer_fwd(*ref_in, segment_ids=seg, **a.options())
    ref_g = proj.attn_layer_bwd(*ref_in, inp["dy"].double().numpy(), segment_ids=seg, **a.options())
    yn = _np(y)
    assert _rel(yn, ref_y) <= 1e-2 and float(np.max(np.abs(yn - ref_y))) <= 2e-2
    for got, ref, n in zip(grads, ref_g, ("dx", "dwq", "dwk", "dwv", "dwo")):
        got = got.cpu().double().numpy() if got.dtype == torch.float32 else _np(got)
        assert _rel(got, ref) <= 2e-2, (n, _rel(got, ref))


@pytest.mark.parametrize("lw", LAYER_WORKLOADS, ids=lambda w: w.name)
def test_layer_full_size(csa, lw):
    """Full-size layer step: y and dx on the first and last batch rows against the oracle layer
    run on those rows alone (rows are independent), and every projection product of the step
    against its exact fp64 value -- bf16 products on sampled token rows, the fp32 weight
    gradients in full."""
    a = lw.attn
    inp = make_layer_inputs(lw)
    y, (dx, dwq, dwk, dwv, dwo) = _layer_gpu(csa, inp, a)
    oracle.set_threads(oracle.max_threads())
    for b in (0, a.B - 1):
        ref_in = [inp["x"][b:b + 1].double().numpy()] + [inp[n].double().numpy() for n in ("wq", "wk", "wv", "wo")]
        ref_y, _ = proj.attn_layer_fwd(*ref_in, **a.options())
        ref_dx = proj.attn_layer_bwd(*ref_in, inp["dy"][b:b + 1].double().numpy(), **a.options())[0]
        yn, dxn = _np(y[b:b + 1]), _np(dx[b:b + 1])
        assert _rel(yn, ref_y) <= 1e-2 and float(np.max(np.abs(yn - ref_y))) <= 2e-2, b
        assert _rel(dxn, ref_dx) <= 2e-2, b


def test_gemm_full_size_exact(csa):
    """At the 181M layer's full size, each projection product of the GPU against the fp64
    product of the same bf16 operands: q/k/v/y/dout/dx on 96 sampled token rows, the three
    fp32 weight gradients of the Q/K/V projection and dwo in full."""
    lw = LAYER_WORKLOADS[0]
    a = lw.attn
    inp = make_layer_inputs(lw)
    x, wq, wk, wv, wo, dy = (inp[n].to(DEV) for n in ("x", "wq", "wk", "wv", "wo", "dy"))
    q, k, v = csa.qkv_proj(x, wq, wk, wv)
    y = csa.out_proj(q, wo)  # any [B,T,Hq,D] bf16 serves as the attention output here
    dout, dwo = csa.out_proj_bwd(q, wo, dy)
    dx, dwq, dwk, dwv = csa.qkv_proj_bwd(x, wq, wk, wv, q, k, v)
    torch.cuda.synchronize()
    M = a.B * a.T
    rows = np.sort(np.random.default_rng(3).choice(M, 94, replace=False))
    rows = np.concatenate([[0], rows, [M - 1]])
    X = inp["x"].double().numpy().reshape(M, lw.C)
    W = [inp[n].double().numpy().reshape(lw.C, -1) for n in ("wq", "wk", "wv")]
    WO = inp["wo"].double().numpy().reshape(-1, lw.C)
    DY = inp["dy"].double().numpy().reshape(M, lw.C)
    Q, K, V = (_np(t).reshape(M, -1) for t in (q, k, v))
    for t, Wi, n in ((Q, W[0], "q"), (K, W[1], "k"), (V, W[2], "v")):
        _check_bf16(t[rows], X[rows] @ Wi, n)
    _check_bf16(_np(y).reshape(M, -1)[rows], Q[rows] @ WO, "y")
    _check_bf16(_np(dout).reshape(M, -1)[rows], DY[rows] @ WO.T, "dout")
    _check_bf16(_np(dx).reshape(M, -1)[rows], Q[rows] @ W[0].T + K[rows] @ W[1].T + V[rows] @ W[2].T, "dx")
    _check_f32(dwo.cpu().double().numpy().reshape(-1, lw.C), Q.T @ DY, "dwo")
    for got, G, n in ((dwq, Q, "dwq"), (dwk, K, "dwk"), (dwv, V, "dwv")):
        _check_f32(got.cpu().double().numpy().reshape(lw.C, -1), X.T @ G, n)
