"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded bf16 inputs.

Tolerances (stated for the bf16 path): O relative L2 <= 1e-2 and max-abs <= 2e-2;
dQ, dK, dV relative L2 <= 2e-2 each; LSE max-abs <= 1e-2 (internal).
Small shapes cover every option, ragged tails (T not a multiple of the 128-row tile),
T = 1, odd group sizes and windows that bind.  The named workloads run at full size
in the call sequence and launch configuration the benchmark times (forward, then the
backward that reuses the forward's workspace): O and LSE on every batch row, gradients per
head on the first, middle and last rows (batch rows are independent, so a row's outputs and
gradients are exact oracle targets).
"""
import numpy as np
import pytest
import torch

from causal_self_attention_gqa_b200.workloads import WORKLOADS, Workload, make_inputs, packed_segment_ids

pytestmark = pytest.mark.gpu

O_REL, O_ABS, G_REL, LSE_ABS = 1e-2, 2e-2, 2e-2, 1e-2


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding
    return _binding


@pytest.fixture(scope="module")
def ora():
    import oracle
    oracle.build()
    return oracle


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run_gpu(csa, inp, opts, backward=True, after_fwd=False):
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    seg = inp["segment_ids"].to(dev) if inp["segment_ids"] is not None else None
    ws = csa.workspace_for(q, k, True, **opts)
    o, lse = csa.attn_fwd(q, k, v, segment_ids=seg, workspace=ws, **opts)
    out = dict(o=o, lse=lse)
    if backward:
        do = inp["do"].to(dev)
        dq, dk, dv = csa.attn_bwd(q, k, v, o, do, lse, segment_ids=seg, workspace=ws, after_fwd=after_fwd, **opts)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert csa.device_status(ws) == 0
    return {n: t.float().cpu().numpy() for n, t in out.items()}


def check(gpu, ref_o, ref_lse, ref_g=None, rows=None):
    sl = slice(None) if rows is None else rows
    o = gpu["o"][sl]
    assert np.all(np.isfinite(o))
    r = rel_l2(o, ref_o)
    m = float(np.max(np.abs(o - ref_o)))
    assert r <= O_REL and m <= O_ABS, (r, m)
    lse_err = float(np.max(np.abs(gpu["lse"][sl] - ref_lse)))
    assert lse_err <= LSE_ABS, lse_err
    if ref_g is not None:
        for name, ref in zip(("dq", "dk", "dv"), ref_g):
            g = gpu[name][sl]
            assert np.all(np.isfinite(g)), name
            e = rel_l2(g, ref)
            assert e <= G_REL, (name, e)


def _small(B, T, Hq, Hkv, D, seed, seg=None, **opts):
    w = Workload("t", B=B, T=T, Hq=Hq, Hkv=Hkv, D=D, seed=seed, **opts)
    inp = make_inputs(w)
    if seg is not None:
        inp["segment_ids"] = torch.from_numpy(packed_segment_ids(B, T, seg[0], seg[1], seed))
    return w, inp


SMALL = [
    # (B, T, Hq, Hkv, D, options, segments)
    (1, 1, 2, 1, 32, dict(), None),
    (2, 17, 2, 2, 32, dict(), None),
    (2, 128, 4, 2, 64, dict(), None),
    (1, 129, 2, 1, 128, dict(), None),
    (2, 300, 4, 2, 96, dict(), None),
    (1, 300, 3, 1, 128, dict(), None),                      # odd group size (G = 3)
    (2, 260, 2, 2, 32, dict(), None),                       # G = 1, odd number of query tiles
    (1, 256, 4, 2, 128, dict(rope_base=10000.0), None),
    (1, 256, 4, 2, 96, dict(qk_norm=True), None),
    (2, 200, 4, 2, 64, dict(rope_base=10000.0, qk_norm=True), None),
    (1, 300, 2, 1, 128, dict(rope_base=10000.0, qk_norm=True, softcap=50.0), None),
    (1, 300, 2, 1, 64, dict(softcap=5.0), None),            # cap that binds (no norm)
    # QK-norm with a cap too tight for the series tanh (D scale / cap > 1/4): hardware tanh
    (1, 300, 4, 2, 128, dict(rope_base=10000.0, qk_norm=True, softcap=20.0), None),
    (2, 200, 2, 1, 64, dict(qk_norm=True, softcap=50.0), None),  # series tanh at D = 64
    (1, 520, 2, 1, 96, dict(window=100), None),             # window that binds, ragged
    (2, 384, 4, 2, 128, dict(rope_base=10000.0, qk_norm=True, window=200), (20, 150)),
    (1, 300, 2, 2, 32, dict(), (1, 40)),                    # segments, single-token documents
    (1, 257, 4, 2, 64, dict(causal=False), None),
    (1, 300, 2, 1, 128, dict(causal=False, window=64), None),
    (2, 200, 2, 1, 96, dict(causal=False, rope_base=10000.0), (30, 90)),
    (1, 200, 2, 2, 64, dict(scale=0.05), None),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}x{c[3]}D{c[4]}"
                         + "".join(f"-{k}{v}" for k, v in c[5].items()) + ("-seg" if c[6] else ""))
def test_small_shapes_match_oracle(csa, ora, case):
    B, T, Hq, Hkv, D, opts, seg = case
    w, inp = _small(B, T, Hq, Hkv, D, seed=7 + T + D, seg=seg, **opts)
    kw = dict(w.options())
    gpu = run_gpu(csa, inp, kw)
    ref_o, ref_lse = ora.attn_fwd(inp["q"], inp["k"], inp["v"], segment_ids=inp["segment_ids"], **kw)
    ref_g = ora.attn_bwd(inp["q"], inp["k"], inp["v"], inp["do"], segment_ids=inp["segment_ids"], **kw)
    check(gpu, ref_o, ref_lse, ref_g)


@pytest.mark.parametrize("case", [SMALL[i] for i in (2, 8, 10, 12, 15, 19)],
                         ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}x{c[3]}D{c[4]}"
                         + "".join(f"-{k}{v}" for k, v in c[5].items()) + ("-seg" if c[6] else ""))
def test_backward_after_forward_reuses_the_workspace(csa, ora, case):
    """csa_attn_bwd_after_fwd (q', k' and segment bounds from the forward's workspace, no
    prologue) against the oracle: with and without norm / RoPE / segments."""
    B, T, Hq, Hkv, D, opts, seg = case
    w, inp = _small(B, T, Hq, Hkv, D, seed=11 + T + D, seg=seg, **opts)
    kw = dict(w.options())
    gpu = run_gpu(csa, inp, kw, after_fwd=True)
    ref_o, ref_lse = ora.attn_fwd(inp["q"], inp["k"], inp["v"], segment_ids=inp["segment_ids"], **kw)
    ref_g = ora.attn_bwd(inp["q"], inp["k"], inp["v"], inp["do"], segment_ids=inp["segment_ids"], **kw)
    check(gpu, ref_o, ref_lse, ref_g)


def grad_rows(w):
    """Batch rows whose gradients the full-size tests compare: first, middle and last."""
    return sorted({0, w.B // 2, w.B - 1})


def check_per_head(name, got, ref, tol):
    """Relative L2 per (batch row, head) of [rows, T, H, D] gradients: a single wrong head
    cannot hide inside a norm taken over the whole tensor."""
    assert np.all(np.isfinite(got)), name
    for r in range(got.shape[0]):
        for h in range(got.shape[2]):
            e = rel_l2(got[r, :, h], ref[r, :, h])
            assert e <= tol, (name, r, h, e)


@pytest.mark.parametrize("widx", range(len(WORKLOADS)), ids=[w.name for w in WORKLOADS])
def test_benchmarked_step_full_size(csa, ora, widx):
    """The exact sequence the benchmark times, at full size: csa_attn_fwd, then
    csa_attn_bwd_after_fwd on the same workspace (q', k', segment bounds and whatever else
    the forward left there).  O and LSE are compared with the oracle on EVERY batch row;
    dQ, dK, dV on the first, middle and last rows, per head."""
    w = WORKLOADS[widx]
    inp = make_inputs(w)
    kw = dict(w.options())
    gpu = run_gpu(csa, inp, kw, after_fwd=True)
    ref_o, ref_lse = ora.attn_fwd(inp["q"], inp["k"], inp["v"], segment_ids=inp["segment_ids"], **kw)
    for b in range(w.B):
        check(gpu, ref_o[b:b + 1], ref_lse[b:b + 1], rows=slice(b, b + 1))
    rows = grad_rows(w)
    seg = inp["segment_ids"][rows] if inp["segment_ids"] is not None else None
    ref_g = ora.attn_bwd(inp["q"][rows], inp["k"][rows], inp["v"][rows], inp["do"][rows], segment_ids=seg, **kw)
    for name, ref in zip(("dq", "dk", "dv"), ref_g):
        check_per_head(name, gpu[name][rows], ref, G_REL)


@pytest.mark.parametrize("widx", range(len(WORKLOADS)), ids=[w.name for w in WORKLOADS])
def test_stateless_backward_full_size(csa, ora, widx):
    """csa_attn_bwd (the stateless backward, which reruns the prologue itself) at full size,
    against the oracle on the last batch row, per head."""
    w = WORKLOADS[widx]
    inp = make_inputs(w)
    kw = dict(w.options())
    gpu = run_gpu(csa, inp, kw)
    b = w.B - 1
    sl = slice(b, b + 1)
    seg = inp["segment_ids"][sl] if inp["segment_ids"] is not None else None
    args = (inp["q"][sl], inp["k"][sl], inp["v"][sl])
    ref_o, ref_lse = ora.attn_fwd(*args, segment_ids=seg, **kw)
    check(gpu, ref_o, ref_lse, rows=sl)
    ref_g = ora.attn_bwd(*args, inp["do"][sl], segment_ids=seg, **kw)
    for name, ref in zip(("dq", "dk", "dv"), ref_g):
        check_per_head(name, gpu[name][sl], ref, G_REL)


def test_causal_outputs_ignore_future_tokens(csa):
    """Masking is exact: changing tokens after position c leaves rows <= c bit-identical."""
    w = Workload("t", B=1, T=384, Hq=4, Hkv=2, D=128, rope_base=10000.0, qk_norm=True, seed=3)
    inp = make_inputs(w)
    kw = w.options()
    a = run_gpu(csa, inp, kw, backward=False)
    cut = 200
    inp2 = {k: (v.clone() if v is not None else None) for k, v in inp.items()}
    for n in ("q", "k", "v"):
        inp2[n][:, cut:] = -inp2[n][:, cut:]
    b = run_gpu(csa, inp2, kw, backward=False)
    assert np.array_equal(a["o"][:, :cut], b["o"][:, :cut])
    assert np.array_equal(a["lse"][:, :, :cut], b["lse"][:, :, :cut])


def test_repeated_calls_are_deterministic_in_forward(csa):
    w = WORKLOADS[3].with_(B=2)
    inp = make_inputs(w)
    a = run_gpu(csa, inp, w.options(), backward=False)
    b = run_gpu(csa, inp, w.options(), backward=False)
    assert np.array_equal(a["o"], b["o"])
