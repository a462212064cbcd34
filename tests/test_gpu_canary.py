"""Every output and the workspace sit inside larger buffers filled with a sentinel byte; after
the forward and both backward entry points the bytes before and after each tensor must be
untouched.  Ragged T (129, 300: the last 128-row tile is partly outside the tensor) checks
that the TMA stores of O, dV and dK, the LSE writes, the dQ reduce-adds and the finalize
kernel never write past a tensor's end (every tensor is allocated exactly to size, so an
overrun would otherwise corrupt a neighbouring allocation silently)."""
import numpy as np
import pytest
import torch

from causal_self_attention_gqa_b200.workloads import Workload, make_inputs, packed_segment_ids

pytestmark = pytest.mark.gpu

PAD = 4096
SENTINEL = 0x5A


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding
    return _binding


class Guarded:
    """A tensor of the given shape and dtype placed PAD bytes into a sentinel-filled buffer."""

    def __init__(self, shape, dtype, dev):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((PAD + n + PAD,), SENTINEL, dtype=torch.uint8, device=dev)
        self.t = self.buf[PAD:PAD + n].view(dtype).view(*shape)

    def intact(self):
        b = self.buf.cpu().numpy()
        return bool(np.all(b[:PAD] == SENTINEL) and np.all(b[PAD + self.n:] == SENTINEL))


CASES = [
    # (B, T, Hq, Hkv, D, options, segments)
    (2, 129, 4, 2, 96, dict(rope_base=10000.0, qk_norm=True), None),
    (2, 300, 6, 3, 128, dict(rope_base=10000.0, qk_norm=True, softcap=50.0), None),
    (1, 300, 2, 2, 64, dict(), None),                       # no prologue: dK stored as bf16 by the kernel
    (2, 129, 2, 1, 32, dict(rope_base=10000.0, window=50), (10, 70)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}x{c[3]}D{c[4]}"
                         + "".join(f"-{k}{v}" for k, v in c[5].items()) + ("-seg" if c[6] else ""))
@pytest.mark.parametrize("after_fwd", [False, True])
def test_outputs_and_workspace_stay_in_bounds(csa, case, after_fwd):
    B, T, Hq, Hkv, D, opts, seg_len = case
    w = Workload("canary", B=B, T=T, Hq=Hq, Hkv=Hkv, D=D, seed=31 + T, **opts)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    seg = None
    if seg_len is not None:
        seg = torch.from_numpy(packed_segment_ids(B, T, seg_len[0], seg_len[1], 31)).to(dev)
    kw = w.options()
    ws_bytes = csa.workspace_size(csa.make_params(B, T, Hq, Hkv, D, **kw), True)
    ws = Guarded((ws_bytes,), torch.uint8, dev)
    o = Guarded((B, T, Hq, D), torch.bfloat16, dev)
    lse = Guarded((B, Hq, T), torch.float32, dev)
    dq = Guarded((B, T, Hq, D), torch.bfloat16, dev)
    dk = Guarded((B, T, Hkv, D), torch.bfloat16, dev)
    dv = Guarded((B, T, Hkv, D), torch.bfloat16, dev)
    csa.attn_fwd(q, k, v, segment_ids=seg, out=o.t, lse=lse.t, workspace=ws.t, **kw)
    csa.attn_bwd(q, k, v, o.t, do, lse.t, segment_ids=seg, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t,
                 after_fwd=after_fwd, **kw)
    torch.cuda.synchronize()
    assert csa.device_status(ws.t) == 0
    for name, g in (("workspace", ws), ("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert g.intact(), name
    # the guarded outputs are the real results: finite everywhere
    for name, g in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.isfinite(g.t.float()).all(), name


PROJ_CASES = [
    # (B, T, C, Hq, Hkv, D): a single-CTA shape with a ragged 128-row tile, and a CTA-pair
    # shape whose last 256-row tile and last 256-column tile are partly outside the tensors
    (1, 300, 256, 4, 2, 64),
    (1, 19044, 320, 5, 1, 64),
]


@pytest.mark.parametrize("case", PROJ_CASES, ids=lambda c: "B%dT%dC%dH%dx%dD%d" % c)
def test_projection_outputs_stay_in_bounds(csa, case):
    """The TMA stores (bf16 products) and reduce-adds (fp32 weight gradients) of the four
    projection calls never write outside their tensors."""
    B, T, C, Hq, Hkv, D = case
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(T)

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(dev)

    x, dy = rnd(B, T, C), rnd(B, T, C)
    wq, wk, wv = rnd(C, Hq, D, std=C ** -0.5), rnd(C, Hkv, D, std=C ** -0.5), rnd(C, Hkv, D, std=C ** -0.5)
    wo = rnd(Hq, D, C, std=(Hq * D) ** -0.5)
    o = rnd(B, T, Hq, D)
    bf = torch.bfloat16
    gq, gk, gv = (Guarded((B, T, H, D), bf, dev) for H in (Hq, Hkv, Hkv))
    gy, gdx = Guarded((B, T, C), bf, dev), Guarded((B, T, C), bf, dev)
    gdo = Guarded((B, T, Hq, D), bf, dev)
    gdwo = Guarded((Hq, D, C), torch.float32, dev)
    gdw = [Guarded((C, H, D), torch.float32, dev) for H in (Hq, Hkv, Hkv)]
    for t in [gdwo] + gdw:
        t.t.zero_()
    csa.qkv_proj(x, wq, wk, wv, q=gq.t, k=gk.t, v=gv.t)
    csa.out_proj(o, wo, y=gy.t)
    csa.out_proj_bwd(o, wo, dy, dout=gdo.t, dwo=gdwo.t)
    csa.qkv_proj_bwd(x, wq, wk, wv, gq.t, gk.t, gv.t, dx=gdx.t, dwq=gdw[0].t, dwk=gdw[1].t, dwv=gdw[2].t)
    torch.cuda.synchronize()
    for name, t in (("q", gq), ("k", gk), ("v", gv), ("y", gy), ("dout", gdo), ("dx", gdx), ("dwo", gdwo),
                    ("dwq", gdw[0]), ("dwk", gdw[1]), ("dwv", gdw[2])):
        assert t.intact(), name
    # and the products are there (not a silent no-op)
    assert float(gq.t.float().abs().sum()) > 0 and float(gdw[2].t.abs().sum()) > 0
