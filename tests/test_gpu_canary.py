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
