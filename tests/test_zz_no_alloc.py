"""csa_attn_fwd_static_scratch: the forward for callers that cannot allocate device memory
(a host framework that owns every device allocation, or a latency-critical loop that cannot
afford cudaMalloc's implicit synchronisation).  Its scratch is a fixed array inside the
library, so the test checks it against the ordinary workspace forward on two calls in a
row: the second call must not be disturbed by what the first left in the shared array.
Collected last on purpose (file name), so a failure here cannot hide other results."""
import ctypes

import numpy as np
import pytest
import torch

from causal_self_attention_gqa_b200.workloads import Workload, make_inputs, packed_segment_ids

O_REL, O_ABS, LSE_ABS = 1e-2, 2e-2, 1e-2


def _call_static(csa, p, q, k, v, seg, o, lse, status):
    return csa.lib.csa_attn_fwd_static_scratch(
        ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(), None if seg is None else seg.data_ptr(),
        o.data_ptr(), lse.data_ptr(), None if status is None else status.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_static_scratch_forward_matches_workspace_forward_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding as csa
    dev = torch.device("cuda:0")
    cases = [
        # packed rows with RoPE + QK-norm + cap + window: every part of the scratch in use
        (Workload("a", B=2, T=300, Hq=4, Hkv=2, D=64, rope_base=10000.0, qk_norm=True, softcap=50.0,
                  window=160, seed=21), (40, 200), True),
        # then a different shape with no segments and no prologue: stale scratch must not leak in
        (Workload("b", B=4, T=257, Hq=6, Hkv=3, D=96, seed=22), None, True),
        # no status pointer: the device-side status then stays inside the library's array
        (Workload("c", B=1, T=200, Hq=2, Hkv=1, D=128, rope_base=10000.0, qk_norm=True, seed=23), None, False),
    ]
    for w, seg_len, with_status in cases:
        inp = make_inputs(w, need_grad_input=False)
        q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
        seg = None
        if seg_len is not None:
            seg = torch.from_numpy(packed_segment_ids(w.B, w.T, seg_len[0], seg_len[1], w.seed)).to(dev)
        kw = w.options()
        o_ref, lse_ref = csa.attn_fwd(q, k, v, segment_ids=seg, **kw)
        p = csa.make_params(w.B, w.T, w.Hq, w.Hkv, w.D, **kw)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((w.B, w.Hq, w.T), float("nan"), dtype=torch.float32, device=dev)
        status = torch.full((1,), -1, dtype=torch.int32, device=dev) if with_status else None
        rc = _call_static(csa, p, q, k, v, seg, o, lse, status)
        assert rc == 0, csa.status_string(rc)
        torch.cuda.synchronize()
        if with_status:
            assert int(status.item()) == 0
        a, r = o.float().cpu().numpy(), o_ref.float().cpu().numpy()
        assert np.all(np.isfinite(a))
        rel = np.linalg.norm(a - r) / np.linalg.norm(r)
        assert rel <= O_REL and np.max(np.abs(a - r)) <= O_ABS, rel
        assert np.max(np.abs(lse.cpu().numpy() - lse_ref.cpu().numpy())) <= LSE_ABS


def test_static_scratch_rejects_problems_beyond_its_size():
    """Checked on the host before any device work (no GPU needed)."""
    from causal_self_attention_gqa_b200 import build
    build.build()  # this file may run alone, before any other test has built the library
    from causal_self_attention_gqa_b200 import _binding as csa
    # the 181M-model shape needs ~75 MiB of normalised q/k copies: more than the 16 MiB array
    p = csa.make_params(16, 2048, 8, 4, 96, rope_base=10000.0, qk_norm=True)
    fake = 0x10000  # never dereferenced: the size check fails first
    rc = csa.lib.csa_attn_fwd_static_scratch(ctypes.byref(p), fake, fake, fake, None, fake, fake, None, None)
    assert rc == csa.CSA_ERR_WORKSPACE
