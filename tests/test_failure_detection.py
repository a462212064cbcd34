"""Failure detection without a GPU fault.  Every wait inside the library's kernels is a
bounded mbarrier wait: it gives up after about a second of SM clocks (or when another role
of the CTA has given up), records CSA_ERR_DEVICE_TIMEOUT in the status word and lets the
kernel unwind and exit.  Here a kernel waits on barrier phases that nothing will complete;
the test checks that every thread gave up, that the status reads back as a timeout, that
the wait was bounded, and that the device keeps working afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding as csa
    rc, gave_up, cycles = csa.selftest_bounded_wait()
    assert rc == csa.CSA_ERR_DEVICE_TIMEOUT, csa.status_string(rc)
    assert all(g == 1 for g in gave_up)
    # bounded: about 2e9 SM clocks (~1 s), never unbounded
    assert max(cycles) < 8e9
    # the device still works: a normal call afterwards succeeds with status OK
    from causal_self_attention_gqa_b200.workloads import Workload, make_inputs
    w = Workload("t", B=1, T=128, Hq=2, Hkv=1, D=64, seed=1)
    inp = make_inputs(w, need_grad_input=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    ws = csa.workspace_for(q, k, False)
    o, _ = csa.attn_fwd(q, k, v, workspace=ws)
    assert csa.device_status(ws) == 0
    assert torch.isfinite(o.float()).all()
