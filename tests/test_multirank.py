"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU.  The
attention shards into independent problems (batch rows), so N ranks run N independent
batches and exchange nothing but the timing: the job time is the slowest rank's, and the
job throughput counts the work of every rank."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from causal_self_attention_gqa_b200.workloads import WORKLOADS, make_inputs
        w = bench.rank_workload(WORKLOADS[0].with_(B=1, T=16), rank)
        inp = make_inputs(w)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, torch.device("cpu"))
        value = bench.job_tflops(1e9, world, 4, ms_max)
        q.put((rank, w.seed, float(inp["q"].float().sum()), ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_job_timing_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, sum0, max0, val0), (r1, seed1, sum1, max1, val1) = out
    assert seed0 != seed1 and sum0 != sum1          # each rank has its own batch
    assert max0 == max1 == 15.0                     # slowest rank's time on both
    assert val0 == val1 == pytest.approx(1e9 * 2 * 4 / 15e-3 / 1e12)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_tflops(2e12, 1, 1, 1000.0) == pytest.approx(2.0)
