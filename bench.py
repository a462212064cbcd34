#!/usr/bin/env python
"""Attention forward+backward throughput on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the whole path over one batch: csa_attn_fwd (segment bounds / RoPE
table, QK-norm+RoPE prologue, flash forward) then csa_attn_bwd_after_fwd (delta
preprocess, flash backward, dQ/dK finalize; it reads the forward's q', k' from the shared
workspace, as a training step would, instead of recomputing the prologue), inputs resident
in HBM.  The default
workload is the 181M-model GQA shape (B=16, T=2048, 8 query / 4 KV heads, head dim 96,
RoPE, QK-norm), the largest of the five shapes.  FLOPs are algorithmic: only the
(query, key) pairs the mask keeps count, 4*D per pair per head forward, 10*D backward.

Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the launch stream
with an L2 flush (256 MiB write) between steps outside the events; a barrier and a
device synchronize on both sides; the max over ranks.  With N > 1 every rank runs its own
batch (independent problems, weak scaling); the only collective is the timing reduction.
`--impl reference` times the fp64 CPU oracle (the reference arm) on a bounded sample.

At N = 1 the line also carries `per_workload`: the same step, steps and warm-up for every
named workload (ms/step, TFLOP/s, tokens/s, % of the measured burst peak, forward and
backward kernel TFLOP/s, kernel shares), plus the KV-cache decode leg (GB/s against HBM)
and the chunked-prefill leg (TFLOP/s).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from causal_self_attention_gqa_b200.workloads import (BY_NAME, DECODE_WORKLOADS, LAYER_WORKLOADS,  # noqa: E402
                                                      WORKLOADS, LayerWorkload, make_decode_inputs, make_inputs)

DEFAULT_WORKLOAD = WORKLOADS[3].name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def visible_pairs(w, segment_ids) -> int:
    """Number of unmasked (query, key) pairs summed over batch rows, per head."""
    T, W = w.T, w.window
    total = 0
    for b in range(w.B):
        if segment_ids is not None:
            ids = np.asarray(segment_ids[b])
            starts = np.concatenate([[0], np.nonzero(np.diff(ids))[0] + 1])
            ends = np.concatenate([starts[1:], [T]])
        else:
            starts, ends = np.array([0]), np.array([T])
        for s, e in zip(starts, ends):
            L = int(e - s)
            i = np.arange(L)
            if w.causal:
                cnt = i + 1
                if W > 0:
                    cnt = np.minimum(cnt, W)
            else:
                lo = np.maximum(0, i - W + 1) if W > 0 else np.zeros_like(i)
                hi = np.minimum(L - 1, i + W - 1) if W > 0 else np.full_like(i, L - 1)
                cnt = hi - lo + 1
            total += int(cnt.sum())
    return total


def flops(w, segment_ids):
    pairs = visible_pairs(w, segment_ids)
    fwd = 4.0 * w.Hq * w.D * pairs
    bwd = 10.0 * w.Hq * w.D * pairs
    return fwd, bwd, pairs


def rank_workload(w, rank: int):
    """The batch rank `rank` runs: same shape, its own seed (independent problems, weak scaling)."""
    return w.with_(seed=w.seed + 7919 * rank)


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step: float, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: the work of every rank over the slowest rank's time."""
    return flops_per_rank_step * world * steps / (ms_max * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    return FALLBACK_PEAKS, "fallback (no MEASURED_PEAKS.json)"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel source is
    unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                a, b = line.strip().split("=", 1)
                kv[a.strip()] = b.strip()
    src = os.path.join(ROOT, "causal_self_attention_gqa_b200", "csrc", kv.get("source", ""))
    if not os.path.exists(src) or "source_sha256" not in kv:
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != kv["source_sha256"]:
            return None
    try:
        return float(kv["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark(self, which):
        if which == "begin":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append(dict(ts=ts, sm=float(parts[2]), smax=float(parts[3]), active=parts[5],
                                     hw=parts[6], hwt=parts[7], swt=parts[8], pcap=parts[9]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        if not rows:
            return {"samples": 0}
        inside = [r for r in rows if self.t0 - 0.05 <= r["ts"] <= self.t1 + 0.05] or rows
        reasons = set()
        for r in inside:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in inside), "sm_max_mhz": max(r["smax"] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside),
                "samples_in_timed_region": sum(1 for r in rows if self.t0 <= r["ts"] <= self.t1)}


# ----------------------------------------------------------------------------- oracle arm
def oracle_units(w, start: int, n: int):
    """The (batch row, key/value-head group) units start .. start+n-1 of the workload, in
    row-major order (wrapping): the oracle's own work units (its backward runs OpenMP over
    them, its forward over their query heads)."""
    total = w.B * w.Hkv
    return [((start + i) % total // w.Hkv, (start + i) % total % w.Hkv) for i in range(n)]


def oracle_sample(w, inp, units, threads: int):
    """fwd + bwd of the CPU oracle, as it stands, on the given (b, group) units run as one
    batch on `threads` OpenMP threads.  Returns (TFLOP/s, seconds, FLOPs)."""
    import oracle
    oracle.build()
    oracle.set_threads(threads)
    G = w.Hq // w.Hkv
    q = torch.stack([inp["q"][b, :, g * G:(g + 1) * G] for b, g in units])
    k = torch.stack([inp["k"][b, :, g:g + 1] for b, g in units])
    v = torch.stack([inp["v"][b, :, g:g + 1] for b, g in units])
    do = torch.stack([inp["do"][b, :, g * G:(g + 1) * G] for b, g in units])
    seg = torch.stack([inp["segment_ids"][b] for b, _ in units]) if inp["segment_ids"] is not None else None
    kw = w.options()
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, segment_ids=seg, **kw)
    oracle.attn_bwd(q, k, v, do, segment_ids=seg, **kw)
    dt = time.perf_counter() - t0
    sub = w.with_(B=len(units), Hq=G, Hkv=1)
    f, bw, _ = flops(sub, seg.numpy() if seg is not None else None)
    return (f + bw) / dt / 1e12, dt, f + bw


def host_cores() -> int:
    return len(os.sched_getaffinity(0))


def run_reference(args, w):
    """The reference arm: the fp64 oracle on the host's cores.  Step i is the oracle's
    forward + backward of one (batch row, key/value-head group) unit of the workload; the
    W warm-up units, then the K timed units, each run as one batch on every core, so the
    whole run stays within minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = make_inputs(w)
    cores = host_cores()
    oracle_sample(w, inp, oracle_units(w, 0, max(args.warmup, 1)), cores)
    value, dt, _ = oracle_sample(w, inp, oracle_units(w, args.warmup, args.steps), cores)
    sample = (f"{args.steps} units of one batch row x one KV-head group ({w.Hq // w.Hkv} query heads) of "
              f"{w.name}, fwd+bwd in fp64, run as one batch on {cores} threads")
    line = {"impl": "reference", "metric": metric_name(), "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "threads": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def metric_name():
    return "causal attn fwd+bwd TFLOP/s and tokens/s on 1 B200; % of dense BF16 peak"


def config_dict(w, n):
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "options": {k: v for k, v in w.options().items()},
            "packed_segments": None if w.seg_len is None else list(w.seg_len),
            "global_batch": w.B * n, "seq_len": w.T, "parallelism": f"dp{n}" if n > 1 else "single",
            "l2": "flushed between timed steps (256 MiB write, outside the events)"}


def profile_step(w):
    """Warm-up step + one step of the path on cuda:0, for an ncu capture (-s/-c select it)."""
    from causal_self_attention_gqa_b200 import _binding as csa
    dev = torch.device("cuda:0")
    inp = make_inputs(w)
    kw = w.options()
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    seg = inp["segment_ids"].to(dev) if inp["segment_ids"] is not None else None
    ws = csa.workspace_for(q, k, True, **kw)
    for _ in range(2):
        o, lse = csa.attn_fwd(q, k, v, segment_ids=seg, workspace=ws, **kw)
        csa.attn_bwd(q, k, v, o, do, lse, segment_ids=seg, workspace=ws, after_fwd=True, **kw)
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    print(json.dumps({"profile_step": w.name, "B": w.B, "status": rc}))
    return 0 if rc == 0 else 1


def measure_decode(steps: int, warmup: int, batch: int = 0) -> dict:
    """KV-cache decoding (csa_attn_decode), 1 GPU: cache bytes read per second against the
    measured HBM copy bandwidth.  The K/V cache (201 MB at the default shape) is larger than
    L2, so every step streams it from HBM; no flush is needed between steps."""
    from causal_self_attention_gqa_b200 import _binding as csa
    w = DECODE_WORKLOADS[0]
    if batch > 0:
        w = w.with_(B=batch)
    dev = torch.device("cuda:0")
    inp = make_decode_inputs(w)
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    kw = w.options()
    p = csa.make_params(w.B, w.Tk, w.Hq, w.Hkv, w.D, **kw)
    ws = torch.empty(csa.decode_workspace_size(p, w.Tq), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(warmup, 3)):
        csa.attn_decode(q, kc, vc, out=o, lse=lse, workspace=ws, **kw)
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {csa.status_string(rc)}")
    csa.timing_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        csa.attn_decode(q, kc, vc, out=o, lse=lse, workspace=ws, **kw)
    e1.record(stream)
    torch.cuda.synchronize()
    csa.timing_enable(False)
    kt = csa.timing_collect()
    ms = e0.elapsed_time(e1) / steps
    cache_bytes = 2 * w.B * w.Tk * w.Hkv * w.D * 2
    io_bytes = cache_bytes + 2 * q.numel() * 2 + lse.numel() * 4
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    split_ms = kt["k_decode"][0] / max(kt["k_decode"][1], 1)
    gbs = io_bytes / (ms * 1e-3) / 1e9
    split_gbs = cache_bytes / (split_ms * 1e-3) / 1e9
    line = {
        "metric": "KV-cache decode step: bytes read per second (cache + queries + outputs)", "value": gbs,
        "unit": "GB/s", "n_gpus": 1, "steps": steps, "warmup": max(warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; see workloads.py)",
        "config": {"workload": w.name, "B": w.B, "Tk": w.Tk, "Tq": w.Tq, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "options": kw, "l2": "cache larger than L2, streamed every step"},
        "tokens_per_s": w.B * w.Tq / (ms * 1e-3),
        "kernels": {n: {"ms_avg": t / c if c else 0.0, "launches": c} for n, (t, c) in kt.items() if c},
        "roofline": {"bound": "hbm", "achieved": split_gbs, "peak": hbm, "unit": "GB/s", "frac": split_gbs / hbm,
                     "traffic": recorded_traffic("k_decode", w.name) if batch <= 0 else None,
                     "kernel": "k_decode", "peak_source": f"{src}, hbm_gbs"},
        "gpu_launches": sum(c for _, c in kt.values()),
    }
    return line


def measure_prefill(steps: int, warmup: int, batch: int = 0) -> dict:
    """Forward over a KV cache (csa_attn_prefill): a 2048-token chunk at the end of an
    8192-entry cache, 181M shape, batch 4; algorithmic TFLOP/s (4 D per visible pair and query
    head) against the measured bf16 peak.  The caches (101 MB) and queries exceed L2 together."""
    from causal_self_attention_gqa_b200 import _binding as csa
    from causal_self_attention_gqa_b200.workloads import DecodeWorkload
    w = DecodeWorkload("prefill_gpt181m_gqa8x4_D96_rope_qknorm_chunk2048_cache8192", B=batch or 4, Tk=8192,
                       Tq=2048, Hq=8, Hkv=4, D=96, rope_base=10000.0, qk_norm=True, seed=2001)
    dev = torch.device("cuda:0")
    inp = make_decode_inputs(w)
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    kw = w.options()
    p = csa.make_params(w.B, w.Tk, w.Hq, w.Hkv, w.D, **kw)
    ws = torch.empty(csa.prefill_workspace_size(p, w.Tq), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Tq), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(warmup, 3)):
        csa.attn_prefill(q, kc, vc, out=o, lse=lse, workspace=ws, **kw)
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {csa.status_string(rc)}")
    csa.timing_enable(True)
    times = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        csa.attn_prefill(q, kc, vc, out=o, lse=lse, workspace=ws, **kw)
        e1.record(stream)
        times.append((e0, e1))
    torch.cuda.synchronize()
    csa.timing_enable(False)
    kt = {n: tc for n, tc in csa.timing_collect().items() if tc[1] > 0}
    ms = sum(a.elapsed_time(b) for a, b in times) / steps
    off = w.Tk - w.Tq
    pairs = sum(off + i + 1 for i in range(w.Tq))  # causal, per (b, query head)
    flops = 4.0 * w.D * w.Hq * w.B * pairs
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    fwd_ms = kt["k_attn_fwd"][0] / kt["k_attn_fwd"][1]
    line = {
        "metric": "forward over a KV cache (chunked prefill): algorithmic TFLOP/s", "value": flops / (ms * 1e-3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": max(warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; see workloads.py)",
        "config": {"workload": w.name, "B": w.B, "Tk": w.Tk, "Tq": w.Tq, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "options": kw, "l2": "flushed between timed steps (256 MiB write, outside the events)"},
        "tokens_per_s": w.B * w.Tq / (ms * 1e-3),
        "kernels": {n: {"ms_avg": t / c, "launches": c} for n, (t, c) in kt.items()},
        "roofline": {"bound": "tensor", "achieved": flops / (fwd_ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                     "frac": flops / (fwd_ms * 1e-3) / 1e12 / peak, "traffic": None, "kernel": "k_attn_fwd",
                     "peak_source": f"{src}, bf16_tflops"},
        "gpu_launches": sum(c for _, c in kt.values()),
    }
    return line


def measure_training(w, dev, steps: int, warmup: int, flush) -> dict:
    """The training step (csa_attn_fwd, then csa_attn_bwd_after_fwd on the same workspace) of
    workload w on one GPU, timed like the headline: per-step CUDA events, L2 flush between
    steps outside the events, per-kernel library events in the same region."""
    from causal_self_attention_gqa_b200 import _binding as csa
    inp = make_inputs(w)
    seg_np = inp["segment_ids"].numpy() if inp["segment_ids"] is not None else None
    f_fwd, f_bwd, pairs = flops(w, seg_np)
    kw = w.options()
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    seg = inp["segment_ids"].to(dev) if inp["segment_ids"] is not None else None
    ws = csa.workspace_for(q, k, True, **kw)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream()

    def step():
        csa.attn_fwd(q, k, v, segment_ids=seg, out=o, lse=lse, workspace=ws, **kw)
        csa.attn_bwd(q, k, v, o, do, lse, segment_ids=seg, dq=dq, dk=dk, dv=dv, workspace=ws, after_fwd=True,
                     **kw)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"{w.name}: device status after warm-up: {csa.status_string(rc)}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    csa.timing_enable(True)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    csa.timing_enable(False)
    kt = {n: tc for n, tc in csa.timing_collect().items() if tc[1] > 0}
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"{w.name}: device status after the timed steps: {csa.status_string(rc)}")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tot_k = sum(t for t, _ in kt.values()) or 1.0
    fwd_ms = kt["k_attn_fwd"][0] / kt["k_attn_fwd"][1]
    bwd_ms = kt["k_attn_bwd"][0] / kt["k_attn_bwd"][1]
    tflops = (f_fwd + f_bwd) / (ms * 1e-3) / 1e12
    return {"ms_per_step": ms, "tflops": tflops, "tokens_per_s": w.B * w.T / (ms * 1e-3),
            "pct_of_measured_burst": 100.0 * tflops / peak,
            "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12, "bwd_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
            "flops_per_step": f_fwd + f_bwd, "pairs_per_head": pairs, "steps": steps, "warmup": max(warmup, 3),
            "launches_per_step": sum(c for _, c in kt.values()) / steps,
            "kernels": {n: {"ms_avg": t / c, "share": t / tot_k} for n, (t, c) in kt.items()}}


GEMM_KERNELS = ("k_gemm_qkv", "k_gemm_out", "k_gemm_dout", "k_gemm_dwo", "k_gemm_dx", "k_gemm_dw")


def gemm_flops(lw) -> dict:
    """Multiply-adds x 2 of each projection product of one layer step (M = B*T tokens)."""
    a = lw.attn
    M, C, hq, hk = a.B * a.T, lw.C, a.Hq * a.D, a.Hkv * a.D
    qkv = 2.0 * M * C * (hq + 2 * hk)
    out = 2.0 * M * hq * C
    return {"k_gemm_qkv": qkv, "k_gemm_out": out, "k_gemm_dout": out, "k_gemm_dwo": out, "k_gemm_dx": qkv,
            "k_gemm_dw": qkv}


def measure_layer(lw, dev, steps: int, warmup: int, flush) -> dict:
    """The attention layer's training step with its projections, 1 GPU: csa_qkv_proj,
    csa_attn_fwd, csa_out_proj, then csa_out_proj_bwd (with dwo), csa_attn_bwd_after_fwd and
    csa_qkv_proj_bwd (with dwq, dwk, dwv).  Timed like the headline (per-step events, L2
    flushed between steps outside them); TFLOP/s counts the attention's algorithmic FLOPs plus
    2 per multiply-add of the six projection products.  Weight gradients accumulate over the
    steps (the calls add into them), as under gradient accumulation."""
    from causal_self_attention_gqa_b200 import _binding as csa
    from causal_self_attention_gqa_b200.workloads import make_layer_inputs
    a = lw.attn
    inp = make_layer_inputs(lw)
    f_fwd, f_bwd, _ = flops(a, None)
    gf = gemm_flops(lw)
    kw = a.options()
    x, wq, wk, wv, wo, dy = (inp[n].to(dev) for n in ("x", "wq", "wk", "wv", "wo", "dy"))
    q = torch.empty((a.B, a.T, a.Hq, a.D), dtype=torch.bfloat16, device=dev)
    k = torch.empty((a.B, a.T, a.Hkv, a.D), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    o, dout, dq = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dk, dv = torch.empty_like(k), torch.empty_like(k)
    y, dx = torch.empty_like(x), torch.empty_like(x)
    lse = torch.empty((a.B, a.Hq, a.T), dtype=torch.float32, device=dev)
    dwq, dwk, dwv = (torch.zeros(t.shape, dtype=torch.float32, device=dev) for t in (wq, wk, wv))
    dwo = torch.zeros(wo.shape, dtype=torch.float32, device=dev)
    ws = csa.workspace_for(q, k, True, **kw)
    stream = torch.cuda.current_stream()

    def step():
        csa.qkv_proj(x, wq, wk, wv, q=q, k=k, v=v, workspace=ws)
        csa.attn_fwd(q, k, v, out=o, lse=lse, workspace=ws, **kw)
        csa.out_proj(o, wo, y=y, workspace=ws)
        csa.out_proj_bwd(o, wo, dy, dout=dout, dwo=dwo, workspace=ws)
        csa.attn_bwd(q, k, v, o, dout, lse, dq=dq, dk=dk, dv=dv, workspace=ws, after_fwd=True, **kw)
        csa.qkv_proj_bwd(x, wq, wk, wv, dq, dk, dv, dx=dx, dwq=dwq, dwk=dwk, dwv=dwv, workspace=ws)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"{lw.name}: device status after warm-up: {csa.status_string(rc)}")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    csa.timing_enable(True)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    csa.timing_enable(False)
    kt = {n: tc for n, tc in csa.timing_collect().items() if tc[1] > 0}
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"{lw.name}: device status after the timed steps: {csa.status_string(rc)}")
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tot_k = sum(t for t, _ in kt.values()) or 1.0
    gemm = {}
    for n in GEMM_KERNELS:
        t, c = kt[n]
        tf = gf[n] / (t / c * 1e-3) / 1e12
        gemm[n] = {"ms_avg": t / c, "tflops": tf, "frac_of_measured_burst": tf / peak, "flops": gf[n]}
    g_ms = sum(kt[n][0] for n in GEMM_KERNELS) / steps
    g_fl = sum(gf.values())
    top = max(GEMM_KERNELS, key=lambda n: kt[n][0])
    return {"ms_per_step": ms, "tflops": (f_fwd + f_bwd + g_fl) / (ms * 1e-3) / 1e12,
            "tokens_per_s": a.B * a.T / (ms * 1e-3), "flops_per_step": f_fwd + f_bwd + g_fl,
            "projection_flops_per_step": g_fl, "projection_ms_per_step": g_ms,
            "projection_tflops": g_fl / (g_ms * 1e-3) / 1e12, "gemm": gemm,
            "roofline": {"bound": "tensor", "achieved": gemm[top]["tflops"], "peak": peak, "unit": "TFLOP/s",
                         "frac": gemm[top]["tflops"] / peak, "traffic": None, "kernel": top,
                         "peak_source": f"{src}, bf16_tflops"},
            "config": {"workload": lw.name, "B": a.B, "T": a.T, "C": lw.C, "Hq": a.Hq, "Hkv": a.Hkv, "D": a.D,
                       "options": kw},
            "steps": steps, "warmup": max(warmup, 3), "launches_per_step": sum(c for _, c in kt.values()) / steps,
            "kernels": {n: {"ms_avg": t / c, "share": t / tot_k} for n, (t, c) in kt.items()}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-workload map (every named workload, decode and prefill legs)")
    ap.add_argument("--e2e-steps", type=int, default=0, help="steps of the end-to-end leg (default: min(K, 20))")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size (profiling cases)")
    ap.add_argument("--prefill", action="store_true",
                    help="time the forward over a KV cache (csa_attn_prefill) instead of the training step")
    ap.add_argument("--layer", action="store_true",
                    help="time the attention layer with its projections (181M shape, C = 768) instead")
    ap.add_argument("--decode", action="store_true",
                    help="time the KV-cache decode step (csa_attn_decode) instead of the training step")
    ap.add_argument("--profile-step", action="store_true",
                    help="one warm-up step and one plain step, nothing else: a small case for ncu")
    args = ap.parse_args()
    w = BY_NAME[args.workload]
    if args.batch > 0:
        w = w.with_(B=args.batch)
    if args.profile_step:
        return profile_step(w)
    if args.layer:
        lw = LAYER_WORKLOADS[0]
        if args.batch:
            lw = LayerWorkload(lw.name, lw.attn.with_(B=args.batch), C=lw.C, seed=lw.seed)
        dev = torch.device("cuda:0")
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        r = measure_layer(lw, dev, args.steps, args.warmup, flush)
        print(json.dumps({"metric": "attention layer with projections, fwd+bwd: algorithmic TFLOP/s",
                          "value": r["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "higher_is_better": True,
                          "dtype": "bf16", "data": "synthetic (seeded bf16; see workloads.py)", **r}))
        return 0
    if args.decode:
        print(json.dumps(measure_decode(args.steps, args.warmup, args.batch)))
        return 0
    if args.prefill:
        print(json.dumps(measure_prefill(args.steps, args.warmup, args.batch)))
        return 0
    if args.impl == "reference":
        return run_reference(args, w)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from causal_self_attention_gqa_b200 import _binding as csa

    # every rank runs its own batch of the workload (weak scaling)
    wr = rank_workload(w, rank)
    inp = make_inputs(wr)
    seg_np = inp["segment_ids"].numpy() if inp["segment_ids"] is not None else None
    f_fwd, f_bwd, pairs = flops(wr, seg_np)
    kw = wr.options()
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    seg = inp["segment_ids"].to(dev) if inp["segment_ids"] is not None else None
    ws = csa.workspace_for(q, k, True, **kw)
    o = torch.empty_like(q)
    lse = torch.empty((wr.B, wr.Hq, wr.T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        csa.attn_fwd(q, k, v, segment_ids=seg, out=o, lse=lse, workspace=ws, **kw)
        csa.attn_bwd(q, k, v, o, do, lse, segment_ids=seg, dq=dq, dk=dk, dv=dv, workspace=ws, after_fwd=True,
                     **kw)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {csa.status_string(rc)}")

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    csa.timing_enable(True)
    sampler.mark("begin")
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    sampler.mark("end")
    csa.timing_enable(False)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    kt = csa.timing_collect()
    rc = csa.device_status(ws)
    if rc != 0:
        raise RuntimeError(f"device status after the timed region: {csa.status_string(rc)}")
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms_max = max_over_ranks(ms, dev)
    ms_per_step = ms_max / args.steps
    value = job_tflops(f_fwd + f_bwd, world, args.steps, ms_max)
    tokens_per_s = wr.B * wr.T * world * args.steps / (ms_max * 1e-3)

    # per-kernel times (library events on the launch stream, same timed region)
    launches = sum(c for _, c in kt.values())
    kt = {name: tc for name, tc in kt.items() if tc[1] > 0}
    per_kernel = {name: {"ms_avg": (t / c if c else 0.0), "launches": c, "share": 0.0} for name, (t, c) in kt.items()}
    tot_k = sum(t for t, _ in kt.values()) or 1.0
    for name, (t, c) in kt.items():
        per_kernel[name]["share"] = t / tot_k
    fwd_ms = per_kernel["k_attn_fwd"]["ms_avg"]
    bwd_ms = per_kernel["k_attn_bwd"]["ms_avg"]
    dom = max(("k_attn_fwd", "k_attn_bwd"), key=lambda n: kt[n][0])
    dom_flops = f_fwd if dom == "k_attn_fwd" else f_bwd
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = dom_flops / (per_kernel[dom]["ms_avg"] * 1e-3) / 1e12 if per_kernel[dom]["ms_avg"] > 0 else 0.0
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": recorded_traffic(dom, wr.name), "kernel": dom,
                "peak_source": f"{peak_src}, bf16_tflops (burst cuBLAS GEMM)"}

    # end-to-end through the public API from pinned host buffers (rank-local).  Every step
    # copies its inputs host -> device and its outputs device -> host inside the timed region;
    # the copies run on their own streams (one per direction, so both copy engines work) into
    # two alternating device slots, so step i's compute overlaps step i+1's inputs and step
    # i-1's outputs.
    e2e = None
    n_e2e = args.e2e_steps or min(args.steps, 20)
    if n_e2e > 0:
        names_in = ("q", "k", "v", "do")
        host_in = {n: inp[n].pin_memory() for n in names_in}
        hseg = inp["segment_ids"].pin_memory() if inp["segment_ids"] is not None else None
        host_out = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory()
                    for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
        h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + \
            (hseg.numel() * 4 if hseg is not None else 0)
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        slots_in = [{n: torch.empty_like(t, device=dev) for n, t in host_in.items()} for _ in range(2)]
        for sl in slots_in:
            sl["seg"] = torch.empty_like(hseg, device=dev) if hseg is not None else None
        slots_out = [{n: torch.empty_like(t, device=dev) for n, t in host_out.items()} for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]    # slot's inputs landed
        ev_done = [torch.cuda.Event() for _ in range(2)]  # slot's step computed
        ev_out = [torch.cuda.Event() for _ in range(2)]   # slot's outputs read back
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        h2d_s.wait_event(e0)
        d2h_s.wait_event(e0)
        for i in range(n_e2e):
            sl, so = slots_in[i % 2], slots_out[i % 2]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_done[i % 2])  # step i-2 no longer reads this slot
                for n in names_in:
                    sl[n].copy_(host_in[n], non_blocking=True)
                if hseg is not None:
                    sl["seg"].copy_(hseg, non_blocking=True)
                ev_in[i % 2].record(h2d_s)
            stream.wait_event(ev_in[i % 2])
            if i >= 2:
                stream.wait_event(ev_out[i % 2])  # step i-2's outputs have been read back
            csa.attn_fwd(sl["q"], sl["k"], sl["v"], segment_ids=sl["seg"], out=so["o"], lse=so["lse"],
                         workspace=ws, **kw)
            csa.attn_bwd(sl["q"], sl["k"], sl["v"], so["o"], sl["do"], so["lse"], segment_ids=sl["seg"],
                         dq=so["dq"], dk=so["dk"], dv=so["dv"], workspace=ws, after_fwd=True, **kw)
            ev_done[i % 2].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[i % 2])
                for n, t in host_out.items():
                    t.copy_(so[n], non_blocking=True)
                ev_out[i % 2].record(d2h_s)
        stream.wait_event(ev_out[(n_e2e - 1) % 2])  # the read-backs run in order on d2h_s
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": job_tflops(f_fwd + f_bwd, world, n_e2e, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e,
               "copies": "pinned host buffers, one stream per direction, two device slots (overlapped with compute)"}

    # every named workload (same steps, warm-up and timing), then the KV-cache legs; one GPU
    per_workload = None
    if world == 1 and not args.no_per_workload:
        per_workload = {}
        for wk in WORKLOADS:
            if wk.name == wr.name:
                per_workload[wk.name] = {
                    "ms_per_step": ms_per_step, "tflops": value, "tokens_per_s": tokens_per_s,
                    "pct_of_measured_burst": 100.0 * value / float(load_peaks()[0].get("bf16_tflops", 1.0)),
                    "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12, "bwd_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
                    "flops_per_step": f_fwd + f_bwd, "pairs_per_head": pairs, "steps": args.steps,
                    "warmup": max(args.warmup, 3), "launches_per_step": launches / args.steps,
                    "kernels": {n: {"ms_avg": d["ms_avg"], "share": d["share"]} for n, d in per_kernel.items()},
                    "headline": True}
            else:
                per_workload[wk.name] = measure_training(wk, dev, args.steps, args.warmup, flush)
        dl = measure_decode(args.steps, args.warmup)
        per_workload[dl["config"]["workload"]] = {
            "ms_per_step": dl["ms_per_step"], "gbs": dl["value"], "tokens_per_s": dl["tokens_per_s"],
            "roofline": dl["roofline"], "kernels": dl["kernels"], "steps": dl["steps"], "warmup": dl["warmup"]}
        pl = measure_prefill(args.steps, args.warmup)
        per_workload[pl["config"]["workload"]] = {
            "ms_per_step": pl["ms_per_step"], "tflops": pl["value"], "tokens_per_s": pl["tokens_per_s"],
            "roofline": pl["roofline"], "kernels": pl["kernels"], "steps": pl["steps"], "warmup": pl["warmup"]}
        for lw in LAYER_WORKLOADS:
            per_workload[lw.name] = measure_layer(lw, dev, args.steps, args.warmup, flush)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # one unit per core, so every core works: about one unit's time (10-30 s at T = 2048)
        cores = host_cores()
        units = oracle_units(wr, 0, cores)
        val, dt, _ = oracle_sample(wr, inp, units, cores)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cores, "threads": cores, "kind": "oracle",
               "sample": f"{len(units)} units of one batch row x one KV-head group ({wr.Hq // wr.Hkv} query heads) "
                         f"of {wr.name}, fwd+bwd in fp64 on {cores} threads, {dt:.1f} s"}

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    peak_spec = 2250.0
    line = {
        "metric": metric_name(), "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; see workloads.py)",
        "config": config_dict(wr, world),
        "tokens_per_s": tokens_per_s,
        "pct_of_peak": {"measured_burst": 100.0 * value / world / peak, "spec_2250": 100.0 * value / world / peak_spec},
        "fwd_tflops": f_fwd / (fwd_ms * 1e-3) / 1e12 if fwd_ms else None,
        "bwd_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12 if bwd_ms else None,
        "flops_per_step": {"fwd": f_fwd, "bwd": f_bwd, "pairs_per_head": pairs},
        # the common convention that counts causal attention as half of dense: 14 D Hq B T^2 / 2
        "tflops_causal_half_dense": (14.0 * wr.D * wr.Hq * wr.B * world * wr.T * wr.T / 2)
        / (ms_per_step * 1e-3) / 1e12,
        "kernels": per_kernel,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        "per_workload": per_workload,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
