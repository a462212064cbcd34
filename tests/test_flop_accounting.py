"""The benchmark's FLOP accounting (bench.visible_pairs / bench.flops): the number of
unmasked (query, key) pairs must equal a brute-force count of the visibility rule (causal,
window, maximal runs of equal segment ids), since every reported TFLOP/s figure rests on it."""
import numpy as np
import pytest

import bench
from causal_self_attention_gqa_b200.workloads import WORKLOADS, Workload, packed_segment_ids


def brute_pairs(B, T, causal, window, seg):
    total = 0
    for b in range(B):
        for i in range(T):
            for j in range(T):
                if causal and j > i:
                    continue
                if window > 0 and (i - j >= window or (not causal and j - i >= window)):
                    continue
                if seg is not None:
                    lo, hi = min(i, j), max(i, j)
                    if np.any(seg[b, lo:hi + 1] != seg[b, i]):  # same maximal run
                        continue
                total += 1
    return total


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("window", [0, 1, 5, 40])
@pytest.mark.parametrize("packed", [False, True])
def test_visible_pairs_match_brute_force(causal, window, packed):
    B, T = 2, 37
    w = Workload("t", B=B, T=T, Hq=2, Hkv=1, D=32, causal=causal, window=window, seed=3)
    seg = packed_segment_ids(B, T, 3, 12, 3) if packed else None
    assert bench.visible_pairs(w, seg) == brute_pairs(B, T, causal, window, seg)


def test_repeated_ids_in_separate_runs_are_separate_segments():
    seg = np.array([[0, 0, 1, 1, 0, 0]], dtype=np.int32)  # id 0 twice, in two runs
    w = Workload("t", B=1, T=6, Hq=1, Hkv=1, D=32)
    assert bench.visible_pairs(w, seg) == brute_pairs(1, 6, True, 0, seg) == 3 * 3


def test_benchmark_shape_flops():
    w = WORKLOADS[3]  # the benchmark's 181M shape: causal, T = 2048, B = 16
    fwd, bwd, pairs = bench.flops(w, None)
    assert pairs == w.B * w.T * (w.T + 1) // 2 == 33_570_816
    assert fwd == 4.0 * w.Hq * w.D * pairs and bwd == 2.5 * fwd
