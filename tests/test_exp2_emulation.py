"""The FMA-pipe exp2 used for part of the softmax exponentials (exp2_fma2 in ptx.cuh),
replayed step by step in numpy float32 and checked against exp2 in fp64: the same
coefficients, the same rounding trick, the same exponent insertion.  The kernels' parity
tests then cover it on the GPU."""
import re
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "causal_self_attention_gqa_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("exp2_fma2"):]
    body = body[: body.index("return make_float2(__int_as_float")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9][0-9.e+-]*)f, \1f\)", body)]
    return vals  # c4, c3, c2, c1, c0 in Horner order


def _emulate(x):
    x = x.astype(np.float32)
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = [np.float32(v) for v in _coeffs()]
    p = np.full_like(f, c[0])
    for ck in c[1:]:
        p = (p * f + ck).astype(np.float32)
    bits = (t.view(np.int32).astype(np.int64) * 8388608 + p.view(np.int32).astype(np.int64)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_present():
    assert len(_coeffs()) == 5


def test_matches_exp2_within_bound():
    x = np.concatenate([np.linspace(-126.0, 127.0, 2_000_001), np.random.default_rng(0).uniform(-30, 8, 200_000)])
    x = x.astype(np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_integers_and_halves():
    for v in (-126.0, -20.0, -1.0, -0.5, 0.0, 0.5, 1.0, 8.0):
        got = float(_emulate(np.array([v], dtype=np.float32))[0])
        assert abs(got / 2.0 ** v - 1.0) < 4e-6, (v, got)
