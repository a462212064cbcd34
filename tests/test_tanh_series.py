"""The FMA-pipe tanh used for the soft-cap when QK-norm bounds the scores (tanh_series2 in
ptx.cuh), replayed step by step in numpy float32 and checked against tanh in fp64 on its
range |u| <= 1/4: the coefficients are the Maclaurin ones (-1/3, 2/15, -17/315), and the
error stays below the first omitted term (62/2835)|u|^9 plus float rounding."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "causal_self_attention_gqa_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("float2 tanh_series2(float2 u)"):]
    body = body[: body.index("return fmul2(u, p);")]
    return [float(v) for v in re.findall(r"make_float2\((-?[0-9][0-9.e+-]*)f, \1f\)", body)]


def _series(u):
    u = u.astype(np.float32)
    c7, c5, c3, c1 = (np.float32(v) for v in _coeffs())
    u2 = (u * u).astype(np.float32)
    p = (u2 * c7 + c5).astype(np.float32)
    p = (p * u2 + c3).astype(np.float32)
    p = (p * u2 + c1).astype(np.float32)
    return (u * p).astype(np.float32)


def test_coefficients_are_the_maclaurin_ones():
    c = _coeffs()
    assert len(c) == 4
    for got, want in zip(c, (-17.0 / 315.0, 2.0 / 15.0, -1.0 / 3.0, 1.0)):
        assert abs(got - want) <= 1e-7 * abs(want), (got, want)


def test_error_within_the_omitted_term():
    u = np.concatenate([np.linspace(-0.25, 0.25, 1_000_001), np.random.default_rng(1).uniform(-0.25, 0.25, 100_000)])
    u = u.astype(np.float32)
    got = _series(u).astype(np.float64)
    ref = np.tanh(u.astype(np.float64))
    bound = 62.0 / 2835.0 * np.abs(u.astype(np.float64)) ** 9 + 4 * 2.0 ** -24 * np.abs(ref)
    assert np.all(np.abs(got - ref) <= bound + 1e-45)
    rel = np.abs(got - ref)[u != 0] / np.abs(ref[u != 0])
    assert rel.max() < 1e-6, rel.max()


def test_odd_and_exact_at_zero():
    u = np.linspace(0, 0.25, 10001).astype(np.float32)
    assert np.array_equal(_series(-u), -_series(u))
    assert _series(np.zeros(1, np.float32))[0] == 0.0
