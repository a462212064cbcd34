"""The pins must reject a broken oracle: each case below plants one plausible mistake in a
copy of oracle.c (on the CPU, in a temporary directory), builds it, and runs the pin suite
against it in a subprocess; the suite has to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "rope_sign": ("y[d] = a * c - bb * s;", "y[d] = a * c + bb * s;"),
    "rope_freq": ("pow(p->rope_base, -2.0 * d / D);\n            double phi = pos * theta;\n            double c = cos(phi), s = sin(phi);\n            double a = y[d]",
                  "pow(p->rope_base, -1.0 * d / D);\n            double phi = pos * theta;\n            double c = cos(phi), s = sin(phi);\n            double a = y[d]"),
    "gqa_interleaved": ("kvh = h / G;\n    const double sc", "kvh = h % p->Hkv;\n    const double sc"),
    "norm_eps_dropped": ("r = 1.0 / sqrt(ss / D + p->qk_norm_eps);\n    }\n    for", "r = 1.0 / sqrt(ss / D);\n    }\n    for"),
    "norm_bwd_term": ("dx[d] = r * (u[d] - x[d] * r * dot / D);", "dx[d] = r * u[d];"),
    "window_off_by_one": ("if (d >= p->window) return 0; }", "if (d > p->window) return 0; }"),
    "cap_before_scale": ("            s *= sc;\n            if (Sraw)", "            if (Sraw)"),
    "cap_grad": ("g *= 1.0 - th * th;", "g *= 1.0 + th * th;"),
    "softmax_jacobian_sign": ("double g = P[(size_t)i * T + j] * (dP[j] - rowdot);",
                              "double g = P[(size_t)i * T + j] * (dP[j] + rowdot);"),
    "segment_end_ignored": ("if (j < st[i] || j >= en[i]) return 0;", "if (j < st[i]) return 0;"),
    "dk_transposed": ("acc += dS[(size_t)i * T + j] * qp[(size_t)i * D + d];",
                      "acc += dS[(size_t)j * T + i] * qp[(size_t)i * D + d];"),
    "lse_missing_max": ("if (lse) lse[i] = m + log(l);", "if (lse) lse[i] = log(l);"),
}


# Mistakes in the KV-cache attention (oracle_attn_fwd_cached), against its own pins.
CACHED_MUTANTS = {
    "cached_position_from_zero": ("const int pos = offset + i;", "const int pos = i;"),
    "cached_mask_off_by_one": ("if (p->causal && j > pos) vis = 0;", "if (p->causal && j >= pos) vis = 0;"),
    "cached_window_off_by_one": ("if (dd >= p->window || (!p->causal && -dd >= p->window)) vis = 0;",
                                 "if (dd > p->window || (!p->causal && -dd >= p->window)) vis = 0;"),
    "cached_gqa_interleaved": ("            const int kvh = h / G;\n            double* qp = (double*)malloc(sizeof(double) * (size_t)D);",
                               "            const int kvh = h % Hkv;\n            double* qp = (double*)malloc(sizeof(double) * (size_t)D);"),
    "cached_cap_missing": ("if (p->softcap > 0.0) acc = p->softcap * tanh(acc / p->softcap);", ""),
    "cached_lse_missing_max": ("lse[((size_t)b * Hq + h) * Tq + i] = m + log(l);",
                               "lse[((size_t)b * Hq + h) * Tq + i] = log(l);"),
}


def _run_pins(name, old, new, pin_file, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    mutated = tmp_path / "oracle.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                           str(mutated), "-o", str(lib), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", pin_file)],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.mark.parametrize("name", sorted(CACHED_MUTANTS))
def test_cached_pins_reject_mutant(name, tmp_path):
    old, new = CACHED_MUTANTS[name]
    r = _run_pins(name, old, new, "test_oracle_cached.py", tmp_path)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    r = _run_pins(name, old, new, "test_oracle.py", tmp_path)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
