"""KV-cache decoding (csa_attn_decode, through the C ABI) against the fp64 oracle's cached
attention on the same seeded bf16 inputs.  Same tolerances as the forward: O relative L2
<= 1e-2 and max-abs <= 2e-2; LSE max-abs <= 1e-2.  Cases cover one to sixteen new queries,
caches shorter than one key range and ragged ones, every head dimension, GQA group sizes
1 to 8, binding windows, the cap, bidirectional attention and RoPE at large absolute
positions."""
import numpy as np
import pytest
import torch

from causal_self_attention_gqa_b200.workloads import DECODE_WORKLOADS, DecodeWorkload, make_decode_inputs

pytestmark = pytest.mark.gpu

O_REL, O_ABS, LSE_ABS = 1e-2, 2e-2, 1e-2


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_self_attention_gqa_b200 import _binding
    return _binding


@pytest.fixture(scope="module")
def ora():
    import oracle
    oracle.build()
    return oracle


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run_case(csa, ora, w, rows=None):
    inp = make_decode_inputs(w)
    dev = torch.device("cuda:0")
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    o, lse = csa.attn_decode(q, kc, vc, **w.options())
    torch.cuda.synchronize()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    sl = slice(None) if rows is None else rows
    ref_o, ref_lse = ora.attn_fwd_cached(inp["q"][sl], inp["k_cache"][sl], inp["v_cache"][sl], **w.options())
    o, lse = o[sl], lse[sl]
    assert np.all(np.isfinite(o))
    r, m = rel_l2(o, ref_o), float(np.max(np.abs(o - ref_o)))
    assert r <= O_REL and m <= O_ABS, (r, m)
    assert float(np.max(np.abs(lse - ref_lse))) <= LSE_ABS


CASES = [
    # (B, Tk, Tq, Hq, Hkv, D, options)
    (1, 1, 1, 2, 1, 32, dict()),
    (2, 37, 1, 4, 2, 64, dict()),
    (2, 300, 1, 8, 4, 96, dict(rope_base=10000.0, qk_norm=True)),
    (3, 1000, 4, 6, 3, 128, dict(rope_base=10000.0, qk_norm=True, softcap=50.0)),
    (2, 777, 2, 8, 1, 64, dict(window=200)),
    (1, 2049, 16, 4, 4, 96, dict(qk_norm=True)),
    (2, 513, 3, 4, 2, 32, dict(causal=False, window=100)),
    (1, 640, 8, 2, 1, 128, dict(softcap=5.0, scale=0.05)),
    (2, 100000, 1, 8, 4, 96, dict(rope_base=10000.0, qk_norm=True)),  # RoPE at positions near 1e5
    # several blocks of adjacent kv heads per token (4 + 4, and 2 + 2 + 2)
    (2, 700, 1, 16, 8, 64, dict(rope_base=10000.0, qk_norm=True)),
    (1, 301, 2, 12, 6, 32, dict(window=150)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}Tk{c[1]}Tq{c[2]}H{c[3]}x{c[4]}D{c[5]}"
                         + "".join(f"-{k}{v}" for k, v in c[6].items()))
def test_decode_matches_oracle(csa, ora, case):
    B, Tk, Tq, Hq, Hkv, D, opts = case
    w = DecodeWorkload("t", B=B, Tk=Tk, Tq=Tq, Hq=Hq, Hkv=Hkv, D=D, seed=3 + Tk + D, **opts)
    run_case(csa, ora, w)


def test_decode_workload_full_size_sampled_rows(csa, ora):
    """The benchmarked decode step at full size; oracle on the first and last batch rows."""
    w = DECODE_WORKLOADS[0]
    for b in (0, w.B - 1):
        run_case(csa, ora, w, rows=slice(b, b + 1))


def test_decode_new_query_ignores_cache_entries_it_cannot_see(csa):
    """Causal window: changing cache entries outside every query's window leaves O and LSE
    bit-identical (the masked keys contribute nothing, not even through the key-range merge)."""
    w = DecodeWorkload("t", B=1, Tk=1500, Tq=2, Hq=4, Hkv=2, D=64, window=300, seed=11)
    inp = make_decode_inputs(w)
    dev = torch.device("cuda:0")
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    o1, l1 = csa.attn_decode(q, kc, vc, **w.options())
    kc2, vc2 = kc.clone(), vc.clone()
    cut = w.Tk - w.Tq - w.window + 1  # first key any of the new queries can see
    kc2[:, :cut] = -kc2[:, :cut]
    vc2[:, :cut] = 3 * vc2[:, :cut]
    o2, l2 = csa.attn_decode(q, kc2, vc2, **w.options())
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
