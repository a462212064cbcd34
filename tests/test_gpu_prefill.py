"""Forward over a key/value cache (csa_attn_prefill: a chunk of Tq new queries at the last Tq
positions, on the tensor-core forward) against the fp64 oracle's cached attention, on the same
seeded bf16 inputs and with the forward's tolerances (O relative L2 <= 1e-2, max-abs <= 2e-2;
LSE max-abs <= 1e-2).  Plus the wiring check that a chunk covering the whole cache, without
norm or RoPE, is bit-identical to csa_attn_fwd on the same tensors."""
import numpy as np
import pytest
import torch

from causal_self_attention_gqa_b200.workloads import DecodeWorkload, make_decode_inputs

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


CASES = [
    # (B, Tk, Tq, Hq, Hkv, D, options)
    (2, 300, 300, 4, 2, 64, dict(rope_base=10000.0, qk_norm=True)),
    (1, 1000, 129, 8, 4, 96, dict(rope_base=10000.0, qk_norm=True)),
    (2, 2048, 512, 6, 3, 128, dict(rope_base=10000.0, qk_norm=True, softcap=50.0)),
    (1, 777, 100, 4, 1, 32, dict(window=64)),
    (1, 640, 200, 2, 2, 96, dict(causal=False, window=100)),
    (1, 4096, 1, 8, 4, 96, dict(qk_norm=True)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}Tk{c[1]}Tq{c[2]}H{c[3]}x{c[4]}D{c[5]}"
                         + "".join(f"-{k}{v}" for k, v in c[6].items()))
def test_prefill_matches_oracle(csa, ora, case):
    B, Tk, Tq, Hq, Hkv, D, opts = case
    w = DecodeWorkload("t", B=B, Tk=Tk, Tq=Tq, Hq=Hq, Hkv=Hkv, D=D, seed=5 + Tk + Tq, **opts)
    inp = make_decode_inputs(w)
    dev = torch.device("cuda:0")
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    o, lse = csa.attn_prefill(q, kc, vc, **w.options())
    torch.cuda.synchronize()
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    ref_o, ref_lse = ora.attn_fwd_cached(inp["q"], inp["k_cache"], inp["v_cache"], **w.options())
    assert np.all(np.isfinite(o))
    r = float(np.linalg.norm(o - ref_o) / np.linalg.norm(ref_o))
    m = float(np.max(np.abs(o - ref_o)))
    assert r <= O_REL and m <= O_ABS, (r, m)
    assert float(np.max(np.abs(lse - ref_lse))) <= LSE_ABS


def test_whole_cache_chunk_equals_the_forward(csa):
    w = DecodeWorkload("t", B=2, Tk=520, Tq=520, Hq=4, Hkv=2, D=96, window=300, seed=17)
    inp = make_decode_inputs(w)
    dev = torch.device("cuda:0")
    q, kc, vc = (inp[n].to(dev) for n in ("q", "k_cache", "v_cache"))
    o1, l1 = csa.attn_prefill(q, kc, vc, **w.options())
    o2, l2 = csa.attn_fwd(q, kc, vc, **w.options())
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
