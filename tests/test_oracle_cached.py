"""Pins of the oracle's KV-cache attention (oracle_attn_fwd_cached), following the
GPT-pretraining post (dekermanjian.github.io, llm_gpt_pretrain), section "Bonus: KV Caching":
Tq new queries at absolute positions offset + i, offset = Tk - Tq, over the cached keys and
values; a key j is visible to query i when j <= offset + i.

The cached computation takes its keys already normalised and rotated (as the prologue stores
them) and applies the norm and RoPE to the queries at their absolute positions.  It must give
exactly what the full-sequence forward gives for the last Tq rows: that forward is pinned
elsewhere against a library composition and finite differences, and it recomputes k' from the
raw keys itself, so agreement checks the offset, the positions and the mask of the cached path.
"""
import numpy as np
import pytest
import torch

OPTION_SETS = [
    dict(),
    dict(rope_base=10000.0),
    dict(qk_norm=True),
    dict(rope_base=10000.0, qk_norm=True, softcap=2.0),
    dict(window=4),
    dict(rope_base=500.0, qk_norm=True, window=3),
    dict(causal=False),
    dict(causal=False, window=3),
    dict(scale=0.3),
]


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64).numpy()


def _full(oracle_mod, q, k, v, kw):
    return oracle_mod.attn_fwd(q, k, v, **kw)


@pytest.mark.parametrize("opts", OPTION_SETS, ids=lambda o: ",".join(f"{k}={v}" for k, v in o.items()) or "plain")
@pytest.mark.parametrize("heads", [(2, 2), (4, 2), (6, 2)])
@pytest.mark.parametrize("tq", [1, 3, 13])
def test_cached_equals_last_rows_of_full_forward(oracle_mod, opts, heads, tq):
    Hq, Hkv = heads
    B, T, D = 2, 13, 8
    q, k, v = _rand((B, T, Hq, D), 1), _rand((B, T, Hkv, D), 2), _rand((B, T, Hkv, D), 3)
    o_full, lse_full = _full(oracle_mod, q, k, v, opts)
    kc = oracle_mod.qk_prologue(k, rope_base=opts.get("rope_base", 0.0), qk_norm=opts.get("qk_norm", False))
    o, lse = oracle_mod.attn_fwd_cached(q[:, T - tq:], kc, v, **opts)
    np.testing.assert_allclose(o, o_full[:, T - tq:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_full[:, :, T - tq:], rtol=0, atol=1e-12)


def test_window_of_one_returns_the_newest_value(oracle_mod):
    """Causal window 1: the single new query sees only its own (newest) cache entry."""
    B, Tk, Hq, Hkv, D = 2, 9, 4, 2, 8
    q, kc, vc = _rand((B, 1, Hq, D), 4), _rand((B, Tk, Hkv, D), 5), _rand((B, Tk, Hkv, D), 6)
    o, _ = oracle_mod.attn_fwd_cached(q, kc, vc, window=1)
    for h in range(Hq):
        np.testing.assert_allclose(o[:, 0, h], vc[:, Tk - 1, h // 2], rtol=0, atol=1e-15)


def test_zero_query_gives_mean_of_visible_values(oracle_mod):
    """q = 0 gives equal scores, so each new query averages the values it may see."""
    B, Tk, Tq, Hq, Hkv, D, W = 1, 10, 3, 2, 1, 8, 4
    q = np.zeros((B, Tq, Hq, D))
    kc, vc = _rand((B, Tk, Hkv, D), 7), _rand((B, Tk, Hkv, D), 8)
    o, lse = oracle_mod.attn_fwd_cached(q, kc, vc, window=W)
    for i in range(Tq):
        pos = Tk - Tq + i
        lo = pos - W + 1
        np.testing.assert_allclose(o[0, i, 0], vc[0, lo:pos + 1, 0].mean(axis=0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0, i], np.log(W), rtol=0, atol=1e-14)


def test_rejects_more_queries_than_cache(oracle_mod):
    q, kc = _rand((1, 5, 2, 8), 9), _rand((1, 4, 2, 8), 10)
    with pytest.raises(ValueError):
        oracle_mod.attn_fwd_cached(q, kc, kc)
