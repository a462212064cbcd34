"""Pins of the fp64 oracle against things other than itself (CPU only).

* Library routines: torch's scaled_dot_product_attention (fp64, CPU) with its own
  causal / GQA handling, torch's rms_norm, RoPE written as a complex rotation, and torch
  autograd for every gradient -- an implementation that shares nothing with oracle.c.
* Finite differences of L = sum(O * dO) for every option, soft-capping included.
* Closed forms: a two-token soft-capped example worked by hand; Q = 0 gives the mean of
  the visible values.
* Invariants the pages imply: softmax rows sum to 1, position 0 returns V[0], future
  tokens and other packed documents do not change an output, a packed row equals its
  documents run alone with positions from 0, RoPE preserves norms and only sees relative
  positions, grouped-query attention equals multi-head attention with repeated K/V.
"""
import os
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from causal_self_attention_gqa_b200.workloads import packed_segment_ids

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _segments_brute(ids):
    B, T = ids.shape
    st = np.zeros((B, T), np.int64)
    en = np.zeros((B, T), np.int64)
    for b in range(B):
        for t in range(T):
            s = t
            while s > 0 and ids[b, s - 1] == ids[b, t]:
                s -= 1
            e = t
            while e + 1 < T and ids[b, e + 1] == ids[b, t]:
                e += 1
            st[b, t], en[b, t] = s, e + 1
    return st, en


def _lib_attention(q, k, v, *, causal=True, window=0, rope_base=0.0, qk_norm=False,
                   qk_norm_eps=1e-6, scale=0.0, segment_ids=None):
    """Library composition: rms_norm -> complex-rotation RoPE -> SDPA with a boolean mask."""
    B, T, Hq, D = q.shape
    if segment_ids is not None:
        st, en = _segments_brute(np.asarray(segment_ids))
    else:
        st, en = np.zeros((B, T), np.int64), np.full((B, T), T, np.int64)
    st_t, en_t = torch.from_numpy(st), torch.from_numpy(en)
    if qk_norm:
        q = F.rms_norm(q, (D,), eps=qk_norm_eps)
        k = F.rms_norm(k, (D,), eps=qk_norm_eps)
    if rope_base > 0:
        pos = (torch.arange(T)[None, :] - st_t).double()                   # [B, T]
        freqs = rope_base ** (-torch.arange(0, D, 2, dtype=torch.float64) / D)
        rot = torch.polar(torch.ones(B, T, D // 2, dtype=torch.float64),
                          pos[..., None] * freqs)[:, :, None, :]            # [B, T, 1, D/2]

        def rope(x):
            z = torch.complex(x[..., : D // 2], x[..., D // 2:]) * rot
            return torch.cat([z.real, z.imag], dim=-1)
        q, k = rope(q), rope(k)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = torch.ones(B, T, T, dtype=torch.bool)
    if causal:
        mask &= (j <= i)[None]
    if window > 0:
        mask &= ((i - j) < window)[None]
        if not causal:
            mask &= ((j - i) < window)[None]
    mask &= (j[None] >= st_t[:, :, None]) & (j[None] < en_t[:, :, None])
    sc = scale if scale > 0 else 1.0 / math.sqrt(D)
    o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
                                       attn_mask=mask[:, None], scale=sc, enable_gqa=True)
    G = Hq // k.shape[2]
    kr = k.repeat_interleave(G, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, kr) * sc
    s = s.masked_fill(~mask[:, None], float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.transpose(1, 2), lse


OPTION_SETS = [
    dict(),
    dict(rope_base=10000.0),
    dict(qk_norm=True),
    dict(rope_base=10000.0, qk_norm=True),
    dict(window=3),
    dict(causal=False),
    dict(causal=False, window=2),
    dict(segments=True),
    dict(segments=True, rope_base=500.0, qk_norm=True, window=4),
    dict(segments=True, causal=False, rope_base=10000.0),
    dict(scale=0.3),
]


def _opts(o):
    o = dict(o)
    seg = o.pop("segments", False)
    return o, seg


@pytest.mark.parametrize("opts", OPTION_SETS, ids=lambda o: ",".join(f"{k}={v}" for k, v in o.items()) or "plain")
@pytest.mark.parametrize("heads", [(3, 3), (4, 2), (6, 2)])
def test_forward_and_grads_match_library_composition(oracle_mod, opts, heads):
    Hq, Hkv = heads
    B, T, D = 2, 11, 8
    o, seg = _opts(opts)
    q, k, v, do = (_rand((B, T, Hq, D), 1), _rand((B, T, Hkv, D), 2), _rand((B, T, Hkv, D), 3),
                   _rand((B, T, Hq, D), 4))
    ids = packed_segment_ids(B, T, 2, 5, 7) if seg else None
    O, L = oracle_mod.attn_fwd(q, k, v, segment_ids=ids, **o)
    qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
    O_ref, L_ref = _lib_attention(qq, kk, vv, segment_ids=ids, **o)
    np.testing.assert_allclose(O, O_ref.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, L_ref.detach().numpy(), rtol=0, atol=1e-12)
    (O_ref * do).sum().backward()
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, segment_ids=ids, **o)
    for a, r in ((dq, qq.grad), (dk, kk.grad), (dv, vv.grad)):
        np.testing.assert_allclose(a, r.numpy(), rtol=0, atol=1e-11)


FD_SETS = OPTION_SETS + [dict(softcap=1.5), dict(softcap=2.0, rope_base=100.0, qk_norm=True, window=3,
                                                  segments=True)]


@pytest.mark.parametrize("opts", FD_SETS, ids=lambda o: ",".join(f"{k}={v}" for k, v in o.items()) or "plain")
def test_gradients_match_finite_differences(oracle_mod, opts):
    B, T, Hq, Hkv, D = 1, 7, 4, 2, 6
    o, seg = _opts(opts)
    q, k, v, do = (_rand((B, T, Hq, D), 11).numpy(), _rand((B, T, Hkv, D), 12).numpy(),
                   _rand((B, T, Hkv, D), 13).numpy(), _rand((B, T, Hq, D), 14).numpy())
    ids = packed_segment_ids(B, T, 2, 4, 3) if seg else None
    an = oracle_mod.attn_bwd(q, k, v, do, segment_ids=ids, **o)

    def loss(q_, k_, v_):
        return float((oracle_mod.attn_fwd(q_, k_, v_, segment_ids=ids, **o)[0] * do).sum())

    h = 1e-6
    args = [q, k, v]
    for which in range(3):
        fd = np.zeros_like(args[which])
        it = np.nditer(args[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        err = np.linalg.norm(fd - an[which]) / max(np.linalg.norm(an[which]), 1e-30)
        assert err < 1e-6, (which, err)


def test_softcap_two_token_closed_form(oracle_mod):
    """T=2, one head, D=2, no norm/RoPE, cap c=2, scale 1 -- worked by hand."""
    q = np.array([[[[1.0, 2.0]], [[3.0, -1.0]]]])
    k = np.array([[[[0.5, 1.0]], [[2.0, 0.5]]]])
    v = np.array([[[[1.0, -2.0]], [[4.0, 3.0]]]])
    c = 2.0
    # raw scores: s00 = 0.5+2 = 2.5; s10 = 1.5-1 = 0.5; s11 = 6-0.5 = 5.5
    s00, s10, s11 = (c * math.tanh(x / c) for x in (2.5, 0.5, 5.5))
    w0, w1 = math.exp(s10), math.exp(s11)
    o1 = [(w0 * 1.0 + w1 * 4.0) / (w0 + w1), (w0 * -2.0 + w1 * 3.0) / (w0 + w1)]
    O, L = oracle_mod.attn_fwd(q, k, v, softcap=c, scale=1.0)
    np.testing.assert_allclose(O[0, 0, 0], [1.0, -2.0], atol=1e-15)
    np.testing.assert_allclose(O[0, 1, 0], o1, atol=1e-14)
    np.testing.assert_allclose(L[0, 0], [s00, math.log(w0 + w1)], atol=1e-14)


def test_softcap_limits(oracle_mod):
    B, T, H, D = 1, 9, 2, 8
    q, k, v = _rand((B, T, H, D), 21) * 3, _rand((B, T, H, D), 22) * 3, _rand((B, T, H, D), 23)
    O0, L0 = oracle_mod.attn_fwd(q, k, v)
    O1, L1 = oracle_mod.attn_fwd(q, k, v, softcap=1e9)
    np.testing.assert_allclose(O1, O0, atol=1e-9)
    # a small cap bounds every logit: |LSE_i - log(#visible)| <= c
    c = 0.25
    _, Lc = oracle_mod.attn_fwd(q, k, v, softcap=c)
    nvis = np.arange(1, T + 1)
    assert np.all(np.abs(Lc - np.log(nvis)[None, None, :]) <= c + 1e-12)


@pytest.mark.parametrize("opts", OPTION_SETS + [dict(softcap=3.0)],
                         ids=lambda o: ",".join(f"{k}={v}" for k, v in o.items()) or "plain")
def test_rows_sum_to_one_and_masked_entries_are_zero(oracle_mod, opts):
    B, T, Hq, Hkv, D = 2, 13, 4, 2, 8
    o, seg = _opts(opts)
    q, k = _rand((B, T, Hq, D), 31), _rand((B, T, Hkv, D), 32)
    ids = packed_segment_ids(B, T, 2, 6, 5) if seg else None
    for b, h in [(0, 0), (1, 3)]:
        P = oracle_mod.attn_probs(q, k, b, h, segment_ids=ids, **o)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
        if o.get("causal", True):
            assert np.all(np.triu(P, 1) == 0.0)


def test_first_position_returns_its_own_value(oracle_mod):
    B, T, Hq, Hkv, D = 2, 10, 6, 3, 8
    q, k, v = _rand((B, T, Hq, D), 41), _rand((B, T, Hkv, D), 42), _rand((B, T, Hkv, D), 43)
    ids = packed_segment_ids(B, T, 2, 5, 9)
    for kw in (dict(), dict(rope_base=10000.0, qk_norm=True, softcap=5.0)):
        O, _ = oracle_mod.attn_fwd(q, k, v, **kw)
        for h in range(Hq):
            np.testing.assert_array_equal(O[:, 0, h], v[:, 0, h // 2].numpy())
        O, _ = oracle_mod.attn_fwd(q, k, v, segment_ids=ids, **kw)
        st, _ = oracle_mod.segments(ids)
        for b in range(B):
            for t in range(T):
                if st[b, t] == t:  # first token of a document attends only to itself
                    for h in range(Hq):
                        np.testing.assert_array_equal(O[b, t, h], v[b, t, h // 2].numpy())


def test_future_tokens_do_not_change_earlier_outputs(oracle_mod):
    B, T, Hq, Hkv, D = 1, 12, 4, 2, 8
    q, k, v = _rand((B, T, Hq, D), 51), _rand((B, T, Hkv, D), 52), _rand((B, T, Hkv, D), 53)
    kw = dict(rope_base=10000.0, qk_norm=True, softcap=4.0, window=5)
    O, L = oracle_mod.attn_fwd(q, k, v, **kw)
    cut = 7
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, cut:] = _rand((B, T - cut, Hq, D), 54)
    k2[:, cut:] = _rand((B, T - cut, Hkv, D), 55)
    v2[:, cut:] = _rand((B, T - cut, Hkv, D), 56)
    O2, L2 = oracle_mod.attn_fwd(q2, k2, v2, **kw)
    np.testing.assert_array_equal(O2[:, :cut], O[:, :cut])
    np.testing.assert_array_equal(L2[:, :, :cut], L[:, :, :cut])
    assert not np.allclose(O2[:, cut:], O[:, cut:])


def test_packed_row_equals_documents_run_alone(oracle_mod):
    """Segment isolation and RoPE from in-segment positions: every document of a packed row
    gives the same outputs and gradients as that document alone at positions 0.."""
    B, T, Hq, Hkv, D = 1, 23, 4, 2, 8
    q, k, v, do = (_rand((B, T, Hq, D), 61), _rand((B, T, Hkv, D), 62), _rand((B, T, Hkv, D), 63),
                   _rand((B, T, Hq, D), 64))
    ids = packed_segment_ids(B, T, 3, 9, 2)
    kw = dict(rope_base=10000.0, qk_norm=True, softcap=6.0, window=4)
    O, L = oracle_mod.attn_fwd(q, k, v, segment_ids=ids, **kw)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, segment_ids=ids, **kw)
    for doc in np.unique(ids[0]):
        sel = np.nonzero(ids[0] == doc)[0]
        a, b = sel[0], sel[-1] + 1
        Od, Ld = oracle_mod.attn_fwd(q[:, a:b], k[:, a:b], v[:, a:b], **kw)
        np.testing.assert_allclose(O[:, a:b], Od, atol=1e-13)
        np.testing.assert_allclose(L[:, :, a:b], Ld, atol=1e-13)
        g = oracle_mod.attn_bwd(q[:, a:b], k[:, a:b], v[:, a:b], do[:, a:b], **kw)
        for full, part in zip((dq, dk, dv), g):
            np.testing.assert_allclose(full[:, a:b], part, atol=1e-12)


def test_other_documents_do_not_change_a_document(oracle_mod):
    B, T, Hq, Hkv, D = 1, 20, 2, 1, 8
    q, k, v = _rand((B, T, Hq, D), 71), _rand((B, T, Hkv, D), 72), _rand((B, T, Hkv, D), 73)
    ids = np.array([[0] * 6 + [1] * 9 + [2] * 5], dtype=np.int32)
    kw = dict(causal=False, rope_base=100.0, qk_norm=True)
    O, _ = oracle_mod.attn_fwd(q, k, v, segment_ids=ids, **kw)
    k2, v2 = k.clone(), v.clone()
    k2[:, :6], v2[:, :6] = _rand((B, 6, Hkv, D), 74), _rand((B, 6, Hkv, D), 75)
    k2[:, 15:], v2[:, 15:] = _rand((B, 5, Hkv, D), 76), _rand((B, 5, Hkv, D), 77)
    O2, _ = oracle_mod.attn_fwd(q, k2, v2, segment_ids=ids, **kw)
    np.testing.assert_array_equal(O2[:, 6:15], O[:, 6:15])


def test_rope_preserves_norm_and_sees_only_relative_positions(oracle_mod):
    B, T, H, D = 1, 16, 3, 8
    x = _rand((B, T, H, D), 81)
    y = oracle_mod.qk_prologue(x, rope_base=10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x.numpy(), axis=-1),
                               rtol=1e-14)
    # the same q/k vectors placed at every position: q'_i . k'_j depends on i - j only
    qv, kv_ = _rand((D,), 82), _rand((D,), 83)
    qt = qv.expand(B, T, 1, D).contiguous()
    kt = kv_.expand(B, T, 1, D).contiguous()
    qp = oracle_mod.qk_prologue(qt, rope_base=10000.0)[0, :, 0]
    kp = oracle_mod.qk_prologue(kt, rope_base=10000.0)[0, :, 0]
    S = qp @ kp.T
    for d in range(-T + 1, T):
        diag = np.diagonal(S, offset=d)
        np.testing.assert_allclose(diag, diag[0], rtol=1e-12, atol=1e-12)
    # position 0 is the identity rotation
    np.testing.assert_allclose(y[:, 0], x.numpy()[:, 0], atol=0)


def test_rope_matches_complex_rotation_and_norm_matches_library(oracle_mod):
    B, T, H, D = 2, 9, 2, 10
    x = _rand((B, T, H, D), 84)
    ids = packed_segment_ids(B, T, 2, 5, 1)
    y = oracle_mod.qk_prologue(x, rope_base=77.0, qk_norm=True, qk_norm_eps=1e-6, segment_ids=ids)
    st, _ = _segments_brute(ids)
    pos = np.arange(T)[None, :] - st
    xn = F.rms_norm(x, (D,), eps=1e-6).numpy()
    z = xn[..., : D // 2] + 1j * xn[..., D // 2:]
    ang = pos[:, :, None, None] * (77.0 ** (-np.arange(0, D, 2) / D))[None, None, None, :]
    zr = z * np.exp(1j * ang)
    ref = np.concatenate([zr.real, zr.imag], axis=-1)
    np.testing.assert_allclose(y, ref, atol=1e-14)
    # parameter-free RMSNorm: unit RMS up to eps, invariant to positive rescaling
    yn = oracle_mod.qk_prologue(x, qk_norm=True, qk_norm_eps=0.0)
    np.testing.assert_allclose(np.sqrt((yn ** 2).mean(-1)), 1.0, rtol=1e-14)
    yn2 = oracle_mod.qk_prologue(x * 37.5, qk_norm=True, qk_norm_eps=0.0)
    np.testing.assert_allclose(yn2, yn, rtol=1e-13)


@pytest.mark.parametrize("kw", [dict(), dict(window=3), dict(segments=True, window=5),
                                dict(causal=False, segments=True),
                                dict(rope_base=10000.0, qk_norm=True, softcap=2.0)])
def test_zero_queries_give_mean_of_visible_values(oracle_mod, kw):
    """Q = 0 makes every score 0 (RMSNorm of 0 is 0, RoPE of 0 is 0, cap of 0 is 0), so the
    softmax is uniform over the visible keys and O_i is their plain mean."""
    B, T, Hq, Hkv, D = 2, 14, 2, 1, 8
    kw, seg = _opts(kw)
    q = torch.zeros((B, T, Hq, D), dtype=torch.float64)
    k, v = _rand((B, T, Hkv, D), 91), _rand((B, T, Hkv, D), 92).numpy()
    ids = packed_segment_ids(B, T, 2, 6, 4) if seg else np.zeros((B, T), np.int32)
    O, L = oracle_mod.attn_fwd(q, k, v, segment_ids=ids, **kw)
    st, en = _segments_brute(ids)
    W = kw.get("window", 0)
    causal = kw.get("causal", True)
    for b in range(B):
        for i in range(T):
            lo, hi = st[b, i], (i + 1 if causal else en[b, i])
            if W:
                lo = max(lo, i - W + 1)
                if not causal:
                    hi = min(hi, i + W)
            ref = v[b, lo:hi, 0].mean(axis=0)
            for h in range(Hq):
                np.testing.assert_allclose(O[b, i, h], ref, atol=1e-14)
                assert abs(L[b, h, i] - math.log(hi - lo)) < 1e-14


def test_gqa_equals_mha_with_repeated_kv(oracle_mod):
    B, T, Hq, Hkv, D = 2, 10, 6, 2, 8
    q, k, v, do = (_rand((B, T, Hq, D), 101), _rand((B, T, Hkv, D), 102), _rand((B, T, Hkv, D), 103),
                   _rand((B, T, Hq, D), 104))
    kw = dict(rope_base=10000.0, qk_norm=True, softcap=5.0, window=4)
    G = Hq // Hkv
    kr, vr = k.repeat_interleave(G, dim=2), v.repeat_interleave(G, dim=2)
    O, L = oracle_mod.attn_fwd(q, k, v, **kw)
    Or, Lr = oracle_mod.attn_fwd(q, kr, vr, **kw)
    np.testing.assert_array_equal(O, Or)
    np.testing.assert_array_equal(L, Lr)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, **kw)
    dqr, dkr, dvr = oracle_mod.attn_bwd(q, kr, vr, do, **kw)
    np.testing.assert_allclose(dq, dqr, atol=1e-13)
    np.testing.assert_allclose(dk, dkr.reshape(B, T, Hkv, G, D).sum(3), atol=1e-12)
    np.testing.assert_allclose(dv, dvr.reshape(B, T, Hkv, G, D).sum(3), atol=1e-12)


def test_segments_are_maximal_runs(oracle_mod):
    rng = np.random.default_rng(0)
    for _ in range(20):
        ids = rng.integers(0, 3, size=(3, 17)).astype(np.int32)
        st, en = oracle_mod.segments(ids)
        bst, ben = _segments_brute(ids)
        np.testing.assert_array_equal(st, bst)
        np.testing.assert_array_equal(en, ben)


def test_packed_generator_shapes():
    ids = packed_segment_ids(8, 2048, 64, 768, 1004)
    for b in range(8):
        _, counts = np.unique(ids[b], return_counts=True)
        assert counts.sum() == 2048
        assert np.all(counts[:-1] >= 64) and np.all(counts <= 768)
        assert np.all(np.diff(ids[b]) >= 0)


def test_rejects_bad_head_ratio(oracle_mod):
    q, k = np.zeros((1, 2, 3, 4)), np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):
        oracle_mod.attn_fwd(q, k, k)


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["causal_mha_plain", "gqa_rope_qknorm_softcap", "packed_window"])
def test_oracle_reproduces_golden_fixture(oracle_mod, name):
    import json
    with open(os.path.join(GOLDEN, name + ".json")) as f:
        rec = json.load(f)
    arr = {k: np.array(rec[k]) for k in ("q", "k", "v", "do", "o", "lse", "dq", "dk", "dv")}
    seg = np.array(rec["segment_ids"], dtype=np.int32) if rec["segment_ids"] is not None else None
    o, lse = oracle_mod.attn_fwd(arr["q"], arr["k"], arr["v"], segment_ids=seg, **rec["options"])
    np.testing.assert_allclose(o, arr["o"], atol=1e-13)
    np.testing.assert_allclose(lse, arr["lse"], atol=1e-13)
    g = oracle_mod.attn_bwd(arr["q"], arr["k"], arr["v"], arr["do"], segment_ids=seg, **rec["options"])
    for got, key in zip(g, ("dq", "dk", "dv")):
        np.testing.assert_allclose(got, arr[key], atol=1e-12)
