"""fp64 CPU oracle for causal self-attention (MHA / GQA), forward and backward.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` are the only callers; the product path never imports this package.
It shares no code with the CUDA path: the arithmetic lives in ``oracle.c`` (plain C,
fp64, one full T x T score matrix per (batch, head)), and this module only marshals
numpy arrays into it.

Every function follows the definitions cited at the top of ``oracle.c``: the scaled
dot-product attention equation and the causal mask of the GPT-pretraining page
(section "Multihead Attention"), grouped-query heads, QK-RMSNorm, RoPE from packed
segment positions and score soft-capping from the nanogpt-jax-181m model card
("Architecture"), and the sliding window from the flaxchat README ("Core Features").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no fast-math, no FMA contraction).

    ``ORACLE_LIB`` in the environment names a prebuilt library to load instead; the
    mutation tests use it to check that the pins reject deliberately broken copies."""
    override = os.environ.get("ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
             "-Wall", "-Wextra", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("D", ctypes.c_int), ("causal", ctypes.c_int),
                ("window", ctypes.c_int), ("softcap", ctypes.c_double),
                ("rope_base", ctypes.c_double), ("qk_norm", ctypes.c_int),
                ("qk_norm_eps", ctypes.c_double), ("scale", ctypes.c_double)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        pp = ctypes.POINTER(_Params)
        lib.oracle_attn_fwd.argtypes = [pp, dp, dp, dp, ip, dp, dp]
        lib.oracle_attn_bwd.argtypes = [pp, dp, dp, dp, dp, ip, dp, dp, dp]
        lib.oracle_qk_prologue.argtypes = [pp, ctypes.c_int, dp, ip, dp]
        lib.oracle_attn_probs.argtypes = [pp, dp, dp, ip, ctypes.c_int, ctypes.c_int, dp]
        lib.oracle_attn_fwd_cached.argtypes = [pp, ctypes.c_int, dp, dp, dp, dp, dp]
        lib.oracle_segments.argtypes = [ctypes.c_int, ctypes.c_int, ip, ip, ip]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (any dtype, any device)
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _seg(seg, B, T):
    if seg is None:
        return None, None
    if hasattr(seg, "detach"):
        seg = seg.detach().to("cpu").numpy()
    s = np.ascontiguousarray(seg, dtype=np.int32)
    assert s.shape == (B, T), s.shape
    return s, s.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _params(B, T, Hq, Hkv, D, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale):
    return _Params(B, T, Hq, Hkv, D, int(bool(causal)), int(window), float(softcap),
                   float(rope_base), int(bool(qk_norm)), float(qk_norm_eps), float(scale))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def attn_fwd(q, k, v, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
             qk_norm_eps=1e-6, scale=0.0, segment_ids=None):
    """O [B,T,Hq,D] and LSE [B,Hq,T] (natural log) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    assert k.shape == (B, T, Hkv, D) and v.shape == k.shape
    s, sp = _seg(segment_ids, B, T)
    p = _params(B, T, Hq, Hkv, D, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, T), dtype=np.float64)
    rc = _load().oracle_attn_fwd(ctypes.byref(p), _dptr(q), _dptr(k), _dptr(v), sp, _dptr(o), _dptr(lse))
    if rc:
        raise ValueError("oracle_attn_fwd rejected its arguments")
    return o, lse


def attn_bwd(q, k, v, dout, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
             qk_norm_eps=1e-6, scale=0.0, segment_ids=None):
    """dQ, dK, dV (gradients of sum(O * dO) w.r.t. the raw q, k, v) in fp64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    assert dout.shape == q.shape
    s, sp = _seg(segment_ids, B, T)
    p = _params(B, T, Hq, Hkv, D, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    rc = _load().oracle_attn_bwd(ctypes.byref(p), _dptr(q), _dptr(k), _dptr(v), _dptr(dout), sp,
                                 _dptr(dq), _dptr(dk), _dptr(dv))
    if rc:
        raise ValueError("oracle_attn_bwd rejected its arguments")
    return dq, dk, dv


def attn_fwd_cached(q, k_cache, v_cache, *, causal=True, window=0, softcap=0.0, rope_base=0.0,
                    qk_norm=False, qk_norm_eps=1e-6, scale=0.0):
    """Tq new (raw) queries over a cache of Tk keys (already normalised and rotated, as the
    prologue stores them) and values: O [B,Tq,Hq,D], LSE [B,Hq,Tq], fp64.  Query i sits at
    absolute position Tk - Tq + i."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Tq, Hq, D = q.shape
    Tk, Hkv = kc.shape[1], kc.shape[2]
    assert kc.shape == (B, Tk, Hkv, D) and vc.shape == kc.shape
    p = _params(B, Tk, Hq, Hkv, D, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Tq), dtype=np.float64)
    rc = _load().oracle_attn_fwd_cached(ctypes.byref(p), int(Tq), _dptr(q), _dptr(kc), _dptr(vc), _dptr(o),
                                        _dptr(lse))
    if rc:
        raise ValueError("oracle_attn_fwd_cached rejected its arguments")
    return o, lse


def qk_prologue(x, *, rope_base=0.0, qk_norm=False, qk_norm_eps=1e-6, segment_ids=None):
    """The normalised and rotated copy (Q' or K') of a [B,T,H,D] tensor, fp64."""
    x = _f64(x)
    B, T, H, D = x.shape
    s, sp = _seg(segment_ids, B, T)
    p = _params(B, T, H, H, D, True, 0, 0.0, rope_base, qk_norm, qk_norm_eps, 0.0)
    y = np.zeros_like(x)
    _load().oracle_qk_prologue(ctypes.byref(p), H, _dptr(x), sp, _dptr(y))
    return y


def attn_probs(q, k, b, h, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
               qk_norm_eps=1e-6, scale=0.0, segment_ids=None):
    """The T x T attention-probability matrix of batch row b, query head h (fp64)."""
    q, k = _f64(q), _f64(k)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    s, sp = _seg(segment_ids, B, T)
    p = _params(B, T, Hq, Hkv, D, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale)
    P = np.zeros((T, T), dtype=np.float64)
    _load().oracle_attn_probs(ctypes.byref(p), _dptr(q), _dptr(k), sp, int(b), int(h), _dptr(P))
    return P


def segments(segment_ids):
    """(start, end) int32 [B,T]: the maximal run of equal ids containing each token."""
    s = np.ascontiguousarray(segment_ids, dtype=np.int32)
    B, T = s.shape
    st = np.zeros((B, T), dtype=np.int32)
    en = np.zeros((B, T), dtype=np.int32)
    ip = ctypes.POINTER(ctypes.c_int32)
    _load().oracle_segments(B, T, s.ctypes.data_as(ip), st.ctypes.data_as(ip), en.ctypes.data_as(ip))
    return st, en
