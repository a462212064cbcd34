"""The C ABI without a GPU: the library loads, exports every entry point include/csa.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def b():
    from causal_self_attention_gqa_b200 import build
    build.build()
    from causal_self_attention_gqa_b200 import _binding
    return _binding


def _declared():
    text = open(os.path.join(ROOT, "include", "csa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("csa_attn_fwd", "csa_attn_bwd", "csa_workspace_size", "csa_device_status", "csa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(b):
    lib = ctypes.CDLL(b.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(b.EXPORTED) == _declared()


def test_workspace_size(b):
    p = b.make_params(2, 128, 6, 6, 32)
    f, w = b.workspace_size(p, False), b.workspace_size(p, True)
    assert 0 < f < w
    pr = b.make_params(2, 128, 6, 6, 32, rope_base=10000.0, qk_norm=True)
    assert b.workspace_size(pr, False) > f
    # backward adds delta [B,Hq,T] fp32 and the fp32 dQ accumulator [B,T,Hq,D]
    assert w - f >= 2 * 128 * 6 * 4 + 2 * 128 * 6 * 32 * 4
    for bad in (b.make_params(2, 128, 6, 4, 32), b.make_params(2, 128, 6, 6, 48),
                b.make_params(2, 128, 6, 6, 32, qk_norm=True, qk_norm_eps=0.0),
                b.make_params(-1, 128, 6, 6, 32), b.make_params(1, (1 << 20) + 1, 1, 1, 32),
                b.make_params(1024, 1 << 20, 1, 1, 32)):  # 2^31 rows: past the 31-bit row index
        assert b.workspace_size(bad, False) == 0


# The fake pointers below are never dereferenced: every call here fails a host-side check
# before anything is enqueued.  No call in this file passes all checks.
def _call_fwd(b, p, q=0x1000, k=0x2000, v=0x3000, seg=None, o=0x4000, lse=0x5000, ws=0x10000, nws=1 << 30):
    return b.lib.csa_attn_fwd(ctypes.byref(p), q, k, v, seg, o, lse, ws, nws, None)


def _call_bwd(b, p, ptrs=None, ws=0x10000, nws=1 << 30):
    q, k, v, o, do, lse, dq, dk, dv = ptrs or [0x1000 * (i + 1) for i in range(9)]
    return b.lib.csa_attn_bwd(ctypes.byref(p), q, k, v, o, do, lse, None, dq, dk, dv, ws, nws, None)


def test_invalid_arguments_are_rejected_before_any_device_work(b):
    good = b.make_params(2, 128, 6, 6, 32)
    assert _call_fwd(b, b.make_params(2, 128, 6, 4, 32)) == b.CSA_ERR_INVALID_ARG      # Hq % Hkv
    assert _call_fwd(b, b.make_params(2, 128, 6, 6, 40)) == b.CSA_ERR_INVALID_ARG      # head dim
    assert _call_fwd(b, b.make_params(2, 128, 6, 6, 32, causal=True, qk_norm=True,
                                      qk_norm_eps=-1.0)) == b.CSA_ERR_INVALID_ARG
    bad = b.make_params(2, 128, 6, 6, 32)
    bad.softcap = float("nan")
    assert _call_fwd(b, bad) == b.CSA_ERR_INVALID_ARG
    assert _call_fwd(b, good, q=None) == b.CSA_ERR_INVALID_ARG
    assert _call_fwd(b, good, ws=None) == b.CSA_ERR_INVALID_ARG
    assert _call_fwd(b, good, q=0x1008) == b.CSA_ERR_ALIGNMENT
    assert _call_fwd(b, good, ws=0x10080) == b.CSA_ERR_ALIGNMENT
    assert _call_fwd(b, good, nws=100) == b.CSA_ERR_WORKSPACE
    assert _call_bwd(b, b.make_params(2, 128, 6, 5, 32)) == b.CSA_ERR_INVALID_ARG
    # the reuse entry point runs the same host checks before touching the workspace
    q, k, v, o, do, lse, dq, dk, dv = [0x1000 * (i + 1) for i in range(9)]
    after = b.lib.csa_attn_bwd_after_fwd
    assert after(ctypes.byref(b.make_params(2, 128, 6, 5, 32)), q, k, v, o, do, lse, None, dq, dk, dv, 0x10000,
                 1 << 30, None) == b.CSA_ERR_INVALID_ARG
    assert after(ctypes.byref(good), q, k, v, o, do, lse, None, dq, dk, dv, 0x10001, 1 << 30,
                 None) == b.CSA_ERR_ALIGNMENT
    assert after(ctypes.byref(good), q, k, v, o, do, lse, None, dq, dk, dv, 0x10000, 16,
                 None) == b.CSA_ERR_WORKSPACE
    ptrs = [0x1000 * (i + 1) for i in range(9)]
    ptrs[4] = 0x5004  # dout misaligned
    assert _call_bwd(b, good, ptrs) == b.CSA_ERR_ALIGNMENT
    assert _call_bwd(b, good, nws=b.workspace_size(good, False)) == b.CSA_ERR_WORKSPACE


def test_empty_problem_is_a_no_op(b):
    assert _call_fwd(b, b.make_params(0, 128, 6, 6, 32), q=None, k=None, v=None, o=None, lse=None, ws=None) == 0
    assert _call_fwd(b, b.make_params(2, 0, 6, 6, 32), q=None, k=None, v=None, o=None, lse=None, ws=None) == 0


def test_status_strings(b):
    for code in range(9):
        assert b.status_string(code)
    assert b.status_string(6) == "a bounded wait inside a kernel ran out"
    assert b.kernel_names() == ["k_prep", "k_qk_prologue", "k_attn_fwd", "k_bwd_pre", "k_attn_bwd",
                                "k_grad_finalize", "k_decode", "k_gemm_qkv", "k_gemm_out", "k_gemm_dout",
                                "k_gemm_dwo", "k_gemm_dx", "k_gemm_dw"]


def test_projection_arguments_are_checked_on_the_host(b):
    """csa_qkv_proj / csa_out_proj / csa_out_proj_bwd / csa_qkv_proj_bwd: model width, piece
    alignment, pointers and workspace are rejected before anything is enqueued (fake
    pointers: every call here fails a check)."""
    lib = b.lib
    good = b.make_params(2, 128, 8, 4, 96)
    assert lib.csa_proj_workspace_size() == 256
    P = [0x1000 * (i + 1) for i in range(12)]
    ws = 0x100000

    def qkv(p, C, ptrs=P, w=ws, n=256):
        return lib.csa_qkv_proj(ctypes.byref(p), C, *ptrs[:7], w, n, None)

    assert qkv(good, 96) == b.CSA_ERR_INVALID_ARG        # C not a multiple of 64
    assert qkv(good, 0) == b.CSA_ERR_INVALID_ARG
    assert qkv(b.make_params(2, 128, 2, 1, 32), 128) == b.CSA_ERR_INVALID_ARG  # Hkv * D = 32
    assert qkv(b.make_params(2, 128, 6, 4, 64), 128) == b.CSA_ERR_INVALID_ARG  # Hq % Hkv != 0
    assert qkv(good, 768, w=None) == b.CSA_ERR_INVALID_ARG
    assert qkv(good, 768, w=ws + 16) == b.CSA_ERR_ALIGNMENT
    assert qkv(good, 768, n=128) == b.CSA_ERR_WORKSPACE
    bad = list(P)
    bad[3] = 0x4008  # wv misaligned
    assert qkv(good, 768, ptrs=bad) == b.CSA_ERR_ALIGNMENT
    bad[3] = 0
    assert qkv(good, 768, ptrs=bad) == b.CSA_ERR_INVALID_ARG
    assert lib.csa_out_proj(ctypes.byref(good), 100, *P[:3], ws, 256, None) == b.CSA_ERR_INVALID_ARG
    assert lib.csa_out_proj(ctypes.byref(good), 768, P[0], 0, P[2], ws, 256, None) == b.CSA_ERR_INVALID_ARG
    assert lib.csa_out_proj_bwd(ctypes.byref(good), 768, *P[:4], 0x5004, ws, 256, None) == b.CSA_ERR_ALIGNMENT
    assert lib.csa_qkv_proj_bwd(ctypes.byref(good), 768, *P[:8], P[8], 0, P[10], ws, 256,
                                None) == b.CSA_ERR_INVALID_ARG  # dwk missing while dwq is given


def test_decode_arguments_are_checked_on_the_host(b):
    """csa_attn_decode: Tq range, rows per KV head, alignment and workspace size are
    rejected before anything is enqueued (fake pointers: every call here fails a check)."""
    p = b.make_params(2, 64, 8, 4, 96, rope_base=10000.0, qk_norm=True)
    assert b.decode_workspace_size(p, 1) > 0
    assert b.decode_workspace_size(p, 0) == 0          # Tq < 1
    assert b.decode_workspace_size(p, 17) == 0         # Tq > 16
    assert b.decode_workspace_size(b.make_params(2, 4, 8, 4, 96), 5) == 0   # Tq > cache length
    assert b.decode_workspace_size(b.make_params(2, 64, 32, 1, 64), 1) == 0  # 32 rows per KV head
    dec = b.lib.csa_attn_decode
    ptr = [0x1000 * (i + 1) for i in range(6)]
    assert dec(ctypes.byref(p), 0, *ptr[:5], 0x10000, 1 << 30, None) == b.CSA_ERR_INVALID_ARG
    assert dec(ctypes.byref(b.make_params(2, 64, 32, 1, 64)), 1, *ptr[:5], 0x10000, 1 << 30,
               None) == b.CSA_ERR_NOT_IMPLEMENTED
    assert dec(ctypes.byref(p), 1, 0x1008, *ptr[1:5], 0x10000, 1 << 30, None) == b.CSA_ERR_ALIGNMENT
    assert dec(ctypes.byref(p), 1, *ptr[:5], 0x10000, 64, None) == b.CSA_ERR_WORKSPACE
    assert dec(ctypes.byref(p), 1, None, *ptr[1:5], 0x10000, 1 << 30, None) == b.CSA_ERR_INVALID_ARG


def test_prefill_arguments_are_checked_on_the_host(b):
    """csa_attn_prefill: the chunk length, alignment and workspace size are rejected before
    anything is enqueued (fake pointers: every call here fails a check)."""
    p = b.make_params(2, 512, 8, 4, 96, rope_base=10000.0, qk_norm=True)
    n = b.prefill_workspace_size(p, 128)
    assert n > 0
    # q' of the 128-token chunk (the RoPE angles are formed in the kernels, no table)
    assert n >= 2 * 128 * 8 * 96 * 2
    assert b.prefill_workspace_size(p, 0) == 0
    assert b.prefill_workspace_size(p, 513) == 0
    assert b.prefill_workspace_size(b.make_params(2, 512, 8, 4, 96), 128) < n  # no prologue
    pre = b.lib.csa_attn_prefill
    ptr = [0x1000 * (i + 1) for i in range(6)]
    assert pre(ctypes.byref(p), 513, *ptr[:5], 0x10000, 1 << 30, None) == b.CSA_ERR_INVALID_ARG
    assert pre(ctypes.byref(p), 128, *ptr[:4], 0x5002, 0x10000, 1 << 30, None) == b.CSA_ERR_ALIGNMENT
    assert pre(ctypes.byref(p), 128, *ptr[:5], 0x10000, n - 1, None) == b.CSA_ERR_WORKSPACE
    assert pre(ctypes.byref(p), 128, *ptr[:4], None, 0x10000, 1 << 30, None) == b.CSA_ERR_INVALID_ARG
