"""ctypes binding of libcsa.so (include/csa.h).  Argument marshalling only: every step of
the attention runs in the library's CUDA kernels; torch provides device memory and the
current stream.  Importing this module fails loudly when the library is missing."""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m causal_self_attention_gqa_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

CSA_OK = 0
CSA_ERR_INVALID_ARG = 1
CSA_ERR_ALIGNMENT = 2
CSA_ERR_WORKSPACE = 3
CSA_ERR_ARCH = 4
CSA_ERR_LAUNCH = 5
CSA_ERR_DEVICE_TIMEOUT = 6
CSA_ERR_CUDA = 7
CSA_ERR_NOT_IMPLEMENTED = 8

# every entry point include/csa.h declares
EXPORTED = ["csa_workspace_size", "csa_attn_fwd", "csa_attn_bwd", "csa_device_status",
            "csa_status_string", "csa_timing_enable", "csa_timing_collect", "csa_num_kernels",
            "csa_kernel_name", "csa_attn_fwd_static_scratch", "csa_selftest_bounded_wait",
            "csa_attn_bwd_after_fwd", "csa_decode_workspace_size", "csa_attn_decode",
            "csa_prefill_workspace_size", "csa_attn_prefill", "csa_proj_workspace_size", "csa_qkv_proj",
            "csa_out_proj", "csa_out_proj_bwd", "csa_qkv_proj_bwd"]


class Params(ctypes.Structure):
    """Mirror of csa_params."""
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("causal", ctypes.c_int), ("window", ctypes.c_int),
                ("softcap", ctypes.c_float), ("rope_base", ctypes.c_float), ("qk_norm", ctypes.c_int),
                ("qk_norm_eps", ctypes.c_float), ("scale", ctypes.c_float)]


_vp = ctypes.c_void_p
_lib.csa_workspace_size.argtypes = [ctypes.POINTER(Params), ctypes.c_int]
_lib.csa_workspace_size.restype = ctypes.c_size_t
_lib.csa_attn_fwd.argtypes = [ctypes.POINTER(Params), _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.csa_attn_fwd.restype = ctypes.c_int
_lib.csa_attn_bwd.argtypes = [ctypes.POINTER(Params), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                              ctypes.c_size_t, _vp]
_lib.csa_attn_bwd.restype = ctypes.c_int
_lib.csa_attn_bwd_after_fwd.argtypes = [ctypes.POINTER(Params), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp, ctypes.c_size_t, _vp]
_lib.csa_attn_bwd_after_fwd.restype = ctypes.c_int
_lib.csa_prefill_workspace_size.argtypes = [ctypes.POINTER(Params), ctypes.c_int]
_lib.csa_prefill_workspace_size.restype = ctypes.c_size_t
_lib.csa_attn_prefill.argtypes = [ctypes.POINTER(Params), ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                  _vp]
_lib.csa_attn_prefill.restype = ctypes.c_int
_lib.csa_decode_workspace_size.argtypes = [ctypes.POINTER(Params), ctypes.c_int]
_lib.csa_decode_workspace_size.restype = ctypes.c_size_t
_lib.csa_attn_decode.argtypes = [ctypes.POINTER(Params), ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                 _vp]
_lib.csa_attn_decode.restype = ctypes.c_int
_lib.csa_attn_fwd_static_scratch.argtypes = [ctypes.POINTER(Params), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.csa_attn_fwd_static_scratch.restype = ctypes.c_int
_lib.csa_proj_workspace_size.argtypes = []
_lib.csa_proj_workspace_size.restype = ctypes.c_size_t
_lib.csa_qkv_proj.argtypes = [ctypes.POINTER(Params), ctypes.c_int] + [_vp] * 8 + [ctypes.c_size_t, _vp]
_lib.csa_qkv_proj.restype = ctypes.c_int
_lib.csa_out_proj.argtypes = [ctypes.POINTER(Params), ctypes.c_int] + [_vp] * 4 + [ctypes.c_size_t, _vp]
_lib.csa_out_proj.restype = ctypes.c_int
_lib.csa_out_proj_bwd.argtypes = [ctypes.POINTER(Params), ctypes.c_int] + [_vp] * 6 + [ctypes.c_size_t, _vp]
_lib.csa_out_proj_bwd.restype = ctypes.c_int
_lib.csa_qkv_proj_bwd.argtypes = [ctypes.POINTER(Params), ctypes.c_int] + [_vp] * 12 + [ctypes.c_size_t, _vp]
_lib.csa_qkv_proj_bwd.restype = ctypes.c_int
_lib.csa_selftest_bounded_wait.argtypes = [_vp, ctypes.c_size_t, _vp]
_lib.csa_selftest_bounded_wait.restype = ctypes.c_int
_lib.csa_device_status.argtypes = [_vp, _vp]
_lib.csa_device_status.restype = ctypes.c_int
_lib.csa_status_string.argtypes = [ctypes.c_int]
_lib.csa_status_string.restype = ctypes.c_char_p
_lib.csa_timing_enable.argtypes = [ctypes.c_int]
_lib.csa_timing_enable.restype = ctypes.c_int
_lib.csa_timing_collect.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int), ctypes.c_int]
_lib.csa_timing_collect.restype = ctypes.c_int
_lib.csa_num_kernels.argtypes = []
_lib.csa_num_kernels.restype = ctypes.c_int
_lib.csa_kernel_name.argtypes = [ctypes.c_int]
_lib.csa_kernel_name.restype = ctypes.c_char_p

lib = _lib


class CsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} (code {code})")
        self.code = code


def status_string(code: int) -> str:
    return _lib.csa_status_string(int(code)).decode()


def make_params(B, T, Hq, Hkv, D, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
                qk_norm_eps=1e-6, scale=0.0) -> Params:
    return Params(int(B), int(T), int(Hq), int(Hkv), int(D), int(bool(causal)), int(window), float(softcap),
                  float(rope_base), int(bool(qk_norm)), float(qk_norm_eps), float(scale))


def workspace_size(params: Params, backward: bool) -> int:
    return int(_lib.csa_workspace_size(ctypes.byref(params), int(bool(backward))))


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check_bf16(name, t, shape):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _opts_params(q, k, opts) -> Params:
    B, T, Hq, D = q.shape
    return make_params(B, T, Hq, k.shape[2], D, **opts)


def _seg(segment_ids, B, T):
    if segment_ids is None:
        return None
    if not (segment_ids.is_cuda and segment_ids.dtype == torch.int32 and segment_ids.is_contiguous()
            and tuple(segment_ids.shape) == (B, T)):
        raise ValueError("segment_ids must be a contiguous CUDA int32 tensor of shape (B, T)")
    return segment_ids


def workspace_for(q, k, backward: bool, **opts) -> torch.Tensor:
    """A workspace tensor (uint8, on q's device) big enough for the call."""
    n = workspace_size(_opts_params(q, k, opts), backward)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def attn_fwd(q, k, v, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False, qk_norm_eps=1e-6,
             scale=0.0, segment_ids=None, out=None, lse=None, workspace=None, stream=None):
    """csa_attn_fwd: O [B,T,Hq,D] bf16 and LSE [B,Hq,T] fp32 from raw q, k, v."""
    opts = dict(causal=causal, window=window, softcap=softcap, rope_base=rope_base, qk_norm=qk_norm,
                qk_norm_eps=qk_norm_eps, scale=scale)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    _check_bf16("q", q, (B, T, Hq, D))
    _check_bf16("k", k, (B, T, Hkv, D))
    _check_bf16("v", v, (B, T, Hkv, D))
    seg = _seg(segment_ids, B, T)
    p = _opts_params(q, k, opts)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(q, k, False, **opts)
    rc = _lib.csa_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(seg), _ptr(out), _ptr(lse),
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_attn_fwd")
    return out, lse


def attn_bwd(q, k, v, o, do, lse, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
             qk_norm_eps=1e-6, scale=0.0, segment_ids=None, dq=None, dk=None, dv=None, workspace=None,
             stream=None, after_fwd=False):
    """csa_attn_bwd: dq, dk, dv (bf16) = gradients w.r.t. the raw q, k, v.  after_fwd=True calls
    csa_attn_bwd_after_fwd instead, which reuses q', k' from `workspace` (it must be the one the
    matching attn_fwd call used, untouched since)."""
    opts = dict(causal=causal, window=window, softcap=softcap, rope_base=rope_base, qk_norm=qk_norm,
                qk_norm_eps=qk_norm_eps, scale=scale)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    for name, t, shp in (("q", q, (B, T, Hq, D)), ("k", k, (B, T, Hkv, D)), ("v", v, (B, T, Hkv, D)),
                         ("o", o, (B, T, Hq, D)), ("do", do, (B, T, Hq, D))):
        _check_bf16(name, t, shp)
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, Hq, T)):
        raise ValueError("lse must be a contiguous CUDA fp32 tensor of shape (B, Hq, T)")
    seg = _seg(segment_ids, B, T)
    p = _opts_params(q, k, opts)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        if after_fwd:
            raise ValueError("after_fwd needs the workspace of the matching attn_fwd call")
        workspace = workspace_for(q, k, True, **opts)
    fn = _lib.csa_attn_bwd_after_fwd if after_fwd else _lib.csa_attn_bwd
    rc = fn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(seg),
            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_attn_bwd_after_fwd" if after_fwd else "csa_attn_bwd")
    return dq, dk, dv


def prefill_workspace_size(p: Params, Tq: int) -> int:
    """csa_prefill_workspace_size: bytes of workspace csa_attn_prefill needs (0: invalid)."""
    return int(_lib.csa_prefill_workspace_size(ctypes.byref(p), int(Tq)))


def attn_prefill(q, k_cache, v_cache, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
                 qk_norm_eps=1e-6, scale=0.0, out=None, lse=None, workspace=None, stream=None):
    """csa_attn_prefill: the forward of Tq new raw queries (the last Tq positions) over a cache
    of Tk keys (stored after their own norm and RoPE) and values; o bf16, lse fp32."""
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k_cache.shape[1], k_cache.shape[2]
    _check_bf16("q", q, (B, Tq, Hq, D))
    _check_bf16("k_cache", k_cache, (B, Tk, Hkv, D))
    _check_bf16("v_cache", v_cache, (B, Tk, Hkv, D))
    p = make_params(B, Tk, Hq, Hkv, D, causal=causal, window=window, softcap=softcap, rope_base=rope_base,
                    qk_norm=qk_norm, qk_norm_eps=qk_norm_eps, scale=scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        n = prefill_workspace_size(p, Tq)
        if n == 0:
            raise CsaError(CSA_ERR_INVALID_ARG, "csa_prefill_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    rc = _lib.csa_attn_prefill(ctypes.byref(p), int(Tq), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_attn_prefill")
    return o, lse


def decode_workspace_size(p: Params, Tq: int) -> int:
    """csa_decode_workspace_size: bytes of workspace csa_attn_decode needs (0: invalid)."""
    return int(_lib.csa_decode_workspace_size(ctypes.byref(p), int(Tq)))


def attn_decode(q, k_cache, v_cache, *, causal=True, window=0, softcap=0.0, rope_base=0.0, qk_norm=False,
                qk_norm_eps=1e-6, scale=0.0, out=None, lse=None, workspace=None, stream=None):
    """csa_attn_decode: o [B,Tq,Hq,D] bf16 and lse [B,Hq,Tq] fp32 for Tq new raw queries over a
    cache of Tk keys (stored after their own norm and RoPE) and values."""
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k_cache.shape[1], k_cache.shape[2]
    _check_bf16("q", q, (B, Tq, Hq, D))
    _check_bf16("k_cache", k_cache, (B, Tk, Hkv, D))
    _check_bf16("v_cache", v_cache, (B, Tk, Hkv, D))
    p = make_params(B, Tk, Hq, Hkv, D, causal=causal, window=window, softcap=softcap, rope_base=rope_base,
                    qk_norm=qk_norm, qk_norm_eps=qk_norm_eps, scale=scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        n = decode_workspace_size(p, Tq)
        if n == 0:
            raise CsaError(CSA_ERR_INVALID_ARG, "csa_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    rc = _lib.csa_attn_decode(ctypes.byref(p), int(Tq), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_attn_decode")
    return o, lse


# ------------------------------------------------------------------ projections around attention
def _check_f32(name, t, shape):
    if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name} must be a contiguous CUDA fp32 tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def _proj_ws(workspace, device):
    if workspace is None:
        workspace = torch.zeros(int(_lib.csa_proj_workspace_size()), dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def _proj_shapes(x_shape, wq, wk):
    B, T, C = x_shape
    _, Hq, D = wq.shape
    return B, T, C, Hq, wk.shape[1], D


def qkv_proj(x, wq, wk, wv, *, q=None, k=None, v=None, workspace=None, stream=None):
    """csa_qkv_proj: q = x wq, k = x wk, v = x wv (one launch); x [B,T,C], wq [C,Hq,D],
    wk / wv [C,Hkv,D], all bf16."""
    B, T, C, Hq, Hkv, D = _proj_shapes(x.shape, wq, wk)
    _check_bf16("x", x, (B, T, C))
    _check_bf16("wq", wq, (C, Hq, D))
    _check_bf16("wk", wk, (C, Hkv, D))
    _check_bf16("wv", wv, (C, Hkv, D))
    q = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=x.device) if v is None else v
    ws, nb = _proj_ws(workspace, x.device)
    p = make_params(B, T, Hq, Hkv, D)
    rc = _lib.csa_qkv_proj(ctypes.byref(p), C, _ptr(x), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(q), _ptr(k), _ptr(v),
                           _ptr(ws), nb, _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_qkv_proj")
    return q, k, v


def out_proj(o, wo, *, y=None, workspace=None, stream=None):
    """csa_out_proj: y = o wo; o [B,T,Hq,D], wo [Hq,D,C] bf16 -> y [B,T,C] bf16."""
    B, T, Hq, D = o.shape
    C = wo.shape[2]
    _check_bf16("o", o, (B, T, Hq, D))
    _check_bf16("wo", wo, (Hq, D, C))
    y = torch.empty((B, T, C), dtype=torch.bfloat16, device=o.device) if y is None else y
    ws, nb = _proj_ws(workspace, o.device)
    p = make_params(B, T, Hq, Hq, D)
    rc = _lib.csa_out_proj(ctypes.byref(p), C, _ptr(o), _ptr(wo), _ptr(y), _ptr(ws), nb, _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_out_proj")
    return y


def out_proj_bwd(o, wo, dy, *, dout=None, dwo=None, weight_grad=True, workspace=None, stream=None):
    """csa_out_proj_bwd: dout = dy wo^T (bf16) and, when weight_grad, dwo += o^T dy (fp32;
    a zeroed tensor is allocated when dwo is None)."""
    B, T, Hq, D = o.shape
    C = wo.shape[2]
    _check_bf16("o", o, (B, T, Hq, D))
    _check_bf16("wo", wo, (Hq, D, C))
    _check_bf16("dy", dy, (B, T, C))
    dout = torch.empty_like(o) if dout is None else dout
    if weight_grad:
        dwo = torch.zeros((Hq, D, C), dtype=torch.float32, device=o.device) if dwo is None else dwo
        _check_f32("dwo", dwo, (Hq, D, C))
    else:
        dwo = None
    ws, nb = _proj_ws(workspace, o.device)
    p = make_params(B, T, Hq, Hq, D)
    rc = _lib.csa_out_proj_bwd(ctypes.byref(p), C, _ptr(o), _ptr(wo), _ptr(dy), _ptr(dout), _ptr(dwo), _ptr(ws), nb,
                               _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_out_proj_bwd")
    return dout, dwo


def qkv_proj_bwd(x, wq, wk, wv, dq, dk, dv, *, dx=None, dwq=None, dwk=None, dwv=None, weight_grad=True,
                 workspace=None, stream=None):
    """csa_qkv_proj_bwd: dx = dq wq^T + dk wk^T + dv wv^T (bf16) and, when weight_grad,
    dwq += x^T dq, dwk += x^T dk, dwv += x^T dv (fp32; zeroed tensors allocated when None)."""
    B, T, C, Hq, Hkv, D = _proj_shapes(x.shape, wq, wk)
    _check_bf16("x", x, (B, T, C))
    for name, t, shp in (("wq", wq, (C, Hq, D)), ("wk", wk, (C, Hkv, D)), ("wv", wv, (C, Hkv, D)),
                         ("dq", dq, (B, T, Hq, D)), ("dk", dk, (B, T, Hkv, D)), ("dv", dv, (B, T, Hkv, D))):
        _check_bf16(name, t, shp)
    dx = torch.empty_like(x) if dx is None else dx
    if weight_grad:
        z = lambda t, H: torch.zeros((C, H, D), dtype=torch.float32, device=x.device) if t is None else t  # noqa: E731
        dwq, dwk, dwv = z(dwq, Hq), z(dwk, Hkv), z(dwv, Hkv)
        for name, t, H in (("dwq", dwq, Hq), ("dwk", dwk, Hkv), ("dwv", dwv, Hkv)):
            _check_f32(name, t, (C, H, D))
    else:
        dwq = dwk = dwv = None
    ws, nb = _proj_ws(workspace, x.device)
    p = make_params(B, T, Hq, Hkv, D)
    rc = _lib.csa_qkv_proj_bwd(ctypes.byref(p), C, _ptr(x), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(dx), _ptr(dwq), _ptr(dwk), _ptr(dwv), _ptr(ws), nb, _stream(stream))
    if rc != CSA_OK:
        raise CsaError(rc, "csa_qkv_proj_bwd")
    return dx, dwq, dwk, dwv


def device_status(workspace, stream=None) -> int:
    """csa_device_status: synchronises the stream, returns (and clears) the device-side status."""
    return int(_lib.csa_device_status(_ptr(workspace), _stream(stream)))


def selftest_bounded_wait(device=None):
    """csa_selftest_bounded_wait: runs the never-completing-wait kernel and returns
    (status, gave_up[128], cycles[128]); status is CSA_ERR_DEVICE_TIMEOUT when every
    bounded wait gave up as designed."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    ws = torch.zeros(2048, dtype=torch.uint8, device=dev)
    rc = int(_lib.csa_selftest_bounded_wait(_ptr(ws), ws.numel(), _stream(None)))
    body = ws[256:256 + 128 * 4 + 128 * 8].cpu()
    gave_up = body[:512].view(torch.int32).tolist()
    cycles = body[512:].view(torch.int64).tolist()
    return rc, gave_up, cycles


def timing_enable(on: bool) -> None:
    _lib.csa_timing_enable(int(bool(on)))


def kernel_names() -> list[str]:
    return [_lib.csa_kernel_name(i).decode() for i in range(_lib.csa_num_kernels())]


def timing_collect() -> dict:
    """{kernel name: (total_ms, launches)} for every timed launch since the last collect."""
    n = _lib.csa_num_kernels()
    tot = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    rc = _lib.csa_timing_collect(tot, cnt, n)
    if rc != CSA_OK:
        raise CsaError(rc, "csa_timing_collect")
    return {name: (tot[i], cnt[i]) for i, name in enumerate(kernel_names())}
