"""Causal multi-head / grouped-query self-attention, forward and backward, for B200 (sm_100a).

The work runs in hand-written CUDA kernels inside ``libcsa.so`` (C ABI: include/csa.h);
this package is its Python binding.  Public calls:

    attn_fwd(q, k, v, *, causal, window, softcap, rope_base, qk_norm, qk_norm_eps, scale,
             segment_ids) -> (o, lse)
    attn_bwd(q, k, v, o, do, lse, *, ...same options...) -> (dq, dk, dv)
    device_status(workspace), status_string(code), workspace_size(params, backward)

``workloads`` (seeded synthetic inputs) imports without the library; the attention calls
load it on first use and raise ImportError when it has not been built.
"""
_BOUND = ("attn_fwd", "attn_bwd", "device_status", "status_string", "workspace_size", "workspace_for",
          "make_params", "Params", "CsaError", "timing_enable", "timing_collect", "kernel_names")

__all__ = list(_BOUND) + ["workloads"]


def __getattr__(name):
    if name in _BOUND:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
