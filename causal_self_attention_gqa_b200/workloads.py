"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic.  It only draws inputs, so that the CUDA path
and the fp64 oracle see bit-identical bf16 tensors:

* Q, K, V, dO: fp32 samples of N(0, 1) from a CPU ``torch.Generator`` seeded with
  ``seed`` (drawn in that order), rounded once (round-to-nearest-even) to bf16.
* Packed rows (segment_ids): per batch row, document lengths are drawn from
  ``numpy.random.default_rng(seed)`` as integers uniform on [lo, hi] inclusive and laid
  end to end until the row is full; the last document is cut to fit, there is no
  padding, and the documents of a row get ids 0, 1, 2, ...  This stands in for the
  BestFit-packed instruction-tuning rows of the nanogpt-jax-181m model card (section
  "SFT"), whose data is not available here.

The five named workloads are the model shapes the pages train (MiniGPT page: 6 heads,
embed 192, T=128, batch 32; nanogpt-jax-181m model card: 8/4 GQA heads, head dim 96,
T=2048; flaxchat README: 12L/768d/6h with 3 KV heads) with the options each one uses.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    causal: bool = True
    window: int = 0
    softcap: float = 0.0
    rope_base: float = 0.0
    qk_norm: bool = False
    qk_norm_eps: float = 1e-6
    scale: float = 0.0            # <= 0: 1/sqrt(D)
    seg_len: tuple | None = None  # (lo, hi) document lengths for packed rows
    seed: int = 0

    def options(self) -> dict:
        return dict(causal=self.causal, window=self.window, softcap=self.softcap,
                    rope_base=self.rope_base, qk_norm=self.qk_norm,
                    qk_norm_eps=self.qk_norm_eps, scale=self.scale)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five benchmark-defined workloads, in order, then the short-window layer of an SSSL stack
# (the 181M shape with a window of T/2 that binds on unpacked rows: three of every four layers
# in a short-short-short-long pattern run it); seed = 1000 + index.
WORKLOADS = [
    Workload("pr1_mha_T128_D32", B=2, T=128, Hq=6, Hkv=6, D=32, seed=1000),
    Workload("minigpt_T128_D32_rope_qknorm", B=32, T=128, Hq=6, Hkv=6, D=32,
             rope_base=10000.0, qk_norm=True, seed=1001),
    Workload("depth12_gqa6x3_T2048_D128_rope_qknorm_cap50", B=8, T=2048, Hq=6, Hkv=3, D=128,
             rope_base=10000.0, qk_norm=True, softcap=50.0, seed=1002),
    Workload("gpt181m_gqa8x4_T2048_D96_rope_qknorm", B=16, T=2048, Hq=8, Hkv=4, D=96,
             rope_base=10000.0, qk_norm=True, seed=1003),
    Workload("packed_sft_gqa6x3_T2048_D128_win1024", B=8, T=2048, Hq=6, Hkv=3, D=128,
             rope_base=10000.0, qk_norm=True, window=1024, seg_len=(64, 768), seed=1004),
    Workload("sssl_short_gqa8x4_T2048_D96_rope_qknorm_win1024", B=16, T=2048, Hq=8, Hkv=4, D=96,
             rope_base=10000.0, qk_norm=True, window=1024, seed=1005),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def packed_segment_ids(B: int, T: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """int32 [B, T]: documents of length U[lo, hi] laid end to end, ids 0, 1, 2, ..."""
    rng = np.random.default_rng(seed)
    ids = np.empty((B, T), dtype=np.int32)
    for b in range(B):
        t, doc = 0, 0
        while t < T:
            n = int(rng.integers(lo, hi, endpoint=True))
            n = min(n, T - t)
            ids[b, t:t + n] = doc
            t += n
            doc += 1
    return ids


def make_inputs(w: Workload, *, need_grad_input: bool = True) -> dict:
    """bf16 CPU tensors q [B,T,Hq,D], k/v [B,T,Hkv,D], do [B,T,Hq,D] and int32 segment_ids."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.T, w.Hq, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((w.B, w.T, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((w.B, w.T, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    out = dict(q=q, k=k, v=v, segment_ids=None)
    if need_grad_input:
        out["do"] = torch.randn((w.B, w.T, w.Hq, w.D), generator=g,
                                dtype=torch.float32).to(torch.bfloat16)
    if w.seg_len is not None:
        lo, hi = w.seg_len
        out["segment_ids"] = torch.from_numpy(packed_segment_ids(w.B, w.T, lo, hi, w.seed))
    return out


# KV-cache decoding: B rows of Tq new raw queries over a cache of Tk entries.  The cached keys
# stand for keys already passed through the norm and RoPE: unit-RMS N(0,1) draws, like the
# normalised keys of the QK-norm models.
@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Tk: int
    Tq: int
    Hq: int
    Hkv: int
    D: int
    causal: bool = True
    window: int = 0
    softcap: float = 0.0
    rope_base: float = 0.0
    qk_norm: bool = False
    qk_norm_eps: float = 1e-6
    scale: float = 0.0
    seed: int = 0

    def options(self) -> dict:
        return dict(causal=self.causal, window=self.window, softcap=self.softcap, rope_base=self.rope_base,
                    qk_norm=self.qk_norm, qk_norm_eps=self.qk_norm_eps, scale=self.scale)

    def with_(self, **kw) -> "DecodeWorkload":
        return replace(self, **kw)


# One decoding step of the 181M model on a batch of 16 sequences with 8192 tokens of history.
DECODE_WORKLOADS = [
    DecodeWorkload("decode_gpt181m_gqa8x4_D96_rope_qknorm_cache8192", B=16, Tk=8192, Tq=1, Hq=8, Hkv=4, D=96,
                   rope_base=10000.0, qk_norm=True, seed=2000),
]


def make_decode_inputs(w: DecodeWorkload) -> dict:
    """bf16 CPU tensors q [B,Tq,Hq,D] (raw), k_cache / v_cache [B,Tk,Hkv,D]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.Tq, w.Hq, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    kc = torch.randn((w.B, w.Tk, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((w.B, w.Tk, w.Hkv, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return dict(q=q, k_cache=kc, v_cache=vc)


# The attention layer with its projections (x -> q, k, v -> attention -> y): the attention
# workload's shape plus the model width C.  Weights are drawn like a fan-in initialisation,
# N(0, 1/fan_in), so that q, k, v and y have about unit variance when x does.
@dataclass(frozen=True)
class LayerWorkload:
    name: str
    attn: Workload
    C: int
    seed: int = 0


LAYER_WORKLOADS = [
    LayerWorkload("layer_gpt181m_C768_gqa8x4_T2048_D96_rope_qknorm", WORKLOADS[3], C=768, seed=1100),
    LayerWorkload("layer_depth12_C768_gqa6x3_T2048_D128_rope_qknorm_cap50", WORKLOADS[2], C=768, seed=1101),
]


def make_layer_inputs(w: LayerWorkload) -> dict:
    """bf16 CPU tensors x [B,T,C], wq [C,Hq,D], wk / wv [C,Hkv,D], wo [Hq,D,C], dy [B,T,C]."""
    a = w.attn
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)

    def draw(shape, std):
        return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)

    return dict(
        x=draw((a.B, a.T, w.C), 1.0),
        wq=draw((w.C, a.Hq, a.D), w.C ** -0.5),
        wk=draw((w.C, a.Hkv, a.D), w.C ** -0.5),
        wv=draw((w.C, a.Hkv, a.D), w.C ** -0.5),
        wo=draw((a.Hq, a.D, w.C), (a.Hq * a.D) ** -0.5),
        dy=draw((a.B, a.T, w.C), 1.0),
    )
