"""Writes the regression fixtures in this folder.  Calls only the fp64 oracle.

The pages print no worked numeric example of attention, so these fixtures are not the
pages' numbers: they freeze the pinned oracle's outputs on three tiny seeded cases so
that a later change to its arithmetic shows up as a diff.  Each fixture records the
definition it exercises.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

CASES = {
    "causal_mha_plain": dict(
        shape=(1, 5, 2, 2, 4), opts=dict(), seg=None,
        cite="GPT-pretraining page, section 'Multihead Attention': softmax(QK^T/sqrt(d_k))V "
             "with the upper-triangular -inf mask"),
    "gqa_rope_qknorm_softcap": dict(
        shape=(1, 6, 4, 2, 4), opts=dict(rope_base=10000.0, qk_norm=True, softcap=2.0), seg=None,
        cite="nanogpt-jax-181m model card, section 'Architecture': GQA with RoPE, QK-norm and "
             "logits soft-capping; parameter-free RMSNorm"),
    "packed_window": dict(
        shape=(1, 7, 2, 1, 4), opts=dict(rope_base=10000.0, qk_norm=True, window=2),
        seg=[[0, 0, 0, 1, 1, 1, 1]],
        cite="nanogpt-jax-181m model card, sections 'Architecture' and 'SFT' (RoPE from packed "
             "segment positions, segment_ids); flaxchat README 'Core Features' (sliding window)"),
}


def inputs(shape, seed):
    B, T, Hq, Hkv, D = shape
    rng = np.random.default_rng(seed)
    # small dyadic values: exact in bf16 and in the JSON text
    q = rng.integers(-8, 9, size=(B, T, Hq, D)) / 4.0
    k = rng.integers(-8, 9, size=(B, T, Hkv, D)) / 4.0
    v = rng.integers(-8, 9, size=(B, T, Hkv, D)) / 4.0
    do = rng.integers(-8, 9, size=(B, T, Hq, D)) / 4.0
    return q, k, v, do


def main():
    for i, (name, c) in enumerate(sorted(CASES.items())):
        q, k, v, do = inputs(c["shape"], 100 + i)
        seg = np.array(c["seg"], dtype=np.int32) if c["seg"] is not None else None
        o, lse = oracle.attn_fwd(q, k, v, segment_ids=seg, **c["opts"])
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, segment_ids=seg, **c["opts"])
        rec = dict(name=name, cite=c["cite"], options=c["opts"], segment_ids=c["seg"],
                   q=q.tolist(), k=k.tolist(), v=v.tolist(), do=do.tolist(),
                   o=o.tolist(), lse=lse.tolist(), dq=dq.tolist(), dk=dk.tolist(), dv=dv.tolist())
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(rec, f, indent=None, separators=(",", ":"))
            f.write("\n")


if __name__ == "__main__":
    main()
