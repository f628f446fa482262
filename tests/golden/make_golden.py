"""Writes oracle_small.npz: a small seeded segment-masked case and the fp64
oracle's outputs for it.  Calls only the oracle; a regression fixture that
catches unintended changes to the oracle's arithmetic.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from video_diffusion_transformer_non_b200 import workloads as wl  # noqa: E402


def main():
    B, H, D = 2, 2, 16
    runs = ((70, 0), (21, 1), (9, 2))
    S = sum(n for n, _ in runs)
    seg = wl.segment_ids(runs, B)
    c = wl.make_random(B, H, S, S, D, 2024, seg, seg.copy())
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.npz")
    np.savez_compressed(path, q=c["q"], k=c["k"], v=c["v"], seg_q=c["seg_q"],
                        seg_kv=c["seg_kv"], scale=np.float64(c["scale"]), out=out, lse=lse)
    print("wrote", path)


if __name__ == "__main__":
    main()
