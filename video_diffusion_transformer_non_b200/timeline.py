"""Per-tile timeline of one CTA of the attention kernel, from the trace build.

    python -m video_diffusion_transformer_non_b200.build --trace
    python -m video_diffusion_transformer_non_b200.timeline --D 64 --heads 8 --seq 32768

Loads libvidattn_trace.so (the same kernels with clock64 stamps at each
pipeline event of the CTA in the middle of the grid), runs a few forwards on
random inputs, and prints, for a window of key tiles, the cycles each role
spent between its events.  Events (see VIDATTN_TR in csrc/fwd_kernel.cuh):

  MMA      0 tile start, 1 K ready and S0 free, 2 S0 = Q0 K^T issued,
           3 V and P0 ready, 4 O0 += P0 V issued, 5 S1 free,
           6 S1 = Q1 K^T issued, 7 P1 ready, 8 O1 += P1 V issued
  softmax  0 wait for S, 1 S ready, 2 S in registers, 3 P computed,
           4 P columns free, 5 P written and signalled
"""
from __future__ import annotations

import argparse
import ctypes
import os

import numpy as np


def run(D, heads, seq, batch=1, lib_path=None, reps=3):
    import torch
    here = os.path.dirname(os.path.abspath(__file__))
    lib = ctypes.CDLL(lib_path or os.path.join(here, "csrc", "libvidattn_trace.so"))
    p, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.vidattn_fwd.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, f32, p]
    lib.vidattn_trace_set.argtypes = [p]
    q = torch.randn(batch, heads, seq, D, device="cuda", dtype=torch.bfloat16)
    k, v = torch.randn_like(q), torch.randn_like(q)
    o = torch.empty_like(q)
    lse = torch.empty(batch, heads, seq, device="cuda")
    tr = torch.zeros(4 * 64 * 16, dtype=torch.int64, device="cuda")
    for _ in range(reps):
        tr.zero_()
        lib.vidattn_trace_set(tr.data_ptr())
        st = lib.vidattn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), None, None, o.data_ptr(),
                             lse.data_ptr(), batch, heads, seq, seq, D, D ** -0.5,
                             torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
    lib.vidattn_trace_set(None)
    return tr.cpu().numpy().reshape(4, 64, 16).astype(np.int64)


def summarize(tr, lo=10, hi=18):
    lines = []
    mma = tr[0]
    lines.append("MMA, cycles between events 0>1>2>3>4>5>6>7>8, and the tile period")
    for t in range(lo, hi):
        r = mma[t]
        d = [int(r[e + 1] - r[e]) if r[e + 1] and r[e] else 0 for e in range(8)]
        lines.append(f"  t={t:2d} {d}  period {int(mma[t + 1, 0] - r[0])}")
    for qi in (0, 1):
        sm = tr[1 + qi]
        lines.append(f"softmax {qi}, cycles between events 0>1>2>3>4>5")
        for t in range(lo, hi):
            r = sm[t]
            d = [int(r[e + 1] - r[e]) if r[e + 1] and r[e] else 0 for e in range(5)]
            lines.append(f"  t={t:2d} {d}")
    return "\n".join(lines)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--seq", type=int, default=32768)
    ap.add_argument("--out", default=None, help="save the raw stamps (.npy)")
    a = ap.parse_args(argv)
    tr = run(a.D, a.heads, a.seq)
    if a.out:
        np.save(a.out, tr)
    print(summarize(tr))


if __name__ == "__main__":
    main()
