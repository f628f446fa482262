"""Every kernel family under a forced grid choice: VIDATTN_PERSIST=1 makes
every unsplit launch persistent (one CTA per SM looping over units), =0 one
CTA per unit, whatever the shape.  The library reads the variable once per
process, so each setting runs in a child process that checks its cases
against the fp64 oracle and reports back.  Persistent D = 64 and persistent
launches of long units are never chosen by default; this is where they are
tested."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np
from video_diffusion_transformer_non_b200 import workloads as wl
from _gpu_helpers import check_all_rows
cases = []
for D in (64, 128):
    # more units than SMs (2 x 40 x 4 = 320), short: ids + causal, and plain
    seg = wl.segment_ids(((600, 0), (300, 1), (100, 2)), 2)
    c = wl.make_random(2, 40, 1000, 1000, D, 90 + D, seg, seg.copy())
    check_all_rows(c, what=f"ids+causal D{D}", causal=True)
    c = wl.make_random(2, 40, 1000, 1000, D, 92 + D)
    check_all_rows(c, what=f"plain D{D}")
    # long units (16 key tiles of 2048 keys per unit) and a ragged tail
    c = wl.make_random(1, 40, 700, 2053, D, 94 + D)
    check_all_rows(c, what=f"long units D{D}")
print("child ok")
"""


@pytest.mark.gpu
@pytest.mark.parametrize("persist", ["1", "0"])
def test_forced_grid_choice_matches_oracle(persist):
    env = dict(os.environ, VIDATTN_PERSIST=persist)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "child ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
