"""The pair counts behind the benchmark's FLOP figures, against brute force.

bench.py divides 4*D*H*(allowed pairs) by the kernel's time, so a wrong count
misstates every TFLOP/s it prints.  The counting helpers in workloads.py work
from segment runs and per-axis window lengths; here each is compared with a
count over every (query, key) pair of small workloads of the same kinds: ids
compared token by token, the causal limit applied pair by pair, and for
windows the nonzero entries of the oracle's probability matrix (the oracle's
window rule is pinned on its own in test_window_oracle.py)."""
import numpy as np
import pytest

import oracle
from video_diffusion_transformer_non_b200 import workloads as wl


def _seg_row(w):
    return np.concatenate([np.full(n, sid, np.int32) for n, sid in w.segments])


def _brute_allowed(w, causal=False):
    if w.segments is None:
        ids = np.zeros(w.S, np.int32)
    else:
        ids = _seg_row(w)
    same = ids[:, None] == ids[None, :]
    if causal:
        same &= np.arange(w.S)[None, :] <= np.arange(w.S)[:, None]
    return w.B * int(same.sum())


SEGMENT_CASES = [
    ((7, 0), (3, 1), (2, 2)),          # video / text / pad
    ((5, 0), (4, 1), (3, 0), (2, 1)),  # ids that come back after another run
    ((9, 3),),                         # one id
    ((1, 0), (1, 1), (1, 0), (1, 2), (6, 1)),
]


@pytest.mark.parametrize("runs", SEGMENT_CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_segment_pair_counts(runs, causal):
    S = sum(n for n, _ in runs)
    w = wl.Workload(name="t", B=3, H=2, D=64, segments=runs, S=S, seed=0)
    got = wl.causal_pairs(w) if causal else wl.allowed_pairs(w)
    assert got == _brute_allowed(w, causal)
    assert wl.flops(w, causal) == 4.0 * w.H * w.D * got
    seg = wl.segment_ids(runs, w.B)
    if not causal:
        assert wl.allowed_pairs(seg, seg.copy()) == got


def test_unsegmented_pair_counts():
    w = wl.Workload(name="t", B=2, H=3, D=128, segments=None, S=11, seed=0)
    assert wl.allowed_pairs(w) == _brute_allowed(w)
    assert wl.causal_pairs(w) == _brute_allowed(w, causal=True)


def _window_workload(grid, size, clamped, B=1):
    return wl.Workload(name="win", B=B, H=2, D=128, segments=None, S=int(np.prod(grid)),
                       seed=0, rope_grid=grid, rope_bands=(44, 42, 42), window=size,
                       window_clamped=clamped)


WINDOW_CASES = [
    ((3, 4, 5), (3, 3, 3)),
    ((2, 6, 7), (5, 3, 7)),     # windows wider than an axis
    ((4, 1, 9), (3, 5, 1)),
    ((1, 5, 5), (1, 1, 1)),
    ((3, 3, 4), (7, 7, 9)),     # wider than the volume on every axis
]


@pytest.mark.parametrize("grid,size", WINDOW_CASES)
@pytest.mark.parametrize("clamped", [False, True])
def test_window_pair_counts_equal_the_oracles_window(grid, size, clamped):
    w = _window_workload(grid, size, clamped, B=2)
    c = wl.make_random(1, 1, w.S, w.S, 4, 3, std=0.2)
    win = wl.window_of(w, B=1)
    P = oracle.attn_probs(c["q"], c["k"], window=win)[0, 0]
    visible = P > 0
    assert wl.window_pairs(w) == int(visible.sum())
    assert wl.allowed_pairs(w) == w.B * int(visible.sum())
    rows = np.arange(w.S)
    assert np.array_equal(wl.window_row_counts(w, rows), visible.sum(axis=1))


def test_bench_workloads_window_counts_on_sampled_rows():
    """The window workloads the benchmark runs: per-row counts from the
    helper against the oracle's window on sampled rows (the full matrix is
    too large at 480p), and their sum over all rows against window_pairs."""
    for name in ("window_small", "window_480p"):
        w = wl.WORKLOADS[name]
        rows = np.arange(w.S)
        assert int(wl.window_row_counts(w, rows).sum()) == wl.window_pairs(w)
        rng = np.random.Generator(np.random.PCG64(11))
        sample = np.sort(rng.choice(w.S, 24, replace=False))
        win = wl.window_of(w, B=1)
        c = wl.make_random(1, 1, w.S, w.S, 4, 5, std=0.2)
        for i in sample:          # one query row of the oracle's window at a time
            qi = np.ascontiguousarray(c["q"][:, :, i:i + 1])
            wi = dict(win, coord_q=np.ascontiguousarray(win["coord_q"][:, i:i + 1]))
            p = oracle.attn_probs(qi, c["k"], window=wi)[0, 0, 0]
            assert int((p > 0).sum()) == int(wl.window_row_counts(w, [i])[0]), (name, i)
