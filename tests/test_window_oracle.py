"""Pins for the oracle's 3D neighbourhood window (oracle/attn_oracle.c,
`window` arguments), checked against facts the definitions fix rather than
against the oracle's own code: how many keys each query sees (a product over
axes of interval lengths, centred or clamped), hand-worked 1-D windows, a
window covering the volume reducing to full attention, a 1x1x1 window
reducing to v of the query's own position, torch's fp64 SDPA with an
explicit mask built from coordinate differences, the clamped and centred
windows agreeing away from the borders, permutation of token order, and the
window being the intersection of its three one-axis windows.  Planted
mistakes in copies of the C source must each fail one of these."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from video_diffusion_transformer_non_b200 import workloads as wl

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")


def pack(t, h, w):
    return ((np.asarray(t, np.int64) << 22) | (np.asarray(h, np.int64) << 11)
            | np.asarray(w, np.int64)).astype(np.uint32).view(np.int32)


def volume_coords(T, Hg, Wg, B=1):
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    c = pack(t.ravel(), h.ravel(), w.ravel())
    return np.ascontiguousarray(np.broadcast_to(c, (B, c.size))), (t.ravel(), h.ravel(), w.ravel())


def window(coords, size, extent, clamped):
    return dict(coord_q=coords, coord_kv=coords.copy(), size=size, extent=extent, clamped=clamped)


def case(B, H, S, D, seed, std=1.0):
    return wl.make_random(B, H, S, S, D, seed, std=std)


# ---------------------------------------------------------------- pins


def pin_counts():
    """Keys per query: centred = prod_a (min(c+r, N-1) - max(c-r, 0) + 1);
    clamped = prod_a min(k, N)."""
    T, Hg, Wg = 3, 5, 6
    size = (3, 5, 3)
    coords, (t, h, w) = volume_coords(T, Hg, Wg)
    c = case(1, 1, T * Hg * Wg, 16, 1, std=0.3)
    for clamped in (False, True):
        P = oracle.attn_probs(c["q"], c["k"], window=window(coords, size, (T, Hg, Wg), clamped))
        seen = (P[0, 0] > 0).sum(axis=1)
        want = np.ones_like(seen)
        for cc, k, N in zip((t, h, w), size, (T, Hg, Wg)):
            r = (k - 1) // 2
            want = want * (np.minimum(k, N) if clamped
                           else np.minimum(cc + r, N - 1) - np.maximum(cc - r, 0) + 1)
        assert np.array_equal(seen, want), clamped


def pin_hand_worked_lines():
    """One axis of 7 tokens, window 3: centred {c-1, c, c+1} cut at the ends;
    clamped shifted inside: query 0 sees {0,1,2}, query 6 sees {4,5,6}.
    Window 5 on 4 tokens, clamped: everyone sees all 4."""
    want = {
        (7, 3, False): [{0, 1}, {0, 1, 2}, {1, 2, 3}, {2, 3, 4}, {3, 4, 5}, {4, 5, 6}, {5, 6}],
        (7, 3, True): [{0, 1, 2}, {0, 1, 2}, {1, 2, 3}, {2, 3, 4}, {3, 4, 5}, {4, 5, 6}, {4, 5, 6}],
        (4, 5, True): [{0, 1, 2, 3}] * 4,
        (4, 5, False): [{0, 1, 2}, {0, 1, 2, 3}, {0, 1, 2, 3}, {1, 2, 3}],
    }
    for (N, k, clamped), sets in want.items():
        for axis in range(3):
            ext = [1, 1, 1]
            ext[axis] = N
            size = [1, 1, 1]
            size[axis] = k
            coords, _ = volume_coords(*ext)
            c = case(1, 1, N, 8, 2, std=0.3)
            P = oracle.attn_probs(c["q"], c["k"], window=window(coords, size, ext, clamped))
            got = [set(np.nonzero(P[0, 0, i])[0].tolist()) for i in range(N)]
            assert got == sets, (N, k, clamped, axis)


def pin_covering_window_is_full_attention():
    T, Hg, Wg = 2, 3, 4
    coords, _ = volume_coords(T, Hg, Wg, B=2)
    c = case(2, 2, T * Hg * Wg, 16, 3)
    ref_o, ref_l = oracle.attn_fwd(c["q"], c["k"], c["v"])
    for size, clamped in (((3, 5, 7), False), ((3, 3, 5), True)):
        o, l = oracle.attn_fwd(c["q"], c["k"], c["v"],
                               window=window(coords, size, (T, Hg, Wg), clamped))
        assert np.array_equal(o, ref_o) and np.array_equal(l, ref_l)


def pin_unit_window_is_own_value():
    T, Hg, Wg = 2, 3, 5
    coords, _ = volume_coords(T, Hg, Wg)
    c = case(1, 2, T * Hg * Wg, 16, 4)
    o, l = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=0.25,
                           window=window(coords, (1, 1, 1), (T, Hg, Wg), False))
    q = wl.bf16_bits_to_f32(c["q"]).astype(np.float64)
    k = wl.bf16_bits_to_f32(c["k"]).astype(np.float64)
    v = wl.bf16_bits_to_f32(c["v"]).astype(np.float64)
    assert np.array_equal(o, v)
    assert np.allclose(l, 0.25 * np.einsum("bhsd,bhsd->bhs", q, k), rtol=0, atol=1e-12)


def pin_sdpa_with_explicit_mask():
    """Centred window = |c_i - c_j| <= (k-1)/2 on every axis: torch fp64 SDPA."""
    T, Hg, Wg = 3, 4, 5
    size = (3, 3, 5)
    coords, (t, h, w) = volume_coords(T, Hg, Wg)
    c = case(1, 2, T * Hg * Wg, 16, 5)
    o, l = oracle.attn_fwd(c["q"], c["k"], c["v"], window=window(coords, size, (T, Hg, Wg), False))
    mask = np.ones((t.size, t.size), bool)
    for cc, k in zip((t, h, w), size):
        mask &= np.abs(cc[:, None] - cc[None, :]) <= (k - 1) // 2
    f = lambda a: torch.from_numpy(wl.bf16_bits_to_f32(a).astype(np.float64))
    q, kk, v = f(c["q"]), f(c["k"]), f(c["v"])
    m = torch.from_numpy(mask)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, v, attn_mask=m, scale=0.25)
    o2, _ = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=0.25,
                            window=window(coords, size, (T, Hg, Wg), False))
    assert np.allclose(o2, ref.numpy(), rtol=0, atol=1e-12)
    logits = (q @ kk.transpose(-1, -2)) * 0.25          # the default scale 1/sqrt(16)
    logits = logits.masked_fill(~m, float("-inf"))
    assert np.allclose(l, torch.logsumexp(logits, -1).numpy(), rtol=0, atol=1e-12)


def pin_clamped_equals_centred_inside():
    T, Hg, Wg = 5, 6, 7
    size = (3, 3, 5)
    coords, (t, h, w) = volume_coords(T, Hg, Wg)
    c = case(1, 1, T * Hg * Wg, 16, 6)
    ext = (T, Hg, Wg)
    a, la = oracle.attn_fwd(c["q"], c["k"], c["v"], window=window(coords, size, ext, False))
    b, lb = oracle.attn_fwd(c["q"], c["k"], c["v"], window=window(coords, size, ext, True))
    inside = np.ones(t.size, bool)
    for cc, k, N in zip((t, h, w), size, ext):
        r = (k - 1) // 2
        inside &= (cc - r >= 0) & (cc + r <= N - 1)
    assert inside.any() and (~inside).any()
    assert np.array_equal(a[:, :, inside], b[:, :, inside])
    assert not np.allclose(a[:, :, ~inside], b[:, :, ~inside])


def pin_token_order_does_not_matter():
    """The window follows the coordinates, not the sequence index."""
    T, Hg, Wg = 2, 4, 4
    coords, _ = volume_coords(T, Hg, Wg)
    c = case(1, 2, T * Hg * Wg, 16, 7)
    ext, size = (T, Hg, Wg), (1, 3, 3)
    o, l = oracle.attn_fwd(c["q"], c["k"], c["v"], window=window(coords, size, ext, True))
    perm = np.random.Generator(np.random.PCG64(8)).permutation(T * Hg * Wg)
    pc = np.ascontiguousarray(coords[:, perm])
    po, pl = oracle.attn_fwd(np.ascontiguousarray(c["q"][:, :, perm]),
                             np.ascontiguousarray(c["k"][:, :, perm]),
                             np.ascontiguousarray(c["v"][:, :, perm]),
                             window=window(pc, size, ext, True))
    assert np.allclose(po, o[:, :, perm], rtol=0, atol=1e-12)
    assert np.allclose(pl, l[:, :, perm], rtol=0, atol=1e-12)


def pin_window_is_intersection_of_axis_windows():
    T, Hg, Wg = 3, 4, 5
    coords, _ = volume_coords(T, Hg, Wg)
    c = case(1, 1, T * Hg * Wg, 16, 9, std=0.3)
    ext, size = (T, Hg, Wg), (3, 1, 3)
    for clamped in (False, True):
        full = oracle.attn_probs(c["q"], c["k"], window=window(coords, size, ext, clamped)) > 0
        parts = np.ones_like(full)
        for a in range(3):
            s = [2 * N + 1 for N in ext]
            s[a] = size[a]
            parts &= oracle.attn_probs(c["q"], c["k"], window=window(coords, s, ext, clamped)) > 0
        assert np.array_equal(full, parts)


def pin_window_with_segments_and_batches():
    """Per-sample coordinates and ids: a sample's rows depend only on its own
    coordinates; ids further restrict the window."""
    T, Hg, Wg = 2, 3, 4
    S = T * Hg * Wg
    coords, _ = volume_coords(T, Hg, Wg, B=2)
    coords[1] = coords[1, ::-1]                       # sample 1: reversed order
    seg = np.zeros((2, S), np.int32)
    seg[:, S // 2:] = 1
    c = wl.make_random(2, 1, S, S, 16, 10, seg, seg.copy())
    ext, size = (T, Hg, Wg), (3, 3, 3)
    P = oracle.attn_probs(c["q"], c["k"], c["seg_q"], c["seg_kv"],
                          window=window(coords, size, ext, False))
    Pn = oracle.attn_probs(c["q"], c["k"], window=window(coords, size, ext, False))
    same = seg[:, :, None] == seg[:, None, :]
    assert np.array_equal(P[:, 0] > 0, (Pn[:, 0] > 0) & same)
    # sample 1 holds the volume in reverse order: its rows see the windows of
    # their own coordinates, i.e. sample 0's pattern reversed on both axes
    assert np.array_equal(Pn[1, 0] > 0, (Pn[0, 0] > 0)[::-1, ::-1])


PINS = [pin_counts, pin_hand_worked_lines, pin_covering_window_is_full_attention,
        pin_unit_window_is_own_value, pin_sdpa_with_explicit_mask,
        pin_clamped_equals_centred_inside, pin_token_order_does_not_matter,
        pin_window_is_intersection_of_axis_windows, pin_window_with_segments_and_batches]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_window_pin(pin):
    pin()


def test_bad_window_arguments():
    coords, _ = volume_coords(1, 2, 2)
    c = case(1, 1, 4, 8, 11)
    for size, ext in (((2, 1, 1), (1, 2, 2)), ((0, 1, 1), (1, 2, 2)), ((1, 1, 1), (0, 2, 2))):
        with pytest.raises(RuntimeError):
            oracle.attn_fwd(c["q"], c["k"], c["v"], window=window(coords, size, ext, False))


# ------------------------------------------------------- planted mistakes

MUTATIONS = {
    "window_too_wide": ("if (ck[a] < start || ck[a] > start + w->size[a] - 1) return 0;",
                        "if (ck[a] < start || ck[a] > start + w->size[a]) return 0;"),
    "window_shifted": ("long start = c - (size - 1) / 2;", "long start = c - (size + 1) / 2;"),
    "clamp_missing": ("  if (clamped) {\n", "  if (0) {\n"),
    "clamp_to_end_missing": ("    if (start > extent - size) start = extent - size;\n", ""),
    "h_unpacked_wrong": ("c[1] = (long)((u >> 11) & 2047u);", "c[1] = (long)((u >> 10) & 2047u);"),
    "axis_sizes_swapped": ("long start = window_start(cq[a], w->size[a], w->extent[a], w->clamped);",
                           "long start = window_start(cq[a], w->size[2 - a], w->extent[a], w->clamped);"),
    "window_ignored": ("  if (win != NULL && !in_window(win, S_q, S_kv, b, i, j)) return 0;\n", ""),
    "key_coord_of_query": ("unpack_coord(w->coord_kv[b * S_kv + j], ck);",
                           "unpack_coord(w->coord_kv[b * S_kv + i], ck);"),
    "coords_ignore_batch": ("unpack_coord(w->coord_q[b * S_q + i], cq);",
                            "unpack_coord(w->coord_q[i], cq);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_window_mistake_fails_a_pin(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", str(so),
                    str(path), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle._declare(ctypes.CDLL(str(so))))
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, RuntimeError):
            failed.append(pin.__name__)
    assert failed, f"mutation {name} passes every window pin"
