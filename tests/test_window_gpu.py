"""Parity of 3D neighbourhood attention (vidattn_fwd_window, through the C ABI)
with the fp64 oracle's window rule, under the attention tolerances: centred
and clamped windows, head dims 64 and 128, ragged volumes, windows from
1x1x1 to wider than the volume, per-sample coordinates, shuffled token order,
segment-free joint cases, the window_small workload on every row and the
11x11x11 window over the 480p latent volume on sampled rows.  Guard regions
around out and lse are checked on every call."""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_transformer_non_b200 import binding
from video_diffusion_transformer_non_b200 import workloads as wl

from _gpu_helpers import Guarded, bf16_to_f64, compare, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


def run_window(c, win, scale=None):
    q, k, v = (to_dev_bf16(c[n]) for n in ("q", "k", "v"))
    cq, ck = to_dev_i32(win["coord_q"]), to_dev_i32(win["coord_kv"])
    B, H, S_q, D = c["q"].shape
    S_kv = c["k"].shape[2]
    g = Guarded(B, H, S_q, D)
    sc = c["scale"] if scale is None else scale
    st = binding.vidattn_fwd_window(q, k, v, cq, ck, g.out, g.lse, B, H, S_q, S_kv, D, sc,
                                    *win["size"], *win["extent"],
                                    binding.VIDATTN_WINDOW_CLAMPED if win["clamped"] else 0)
    assert st == 0, binding.status_string(st)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    g.check_guards()
    return g.out, g.lse


def check_window(c, win, what, scale=None):
    out, lse = run_window(c, win, scale)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=c["scale"] if scale is None else scale,
                             window=win)
    return compare(bf16_to_f64(out), lse.double().cpu().numpy(), ro, rl, what)


def volume_case(B, H, D, grid, size, clamped, seed):
    S = int(np.prod(grid))
    c = wl.make_random(B, H, S, S, D, seed)
    coords = wl.raster_coords(grid, B)
    return c, dict(coord_q=coords, coord_kv=coords.copy(), size=size, extent=grid, clamped=clamped)


CASES = {
    # name: (B, H, D, grid, size)
    "d128_small": (1, 2, 128, (4, 8, 16), (3, 5, 5)),
    "d64_small": (1, 2, 64, (4, 8, 16), (3, 5, 5)),
    "ragged_volume": (2, 2, 128, (3, 5, 7), (3, 3, 3)),
    "wide_rows": (1, 2, 128, (2, 6, 130), (1, 3, 9)),
    "window_11": (1, 1, 128, (6, 12, 20), (11, 11, 11)),
    "flat_t": (1, 2, 64, (1, 20, 30), (1, 7, 7)),
    "only_t_axis": (1, 2, 128, (40, 2, 3), (5, 1, 1)),
}


@pytest.mark.parametrize("clamped", [False, True], ids=["centred", "clamped"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_window_matches_oracle(name, clamped):
    B, H, D, grid, size = CASES[name]
    c, win = volume_case(B, H, D, grid, size, clamped, seed=sorted(CASES).index(name))
    check_window(c, win, f"{name} clamped={clamped}")


def test_window_at_the_key_tile_limit():
    """S_kv = 262144 keys (2048 key tiles, the most a window call takes): a
    16 x 128 x 128 volume, window 3 x 3 x 5, queries of two frames."""
    grid = (16, 128, 128)
    ck = wl.raster_coords(grid, 1)
    assert ck.shape[1] == 262144
    cq = np.ascontiguousarray(ck[:, 7 * 16384: 7 * 16384 + 512])   # frame 7, first 4 rows
    c = wl.make_random(1, 1, cq.shape[1], ck.shape[1], 64, 30)
    win = dict(coord_q=cq, coord_kv=ck, size=(3, 3, 5), extent=grid, clamped=True)
    check_window(c, win, "2048 key tiles")


def test_unit_window_returns_own_value():
    c, win = volume_case(1, 2, 128, (3, 10, 20), (1, 1, 1), False, seed=21)
    out, lse = run_window(c, win)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), c["v"])


def test_covering_window_equals_plain_attention():
    """A window wider than the volume is full attention: on a volume of whole
    key tiles (512 tokens) no tile is masked, so the result is vidattn_fwd's
    up to the rounding of the exponentials (the window kernel computes 2 of
    16 on the FMA pipe, the plain kernel 4), and the oracle's."""
    grid = (4, 8, 16)
    c, win = volume_case(1, 2, 128, grid, (7, 15, 31), False, seed=22)
    out, lse = run_window(c, win)
    plain_o, plain_l = binding.attention(to_dev_bf16(c["q"]), to_dev_bf16(c["k"]),
                                         to_dev_bf16(c["v"]), scale=c["scale"])
    torch.cuda.synchronize()
    d = (out.float() - plain_o.float()).abs()
    assert float(d.max()) <= 8e-3 and float(d.mean()) <= 5e-4
    assert float((lse - plain_l).abs().max()) <= 2e-4
    check_window(c, win, "covering, whole tiles")


def test_covering_window_on_a_ragged_volume():
    """The same on 540 tokens: the ragged last key tile is masked (by the
    sequence end), every other tile is full; compared with the oracle."""
    c, win = volume_case(1, 2, 128, (3, 9, 20), (7, 17, 39), False, seed=29)
    check_window(c, win, "covering, ragged")


def test_shuffled_token_order_and_per_sample_coordinates():
    grid = (4, 10, 13)
    S = int(np.prod(grid))
    c = wl.make_random(2, 2, S, S, 128, 23)
    coords = wl.raster_coords(grid, 2).copy()
    rng = np.random.Generator(np.random.PCG64(24))
    coords[1] = coords[1, rng.permutation(S)]
    win = dict(coord_q=coords, coord_kv=coords.copy(), size=(3, 5, 5), extent=grid, clamped=True)
    check_window(c, win, "shuffled sample 1")


def test_raster_and_staged_key_tiles_in_one_call():
    """Keys in raster order except two swapped tokens in the third key tile:
    that tile takes the staged-coordinate mask, the others the raster-order
    mask from the tile index; one call, B = 2 with only sample 0 altered, so
    the two samples' tiles differ too."""
    grid = (3, 12, 24)
    S = int(np.prod(grid))
    c = wl.make_random(2, 2, S, S, 128, 31)
    ck = wl.raster_coords(grid, 2).copy()
    ck[0, [2 * 128 + 5, 2 * 128 + 77]] = ck[0, [2 * 128 + 77, 2 * 128 + 5]]
    cq = wl.raster_coords(grid, 2)
    win = dict(coord_q=cq, coord_kv=ck, size=(3, 5, 7), extent=grid, clamped=True)
    check_window(c, win, "raster with one staged tile")


def test_keys_a_raster_prefix_of_the_volume():
    """Keys are the first 500 tokens of the volume in raster order (a ragged
    last key tile, a last (t, h) row cut short), queries the whole volume:
    raster-order masks end at the sequence, and queries whose window holds
    no key get out = 0, lse = -inf."""
    grid = (3, 12, 24)
    ck_full = wl.raster_coords(grid, 1)
    ck = np.ascontiguousarray(ck_full[:, :500])
    c = wl.make_random(1, 2, ck_full.shape[1], 500, 128, 33)
    win = dict(coord_q=ck_full, coord_kv=ck, size=(1, 3, 5), extent=grid, clamped=False)
    check_window(c, win, "raster prefix keys")


def test_queries_and_keys_from_different_token_sets():
    """S_q != S_kv: queries are one frame, keys the whole volume."""
    grid = (5, 8, 16)
    S_kv = int(np.prod(grid))
    ck = wl.raster_coords(grid, 1)
    cq = np.ascontiguousarray(ck[:, 2 * 128: 3 * 128])        # frame t = 2
    c = wl.make_random(1, 2, cq.shape[1], S_kv, 128, 25)
    win = dict(coord_q=cq, coord_kv=ck, size=(3, 3, 5), extent=grid, clamped=False)
    check_window(c, win, "frame vs volume")


def test_scales():
    c, win = volume_case(1, 2, 128, (4, 8, 16), (3, 5, 5), True, seed=26)
    for sc in (0.0, -0.1, 0.5):
        check_window(c, win, f"scale {sc}", scale=sc)


def test_deterministic():
    c, win = volume_case(1, 2, 128, (4, 8, 16), (3, 5, 5), True, seed=27)
    a, la = run_window(c, win)
    b, lb = run_window(c, win)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)


def test_workload_window_small_all_rows():
    w = wl.WORKLOADS["window_small"]
    inp = wl.make_inputs(w)
    check_window(inp, wl.window_of(w), "window_small")


@pytest.mark.slow
def test_window_480p_sampled_rows():
    """The 11x11x11 window over the 480p latent volume, in the launch the
    benchmark times; 1024 random rows plus every row of the first, middle and
    last query tiles of 2 heads."""
    w = wl.WORKLOADS["window_480p"]
    inp = wl.make_inputs(w)
    win = wl.window_of(w)
    out, lse = run_window(inp, win)
    rng = np.random.Generator(np.random.PCG64(28))
    rows = [np.stack([np.zeros(1024, np.int64), rng.integers(0, w.H, 1024),
                      rng.integers(0, w.S, 1024)], 1)]
    for t in (0, (w.S // 2) // 128, (w.S - 1) // 128):
        i = np.arange(t * 128, min(w.S, t * 128 + 128))
        for h in (0, w.H - 1):
            rows.append(np.stack([np.zeros_like(i), np.full_like(i, h), i], 1))
    rows = np.unique(np.concatenate(rows), axis=0)
    ro, rl = oracle.attn_rows(inp["q"], inp["k"], inp["v"], rows, scale=inp["scale"], window=win)
    idx = torch.from_numpy(rows).cuda()
    go = out[idx[:, 0], idx[:, 1], idx[:, 2]]
    gl = lse[idx[:, 0], idx[:, 1], idx[:, 2]]
    compare(bf16_to_f64(go), gl.double().cpu().numpy(), ro, rl, "window_480p")
