"""Pins for the 3D rotary-embedding oracle (oracle/rope3d.py), checked against
properties that define rotary embeddings rather than against its own formula:
rotations keep every pair's norm, position 0 is the identity, and the dot
product of a rotated query and key depends only on their coordinate offsets
(RoFormer's defining property), per axis.  Planted mistakes must fail."""
import numpy as np
import pytest

from oracle.rope3d import rope3d_f64
from video_diffusion_transformer_non_b200 import workloads as wl


def _rand_bits(shape, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return wl.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def _pairs(D, bands, interleaved):
    out, start = [], 0
    for d in bands:
        for k in range(d // 2):
            out.append((start + 2 * k, start + 2 * k + 1) if interleaved
                       else (start + k, start + k + d // 2))
        start += d
    return out


@pytest.mark.parametrize("interleaved", [True, False])
def test_pair_norms_kept_and_position_zero_is_identity(interleaved):
    grid, bands = (3, 4, 5), (16, 24, 24)
    x = _rand_bits((2, 3, 70, 64), 1)
    y = rope3d_f64(x, grid, bands, interleaved=interleaved, token_offset=5)
    xf = _f64(x)
    for a, b in _pairs(64, bands, interleaved):
        assert np.allclose(np.hypot(y[..., a], y[..., b]), np.hypot(xf[..., a], xf[..., b]),
                           rtol=1e-13, atol=1e-13)
    assert np.array_equal(y[:, :, 5], xf[:, :, 5])                 # video token 0: (0,0,0)
    assert np.array_equal(y[:, :, :5], xf[:, :, :5])               # before the video
    assert np.array_equal(y[:, :, 5 + 60:], xf[:, :, 5 + 60:])     # after the video


@pytest.mark.parametrize("interleaved", [True, False])
def test_dot_products_depend_only_on_coordinate_offsets(interleaved):
    """<R(p) q, R(p') k> = <R(p + d) q, R(p' + d) k> for any shift d of the
    (t, h, w) coordinates: compare token pairs with equal offsets."""
    grid, bands = (4, 5, 6), (8, 12, 12)
    Hg, Wg = grid[1], grid[2]
    idx = lambda t, h, w: (t * Hg + h) * Wg + w
    rng = np.random.Generator(np.random.PCG64(2))
    q1 = wl.f32_to_bf16_bits(rng.standard_normal(32, dtype=np.float32))
    k1 = wl.f32_to_bf16_bits(rng.standard_normal(32, dtype=np.float32))
    n_video = grid[0] * Hg * Wg
    # every token holds the same q (resp. k) vector
    xq = np.broadcast_to(q1, (1, 1, n_video, 32)).copy()
    xk = np.broadcast_to(k1, (1, 1, n_video, 32)).copy()
    rq = rope3d_f64(xq, grid, bands, interleaved=interleaved)[0, 0]
    rk = rope3d_f64(xk, grid, bands, interleaved=interleaved)[0, 0]
    dot = lambda a, b: float(np.dot(rq[a], rk[b]))
    for (p, pk), shift in [(((0, 0, 0), (1, 2, 3)), (2, 1, 1)), (((1, 3, 0), (0, 1, 4)), (1, 0, 1)),
                           (((2, 2, 2), (2, 2, 2)), (1, 2, 3))]:
        a0, b0 = idx(*p), idx(*pk)
        a1 = idx(*(c + s for c, s in zip(p, shift)))
        b1 = idx(*(c + s for c, s in zip(pk, shift)))
        assert abs(dot(a0, b0) - dot(a1, b1)) <= 1e-12
    # and the offset matters: a different offset gives a different dot product
    assert abs(dot(idx(0, 0, 0), idx(1, 2, 3)) - dot(idx(0, 0, 0), idx(1, 2, 4))) > 1e-6


def test_band_of_one_axis_sees_only_that_coordinate():
    """Moving along w changes only the w band; along t only the t band."""
    grid, bands = (3, 3, 3), (8, 8, 16)
    x = _rand_bits((1, 1, 27, 32), 3)
    x[0, 0] = x[0, 0, 0]
    y = rope3d_f64(x, grid, bands)[0, 0]
    assert np.array_equal(y[1, :16], y[0, :16]) and not np.allclose(y[1, 16:], y[0, 16:])
    assert np.array_equal(y[9, 8:], y[0, 8:]) and not np.allclose(y[9, :8], y[0, :8])


def test_row_subset_matches_full_result():
    """Rows computed on their own equal the same rows of the whole sequence."""
    grid, bands = (3, 4, 5), (16, 24, 24)
    x = _rand_bits((2, 2, 75, 64), 6)
    full = rope3d_f64(x, grid, bands, token_offset=9, interleaved=False)
    rows = np.array([0, 8, 9, 10, 33, 68, 69, 74])
    part = rope3d_f64(x[:, :, rows], grid, bands, token_offset=9, interleaved=False, S=75, rows=rows)
    assert np.array_equal(part, full[:, :, rows])


def test_pairings_differ():
    """The two pairings are different rotations (the conventions are not
    interchangeable)."""
    x = _rand_bits((1, 1, 8, 16), 4)
    a = rope3d_f64(x, (2, 2, 2), (4, 4, 8), interleaved=True)
    b = rope3d_f64(x, (2, 2, 2), (4, 4, 8), interleaved=False)
    assert not np.allclose(a, b)


def test_bad_arguments():
    x = _rand_bits((1, 1, 8, 16), 5)
    with pytest.raises(ValueError):
        rope3d_f64(x, (2, 2, 2), (4, 4, 6))
    with pytest.raises(ValueError):
        rope3d_f64(x, (2, 2, 3), (4, 4, 8))


@pytest.mark.parametrize("interleaved", [True, False])
def test_closed_form_rotation_of_unit_vectors(interleaved):
    """theta = 10000 and a band of 8 features give the frequencies 1, 0.1,
    0.01 and 0.001 (10000^(-2k/8)); a unit vector on the first feature of pair
    k at coordinate c comes out as (cos(c f_k), sin(c f_k)) on that pair, the
    counter-clockwise rotation of RoFormer's definition."""
    freqs = (1.0, 0.1, 0.01, 0.001)
    grid, bands = (2, 3, 7), (8, 8, 8)
    S = 2 * 3 * 7
    for band in range(3):
        for k in range(4):
            x = np.zeros((1, 1, S, 24), np.uint16)
            i0 = band * 8 + (2 * k if interleaved else k)
            i1 = i0 + (1 if interleaved else 4)
            x[..., i0] = wl.f32_to_bf16_bits(np.float32([1.0]))[0]
            y = rope3d_f64(x, grid, bands, interleaved=interleaved)[0, 0]
            # the token at (t, h, w) = (1, 2, 6): its coordinate on this band's axis
            n = (1 * 3 + 2) * 7 + 6
            c = (1, 2, 6)[band]
            a = c * freqs[k]
            want = np.zeros(24)
            want[i0], want[i1] = np.cos(a), np.sin(a)
            assert np.allclose(y[n], want, rtol=0, atol=1e-14), (band, k)


# planted mistakes: each must make one of the pins above fail
import inspect
import oracle.rope3d as _rope_mod

ROPE_MUTATIONS = {
    "rotation_sign": ("i0[None, :]] = xa * c - xb * s", "i0[None, :]] = xa * c + xb * s"),
    "rotation_direction": ("i1[None, :]] = xa * s + xb * c", "i1[None, :]] = -xa * s + xb * c"),
    "freq_exponent": ("freq = theta ** (-2.0 * k / d)", "freq = theta ** (-1.0 * k / d)"),
    "freq_over_D": ("freq = theta ** (-2.0 * k / d)", "freq = theta ** (-2.0 * k / D)"),
    "hw_swapped": ("coords = (n // (Hg * Wg), (n // Wg) % Hg, n % Wg)",
                   "coords = (n // (Hg * Wg), n % Wg, (n // Wg) % Hg)"),
    "w_mod_Hg": ("coords = (n // (Hg * Wg), (n // Wg) % Hg, n % Wg)",
                 "coords = (n // (Hg * Wg), (n // Wg) % Hg, n % Hg)"),
    "offset_not_subtracted": ("n = rows[inside] - token_offset", "n = rows[inside]"),
    "range_ignores_offset": ("inside = (rows >= token_offset) & (rows < token_offset + n_video)",
                             "inside = rows < n_video"),
    "pairing_swapped": ("if interleaved:", "if not interleaved:"),
    "half_split_stride": ("i1 = i0 + half", "i1 = i0 + 1"),
    "band_start_not_advanced": ("start += d", "start += 0"),
}

_PINS = [
    lambda: [test_pair_norms_kept_and_position_zero_is_identity(i) for i in (True, False)],
    lambda: [test_dot_products_depend_only_on_coordinate_offsets(i) for i in (True, False)],
    test_band_of_one_axis_sees_only_that_coordinate,
    lambda: [test_closed_form_rotation_of_unit_vectors(i) for i in (True, False)],
]


@pytest.mark.parametrize("name", sorted(ROPE_MUTATIONS))
def test_planted_mistakes_fail_a_pin(name, monkeypatch):
    old, new = ROPE_MUTATIONS[name]
    src = inspect.getsource(_rope_mod)
    assert src.count(old) == 1, name
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    monkeypatch.setitem(globals(), "rope3d_f64", ns["rope3d_f64"])
    failed = 0
    for pin in _PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, f"mutation {name} passes every pin"
