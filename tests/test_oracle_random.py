"""Randomised pins of the oracles (hypothesis, seeded and bounded): on random
small shapes, id layouts, causal limits, windows and rotary conventions, each
oracle agrees with an independent formulation of the same definition — the
pure-Python brute force for attention, torch's fp64 SDPA with a mask built
from coordinate differences for windows, and the relative-offset property
for the rotary embedding."""
import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from oracle.rope3d import rope3d_f64
from video_diffusion_transformer_non_b200 import workloads as wl

from test_oracle_pins import brute_force

SETTINGS = dict(max_examples=40, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.too_slow])


@settings(**SETTINGS)
@given(B=st.integers(1, 2), H=st.integers(1, 2), Sq=st.integers(1, 7), Skv=st.integers(1, 7),
       D=st.integers(1, 5), n_ids=st.integers(0, 3), causal=st.booleans(),
       scale=st.sampled_from([0.0, -0.3, 0.25, 1.0, 3.0]), data_seed=st.integers(0, 10 ** 6))
def test_attention_oracle_equals_brute_force(B, H, Sq, Skv, D, n_ids, causal, scale, data_seed):
    rng = np.random.Generator(np.random.PCG64(data_seed))
    seg_q = seg_kv = None
    if n_ids:
        seg_q = rng.integers(0, n_ids, (B, Sq)).astype(np.int32)
        seg_kv = rng.integers(0, n_ids, (B, Skv)).astype(np.int32)
    c = wl.make_random(B, H, Sq, Skv, D, data_seed, seg_q, seg_kv)
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], scale,
                               causal=causal)
    bo, bl = brute_force(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], scale, causal=causal)
    assert np.array_equal(np.isneginf(lse), np.isneginf(bl))
    fin = ~np.isneginf(bl)
    assert np.allclose(lse[fin], bl[fin], rtol=0, atol=1e-12)
    assert np.allclose(out, bo, rtol=0, atol=1e-12)


@settings(**SETTINGS)
@given(T=st.integers(1, 4), Hg=st.integers(1, 5), Wg=st.integers(1, 6),
       kt=st.sampled_from([1, 3, 5]), kh=st.sampled_from([1, 3, 5]), kw=st.sampled_from([1, 3, 7]),
       data_seed=st.integers(0, 10 ** 6))
def test_centred_window_oracle_equals_masked_sdpa(T, Hg, Wg, kt, kh, kw, data_seed):
    S = T * Hg * Wg
    coords = wl.raster_coords((T, Hg, Wg), 1)
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    c = wl.make_random(1, 1, S, S, 8, data_seed)
    win = dict(coord_q=coords, coord_kv=coords.copy(), size=(kt, kh, kw), extent=(T, Hg, Wg),
               clamped=False)
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=0.35, window=win)
    mask = np.ones((S, S), bool)
    for cc, k in zip((t, h, w), (kt, kh, kw)):
        mask &= np.abs(cc[:, None] - cc[None, :]) <= (k - 1) // 2
    f = lambda a: torch.from_numpy(wl.bf16_bits_to_f32(a).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        f(c["q"]), f(c["k"]), f(c["v"]), attn_mask=torch.from_numpy(mask), scale=0.35)
    assert np.allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    logits = (f(c["q"]) @ f(c["k"]).transpose(-1, -2)) * 0.35
    ref_lse = torch.logsumexp(logits.masked_fill(~torch.from_numpy(mask), float("-inf")), -1)
    assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


@settings(**SETTINGS)
@given(T=st.integers(1, 3), Hg=st.integers(1, 4), Wg=st.integers(1, 5),
       kt=st.sampled_from([1, 3, 5]), kh=st.sampled_from([1, 3]), kw=st.sampled_from([1, 3, 5, 9]))
def test_clamped_window_sees_min_k_n_keys_per_axis(T, Hg, Wg, kt, kh, kw):
    """Neighbourhood attention's clamped window: every query sees exactly
    prod_a min(k_a, extent_a) keys, and always its own position."""
    S = T * Hg * Wg
    coords = wl.raster_coords((T, Hg, Wg), 1)
    c = wl.make_random(1, 1, S, S, 4, 7, std=0.2)
    win = dict(coord_q=coords, coord_kv=coords.copy(), size=(kt, kh, kw), extent=(T, Hg, Wg),
               clamped=True)
    P = oracle.attn_probs(c["q"], c["k"], window=win)[0, 0]
    want = min(kt, T) * min(kh, Hg) * min(kw, Wg)
    assert ((P > 0).sum(axis=1) == want).all()
    assert (np.diag(P) > 0).all()


@settings(**SETTINGS)
@given(T=st.integers(1, 4), Hg=st.integers(1, 4), Wg=st.integers(1, 4),
       bt=st.integers(0, 6), bh=st.integers(0, 6), bw=st.integers(0, 6),
       interleaved=st.booleans(), theta=st.sampled_from([100.0, 1e4, 256.0]),
       shift=st.tuples(st.integers(0, 2), st.integers(0, 2), st.integers(0, 2)),
       data_seed=st.integers(0, 10 ** 6))
def test_rope_dot_products_depend_only_on_offsets(T, Hg, Wg, bt, bh, bw, interleaved, theta,
                                                  shift, data_seed):
    """RoFormer's defining property, per axis, on random grids and bands: the
    dot product of a rotated query and key depends only on their coordinate
    offsets."""
    bands = (2 * bt, 2 * bh, 2 * bw)
    D = sum(bands)
    if D == 0:
        return
    Tt, Hh, Ww = T + shift[0], Hg + shift[1], Wg + shift[2]
    n = Tt * Hh * Ww
    rng = np.random.Generator(np.random.PCG64(data_seed))
    q1 = wl.f32_to_bf16_bits(rng.standard_normal(D, dtype=np.float32))
    k1 = wl.f32_to_bf16_bits(rng.standard_normal(D, dtype=np.float32))
    rq = rope3d_f64(np.broadcast_to(q1, (1, 1, n, D)).copy(), (Tt, Hh, Ww), bands, theta,
                    interleaved)[0, 0]
    rk = rope3d_f64(np.broadcast_to(k1, (1, 1, n, D)).copy(), (Tt, Hh, Ww), bands, theta,
                    interleaved)[0, 0]
    idx = lambda p: (p[0] * Hh + p[1]) * Ww + p[2]
    p0 = (int(rng.integers(0, T)), int(rng.integers(0, Hg)), int(rng.integers(0, Wg)))
    p1 = (int(rng.integers(0, T)), int(rng.integers(0, Hg)), int(rng.integers(0, Wg)))
    moved = lambda p: tuple(a + s for a, s in zip(p, shift))
    a = float(np.dot(rq[idx(p0)], rk[idx(p1)]))
    b = float(np.dot(rq[idx(moved(p0))], rk[idx(moved(p1))]))
    assert abs(a - b) <= 1e-11 * max(1.0, abs(a))
