"""Pins for the fp64 oracle, checked against things other than itself:
brute force on tiny inputs, a library routine on the no-empty-row case,
closed forms, and invariants of softmax attention with segment-equality masks.

What is pinned: exact softmax attention (vidax: A Unified JAX Framework for
Video Generative Models on Accelerator Meshes, §2 "3D RoPE, 3D VAEs, and flash
attention"; FlashAttention, its reference [2]) with the segment-id mask of
Appendix A, Table 4, row "HunyuanVideo-1.5: RESOURCE_EXHAUSTED at 720p".
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from video_diffusion_transformer_non_b200 import workloads as wl

TOL = 1e-12


def bits(x):
    """Exact bf16 bit patterns of values that are representable in bf16."""
    x = np.asarray(x, np.float32)
    b = wl.f32_to_bf16_bits(x)
    assert np.array_equal(wl.bf16_bits_to_f32(b), x), "value not bf16-exact"
    return b


def f64(b):
    return wl.bf16_bits_to_f32(b).astype(np.float64)


def brute_force(q, k, v, seg_q, seg_kv, scale, causal=False):
    """Pure-Python double loop: the full masked score matrix, then normalise.
    causal: key j visible to query i only if j <= i + (S_kv - S_q)."""
    qf, kf, vf = f64(q), f64(k), f64(v)
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    out = np.zeros((B, H, Sq, D))
    lse = np.full((B, H, Sq), -math.inf)
    for b, h, i in itertools.product(range(B), range(H), range(Sq)):
        row = []
        for j in range(Skv):
            if seg_q is not None and seg_q[b, i] != seg_kv[b, j]:
                row.append(None)
                continue
            if causal and j > i + (Skv - Sq):
                row.append(None)
                continue
            row.append(scale * math.fsum(qf[b, h, i, d] * kf[b, h, j, d] for d in range(D)))
        allowed = [s for s in row if s is not None]
        if not allowed:
            continue
        mx = max(allowed)
        w = [0.0 if s is None else math.exp(s - mx) for s in row]
        tot = math.fsum(w)
        for d in range(D):
            out[b, h, i, d] = math.fsum(w[j] * vf[b, h, j, d] for j in range(Skv)) / tot
        lse[b, h, i] = mx + math.log(tot)
    return out, lse


def rand_case(B, H, Sq, Skv, D, seed, n_ids=0, std=1.0):
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    seg_q = seg_kv = None
    if n_ids:
        seg_q = rng.integers(0, n_ids, (B, Sq)).astype(np.int32)
        seg_kv = rng.integers(0, n_ids, (B, Skv)).astype(np.int32)
    return wl.make_random(B, H, Sq, Skv, D, seed, seg_q, seg_kv, std)


def run(case, scale=None):
    return oracle.attn_fwd(case["q"], case["k"], case["v"], case["seg_q"], case["seg_kv"],
                           case["scale"] if scale is None else scale)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("shape,n_ids,seed", [
    ((1, 1, 1, 1, 1), 0, 0),
    ((1, 2, 5, 7, 3), 0, 1),
    ((2, 1, 8, 8, 4), 2, 2),
    ((2, 2, 6, 3, 2), 3, 3),   # some rows see no key
    ((1, 1, 8, 5, 4), 4, 4),
])
def test_brute_force_tiny(shape, n_ids, seed):
    c = rand_case(*shape, seed, n_ids)
    out, lse = run(c)
    ref_out, ref_lse = brute_force(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"])
    assert np.max(np.abs(out - ref_out)) <= TOL
    finite = np.isfinite(ref_lse)
    assert np.array_equal(finite, np.isfinite(lse))
    assert np.max(np.abs(lse[finite] - ref_lse[finite]), initial=0) <= TOL
    assert np.all(out[~finite] == 0.0)
    assert np.all(lse[~finite] == -np.inf)


@pytest.mark.parametrize("shape,n_ids,seed", [
    ((1, 2, 6, 6, 3), 0, 21), ((2, 1, 5, 8, 4), 2, 22), ((1, 1, 8, 3, 2), 0, 23),
    ((2, 2, 7, 7, 3), 3, 24),
])
def test_brute_force_tiny_causal(shape, n_ids, seed):
    c = rand_case(*shape, seed, n_ids)
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"],
                               causal=True)
    ro, rl = brute_force(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"], causal=True)
    fin = np.isfinite(rl)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(out - ro)) <= TOL
    assert np.max(np.abs(lse[fin] - rl[fin]), initial=0) <= TOL


# ------------------------------------------------------------ library routine

@pytest.mark.parametrize("seed,n_ids", [(5, 0), (6, 2), (7, 3)])
def test_matches_torch_sdpa_fp64(seed, n_ids):
    """torch's reference SDPA in fp64 on the CPU, with the boolean mask built
    from segment equality (small sizes, so the dense mask is harmless here)."""
    B, H, Sq, Skv, D = 2, 3, 33, 47, 16
    c = rand_case(B, H, Sq, Skv, D, seed, n_ids, std=2.0)
    q, k, v = (torch.from_numpy(f64(c[n])) for n in ("q", "k", "v"))
    if n_ids:
        mask = torch.from_numpy(c["seg_q"][:, None, :, None] == c["seg_kv"][:, None, None, :])
    else:
        mask = torch.ones(B, 1, Sq, Skv, dtype=torch.bool)
    mask = mask.expand(B, H, Sq, Skv)
    nonempty = mask.any(-1).numpy()
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=mask, scale=c["scale"]).numpy()
    logits = (q @ k.transpose(-1, -2)) * c["scale"]
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).numpy()
    out, lse = run(c)
    assert np.max(np.abs(out[nonempty] - ref[nonempty])) <= 1e-12
    assert np.max(np.abs(lse[nonempty] - ref_lse[nonempty])) <= 1e-12
    assert np.all(out[~nonempty] == 0) and np.all(lse[~nonempty] == -np.inf)


@pytest.mark.parametrize("S_q,S_kv", [(40, 40), (25, 40), (40, 25)])
def test_causal_matches_torch_sdpa_fp64(S_q, S_kv):
    """torch's fp64 SDPA with the bottom-right causal boolean mask."""
    B, H, D = 2, 2, 16
    c = rand_case(B, H, S_q, S_kv, D, 25, 2, std=2.0)
    q, k, v = (torch.from_numpy(f64(c[n])) for n in ("q", "k", "v"))
    i = torch.arange(S_q)[:, None]
    j = torch.arange(S_kv)[None, :]
    causal = j <= i + (S_kv - S_q)
    mask = torch.from_numpy(c["seg_q"][:, None, :, None] == c["seg_kv"][:, None, None, :]) & causal
    mask = mask.expand(B, H, S_q, S_kv)
    nonempty = mask.any(-1).numpy()
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                           scale=c["scale"]).numpy()
    logits = (q @ k.transpose(-1, -2)) * c["scale"]
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1).numpy()
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"],
                               causal=True)
    assert np.max(np.abs(out[nonempty] - ref[nonempty])) <= 1e-12
    assert np.max(np.abs(lse[nonempty] - ref_lse[nonempty])) <= 1e-12
    assert np.all(out[~nonempty] == 0) and np.all(lse[~nonempty] == -np.inf)


def test_causal_prefix_property_and_first_row():
    """Causal row i (S_q = S_kv) is full attention over keys 0..i alone; the
    first row sees only key 0: out = v_0, lse = scale q_0.k_0."""
    B, H, S, D = 1, 2, 12, 8
    c = wl.make_random(B, H, S, S, D, 26)
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=c["scale"], causal=True)
    for i in range(S):
        sub = {x: np.ascontiguousarray(c[x][:, :, :i + 1]) for x in ("k", "v")}
        qi = np.ascontiguousarray(c["q"][:, :, i:i + 1])
        o2, l2 = oracle.attn_fwd(qi, sub["k"], sub["v"], scale=c["scale"])
        assert np.max(np.abs(out[:, :, i] - o2[:, :, 0])) <= TOL
        assert np.max(np.abs(lse[:, :, i] - l2[:, :, 0])) <= TOL
    assert np.array_equal(out[:, :, 0], f64(c["v"])[:, :, 0])
    s00 = c["scale"] * np.sum(f64(c["q"])[:, :, 0] * f64(c["k"])[:, :, 0], -1)
    assert np.max(np.abs(lse[:, :, 0] - s00)) <= 1e-14


def test_causal_with_more_queries_than_keys_has_empty_rows():
    c = wl.make_random(1, 1, 10, 4, 4, 27)
    out, lse = oracle.attn_fwd(c["q"], c["k"], c["v"], scale=c["scale"], causal=True)
    assert np.all(lse[:, :, :6] == -np.inf) and np.all(out[:, :, :6] == 0)
    assert np.all(np.isfinite(lse[:, :, 6:]))


# ----------------------------------------------------------------- closed forms

def test_two_keys_one_to_three():
    """scores 0 and ln 3 (scale = ln 3, q = 1, k = 0 and 1) give weights 1/4 and
    3/4: out = (2 + 3*6)/4 = 5, lse = ln 4."""
    q = bits([[[[1.0]]]])
    k = bits([[[[0.0], [1.0]]]])
    v = bits([[[[2.0], [6.0]]]])
    out, lse = oracle.attn_fwd(q, k, v, scale=math.log(3.0))
    assert abs(out[0, 0, 0, 0] - 5.0) <= 1e-14
    assert abs(lse[0, 0, 0] - math.log(4.0)) <= 1e-15


def test_segments_hand_example():
    """seg_q = [0, 1], seg_kv = [1, 0, 1], scale 1.
    Row 0 sees only key 1: out = v1, lse = q0.k1 = 2.
    Row 1 sees keys 0 and 2 with scores 0 and 2:
    out = (v0 + e^2 v2)/(1 + e^2), lse = ln(1 + e^2)."""
    q = bits([[[[1, 0], [0, 1]]]])
    k = bits([[[[1, 0], [2, 0], [0, 2]]]])
    v = bits([[[[1, 1], [3, 5], [-1, 7]]]])
    sq = np.array([[0, 1]], np.int32)
    sk = np.array([[1, 0, 1]], np.int32)
    out, lse = oracle.attn_fwd(q, k, v, sq, sk, scale=1.0)
    e2 = math.exp(2.0)
    assert np.allclose(out[0, 0, 0], [3.0, 5.0], rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - 2.0) <= 1e-15
    assert np.allclose(out[0, 0, 1], [(1 - e2) / (1 + e2), (1 + 7 * e2) / (1 + e2)], rtol=0, atol=1e-14)
    assert abs(lse[0, 0, 1] - math.log1p(e2)) <= 1e-14


def test_scale_zero_gives_mean_of_allowed_values():
    c = rand_case(2, 2, 9, 13, 8, 11, n_ids=3)
    out, lse = run(c, scale=0.0)
    vf = f64(c["v"])
    for b, h, i in itertools.product(range(2), range(2), range(9)):
        allowed = c["seg_kv"][b] == c["seg_q"][b, i]
        n = int(allowed.sum())
        if n == 0:
            assert lse[b, h, i] == -np.inf and np.all(out[b, h, i] == 0)
            continue
        assert np.max(np.abs(out[b, h, i] - vf[b, h, allowed].mean(0))) <= 1e-14
        assert abs(lse[b, h, i] - math.log(n)) <= 1e-14


def test_identical_keys_give_mean_of_values():
    """Every key of a segment equal: all allowed scores equal s, so out is the
    mean of the allowed v and lse = s + ln |A_i|."""
    c = rand_case(1, 2, 7, 10, 4, 12, n_ids=2)
    k = c["k"].copy()
    for b in range(1):
        for sid in (0, 1):
            idx = np.nonzero(c["seg_kv"][b] == sid)[0]
            if idx.size:
                k[b, :, idx, :] = k[b, :, idx[:1], :]
    c["k"] = k
    out, lse = run(c)
    qf, kf, vf = f64(c["q"]), f64(k), f64(c["v"])
    for h, i in itertools.product(range(2), range(7)):
        allowed = c["seg_kv"][0] == c["seg_q"][0, i]
        if not allowed.any():
            continue
        j0 = np.nonzero(allowed)[0][0]
        s = c["scale"] * float(np.dot(qf[0, h, i], kf[0, h, j0]))
        assert np.max(np.abs(out[0, h, i] - vf[0, h, allowed].mean(0))) <= 1e-14
        assert abs(lse[0, h, i] - (s + math.log(allowed.sum()))) <= 1e-13


def test_single_allowed_key_and_dominant_key():
    # single allowed key: out is exactly that value row
    c = rand_case(1, 1, 4, 6, 8, 13)
    c["seg_q"] = np.array([[0, 1, 2, 3]], np.int32)
    c["seg_kv"] = np.array([[9, 2, 9, 0, 1, 3]], np.int32)
    out, lse = run(c)
    vf, qf, kf = f64(c["v"]), f64(c["q"]), f64(c["k"])
    for i, j in enumerate([3, 4, 1, 5]):
        assert np.array_equal(out[0, 0, i], vf[0, 0, j])
        assert abs(lse[0, 0, i] - c["scale"] * float(np.dot(qf[0, 0, i], kf[0, 0, j]))) <= 1e-14
    # one dominant key: q = 8 e_0, k_3 = 8 e_0, other keys 0 => s_3 - s_j = 64*scale
    D = 4
    q = np.zeros((1, 1, 1, D), np.float32); q[..., 0] = 8
    k = np.zeros((1, 1, 5, D), np.float32); k[0, 0, 3, 0] = 8
    v = np.arange(5 * D, dtype=np.float32).reshape(1, 1, 5, D)
    out, lse = oracle.attn_fwd(bits(q), bits(k), bits(v), scale=1.0)
    assert np.max(np.abs(out[0, 0, 0] - v[0, 0, 3])) <= 1e-15 * 100   # weight of others ~ 4e-28
    assert abs(lse[0, 0, 0] - (64.0 + math.log1p(4 * math.exp(-64.0)))) <= 1e-13


# ----------------------------------------------------------------- invariants

def test_probability_rows_sum_to_one_and_reproduce_output():
    c = rand_case(2, 2, 11, 17, 8, 14, n_ids=3)
    P = oracle.attn_probs(c["q"], c["k"], c["seg_q"], c["seg_kv"], c["scale"])
    out, _ = run(c)
    sums = P.sum(-1)
    nonempty = (c["seg_q"][:, :, None] == c["seg_kv"][:, None, :]).any(-1)  # [B,Sq]
    ne = np.broadcast_to(nonempty[:, None, :], sums.shape)
    assert np.max(np.abs(sums[ne] - 1.0)) <= 1e-14
    assert np.all(sums[~ne] == 0)
    masked = c["seg_q"][:, None, :, None] != c["seg_kv"][:, None, None, :]
    assert np.all(P[np.broadcast_to(masked, P.shape)] == 0)
    assert np.all(P >= 0)
    assert np.max(np.abs(P @ f64(c["v"]) - out)) <= 1e-13


def test_key_value_permutation_equivariance():
    c = rand_case(2, 3, 12, 29, 8, 15, n_ids=3)
    out, lse = run(c)
    perm = np.random.Generator(np.random.PCG64(99)).permutation(29)
    c2 = dict(c, k=np.ascontiguousarray(c["k"][:, :, perm]),
              v=np.ascontiguousarray(c["v"][:, :, perm]),
              seg_kv=np.ascontiguousarray(c["seg_kv"][:, perm]))
    out2, lse2 = run(c2)
    assert np.max(np.abs(out - out2)) <= TOL
    fin = np.isfinite(lse)
    assert np.array_equal(fin, np.isfinite(lse2))
    assert np.max(np.abs(lse[fin] - lse2[fin])) <= TOL


def test_query_permutation_equivariance():
    c = rand_case(1, 2, 21, 15, 8, 16, n_ids=2)
    out, lse = run(c)
    perm = np.random.Generator(np.random.PCG64(7)).permutation(21)
    c2 = dict(c, q=np.ascontiguousarray(c["q"][:, :, perm]),
              seg_q=np.ascontiguousarray(c["seg_q"][:, perm]))
    out2, lse2 = run(c2)
    assert np.array_equal(out[:, :, perm], out2)
    assert np.array_equal(lse[:, :, perm], lse2)


def test_segment_decomposition_equals_separate_attention():
    """Joint masked attention over a video/text/pad sequence equals attention
    run on each segment's sub-sequence alone, with no ids."""
    B, H, D = 2, 2, 8
    runs = ((40, 0), (9, 1), (5, 2))
    S = sum(n for n, _ in runs)
    seg = wl.segment_ids(runs, B)
    c = wl.make_random(B, H, S, S, D, 17, seg, seg.copy())
    out, lse = run(c)
    start = 0
    for n, _ in runs:
        sl = slice(start, start + n)
        sub = {x: np.ascontiguousarray(c[x][:, :, sl]) for x in ("q", "k", "v")}
        o2, l2 = oracle.attn_fwd(sub["q"], sub["k"], sub["v"], scale=c["scale"])
        assert np.max(np.abs(out[:, :, sl] - o2)) <= TOL
        assert np.max(np.abs(lse[:, :, sl] - l2)) <= TOL
        start += n


def test_cross_sample_and_head_independence():
    """Changing sample 1 / head 1 leaves sample 0 / head 0 untouched."""
    c = rand_case(2, 2, 10, 10, 4, 18, n_ids=2)
    out, lse = run(c)
    c2 = dict(c)
    for x in ("q", "k", "v"):
        a = c[x].copy(); a[1] = a[1][..., ::-1]; a[0, 1] = 0; c2[x] = a
    out2, lse2 = run(c2)
    assert np.array_equal(out[0, 0], out2[0, 0]) and np.array_equal(lse[0, 0], lse2[0, 0])


def test_rows_entry_matches_full():
    c = rand_case(2, 3, 37, 23, 16, 19, n_ids=3)
    out, lse = run(c)
    rows = np.array([[0, 0, 0], [1, 2, 36], [0, 1, 17], [1, 0, 5]], np.int64)
    o, l = oracle.attn_rows(c["q"], c["k"], c["v"], rows, c["seg_q"], c["seg_kv"], c["scale"])
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(o[r], out[b, h, i])
        assert l[r] == lse[b, h, i]


def test_all_masked_rows_and_empty_sizes():
    c = rand_case(1, 1, 4, 4, 4, 20)
    c["seg_q"] = np.array([[5, 5, 5, 5]], np.int32)
    c["seg_kv"] = np.array([[1, 2, 3, 4]], np.int32)
    out, lse = run(c)
    assert np.all(out == 0) and np.all(lse == -np.inf)
    # S_q = 0 and S_kv = 0
    z = wl.make_random(1, 1, 0, 3, 4, 0)
    o, l = oracle.attn_fwd(z["q"], z["k"], z["v"])
    assert o.shape == (1, 1, 0, 4) and l.shape == (1, 1, 0)
    z = wl.make_random(1, 1, 3, 0, 4, 0)
    o, l = oracle.attn_fwd(z["q"], z["k"], z["v"])
    assert np.all(o == 0) and np.all(l == -np.inf)


def test_oracle_regression_fixture():
    """Outputs stored by tests/golden/make_golden.py (which calls only the
    oracle) are reproduced bit for bit."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.npz")
    g = np.load(path)
    out, lse = oracle.attn_fwd(g["q"], g["k"], g["v"], g["seg_q"], g["seg_kv"], float(g["scale"]))
    assert np.array_equal(out, g["out"])
    assert np.array_equal(lse, g["lse"])


# ---------------------------------------------------------------- workloads

def test_workload_shapes_and_pair_counts():
    w = wl.WORKLOADS
    assert wl.allowed_pairs(w["joint_small"]) == 2 * (4096 ** 2 + 256 ** 2 + 37 ** 2)
    assert abs(wl.flops(w["joint_small"]) - 2.070e11) / 2.070e11 < 1e-3
    assert abs(wl.flops(w["video_480p"]) - 2.198e13) / 2.198e13 < 1e-3
    assert abs(wl.flops(w["cogvideox_joint"]) - 7.766e12) / 7.766e12 < 1e-3
    assert abs(wl.flops(w["video_720p"]) - 1.734e14) / 1.734e14 < 1e-3
    seg = wl.segment_ids(w["cogvideox_joint"].segments, 2)
    assert wl.allowed_pairs(seg, seg, B=2) == wl.allowed_pairs(w["cogvideox_joint"])


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], np.float32)
    got = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(got, ref)
    r = np.random.Generator(np.random.PCG64(3)).standard_normal(100000, dtype=np.float32)
    ref = torch.from_numpy(r).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(r)), ref)
