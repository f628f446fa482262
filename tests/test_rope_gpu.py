"""Parity of the 3D rotary-embedding kernel (vidattn_rope3d, through the C ABI)
with the fp64 oracle (oracle/rope3d.py) on seeded inputs: both pairings,
head dims 64 and 128, text or padding around the video tokens, empty bands,
long axes (large angles), strided [B,S,H,D] input, in place, ragged token
counts, guard regions around the outputs, and the full 480p q/k on sampled
tokens.

Bar: every element within half a bf16 ulp of the exact value plus fp32
arithmetic slack (2^-8 |exact| + 1e-5 x the largest input of its row), at
least 99.8% of elements equal to the correctly rounded exact value, and
bit-for-bit copies where the rotation is the identity (tokens outside the
video, coordinate 0)."""
import numpy as np
import pytest
import torch

from oracle.rope3d import rope3d_f64
from video_diffusion_transformer_non_b200 import binding
from video_diffusion_transformer_non_b200 import workloads as wl

from _gpu_helpers import GUARD, SENTINEL_BF16, to_dev_bf16

pytestmark = pytest.mark.gpu


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def nearest_bf16_bits(ref: np.ndarray) -> np.ndarray:
    """The bf16 nearest to each fp64 value (ties: either)."""
    f = ref.astype(np.float32)
    lo = (f.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    lo_bits = (lo.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    hi_bits = lo_bits + np.uint16(1)          # next bf16 away from zero
    hi = wl.bf16_bits_to_f32(hi_bits).astype(np.float64)
    pick_hi = np.abs(hi - ref) < np.abs(lo.astype(np.float64) - ref)
    return np.where(pick_hi, hi_bits, lo_bits)


def check(got_bits, x_bits, ref, what):
    got = wl.bf16_bits_to_f32(got_bits).astype(np.float64)
    x = wl.bf16_bits_to_f32(x_bits).astype(np.float64)
    assert np.isfinite(got).all(), what
    rowmax = np.abs(x).max(axis=-1, keepdims=True)
    err = np.abs(got - ref)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * rowmax
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), f"{what}: err {err[worst]:.3e} > tol {tol[worst]:.3e} at {worst}"
    exact = np.mean(got_bits == nearest_bf16_bits(ref))
    assert exact >= 0.998, f"{what}: only {exact:.4%} correctly rounded"


class GuardedOut:
    """bf16 [B,H,S,D] output inside a buffer with sentinel margins; NaN inside."""

    def __init__(self, shape):
        n = int(np.prod(shape))
        self.buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=torch.bfloat16, device="cuda")
        self.buf.view(torch.int16)[:GUARD] = SENTINEL_BF16
        self.buf.view(torch.int16)[GUARD + n:] = SENTINEL_BF16
        self.t = self.buf[GUARD:GUARD + n].view(*shape)
        self.n = n

    def check(self):
        b = self.buf.view(torch.int16)
        assert bool((b[:GUARD] == SENTINEL_BF16).all()), "written before the output"
        assert bool((b[GUARD + self.n:] == SENTINEL_BF16).all()), "written past the output"
        assert not bool(torch.isnan(self.t).any()), "an output element was never written"


def run(xq, xk, grid, bands, interleaved, offset, theta=10000.0):
    """xq, xk: bf16 bits [B,H,S,D] (xk may be None).  Returns output bits."""
    q = to_dev_bf16(xq)
    k = None if xk is None else to_dev_bf16(xk)
    oq = GuardedOut(xq.shape)
    ok = None if xk is None else GuardedOut(xk.shape)
    binding.rope3d(q, k, grid, bands, theta=theta, interleaved=interleaved, token_offset=offset,
                   out_q=oq.t, out_k=None if ok is None else ok.t)
    torch.cuda.synchronize()
    oq.check()
    if ok is not None:
        ok.check()
    return bits_of(oq.t), None if ok is None else bits_of(ok.t)


def rand_bits(shape, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return wl.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


CASES = {
    # name: (B, H, D, grid, bands, offset, S, interleaved)
    "d128_interleaved": (1, 3, 128, (3, 5, 7), (44, 42, 42), 0, 105, True),
    "d128_half_split": (1, 3, 128, (3, 5, 7), (44, 42, 42), 0, 105, False),
    "d64_text_first_half_split": (2, 2, 64, (2, 6, 9), (16, 24, 24), 13, 128, False),
    "d64_text_first_interleaved": (2, 2, 64, (2, 6, 9), (16, 24, 24), 13, 128, True),
    "no_t_band": (1, 2, 128, (1, 8, 8), (0, 64, 64), 0, 67, True),
    "only_t_band": (1, 2, 64, (7, 1, 1), (64, 0, 0), 0, 7, False),
    "long_w_axis": (1, 1, 64, (1, 1, 5000), (0, 0, 64), 0, 5000, True),
    "long_t_axis_half_split": (1, 1, 128, (3000, 1, 1), (128, 0, 0), 5, 3006, False),
    "ragged_many_slabs": (3, 5, 128, (2, 3, 3), (40, 44, 44), 2, 21, True),
    "one_token": (1, 1, 64, (1, 1, 1), (16, 24, 24), 0, 1, False),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_rope_matches_oracle(name):
    B, H, D, grid, bands, off, S, inter = CASES[name]
    xq = rand_bits((B, H, S, D), 100 + len(name))
    xk = rand_bits((B, H, S, D), 200 + len(name))
    gq, gk = run(xq, xk, grid, bands, inter, off)
    for x, g, what in ((xq, gq, "q"), (xk, gk, "k")):
        ref = rope3d_f64(x, grid, bands, interleaved=inter, token_offset=off)
        check(g, x, ref, f"{name} {what}")
        n_video = int(np.prod(grid))
        # identity where nothing turns: outside the video and at (0, 0, 0)
        assert np.array_equal(g[:, :, :off], x[:, :, :off])
        assert np.array_equal(g[:, :, off + n_video:], x[:, :, off + n_video:])
        assert np.array_equal(g[:, :, off], x[:, :, off])


def test_theta_other_than_ten_thousand():
    xq = rand_bits((1, 2, 60, 64), 7)
    gq, _ = run(xq, None, (3, 4, 5), (16, 24, 24), True, 0, theta=500.0)
    check(gq, xq, rope3d_f64(xq, (3, 4, 5), (16, 24, 24), theta=500.0), "theta 500")


def test_q_only():
    xq = rand_bits((2, 3, 40, 128), 8)
    gq, gk = run(xq, None, (2, 4, 5), (44, 42, 42), False, 0)
    assert gk is None
    check(gq, xq, rope3d_f64(xq, (2, 4, 5), (44, 42, 42), interleaved=False), "q only")


@pytest.mark.parametrize("interleaved", [True, False])
def test_strided_bshd_input(interleaved):
    """The projection's [B,S,H,D] layout, read through strides; the output is
    [B,H,S,D]."""
    B, S, H, D = 2, 90, 3, 128
    grid, bands = (2, 5, 9), (44, 42, 42)
    xs = rand_bits((B, S, H, D), 9)
    ks = rand_bits((B, S, H, D), 10)
    q = to_dev_bf16(xs).transpose(1, 2)
    k = to_dev_bf16(ks).transpose(1, 2)
    oq, ok = binding.rope3d(q, k, grid, bands, interleaved=interleaved)
    torch.cuda.synchronize()
    for src, o, what in ((xs, oq, "q"), (ks, ok, "k")):
        x = np.ascontiguousarray(src.transpose(0, 2, 1, 3))
        check(bits_of(o), x, rope3d_f64(x, grid, bands, interleaved=interleaved), f"bshd {what}")


@pytest.mark.parametrize("interleaved", [True, False])
def test_in_place_equals_out_of_place(interleaved):
    xq = rand_bits((2, 4, 131, 128), 11)
    xk = rand_bits((2, 4, 131, 128), 12)
    a_q, a_k = run(xq, xk, (3, 6, 7), (44, 42, 42), interleaved, 5)
    q, k = to_dev_bf16(xq), to_dev_bf16(xk)
    binding.rope3d(q, k, (3, 6, 7), (44, 42, 42), interleaved=interleaved, token_offset=5,
                   out_q=q, out_k=k)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(q), a_q) and np.array_equal(bits_of(k), a_k)


def test_deterministic():
    xq = rand_bits((1, 8, 1000, 64), 13)
    grid, bands = (10, 10, 10), (16, 24, 24)
    a, _ = run(xq, None, grid, bands, False, 0)
    b, _ = run(xq, None, grid, bands, False, 0)
    assert np.array_equal(a, b)


@pytest.mark.slow
@pytest.mark.parametrize("interleaved", [True, False])
def test_full_480p_q_k_sampled_tokens(interleaved):
    """The 480p video latent (21 x 30 x 52 tokens, 40 heads of 128), q and k
    in one launch as the benchmark runs it; every head of 96 sampled tokens
    (first, last, tile edges and random) against the oracle."""
    w = wl.WORKLOADS["video_480p"]
    inp = wl.make_inputs(w)
    grid, bands = (21, 30, 52), (44, 42, 42)
    q, k = to_dev_bf16(inp["q"]), to_dev_bf16(inp["k"])
    oq, ok = binding.rope3d(q, k, grid, bands, interleaved=interleaved)
    torch.cuda.synchronize()
    rng = np.random.Generator(np.random.PCG64(14))
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 4, 1559, 1560, w.S - 5, w.S - 1],
                                     rng.integers(0, w.S, 87)]))
    idx = torch.from_numpy(rows).cuda()
    for x, o, what in ((inp["q"], oq, "q"), (inp["k"], ok, "k")):
        got = bits_of(o.index_select(2, idx))
        xs = np.ascontiguousarray(x[:, :, rows])
        ref = rope3d_f64(xs, grid, bands, interleaved=interleaved, S=w.S, rows=rows)
        check(got, xs, ref, f"480p {what}")


@pytest.mark.parametrize("interleaved", [True, False])
def test_rope_then_attention_matches_oracle(interleaved):
    """The benchmark's --rope step on a small case: q and k rotated on the
    GPU, then attention on the rotated tensors, against the oracle's
    attention on the oracle's rotation rounded to bf16 (the rotation's output
    precision), under the attention tolerances."""
    import oracle
    from _gpu_helpers import bf16_to_f64, compare
    grid, bands = (2, 6, 9), (44, 42, 42)
    S = 108 + 20                                  # video tokens, then 20 text tokens
    c = wl.make_random(1, 2, S, S, 128, 50)
    q, k, v = to_dev_bf16(c["q"]), to_dev_bf16(c["k"]), to_dev_bf16(c["v"])
    qr, kr = binding.rope3d(q, k, grid, bands, interleaved=interleaved)
    out, lse = binding.attention(qr, kr, v, scale=c["scale"])
    torch.cuda.synchronize()
    to_bits = lambda x: wl.f32_to_bf16_bits(x.astype(np.float32))
    rq = to_bits(rope3d_f64(c["q"], grid, bands, interleaved=interleaved))
    rk = to_bits(rope3d_f64(c["k"], grid, bands, interleaved=interleaved))
    ro, rl = oracle.attn_fwd(rq, rk, c["v"], scale=c["scale"])
    compare(bf16_to_f64(out), lse.double().cpu().numpy(), ro, rl, "rope then attention")
