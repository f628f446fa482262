"""Shared helpers for the GPU tests: upload seeded inputs, run the CUDA path
through the C ABI with guard regions around the outputs, sample rows, and
compare with the fp64 oracle under the parity tolerances."""
import numpy as np
import torch

import oracle
from video_diffusion_transformer_non_b200 import binding

# Parity bar for N(0,1) inputs: bf16 output, fp32 statistics.
TOL_MAX_OUT = 2e-2
TOL_MEAN_OUT = 2e-3
TOL_LSE = 1e-3

GUARD = 64                 # elements of guard on each side (keeps 16-byte alignment)
SENTINEL_BF16 = 0x7F7F     # a finite bf16 the kernel never writes as a pattern
SENTINEL_F32 = 1.2345e30


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_i32(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a).copy()).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class Guarded:
    """out bf16 [B,H,S_q,D] and lse fp32 [B,H,S_q] inside larger buffers whose
    margins hold a sentinel; the interior starts as NaN."""

    def __init__(self, B, H, S_q, D):
        n_out = B * H * S_q * D
        n_lse = B * H * S_q
        self.out_buf = torch.full((n_out + 2 * GUARD,), float("nan"), dtype=torch.bfloat16,
                                  device="cuda")
        self.out_buf.view(torch.int16)[:GUARD] = SENTINEL_BF16
        self.out_buf.view(torch.int16)[GUARD + n_out:] = SENTINEL_BF16
        self.lse_buf = torch.full((n_lse + 2 * GUARD,), float("nan"), dtype=torch.float32,
                                  device="cuda")
        self.lse_buf[:GUARD] = SENTINEL_F32
        self.lse_buf[GUARD + n_lse:] = SENTINEL_F32
        self.out = self.out_buf[GUARD:GUARD + n_out].view(B, H, S_q, D)
        self.lse = self.lse_buf[GUARD:GUARD + n_lse].view(B, H, S_q)
        self.n_out, self.n_lse = n_out, n_lse

    def check_guards(self):
        o = self.out_buf.view(torch.int16)
        assert bool((o[:GUARD] == SENTINEL_BF16).all()), "out written before its start"
        assert bool((o[GUARD + self.n_out:] == SENTINEL_BF16).all()), "out written past its end"
        assert bool((self.lse_buf[:GUARD] == SENTINEL_F32).all()), "lse written before its start"
        assert bool((self.lse_buf[GUARD + self.n_lse:] == SENTINEL_F32).all()), "lse written past end"
        assert not bool(torch.isnan(self.out).any()), "some out element was never written"
        assert not bool(torch.isnan(self.lse).any()), "some lse element was never written"


def run_gpu(case, scale=None, check=True, causal=False, flags=0):
    """case: dict of numpy inputs (q, k, v bf16 bits; seg_q, seg_kv int32 or None).
    flags: extra vidattn_fwd_ex flags (a VIDATTN_SPLIT_KV request)."""
    q, k, v = (to_dev_bf16(case[n]) for n in ("q", "k", "v"))
    sq, sk = to_dev_i32(case.get("seg_q")), to_dev_i32(case.get("seg_kv"))
    B, H, S_q, D = case["q"].shape
    S_kv = case["k"].shape[2]
    g = Guarded(B, H, S_q, D)
    sc = case["scale"] if scale is None else scale
    st = binding.vidattn_fwd_ex(q, k, v, sq, sk, g.out, g.lse, B, H, S_q, S_kv, D, sc,
                                (binding.VIDATTN_CAUSAL if causal else 0) | flags)
    assert st == 0, binding.status_string(st)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    if check:
        g.check_guards()
    return g.out, g.lse


def compare(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    """out_gpu, out_ref: [..., D] float64; lse_*: [...]."""
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{what}: empty-row pattern differs"
    assert np.all(out_gpu[empty] == 0.0), f"{what}: empty rows must be exactly 0"
    ne = ~empty
    if ne.any():
        d = np.abs(out_gpu[ne] - out_ref[ne])
        dl = np.abs(lse_gpu[ne] - lse_ref[ne])
        assert np.isfinite(out_gpu[ne]).all() and np.isfinite(lse_gpu[ne]).all(), what
        stats = dict(max_out=float(d.max()), mean_out=float(d.mean()), max_lse=float(dl.max()))
        assert stats["max_out"] <= TOL_MAX_OUT, (what, stats)
        assert stats["mean_out"] <= TOL_MEAN_OUT, (what, stats)
        assert stats["max_lse"] <= TOL_LSE, (what, stats)
        return stats
    return {}


def check_all_rows(case, scale=None, what="", causal=False, flags=0):
    out, lse = run_gpu(case, scale, causal=causal, flags=flags)
    ro, rl = oracle.attn_fwd(case["q"], case["k"], case["v"], case.get("seg_q"),
                             case.get("seg_kv"), case["scale"] if scale is None else scale,
                             causal=causal)
    return compare(bf16_to_f64(out), lse.double().cpu().numpy(), ro, rl, what)


def sample_rows(B, H, S_q, seg_runs=None, n_random=4096, n_heads_full=8, seed=0):
    """The rows compared at full size: seeded random (b,h,i) rows plus, for
    n_heads_full heads, every row of the first and last query tile and of
    every tile holding a segment boundary or padding."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = [np.stack([rng.integers(0, B, n_random), rng.integers(0, H, n_random),
                      rng.integers(0, S_q, n_random)], 1)]
    tiles = {0, (S_q - 1) // 128}
    if seg_runs is not None:
        start = 0
        for n, _ in seg_runs[:-1]:
            start += n
            tiles.add(start // 128)
            tiles.add((start - 1) // 128)
        tiles.add((S_q - seg_runs[-1][0]) // 128)
    heads = rng.choice(H, size=min(H, n_heads_full), replace=False)
    for t in sorted(tiles):
        i = np.arange(t * 128, min(S_q, t * 128 + 128))
        for b in range(B):
            for h in heads:
                rows.append(np.stack([np.full_like(i, b), np.full_like(i, h), i], 1))
    rows = np.unique(np.concatenate(rows).astype(np.int64), axis=0)
    return rows
