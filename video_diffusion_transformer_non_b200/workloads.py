"""Seeded synthetic inputs for the attention forward: shapes, segment layouts
and random values.  Shared by the tests and the benchmark for both the CUDA
path and the CPU oracle.  This module holds none of the attention arithmetic.

Recipe (every tensor is seeded; nothing is loaded from disk):

* one ``numpy.random.Generator(PCG64(seed))`` per workload;
* for workloads with per-head scaling, first ``a = uniform(0.5, 2, H)`` (for q)
  then ``b = uniform(0.5, 2, H)`` (for k);
* then q, k and v, in that order, each drawn as ``standard_normal`` float32,
  one (b, h) slab of shape [S, D] at a time in (b, h) order; q and k slabs are
  multiplied by a[h] and b[h] in fp32 when the workload scales heads;
* every fp32 value is rounded to bf16 with round-to-nearest-even; the arrays
  returned are the bf16 bit patterns (uint16), so the GPU path and the oracle
  see bit-identical inputs;
* segment ids are int32 [B, S]: contiguous runs in the order video, text, pad.

The first five named workloads follow the token counts of the video latents in the
paper's benchmark families (vidax: A Unified JAX Framework for Video Generative
Models on Accelerator Meshes, Fig. 1 and Tables 2 and 5: 480p and 720p
Wan/HunyuanVideo grids, CogVideoX 720x480x49 with a 226-token T5 prompt), and
stand in for them; the head counts and head dims are those of the named DiT
families.

The two window workloads stand in for the 3D neighbourhood attention of the
LTX-2.5 VAE decoder (same paper, Appendix A, Table 4, group 4: an 11 x 11 x 11
window); the paper gives neither its volume nor its heads, so window_480p
runs that window over the 480p latent volume with 16 heads of 128, and
window_small is the quick case.  Their tokens are the volume in raster order.

The rotary-embedding conventions attached to each workload (the paper names
3D RoPE per family but prints none) are taken from the families' public
releases: Wan's split of a 128-wide head into t/h/w bands of 44/42/42
features with theta 10000, CogVideoX's 16/24/24 of a 64-wide head with theta
10000, HunyuanVideo's 16/56/56 with theta 256; all pair features 2k and 2k+1.
Positions are the integer (t, h, w) indices of the latent grid.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    # runs of (n_tokens, segment id) in sequence order; None => single segment
    segments: tuple | None
    S: int
    seed: int
    head_scaling: bool = False
    description: str = ""
    # 3D rotary embedding of q and k ahead of the attention: the video tokens'
    # (T, Hg, Wg) grid, where they start, the (d_t, d_h, d_w) feature bands,
    # theta, and the pairing (True: features 2k, 2k+1; False: k, k + d/2)
    rope_grid: tuple | None = None
    rope_offset: int = 0
    rope_bands: tuple | None = None
    rope_theta: float = 10000.0
    rope_interleaved: bool = True
    # 3D neighbourhood attention over the rope_grid volume (all S tokens are
    # video tokens in raster order): odd window size per axis, clamped or not
    window: tuple | None = None
    window_clamped: bool = True

    @property
    def S_q(self) -> int:
        return self.S

    @property
    def S_kv(self) -> int:
        return self.S

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


def _runs_total(runs):
    return sum(n for n, _ in runs)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", B=1, H=2, D=64, segments=None, S=512, seed=0,
        description="B1 H2 D64 S512 (latent 2x16x16), one segment",
        rope_grid=(2, 16, 16), rope_bands=(16, 24, 24)),
    "joint_small": Workload(
        name="joint_small", B=2, H=12, D=128,
        segments=((4096, 0), (256, 1), (37, 2)), S=4389, seed=1,
        description="B2 H12 D128: 4096 video (4x32x32) + 256 text + 37 pad; ids video 0, text 1, pad 2",
        rope_grid=(4, 32, 32), rope_bands=(44, 42, 42)),
    "video_480p": Workload(
        name="video_480p", B=1, H=40, D=128, segments=None, S=32760, seed=2,
        head_scaling=True,
        description="B1 H40 D128 S32760 (21x30x52), one segment, q/k per-head scaled by U[0.5,2]",
        rope_grid=(21, 30, 52), rope_bands=(44, 42, 42)),
    "cogvideox_joint": Workload(
        name="cogvideox_joint", B=2, H=48, D=64,
        segments=((17550 + 226, 0), (16, 1)), S=17792, seed=3,
        description="B2 H48 D64: 17550 video (13x30x45) + 226 text share id 0; 16 pad tokens id 1",
        rope_grid=(13, 30, 45), rope_bands=(16, 24, 24)),
    "video_720p": Workload(
        name="video_720p", B=1, H=24, D=128,
        segments=((118800, 0), (256, 1), (112, 2)), S=119168, seed=4,
        description="B1 H24 D128: 118800 video (33x45x80) + 256 text + 112 pad; ids video 0, text 1, pad 2",
        rope_grid=(33, 45, 80), rope_bands=(16, 56, 56), rope_theta=256.0),
    "window_small": Workload(
        name="window_small", B=2, H=4, D=128, segments=None, S=2048, seed=5,
        description="B2 H4 D128: 3D neighbourhood attention over an 8x16x16 volume, "
                    "window 5x5x5 clamped",
        rope_grid=(8, 16, 16), rope_bands=(44, 42, 42), window=(5, 5, 5)),
    "window_480p": Workload(
        name="window_480p", B=1, H=16, D=128, segments=None, S=32760, seed=6,
        description="B1 H16 D128: 3D neighbourhood attention over the 21x30x52 latent volume, "
                    "window 11x11x11 clamped",
        rope_grid=(21, 30, 52), rope_bands=(44, 42, 42), window=(11, 11, 11)),
}

for _w in WORKLOADS.values():
    assert _w.segments is None or _runs_total(_w.segments) == _w.S, _w.name
    assert _w.rope_offset + int(np.prod(_w.rope_grid)) <= _w.S and sum(_w.rope_bands) == _w.D, _w.name


def pack_coords(t, h, w) -> np.ndarray:
    """Per-token coordinates packed t << 22 | h << 11 | w, as int32."""
    return ((np.asarray(t, np.int64) << 22) | (np.asarray(h, np.int64) << 11)
            | np.asarray(w, np.int64)).astype(np.uint32).view(np.int32)


def raster_coords(grid, B: int) -> np.ndarray:
    """int32 [B, T*Hg*Wg]: the packed (t, h, w) of each token of a T x Hg x Wg
    volume in raster order (w fastest), the same for every sample."""
    T, Hg, Wg = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    c = pack_coords(t.ravel(), h.ravel(), w.ravel())
    return np.ascontiguousarray(np.broadcast_to(c, (B, c.size)))


def window_of(w: Workload, B: int | None = None) -> dict:
    """The window description of a windowed workload (oracle and binding form)."""
    c = raster_coords(w.rope_grid, w.B if B is None else B)
    return dict(coord_q=c, coord_kv=c.copy(), size=w.window, extent=w.rope_grid,
                clamped=w.window_clamped)


def window_pairs(w: Workload) -> int:
    """(query, key) pairs inside the windows over the whole volume, per sample
    and head: the per-axis counts multiply, so the total is the product over
    axes of the sum over coordinates of the window length on that axis."""
    total = 1
    for k, N in zip(w.window, w.rope_grid):
        r = (k - 1) // 2
        c = np.arange(N)
        if w.window_clamped:
            per = np.full(N, min(k, N))
        else:
            per = np.minimum(c + r, N - 1) - np.maximum(c - r, 0) + 1
        total *= int(per.sum())
    return total


def window_row_counts(w: Workload, rows) -> np.ndarray:
    """Keys inside the window of each query row (sequence index, raster order)."""
    T, Hg, Wg = w.rope_grid
    rows = np.asarray(rows, np.int64)
    coords = (rows // (Hg * Wg), (rows // Wg) % Hg, rows % Wg)
    n = np.ones(rows.shape, np.int64)
    for c, k, N in zip(coords, w.window, w.rope_grid):
        r = (k - 1) // 2
        n *= (np.full(c.shape, min(k, N)) if w.window_clamped
              else np.minimum(c + r, N - 1) - np.maximum(c - r, 0) + 1)
    return n


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bits.
    Inputs here are finite and far from the fp32 overflow threshold."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def segment_ids(runs, B: int) -> np.ndarray:
    """int32 [B, S] from runs of (count, id), the same for every sample."""
    row = np.concatenate([np.full(n, sid, np.int32) for n, sid in runs])
    return np.ascontiguousarray(np.broadcast_to(row, (B, row.size)))


def random_bf16(rng: np.random.Generator, B, H, S, D, head_scale=None) -> np.ndarray:
    """bf16 bits [B,H,S,D] of N(0,1) draws, one [S,D] slab per (b,h)."""
    out = np.empty((B, H, S, D), np.uint16)
    for b in range(B):
        for h in range(H):
            slab = rng.standard_normal((S, D), dtype=np.float32)
            if head_scale is not None:
                slab *= np.float32(head_scale[h])
            out[b, h] = f32_to_bf16_bits(slab)
    return out


def make_inputs(w: Workload, seed_offset: int = 0):
    """Returns dict(q, k, v: uint16 bf16 bits [B,H,S,D]; seg_q, seg_kv: int32
    [B,S] or None; scale: float)."""
    rng = np.random.Generator(np.random.PCG64(w.seed + seed_offset))
    a = b = None
    if w.head_scaling:
        a = rng.uniform(0.5, 2.0, w.H).astype(np.float32)
        b = rng.uniform(0.5, 2.0, w.H).astype(np.float32)
    q = random_bf16(rng, w.B, w.H, w.S_q, w.D, a)
    k = random_bf16(rng, w.B, w.H, w.S_kv, w.D, b)
    v = random_bf16(rng, w.B, w.H, w.S_kv, w.D)
    seg = None if w.segments is None else segment_ids(w.segments, w.B)
    return dict(q=q, k=k, v=v, seg_q=seg, seg_kv=None if seg is None else seg.copy(),
                scale=w.scale)


def make_random(B, H, S_q, S_kv, D, seed, seg_q=None, seg_kv=None, std=1.0):
    """Small seeded case for tests: N(0, std^2) q, k, v as bf16 bits."""
    rng = np.random.Generator(np.random.PCG64(seed))
    def draw(S):
        x = rng.standard_normal((B, H, S, D), dtype=np.float32) * np.float32(std)
        return f32_to_bf16_bits(x)
    q = draw(S_q)
    k = draw(S_kv)
    v = draw(S_kv)
    return dict(q=q, k=k, v=v,
                seg_q=None if seg_q is None else np.ascontiguousarray(seg_q, np.int32),
                seg_kv=None if seg_kv is None else np.ascontiguousarray(seg_kv, np.int32),
                scale=1.0 / float(np.sqrt(D)))


def allowed_pairs(w_or_seg_q, seg_kv=None, S_q=None, S_kv=None, B=None) -> int:
    """Number of (b, i, j) pairs whose segment ids match (all pairs when no ids).
    Counted from the runs, without building any mask."""
    if isinstance(w_or_seg_q, Workload):
        w = w_or_seg_q
        if w.window is not None:
            return w.B * window_pairs(w)
        if w.segments is None:
            return w.B * w.S_q * w.S_kv
        per_id = {}
        for n, sid in w.segments:
            per_id[sid] = per_id.get(sid, 0) + n
        return w.B * sum(n * n for n in per_id.values())
    seg_q = w_or_seg_q
    if seg_q is None:
        return B * S_q * S_kv
    total = 0
    for b in range(seg_q.shape[0]):
        ids_q, cnt_q = np.unique(seg_q[b], return_counts=True)
        ids_k, cnt_k = np.unique(seg_kv[b], return_counts=True)
        ck = dict(zip(ids_k.tolist(), cnt_k.tolist()))
        total += sum(c * ck.get(i, 0) for i, c in zip(ids_q.tolist(), cnt_q.tolist()))
    return int(total)


def causal_pairs(w: Workload) -> int:
    """Allowed pairs under the causal limit (key j <= query i, S_q = S_kv) and
    segment equality: n (n + 1) / 2 per id holding n tokens, per sample."""
    if w.segments is None:
        return w.B * w.S_q * (w.S_q + 1) // 2
    per_id = {}
    for n, sid in w.segments:
        per_id[sid] = per_id.get(sid, 0) + n
    return w.B * sum(n * (n + 1) // 2 for n in per_id.values())


def flops(w: Workload, causal: bool = False) -> float:
    """4*D flops per allowed (query, key) pair per head: QK^T and PV."""
    return 4.0 * w.H * w.D * (causal_pairs(w) if causal else allowed_pairs(w))
