"""Test infrastructure only: fp64 oracle of the 3D rotary position embedding
applied to q and k before attention.

The vidax paper (§2, "3D RoPE, 3D VAEs, and flash attention") applies rotary
position embedding over the time, height and width axes of the video latent
and keeps each model family's own convention, the conventions being
"mathematically non-interchangeable"; it gives no formula.  This oracle takes
the published rotary embedding (RoFormer, Su et al. 2021: rotate feature
pair k by the angle pos * theta^(-2k/d)) and applies it per axis:

* the head dim D is split into three contiguous bands of d_t, d_h, d_w
  features (d_t + d_h + d_w = D), driven by the token's t, h and w
  coordinates;
* video token n (n = 0 .. T*Hg*Wg - 1, at sequence index token_offset + n)
  has coordinates t = n // (Hg*Wg), h = (n // Wg) % Hg, w = n % Wg;
* inside a band of d features, pair k (k < d/2) is either (2k, 2k+1)
  ("interleaved") or (k, k + d/2) ("half-split"), and is rotated by
  angle = coord * theta^(-2k/d):  (x, y) -> (x cos a - y sin a, x sin a + y cos a);
* tokens outside the video range (text, padding) are left unchanged.

Computed in float64 from the exact bf16 inputs; the GPU path rounds its
result to bf16 once.
"""
from __future__ import annotations

import numpy as np


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rope3d_f64(x_bits: np.ndarray, grid, bands, theta: float = 10000.0,
               interleaved: bool = True, token_offset: int = 0, S: int | None = None,
               rows=None) -> np.ndarray:
    """x_bits: uint16 bf16 bits [B, H, S, D].  grid = (T, Hg, Wg);
    bands = (d_t, d_h, d_w).  Returns float64 [B, H, S, D].

    With ``rows`` (sequence indices, ascending) x_bits holds only those tokens,
    [B, H, len(rows), D], of a sequence of ``S`` tokens; the result is the
    same rows of the full result."""
    x = _bf16_to_f64(x_bits)
    B, H, n_rows, D = x.shape
    if rows is None:
        rows = np.arange(n_rows)
        S = n_rows
    rows = np.asarray(rows, dtype=np.int64)
    if rows.shape != (n_rows,) or S is None:
        raise ValueError("rows must name one sequence index per token, with S given")
    T, Hg, Wg = grid
    if sum(bands) != D or any(d % 2 for d in bands):
        raise ValueError("bands must be even and sum to D")
    n_video = T * Hg * Wg
    if token_offset < 0 or token_offset + n_video > S:
        raise ValueError("video tokens must lie inside the sequence")
    out = x.copy()
    inside = (rows >= token_offset) & (rows < token_offset + n_video)
    n = rows[inside] - token_offset
    coords = (n // (Hg * Wg), (n // Wg) % Hg, n % Wg)
    tok = np.nonzero(inside)[0]
    start = 0
    for d, coord in zip(bands, coords):
        half = d // 2
        k = np.arange(half)
        freq = theta ** (-2.0 * k / d)                    # [half]
        angle = coord[:, None].astype(np.float64) * freq[None, :]   # [tokens, half]
        c, s = np.cos(angle), np.sin(angle)
        if interleaved:
            i0 = start + 2 * k
            i1 = i0 + 1
        else:
            i0 = start + k
            i1 = i0 + half
        xa = x[:, :, tok][..., i0]
        xb = x[:, :, tok][..., i1]
        out[:, :, tok[:, None], i0[None, :]] = xa * c - xb * s
        out[:, :, tok[:, None], i1[None, :]] = xa * s + xb * c
        start += d
    return out
