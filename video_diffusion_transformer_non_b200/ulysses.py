"""Sequence-parallel attention across GPUs (DeepSpeed-Ulysses layout).

The vidax paper (§2, "Spatiotemporal tensor and sequence sharding") shards
video tokens across devices between attention layers and, for attention only,
transposes to a head-sharded view with all_to_all and back; CogVideoX1.5's
~45k-token joint sequence needs four such devices (§4 and Table 2).  Here:

* every rank holds q, k, v for its contiguous 1/P of the sequence and all H
  heads, bf16 [B, H, S/P, D], and its slice of the segment ids, int32 [B, S/P];
* one all_to_all per tensor gives each rank all S tokens of H/P heads
  (rank r gets heads [r H/P, (r+1) H/P)), the ids are all_gathered;
* the attention runs on that head shard through the library's C ABI
  (``vidattn_fwd_ex``), every key of the full sequence visible to every query;
* one all_to_all returns out [B, H, S/P, D] and lse [B, H, S/P] to the
  sequence-sharded layout.

With ``n_chunks > 1`` the heads of the shard are processed in chunks so the
exchange of one chunk overlaps the attention of the previous one (NCCL runs
the collectives on its own stream).  The collective is torch.distributed's
(NCCL over NVLink on GPUs, gloo on CPU for the tests); the data-path kernel is
vidattn's.  `attn_fn` replaces the attention call (tests on CPU).

The other attention forms go through the same exchange: a 3D neighbourhood
window (each rank's token coordinates are all-gathered like the ids) and the
3D rotary embedding, which is applied after the exchange, where each rank
holds the whole sequence of its heads, so positions are the global ones;
`rope_fn` replaces the rotation (tests on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


class _Exchange:
    """One all_to_all in flight and the layout change that follows it.

    `send` is contiguous with the destination rank outermost.  `recv` is
    where the collective lands (it may be the caller's final buffer, then
    `finish` is None and nothing is copied afterwards); `finish(recv)` makes
    the final layout (at most one copy)."""

    def __init__(self, send, recv, finish, P, group):
        self.recv, self.finish = recv, finish
        self.work = None
        if P > 1:
            self.work = dist.all_to_all_single(recv, send, group=group, async_op=True)
        elif recv.data_ptr() != send.data_ptr():
            recv.copy_(send)

    def result(self):
        if self.work is not None:
            self.work.wait()
        return self.recv if self.finish is None else self.finish(self.recv)


def _seq_to_heads(x: torch.Tensor, P: int, group) -> _Exchange:
    """[B, H, Sl, *r] sequence shard -> [B, H/P, P*Sl, *r] head shard.

    Copies: the send side is a view of x when B == 1 and x is contiguous (the
    rank-major order is then x's own), else one copy; the receive side is one
    copy, recv [P, B, H/P, Sl] -> [B, H/P, P, Sl], into the result."""
    B, H, Sl = x.shape[:3]
    rest = tuple(x.shape[3:])
    Hp = H // P
    send = x.reshape(B, P, Hp, Sl, *rest).movedim(1, 0)
    if not send.is_contiguous():
        send = send.contiguous()
    if P == 1:
        # nothing moves: the head shard is the sequence shard
        return _Exchange(send, send, lambda r: r.reshape(B, H, Sl, *rest), P, group)
    recv = torch.empty_like(send)

    def finish(r):
        out = torch.empty((B, Hp, P * Sl, *rest), dtype=x.dtype, device=x.device)
        # recv[p] = this rank's heads of sequence shard p
        out.view(B, Hp, P, Sl, *rest).copy_(r.permute(1, 2, 0, *range(3, 4 + len(rest))))
        return out

    return _Exchange(send, recv, finish, P, group)


def _heads_to_seq(y: torch.Tensor, P: int, group, dst: torch.Tensor) -> _Exchange:
    """[B, H/P, S, *r] head shard -> dst [B, H, S/P, *r] sequence shard.

    Copies: the send side is one copy, y [B, H/P, P, Sl] -> [P, B, H/P, Sl];
    the collective lands in dst directly when B == 1 (the receive order,
    source rank = head group outermost, is then dst's own), else in a buffer
    copied into dst once."""
    B, Hl, S = y.shape[:3]
    rest = tuple(y.shape[3:])
    Sl = S // P
    send = y.reshape(B, Hl, P, Sl, *rest).movedim(2, 0)
    if not send.is_contiguous():
        send = send.contiguous()
    direct = dst.reshape(B, P, Hl, Sl, *rest).movedim(1, 0)   # dst in receive order
    if direct.is_contiguous():
        return _Exchange(send, direct, None, P, group)
    recv = torch.empty_like(send)

    def finish(r):
        # recv[p] = this rank's sequence shard of head group p
        dst.view(B, P, Hl, Sl, *rest).copy_(r.movedim(0, 1))
        return dst

    return _Exchange(send, recv, finish, P, group)


def _cuda_attention(q, k, v, seg_q, seg_kv, scale, causal, window=None):
    if window is not None:
        return binding.attention_window(q, k, v, window["coords"], window["coords"],
                                        window["size"], window["extent"], window["clamped"],
                                        scale)
    return binding.attention(q, k, v, seg_q, seg_kv, scale, causal=causal)


def _cuda_rope(q, k, rope):
    # out of place: without an exchange (one rank) q and k are views of the
    # caller's tensors, which must not change
    return binding.rope3d(q, k, rope["grid"], rope["bands"], theta=rope.get("theta", 10000.0),
                          interleaved=rope.get("interleaved", True),
                          token_offset=rope.get("offset", 0))


def _all_gather_seq(x, P, group):
    """[B, S/P] per rank -> [B, S] in rank order."""
    if P == 1:
        return x.contiguous()
    parts = [torch.empty_like(x) for _ in range(P)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.cat(parts, dim=1).contiguous()


def ulysses_attention(q, k, v, seg=None, scale=None, causal=False, group=None, n_chunks=1,
                      attn_fn=None, window=None, rope=None, rope_fn=None):
    """Attention over a sequence sharded across the ranks of `group`.

    q, k, v: [B, H, S/P, D] (this rank's contiguous sequence shard; H divisible
    by P * n_chunks); seg: int32 [B, S/P] or None.  window: dict(coords=int32
    [B, S/P] packed t << 22 | h << 11 | w of this rank's tokens, size, extent,
    clamped) for 3D neighbourhood attention, or None.  rope: dict(grid, bands,
    theta, interleaved, offset) to rotate q and k (global positions) before
    the attention, or None.  Returns (out [B, H, S/P, D], lse fp32 [B, H, S/P])
    for this rank's shard, equal to the corresponding rows of single-device
    attention over the whole sequence.  Head chunk c's attention starts once
    its own inputs have arrived, while later chunks' exchanges are still in
    flight."""
    P = _world(group)
    B, H, Sl, D = q.shape
    if H % (P * n_chunks):
        raise ValueError(f"H={H} must be divisible by world size {P} x chunks {n_chunks}")
    if scale is None:
        scale = D ** -0.5
    if window is not None and (seg is not None or causal):
        raise ValueError("a window goes without ids and without the causal limit")
    attn = attn_fn or _cuda_attention
    turn = rope_fn or _cuda_rope
    seg_full = None if seg is None else _all_gather_seq(seg, P, group)
    win_full = None
    if window is not None:
        win_full = dict(window, coords=_all_gather_seq(window["coords"], P, group))
    Hc = H // n_chunks
    inputs = []
    for c in range(n_chunks):          # every input exchange goes out first
        hs = slice(c * Hc, (c + 1) * Hc)
        inputs.append([_seq_to_heads(t[:, hs], P, group) for t in (q, k, v)])
    # the results land in out and lse (allocated as the attention's results
    # are typed), chunk c in heads [c Hc, (c+1) Hc)
    out = lse = None
    pending = []
    for c in range(n_chunks):
        qh, kh, vh = (x.result() for x in inputs[c])
        if rope is not None:
            qh, kh = turn(qh, kh, rope)
        if win_full is not None:
            o, l = attn(qh, kh, vh, None, None, scale, False, window=win_full)
        else:
            o, l = attn(qh, kh, vh, seg_full, seg_full, scale, causal)
        if out is None:
            out = torch.empty((B, H, Sl, D), dtype=o.dtype, device=o.device)
            lse = torch.empty((B, H, Sl), dtype=l.dtype, device=l.device)
        hs = slice(c * Hc, (c + 1) * Hc)
        pending += [_heads_to_seq(o, P, group, out[:, hs]), _heads_to_seq(l, P, group, lse[:, hs])]
    for x in pending:
        x.result()
    return out, lse
