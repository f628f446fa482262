"""Sequence-parallel (Ulysses) attention: the all_to_all layout changes around
the attention call.  CPU: world size 2 and 4 with gloo, the fp64 oracle as the
per-shard attention, compared with the oracle on the whole sequence.  GPU: a
world of one over NCCL through the CUDA kernel, compared with vidattn_fwd."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_attn(q, k, v, seg_q, seg_kv, scale, causal):
    """Per-shard attention on the CPU for the test: the fp64 oracle on the
    bf16 inputs (bit patterns carried in float16-typed tensors)."""
    import oracle
    to_bits = lambda t: t.numpy().view(np.uint16)
    sq = None if seg_q is None else seg_q.numpy()
    sk = None if seg_kv is None else seg_kv.numpy()
    out, lse = oracle.attn_fwd(to_bits(q), to_bits(k), to_bits(v), sq, sk, scale, causal=causal)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _rank_main(rank, world, port, case, n_chunks, causal, q_out):
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        S = case["q"].shape[2]
        Sl = S // world
        sl = slice(rank * Sl, (rank + 1) * Sl)
        # bf16 bit patterns travel as a float16 view (the exchange never looks
        # at values; gloo has no 16-bit integer all_to_all)
        shard = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, sl]).view(np.float16))
        seg = None if case["seg_q"] is None else torch.from_numpy(
            np.ascontiguousarray(case["seg_q"][:, sl]))
        out, lse = ulysses_attention(shard(case["q"]), shard(case["k"]), shard(case["v"]), seg,
                                     case["scale"], causal, None, n_chunks, _oracle_attn)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n_chunks,with_ids,causal", [
    (2, 1, False, False), (2, 2, True, False), (4, 1, True, False), (2, 1, True, True),
])
def test_ulysses_matches_whole_sequence_attention(world, n_chunks, with_ids, causal):
    import oracle
    from video_diffusion_transformer_non_b200 import workloads as wl
    B, H, S, D = 2, 8, 96, 16
    seg = wl.segment_ids(((60, 0), (24, 1), (12, 2)), B) if with_ids else None
    case = wl.make_random(B, H, S, S, D, 61, seg, None if seg is None else seg.copy())
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, n_chunks, causal, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=60) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    out = np.concatenate([r[1] for r in res], axis=2)
    lse = np.concatenate([r[2] for r in res], axis=2)
    ro, rl = oracle.attn_fwd(case["q"], case["k"], case["v"], case["seg_q"], case["seg_kv"],
                             case["scale"], causal=causal)
    assert np.max(np.abs(out - ro)) <= 1e-12
    fin = np.isfinite(rl)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.max(np.abs(lse[fin] - rl[fin]), initial=0) <= 1e-12


def test_head_count_must_divide():
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    x = torch.zeros(1, 6, 8, 4, dtype=torch.int16)
    with pytest.raises(ValueError):
        ulysses_attention(x, x, x, n_chunks=4, attn_fn=_oracle_attn)


@pytest.mark.gpu
def test_ulysses_single_gpu_world_equals_kernel():
    """World of one over NCCL: the layout changes are identities and the result
    is bitwise the kernel's."""
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200 import binding
    from video_diffusion_transformer_non_b200 import workloads as wl
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        B, H, S, D = 1, 4, 700, 128
        seg = wl.segment_ids(((500, 0), (200, 1)), B)
        c = wl.make_random(B, H, S, S, D, 62, seg, seg.copy())
        up = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = up(c["q"]), up(c["k"]), up(c["v"])
        sg = torch.from_numpy(seg.copy()).cuda()
        o1, l1 = ulysses_attention(q, k, v, sg, c["scale"], n_chunks=2)
        o2, l2 = binding.attention(q, k, v, sg, sg, c["scale"])
        torch.cuda.synchronize()
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        assert torch.equal(l1, l2)
    finally:
        dist.destroy_process_group()
