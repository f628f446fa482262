"""Sequence-parallel (Ulysses) attention: the all_to_all layout changes around
the attention call.  CPU: world size 2 and 4 with gloo, the fp64 oracle as the
per-shard attention, compared with the oracle on the whole sequence.  GPU:
(a) a world of one over NCCL through the CUDA kernel, compared with the
direct calls bit for bit and with the fp64 oracle under the parity
tolerances; (b) world size 2 as two processes exchanging over gloo, each
running its head shard's attention (and rotation) with the CUDA kernels on
the one GPU (independent launches: no kernel waits on another process),
compared with the fp64 oracle over the whole sequence, for B = 1 (the
exchange lands in the result directly) and B = 2 (through a buffer)."""
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
        import oracle
        from _gpu_helpers import compare
        for causal in (False, True):
            o1, l1 = ulysses_attention(q, k, v, sg, c["scale"], causal=causal, n_chunks=2)
            o2, l2 = binding.attention(q, k, v, sg, sg, c["scale"], causal=causal)
            torch.cuda.synchronize()
            assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
            assert torch.equal(l1, l2)
            ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], seg, seg.copy(), c["scale"],
                                     causal=causal)
            compare(o1.double().cpu().numpy(), l1.double().cpu().numpy(), ro, rl,
                    f"ulysses world 1, causal={causal}")
    finally:
        dist.destroy_process_group()


def _oracle_attn_win(q, k, v, seg_q, seg_kv, scale, causal, window=None):
    """Per-shard window attention on the CPU: the fp64 oracle's window rule."""
    import oracle
    to_bits = lambda t: t.numpy().view(np.uint16)
    c = window["coords"].numpy()
    win = dict(coord_q=c, coord_kv=c.copy(), size=window["size"], extent=window["extent"],
               clamped=window["clamped"])
    out, lse = oracle.attn_fwd(to_bits(q), to_bits(k), to_bits(v), None, None, scale,
                               window=win)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_rope(q, k, rope):
    """Per-shard rotation on the CPU: the fp64 oracle, rounded to bf16 as the
    kernel stores it (bit patterns carried in float16-typed tensors)."""
    from oracle.rope3d import rope3d_f64
    from video_diffusion_transformer_non_b200 import workloads as wl
    out = []
    for t in (q, k):
        r = rope3d_f64(t.numpy().view(np.uint16), rope["grid"], rope["bands"],
                       rope.get("theta", 10000.0), rope.get("interleaved", True),
                       rope.get("offset", 0))
        out.append(torch.from_numpy(wl.f32_to_bf16_bits(r.astype(np.float32)).view(np.float16)))
    return out[0], out[1]


def _rank_main_win(rank, world, port, case, coords, window, rope, n_chunks, q_out):
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        S = case["q"].shape[2]
        Sl = S // world
        sl = slice(rank * Sl, (rank + 1) * Sl)
        shard = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, sl]).view(np.float16))
        win = dict(window, coords=torch.from_numpy(np.ascontiguousarray(coords[:, sl])))
        out, lse = ulysses_attention(shard(case["q"]), shard(case["k"]), shard(case["v"]), None,
                                     case["scale"], False, None, n_chunks, _oracle_attn_win,
                                     window=win, rope=rope, rope_fn=_oracle_rope)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n_chunks,clamped", [(2, 1, True), (4, 2, False)])
def test_ulysses_window_with_rope_matches_whole_sequence(world, n_chunks, clamped):
    """3D neighbourhood attention of rotated q and k under sequence
    parallelism equals the whole-sequence computation (rotation at global
    positions, windows over all tokens)."""
    import oracle
    from oracle.rope3d import rope3d_f64
    from video_diffusion_transformer_non_b200 import workloads as wl
    grid, bands = (2, 4, 6), (4, 6, 6)
    B, H, D = 1, 8, 16
    S = int(np.prod(grid))
    case = wl.make_random(B, H, S, S, D, 62)
    coords = wl.raster_coords(grid, B)
    window = dict(size=(3, 3, 3), extent=grid, clamped=clamped)
    rope = dict(grid=grid, bands=bands, theta=10000.0, interleaved=True, offset=0)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_win,
                         args=(r, world, port, case, coords, window, rope, n_chunks, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=60) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    out = np.concatenate([r[1] for r in res], axis=2)
    lse = np.concatenate([r[2] for r in res], axis=2)
    rot = lambda x: wl.f32_to_bf16_bits(rope3d_f64(x, grid, bands).astype(np.float32))
    win = dict(coord_q=coords, coord_kv=coords.copy(), size=window["size"], extent=grid,
               clamped=clamped)
    ro, rl = oracle.attn_fwd(rot(case["q"]), rot(case["k"]), case["v"], scale=case["scale"],
                             window=win)
    assert np.max(np.abs(out - ro)) <= 1e-12
    assert np.max(np.abs(lse - rl)) <= 1e-12


@pytest.mark.gpu
def test_ulysses_single_gpu_window_with_rope_equals_direct_calls():
    """World of one over NCCL, window + rotary embedding: bitwise the RoPE
    pass followed by the window kernel."""
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200 import binding
    from video_diffusion_transformer_non_b200 import workloads as wl
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        grid, bands = (3, 8, 20), (44, 42, 42)
        B, H, D = 1, 4, 128
        S = int(np.prod(grid))
        c = wl.make_random(B, H, S, S, D, 63)
        up = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = up(c["q"]), up(c["k"]), up(c["v"])
        co = torch.from_numpy(wl.raster_coords(grid, B).copy()).cuda()
        window = dict(coords=co, size=(3, 5, 5), extent=grid, clamped=True)
        rope = dict(grid=grid, bands=bands)
        q0, k0 = q.clone(), k.clone()
        o1, l1 = ulysses_attention(q, k, v, None, c["scale"], n_chunks=2, window=window,
                                   rope=rope)
        torch.cuda.synchronize()
        assert torch.equal(q, q0) and torch.equal(k, k0)     # the inputs are left as they were
        qr, kr = binding.rope3d(q, k, grid, bands)
        o2, l2 = binding.attention_window(qr, kr, v, co, co, (3, 5, 5), grid, True, c["scale"])
        torch.cuda.synchronize()
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        assert torch.equal(l1, l2)
        # against the oracle: fp64 rotation rounded to bf16, then the window rule
        import oracle
        from oracle.rope3d import rope3d_f64
        from _gpu_helpers import compare
        rot = lambda x: wl.f32_to_bf16_bits(rope3d_f64(x, grid, bands).astype(np.float32))
        coords = wl.raster_coords(grid, B)
        win = dict(coord_q=coords, coord_kv=coords.copy(), size=(3, 5, 5), extent=grid,
                   clamped=True)
        ro, rl = oracle.attn_fwd(rot(c["q"]), rot(c["k"]), c["v"], scale=c["scale"], window=win)
        compare(o1.double().cpu().numpy(), l1.double().cpu().numpy(), ro, rl,
                "ulysses world 1, window + rope")
    finally:
        dist.destroy_process_group()


# --------------------------------------------- world 2 over gloo, CUDA per rank

def _to_gpu_bf16(t):
    """bf16 bit patterns carried in a float16-typed CPU tensor -> bf16 on cuda:0."""
    return t.contiguous().view(torch.bfloat16).cuda()


def _from_gpu_bf16(t):
    return t.cpu().view(torch.float16)


def _cuda_attn_gloo(q, k, v, seg_q, seg_kv, scale, causal, window=None):
    """A rank's head-shard attention with the CUDA kernel; the exchange around
    it stays on the CPU (gloo), in float16-typed tensors holding bf16 bits."""
    from video_diffusion_transformer_non_b200 import binding
    qd, kd, vd = _to_gpu_bf16(q), _to_gpu_bf16(k), _to_gpu_bf16(v)
    if window is not None:
        co = window["coords"].cuda()
        o, l = binding.attention_window(qd, kd, vd, co, co, window["size"], window["extent"],
                                        window["clamped"], scale)
    else:
        sq = None if seg_q is None else seg_q.cuda()
        o, l = binding.attention(qd, kd, vd, sq, sq, scale, causal=causal)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    return _from_gpu_bf16(o), l.cpu()


def _cuda_rope_gloo(q, k, rope):
    from video_diffusion_transformer_non_b200 import binding
    qr, kr = binding.rope3d(_to_gpu_bf16(q), _to_gpu_bf16(k), rope["grid"], rope["bands"],
                            theta=rope.get("theta", 10000.0))
    torch.cuda.synchronize()
    return _from_gpu_bf16(qr), _from_gpu_bf16(kr)


def _rank_main_cuda(rank, world, port, case, coords, opts, q_out):
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200.ulysses import ulysses_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        S = case["q"].shape[2]
        Sl = S // world
        sl = slice(rank * Sl, (rank + 1) * Sl)
        shard = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, sl]).view(np.float16))
        seg = None if case["seg_q"] is None else torch.from_numpy(
            np.ascontiguousarray(case["seg_q"][:, sl]))
        win = None
        if opts.get("window") is not None:
            win = dict(opts["window"], coords=torch.from_numpy(np.ascontiguousarray(coords[:, sl])))
        out, lse = ulysses_attention(shard(case["q"]), shard(case["k"]), shard(case["v"]), seg,
                                     case["scale"], opts.get("causal", False), None,
                                     opts["n_chunks"], _cuda_attn_gloo, window=win,
                                     rope=opts.get("rope"), rope_fn=_cuda_rope_gloo)
        q_out.put((rank, out.view(torch.bfloat16).double().numpy(), lse.double().numpy()))
    finally:
        dist.destroy_process_group()


def _run_world(world, case, coords, opts):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_cuda, args=(r, world, port, case, coords, opts, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return (np.concatenate([r[1] for r in res], axis=2),
            np.concatenate([r[2] for r in res], axis=2))


@pytest.mark.gpu
@pytest.mark.parametrize("B,causal", [(1, False), (2, True)])
def test_ulysses_world2_cuda_attention_matches_oracle(B, causal):
    """Two ranks exchange over gloo; each runs its head shard on the GPU with
    the CUDA kernel (ids, optionally the causal limit, two head chunks); the
    gathered shards match the fp64 oracle over the whole sequence."""
    import oracle
    from _gpu_helpers import compare
    from video_diffusion_transformer_non_b200 import workloads as wl
    H, D = 8, 128
    seg = wl.segment_ids(((900, 0), (200, 1), (100, 2)), B)
    S = seg.shape[1]
    case = wl.make_random(B, H, S, S, D, 64, seg, seg.copy())
    out, lse = _run_world(2, case, None, dict(n_chunks=2, causal=causal))
    ro, rl = oracle.attn_fwd(case["q"], case["k"], case["v"], seg, seg.copy(), case["scale"],
                             causal=causal)
    compare(out, lse, ro, rl, f"ulysses world 2 (gloo), CUDA attention, B={B}")


@pytest.mark.gpu
def test_ulysses_world2_cuda_window_with_rope_matches_oracle():
    """The same with the 3D RoPE pass (global positions) and a clamped 3D
    neighbourhood window, both on the GPU per rank."""
    import oracle
    from oracle.rope3d import rope3d_f64
    from _gpu_helpers import compare
    from video_diffusion_transformer_non_b200 import workloads as wl
    grid, bands = (4, 8, 20), (44, 42, 42)
    B, H, D = 1, 4, 128
    S = int(np.prod(grid))
    case = wl.make_random(B, H, S, S, D, 65)
    coords = wl.raster_coords(grid, B)
    window = dict(size=(3, 5, 5), extent=grid, clamped=True)
    out, lse = _run_world(2, case, coords, dict(n_chunks=2, window=window,
                                                rope=dict(grid=grid, bands=bands)))
    rot = lambda x: wl.f32_to_bf16_bits(rope3d_f64(x, grid, bands).astype(np.float32))
    win = dict(coord_q=coords, coord_kv=coords.copy(), size=(3, 5, 5), extent=grid, clamped=True)
    ro, rl = oracle.attn_fwd(rot(case["q"]), rot(case["k"]), case["v"], scale=case["scale"],
                             window=win)
    compare(out, lse, ro, rl, "ulysses world 2 (gloo), CUDA window + rope")
