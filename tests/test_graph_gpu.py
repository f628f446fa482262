"""CUDA graph capture of the library's calls (the header's capture rules:
after a first call of the largest shape on the capturing stream, the entry
points only enqueue kernel launches).  A graph holding the 3D RoPE pass and
the attention with segment ids (and, in the second case, a split launch with
its merge) is captured on a side stream, replayed twice, and must equal the
direct calls bit for bit."""
import numpy as np
import pytest
import torch

from video_diffusion_transformer_non_b200 import binding
from video_diffusion_transformer_non_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S_kv,n_split", [(700, 0), (4096, 8)])
def test_graph_replay_equals_direct_calls(S_kv, n_split):
    B, H, S_q, D = 1, 4, 700, 128
    seg_q = wl.segment_ids(((500, 0), (200, 1)), B)
    seg_kv = np.zeros((B, S_kv), np.int32)
    seg_kv[:, S_kv - 200:] = 1
    c = wl.make_random(B, H, S_q, S_kv, D, 81, seg_q, seg_kv)
    up = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = up(c["q"]), up(c["k"]), up(c["v"])
    sq = torch.from_numpy(seg_q.copy()).cuda()
    sk = torch.from_numpy(seg_kv.copy()).cuda()
    grid, bands = (5, 10, 10), (44, 42, 42)
    flags = binding.VIDATTN_SPLIT_KV(n_split)
    qr, kr = torch.empty_like(q), torch.empty_like(k)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device="cuda")

    def step(stream):
        h = stream.cuda_stream
        for x, y, S in ((q, qr, S_q), (k, kr, S_kv)):
            st = binding.vidattn_rope3d(x, None, y, None, B, H, S, D, *x.stride()[:3], *grid, 0,
                                        *bands, 10000.0, 0, h)
            assert st == 0
        st = binding.vidattn_fwd_ex(qr, kr, v, sq, sk, out, lse, B, H, S_q, S_kv, D,
                                    c["scale"], flags, h)
        assert st == 0

    # direct calls on the default stream
    step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    ref_out, ref_lse = out.clone(), lse.clone()
    if n_split:
        assert binding.split_count(sq, B, H, S_q, S_kv, flags) == n_split

    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        step(side)                       # set-up call on the capturing stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(side)
    for _ in range(2):
        out.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
