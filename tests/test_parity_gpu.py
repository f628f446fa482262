"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small and medium cases compare every row; the full-size workloads compare a
seeded sample of rows (rows are independent, so each sampled row is an exact
check of that row).  Tolerances: max |dout| <= 2e-2, mean |dout| <= 2e-3,
|dlse| <= 1e-3; rows that see no key must give out == 0 and lse == -inf
exactly.  Every call also checks guard regions around out and lse and that no
output element is left unwritten."""
import numpy as np
import pytest
import torch

import oracle
from video_diffusion_transformer_non_b200 import binding
from video_diffusion_transformer_non_b200 import workloads as wl

from _gpu_helpers import (bf16_to_f64, check_all_rows, compare, run_gpu, sample_rows,
                          to_dev_bf16, to_dev_i32)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------ shapes, no ids

@pytest.mark.parametrize("n_split", [0, 1])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B,H,S_q,S_kv", [
    (1, 1, 1, 1), (1, 2, 128, 128), (1, 2, 127, 129), (2, 2, 129, 127),
    (1, 3, 300, 77), (1, 2, 256, 1000), (2, 1, 513, 384), (1, 1, 640, 2053),
])
def test_shapes_single_segment(B, H, S_q, S_kv, D, n_split):
    """n_split 0: the launch's own choice (these short calls mostly split
    their keys); 1: no split, every key tile of a query block in one unit."""
    c = wl.make_random(B, H, S_q, S_kv, D, seed=S_q * 7 + S_kv + D)
    check_all_rows(c, what=f"B{B} H{H} Sq{S_q} Skv{S_kv} D{D} split {n_split}",
                   flags=binding.VIDATTN_SPLIT_KV(n_split))


# ------------------------------------------------------------- key splits
# The launch splits each 256-row query block's keys into ranges when a call
# has few query blocks (vidattn_split_count); VIDATTN_SPLIT_KV(n) forces n.
# Every count must give the oracle's result: splits with no key, splits of
# one tile, ids whose rows see no key of a split, the causal limit.

@pytest.mark.parametrize("n_split", [1, 2, 3, 5, 8, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_key_splits_single_segment(n_split, D):
    c = wl.make_random(1, 2, 640, 1100, D, seed=900 + n_split + D)
    check_all_rows(c, what=f"split {n_split} D{D}", flags=binding.VIDATTN_SPLIT_KV(n_split))


@pytest.mark.parametrize("n_split", [1, 2, 7])
def test_key_splits_with_ids(n_split):
    c = runs_case(2, 3, ((700, 0), (140, 1), (37, 2)), 128, 34)
    check_all_rows(c, what=f"ids, split {n_split}", flags=binding.VIDATTN_SPLIT_KV(n_split))


@pytest.mark.parametrize("n_split", [1, 3])
def test_key_splits_causal(n_split):
    c = wl.make_random(1, 2, 300, 1000, 128, seed=35)
    check_all_rows(c, what=f"causal, split {n_split}", causal=True,
                   flags=binding.VIDATTN_SPLIT_KV(n_split))


def test_key_splits_more_than_key_tiles():
    """Two key tiles split five ways: three ranges are empty."""
    c = wl.make_random(1, 1, 200, 129, 64, seed=36)
    check_all_rows(c, what="split 5 over 2 tiles", flags=binding.VIDATTN_SPLIT_KV(5))


def test_auto_split_long_keys():
    """A few query blocks over many keys (4 units, 64 key tiles): the
    heuristic splits the keys 8 ways; the result matches the oracle and the
    unsplit launch to within bf16 rounding."""
    c = wl.make_random(1, 2, 512, 8192, 64, seed=37)
    assert binding.split_count(None, 1, 2, 512, 8192) == 8
    o1, l1 = run_gpu(c)
    ro, rl = oracle.attn_fwd(c["q"], c["k"], c["v"], None, None, c["scale"])
    compare(bf16_to_f64(o1), l1.double().cpu().numpy(), ro, rl, "auto split 8")
    o2, l2 = run_gpu(c, flags=binding.VIDATTN_SPLIT_KV(1))
    d = (o1.double() - o2.double()).abs()
    assert float(d.max()) <= 1e-2 and float((l1 - l2).abs().max()) <= 1e-4


def test_launch_plan_matches_the_heuristic():
    """What vidattn_launch_plan reports for the workloads (148 SMs)."""
    seg = np.zeros((2, 4389), np.int32)
    sq = to_dev_i32(seg)
    plan = binding.launch_plan
    assert plan(None, 1, 2, 512, 512, 64) == dict(grid_ctas=4, key_splits=1, persistent=False)
    assert plan(sq, 2, 12, 4389, 4389, 128) == dict(grid_ctas=148, key_splits=1, persistent=True)
    assert plan(None, 1, 40, 32760, 32760, 128) == dict(grid_ctas=5120, key_splits=1,
                                                        persistent=False)
    assert plan(None, 2, 48, 17792, 17792, 64) == dict(grid_ctas=6720, key_splits=1,
                                                       persistent=False)
    assert plan(None, 1, 2, 512, 131072, 128) == dict(grid_ctas=64, key_splits=16,
                                                      persistent=False)


# ------------------------------------------------ persistent launches
# Many short units (more than the 148 SMs, few key tiles each): the launch
# is persistent, so every CTA carries its barrier phases, Q buffers and
# tile lists across several units.

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", ["plain", "ids", "causal"])
def test_persistent_many_short_units(D, mode):
    B, H, S = 2, 40, 1000       # 2 x 40 x 4 = 320 units of 8 key tiles
    seg = None
    if mode == "ids":
        seg = wl.segment_ids(((700, 0), (200, 1), (100, 2)), B)
    c = wl.make_random(B, H, S, S, D, 38 + D, seg, None if seg is None else seg.copy())
    check_all_rows(c, what=f"persistent {mode} D{D}", causal=(mode == "causal"))


# ----------------------------------------------------------- segment layouts

def runs_case(B, H, runs, D, seed):
    seg = wl.segment_ids(runs, B)
    S = seg.shape[1]
    return wl.make_random(B, H, S, S, D, seed, seg, seg.copy())


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("n_split", [0, 1])
def test_video_text_pad_segments(D, n_split):
    c = runs_case(2, 3, ((700, 0), (140, 1), (37, 2)), D, 31)
    check_all_rows(c, what=f"video/text/pad split {n_split}", flags=binding.VIDATTN_SPLIT_KV(n_split))


@pytest.mark.parametrize("D", [64, 128])
def test_text_and_video_shared_id_with_pad(D):
    c = runs_case(1, 2, ((600, 0), (26, 0), (14, 1)), D, 32)
    check_all_rows(c, what="shared id + pad")


def test_alternating_ids_every_tile_mixed():
    B, H, S, D = 1, 2, 515, 128
    seg = (np.arange(S) % 2).astype(np.int32)[None]
    c = wl.make_random(B, H, S, S, D, 33, seg, seg.copy())
    check_all_rows(c, what="alternating")


def test_ids_differ_between_samples_and_random_ids():
    B, H, S, D = 3, 2, 400, 64
    rng = np.random.Generator(np.random.PCG64(34))
    seg_q = np.stack([np.sort(rng.integers(0, 4, S)), rng.integers(0, 3, S),
                      np.full(S, 7)]).astype(np.int32)
    seg_kv = np.stack([np.sort(rng.integers(0, 4, S)), rng.integers(0, 3, S),
                       np.where(np.arange(S) < 200, 7, 8)]).astype(np.int32)
    c = wl.make_random(B, H, S, S, D, 34, seg_q, seg_kv)
    check_all_rows(c, what="per-sample ids")


def test_rows_with_no_visible_key():
    B, H, S_q, S_kv, D = 1, 2, 300, 260, 128
    seg_q = np.where(np.arange(S_q) < 150, 5, 9).astype(np.int32)[None]   # id 9 absent
    seg_kv = np.full((1, S_kv), 5, np.int32)
    c = wl.make_random(B, H, S_q, S_kv, D, 35, seg_q, seg_kv)
    stats = check_all_rows(c, what="empty rows")
    assert stats
    # a whole CTA with no visible key
    seg_q2 = np.full((1, S_q), 3, np.int32)
    c2 = wl.make_random(B, H, S_q, S_kv, D, 36, seg_q2, seg_kv)
    out, lse = run_gpu(c2)
    assert bool((out.float() == 0).all()) and bool(torch.isneginf(lse).all())


def test_large_negative_and_positive_ids():
    B, H, S, D = 1, 1, 384, 64
    ids = np.array([-2 ** 31, 2 ** 31 - 1, 0], np.int64)
    seg = ids[(np.arange(S) // 128) % 3].astype(np.int32)[None]
    c = wl.make_random(B, H, S, S, D, 37, seg, seg.copy())
    check_all_rows(c, what="extreme ids")


# ------------------------------------------------------------------ scales

@pytest.mark.parametrize("scale", [0.0, -0.125, 0.5, 1e-3])
def test_scales(scale):
    c = wl.make_random(1, 2, 300, 400, 128, 38)
    check_all_rows(c, scale=scale, what=f"scale {scale}")


def test_peaked_softmax_with_head_scaling():
    """q and k scaled by 2 each, v ~ N(0,1) (the extreme of the 480p
    workload's per-head scaling): near one-hot rows."""
    c = wl.make_random(1, 2, 512, 1024, 128, 39)
    for n in ("q", "k"):
        c[n] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(c[n]) * np.float32(2.0))
    check_all_rows(c, what="peaked")


@pytest.mark.parametrize("n_split", [0, 1])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("with_ids", [False, True])
@pytest.mark.parametrize("pattern", ["per_tile", "within_tile"])
def test_running_offset_overflow_takes_exact_path(D, with_ids, pattern, n_split):
    """Keys scaled so that scores grow along the sequence: the offset a row
    takes from its first key tile goes stale by far more than 2^32 in P, and
    the kernel must fall back to the exact path (tile max, rescale of O and
    the row sum) and still match the oracle.  per_tile: 128-key tiles scaled
    0.05x .. 16x (the whole tile overflows).  within_tile: 64-key halves
    scaled so that only the second half of a tile overflows.  n_split 1
    keeps every key tile of a row in one unit (the launch would split this
    short call otherwise, 0), so the running offset meets the later tiles."""
    B, H, S_q, S_kv = 1, 2, 300, 640
    rng = np.random.Generator(np.random.PCG64(46 + D))
    q = rng.standard_normal((B, H, S_q, D), dtype=np.float32)
    k = rng.standard_normal((B, H, S_kv, D), dtype=np.float32)
    v = rng.standard_normal((B, H, S_kv, D), dtype=np.float32)
    if pattern == "per_tile":
        blocks, factors = 128, [0.05, 0.5, 2.0, 8.0, 16.0]
    else:
        blocks, factors = 64, [0.05, 0.05, 0.5, 0.5, 2.0, 2.0, 2.0, 8.0, 8.0, 16.0]
    for j, f in enumerate(factors):
        k[:, :, blocks * j:blocks * (j + 1)] *= np.float32(f)
    c = dict(q=wl.f32_to_bf16_bits(q), k=wl.f32_to_bf16_bits(k), v=wl.f32_to_bf16_bits(v),
             seg_q=None, seg_kv=None, scale=1.0 / np.sqrt(D))
    if with_ids:   # one id everywhere: the listed-tile path, same result
        c["seg_q"] = np.zeros((B, S_q), np.int32)
        c["seg_kv"] = np.zeros((B, S_kv), np.int32)
    check_all_rows(c, what=f"stale offset {pattern} D{D} ids={with_ids} split={n_split}",
                   flags=binding.VIDATTN_SPLIT_KV(n_split))


def test_scale_zero_with_segments_gives_segment_means():
    c = runs_case(1, 2, ((200, 0), (100, 1), (20, 2)), 128, 40)
    check_all_rows(c, scale=0.0, what="scale 0 + ids")


# ------------------------------------- more than 2048 key tiles with ids

@pytest.mark.parametrize("causal", [False, True])
def test_ids_beyond_the_listed_tile_limit(causal):
    """S_kv > 262144 (2048 key tiles) with ids: the roles walk the tile
    summaries in global memory instead of a shared-memory list.  Queries
    from every key segment plus an absent id; all rows against the oracle."""
    B, H, D = 1, 2, 64
    S_kv = 270000
    seg_kv = np.concatenate([np.full(100000, 0), np.full(150000, 1),
                             np.full(S_kv - 250000, 2)]).astype(np.int32)[None]
    S_q = 600 if causal else 300
    seg_q = np.array([0, 1, 2, 7])[np.arange(S_q) * 4 // S_q].astype(np.int32)[None]
    c = wl.make_random(B, H, S_q, S_kv, D, 48, seg_q, seg_kv)
    check_all_rows(c, what=f"beyond listed tiles causal={causal}", causal=causal)


def test_ids_beyond_the_listed_tile_limit_two_samples():
    B, H, D, S_q, S_kv = 2, 1, 128, 256, 263000
    seg_kv = np.zeros((B, S_kv), np.int32)
    seg_kv[0, 200000:] = 1
    seg_kv[1, :1000] = 1
    seg_q = np.zeros((B, S_q), np.int32)
    seg_q[:, S_q // 2:] = 1
    c = wl.make_random(B, H, S_q, S_kv, D, 49, seg_q, seg_kv)
    check_all_rows(c, what="beyond listed tiles, B=2")


# -------------------------------------------------------------- edge cases

def test_empty_key_sequence():
    c = wl.make_random(1, 2, 200, 0, 64, 41)
    out, lse = run_gpu(c)
    assert bool((out.float() == 0).all()) and bool(torch.isneginf(lse).all())


def test_empty_query_sequence_is_a_no_op():
    q = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 10, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(4, dtype=torch.float32, device="cuda")
    assert binding.vidattn_fwd(k, k, k, None, None, out, lse, 1, 2, 0, 10, 64, 0.1) == 0
    torch.cuda.synchronize()


def test_deterministic():
    c = runs_case(2, 2, ((500, 0), (60, 1), (9, 2)), 128, 42)
    o1, l1 = run_gpu(c)
    o2, l2 = run_gpu(c)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_host_buffer_entry_point_matches_device_entry_point():
    c = runs_case(1, 2, ((300, 0), (50, 1), (10, 2)), 128, 43)
    out_d, lse_d = run_gpu(c)
    B, H, S, D = c["q"].shape
    pin = lambda a: torch.from_numpy(a if a.flags.writeable else a.copy()).pin_memory()
    hq, hk, hv = (pin(c[n].view(np.int16)) for n in ("q", "k", "v"))
    hsq, hsk = pin(c["seg_q"]), pin(c["seg_kv"])
    hout = torch.empty((B, H, S, D), dtype=torch.int16).pin_memory()
    hlse = torch.empty((B, H, S), dtype=torch.float32).pin_memory()
    dq, dk, dv = (torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    dsq, dsk = (torch.empty((B, S), dtype=torch.int32, device="cuda") for _ in range(2))
    dout = torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda")
    dlse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    st = binding.vidattn_fwd_host(hq, hk, hv, hsq, hsk, hout, hlse, dq, dk, dv, dsq, dsk,
                                  dout, dlse, B, H, S, S, D, c["scale"])
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(hout, out_d.view(torch.int16).cpu())
    assert torch.equal(hlse, lse_d.cpu())


@pytest.mark.parametrize("with_ids,S_q,S_kv", [(True, 8192, 8192), (False, 6000, 9000)])
def test_pipelined_host_entry_point_matches_device_entry_point(with_ids, S_q, S_kv):
    """Over 64 MiB of copies: vidattn_fwd_host pipelines chunks of heads
    (B = 2, H = 5: chunks of 2, 2 and 1 heads per batch entry) across its
    copy streams; the outputs equal the device entry point's bit for bit."""
    B, H, D = 2, 5, 128
    seg_q = seg_kv = None
    if with_ids:
        seg_q = np.zeros((B, S_q), np.int32)
        seg_q[:, S_q - 300:] = 1
        seg_q[1, :1000] = 2
        seg_kv = seg_q.copy()
    c = wl.make_random(B, H, S_q, S_kv, D, 44, seg_q, seg_kv)
    out_d, lse_d = run_gpu(c, check=False)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hq, hk, hv = (pin(c[n].view(np.int16)) for n in ("q", "k", "v"))
    hsq = hsk = dsq = dsk = None
    if with_ids:
        hsq, hsk = pin(c["seg_q"]), pin(c["seg_kv"])
        dsq = torch.empty((B, S_q), dtype=torch.int32, device="cuda")
        dsk = torch.empty((B, S_kv), dtype=torch.int32, device="cuda")
    hout = torch.empty((B, H, S_q, D), dtype=torch.int16).pin_memory()
    hlse = torch.empty((B, H, S_q), dtype=torch.float32).pin_memory()
    dq = torch.empty((B, H, S_q, D), dtype=torch.bfloat16, device="cuda")
    dk, dv = (torch.empty((B, H, S_kv, D), dtype=torch.bfloat16, device="cuda") for _ in range(2))
    dout = torch.empty_like(dq)
    dlse = torch.empty((B, H, S_q), dtype=torch.float32, device="cuda")
    st = binding.vidattn_fwd_host(hq, hk, hv, hsq, hsk, hout, hlse, dq, dk, dv, dsq, dsk,
                                  dout, dlse, B, H, S_q, S_kv, D, c["scale"])
    assert st == 0
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    assert torch.equal(hout, out_d.view(torch.int16).cpu())
    assert torch.equal(hlse, lse_d.cpu())


def test_kernel_wait_timeout_is_reported_not_hung():
    """A kernel whose barrier never completes gives up after its time limit and
    reports through the device error word; the context stays usable."""
    assert binding.device_status() == 0
    assert binding.selftest_timeout(20000) == 0
    assert binding.device_status() == 6          # VIDATTN_ERR_TIMEOUT
    assert binding.device_status() == 0          # cleared
    c = wl.make_random(1, 1, 128, 128, 64, 44)
    check_all_rows(c, what="after timeout")


def test_streams_other_than_the_current_one():
    c = runs_case(1, 2, ((260, 0), (40, 1)), 64, 45)
    ref_out, ref_lse = run_gpu(c)
    s = torch.cuda.Stream()
    q, k, v = (to_dev_bf16(c[n]) for n in ("q", "k", "v"))
    sq, sk = to_dev_i32(c["seg_q"]), to_dev_i32(c["seg_kv"])
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out, lse = binding.attention(q, k, v, sq, sk, c["scale"], stream=s)
    s.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse, ref_lse)


# ------------------------------------------------------------------ causal

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S_q,S_kv", [(128, 128), (300, 300), (257, 513), (513, 257),
                                      (1000, 1000), (100, 700)])
@pytest.mark.parametrize("n_split", [0, 1])
def test_causal_shapes(S_q, S_kv, D, n_split):
    c = wl.make_random(2, 2, S_q, S_kv, D, seed=S_q + 3 * S_kv + D)
    check_all_rows(c, causal=True, what=f"causal Sq{S_q} Skv{S_kv} D{D} split {n_split}",
                   flags=binding.VIDATTN_SPLIT_KV(n_split))


@pytest.mark.parametrize("D", [64, 128])
def test_causal_with_segments(D):
    c = runs_case(2, 2, ((500, 3), (300, 1), (77, 5)), D, 47)
    check_all_rows(c, causal=True, what=f"causal + ids D{D}")
    rng = np.random.Generator(np.random.PCG64(48))
    seg = rng.integers(0, 3, (1, 640)).astype(np.int32)
    c = wl.make_random(1, 2, 640, 640, D, 49, seg, seg.copy())
    check_all_rows(c, causal=True, what=f"causal + random ids D{D}")


def test_causal_full_size_480p_sampled_rows():
    w = wl.WORKLOADS["video_480p"]
    c = wl.make_inputs(w)
    out, lse = run_gpu(c, causal=True)
    rows = sample_rows(w.B, w.H, w.S_q, None, n_random=1024, n_heads_full=2)
    ro, rl = oracle.attn_rows(c["q"], c["k"], c["v"], rows, None, None, c["scale"], causal=True)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    idx = torch.from_numpy(((b * w.H + h) * w.S_q + i).astype(np.int64)).cuda()
    compare(bf16_to_f64(out.reshape(-1, w.D)[idx]), lse.reshape(-1)[idx].double().cpu().numpy(),
            ro, rl, what="causal 480p")


# ---------------------------------------------------- the named workloads

def test_workload_tiny_all_rows():
    w = wl.WORKLOADS["tiny"]
    check_all_rows(wl.make_inputs(w), what=w.name)


def test_workload_joint_small_all_rows():
    w = wl.WORKLOADS["joint_small"]
    check_all_rows(wl.make_inputs(w), what=w.name)


@pytest.mark.parametrize("name", ["video_480p", "cogvideox_joint", "video_720p"])
def test_full_size_workload_sampled_rows(name):
    w = wl.WORKLOADS[name]
    c = wl.make_inputs(w)
    out, lse = run_gpu(c)
    rows = sample_rows(w.B, w.H, w.S_q, w.segments, n_random=4096, n_heads_full=8, seed=0)
    ro, rl = oracle.attn_rows(c["q"], c["k"], c["v"], rows, c["seg_q"], c["seg_kv"], c["scale"])
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    idx = torch.from_numpy(((b * w.H + h) * w.S_q + i).astype(np.int64)).cuda()
    og = bf16_to_f64(out.reshape(-1, w.D)[idx])
    lg = lse.reshape(-1)[idx].double().cpu().numpy()
    compare(og, lg, ro, rl, what=name)
