"""Host logic of the multi-GPU benchmark path, on CPU: two `gloo` ranks take
the max of their timings and compute the weak-scaling (replica) value; the
reference arm runs on rank 0 only and prints the contract's line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(times[rank], world)
        v = bench.weak_scaling_value(2.0e12, 10, world, m)
        out_q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_gloo():
    world = 2
    times = [120.0, 150.0]      # ms for 10 steps on each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, v in res:
        assert m == 150.0
        # 2 ranks x 10 steps x 2e12 FLOP in 0.150 s = 266.67 TFLOP/s
        assert abs(v - 2 * 10 * 2.0e12 / 0.150 / 1e12) < 1e-9


def test_single_rank_shortcuts():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert abs(bench.weak_scaling_value(1e12, 4, 1, 1000.0) - 4.0) < 1e-12


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank0_prints_contract_line():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                    "--warmup", "3", "--ref-seconds", "2"], {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["higher_is_better"] is True


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--workload", "video_720p",
                    "--steps", "2", "--warmup", "3"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_warmup_below_three_is_rejected():
    r = _run_bench(["--warmup", "2"], {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode != 0
