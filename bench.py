"""Benchmark of the segment-masked attention forward on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one vidattn_fwd call (segment classification when ids are given,
then the attention kernel) over one batch of the chosen workload, inputs
already resident in HBM.  Default workload: video_720p (B1 H24 D128,
S = 119168 tokens: 118800 video, 256 text and 112 padding tokens in three
segments), the largest single-GPU configuration and one of the >=32k-token
configurations the >=60%-of-peak target is quoted on; video_480p and the
others are reachable with --workload.  Its inputs (~2.2 GB per step) are
larger than the 126 MB L2, so no flush is needed between steps.

Under torchrun (N > 1) every rank runs its own replica (independent problem,
seeded by rank): weak scaling, no collective on the data path.  Timing is on
the device with CUDA events, bracketed by a barrier and synchronisation, and
the max over ranks is reported.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the only place besides the cpu_baseline leg where
this script runs the oracle).
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bf16 video-DiT attention fwd TFLOP/s and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(bf16=float(d["bf16_tflops"]), bf16_sustained=float(d["bf16_tflops_sustained"]),
                    hbm=float(d["hbm_gbs"]), source="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# device sources of the kernels whose DRAM traffic profiles/ records
KERNEL_SOURCES = ["fwd_kernel.cuh", "ptx.cuh", "classify.cuh"]
ROPE_SOURCES = ["rope3d.cuh", "ptx.cuh"]


def code_only(src: str) -> str:
    """C++ source without comments and blank lines: what the compiler sees."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def measured_traffic(w, summary=None, sources=KERNEL_SOURCES):
    """DRAM bytes per launch from the committed ncu summary of this workload's
    kernel, or None when there is none or the kernel's code changed since
    (sha256 over its device sources with comments removed)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary or traffic_summary(w))
    if not os.path.exists(path):
        return None
    text = open(path).read()
    sha = re.search(r"kernel_sources_sha256:\s*([0-9a-f]{64})", text)
    val = re.search(r"traffic_bytes_per_full_launch:\s*(\d+)", text)
    if not sha or not val:
        return None
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "video_diffusion_transformer_non_b200", "csrc")
    for f in sources:
        with open(os.path.join(csrc, f)) as fh:
            h.update(code_only(fh.read()).encode())
    return int(val.group(1)) if h.hexdigest() == sha.group(1) else None


def traffic_summary(w, causal=False) -> str:
    """Name of the committed ncu summary that holds the DRAM traffic of this
    workload's attention launch (the causal limit has its own capture)."""
    return f"vidattn_fwd_kernel_d{w.D}__{w.name}{'_causal' if causal else ''}_h8.md"


def algorithmic_bytes(w) -> int:
    """Q, K, V read once, out and lse written once, segment ids read once."""
    b = 2 * w.B * w.H * w.D * (2 * w.S_q + 2 * w.S_kv) + 4 * w.B * w.H * w.S_q
    if w.segments is not None:
        b += 4 * w.B * (w.S_q + w.S_kv)
    return b


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampled every 20 ms while the timed region runs (read only:
    no clock or power setting is touched)."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 11:
                    continue
                if self.uuid and self.uuid not in parts[1]:
                    continue
                rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        util = [num(r[5]) or 0 for r in rows]
        loaded = [num(r[2]) for r, u in zip(rows, util) if u and u > 50 and num(r[2])]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, val in zip(names, r[7:11]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(loaded or sm), "sm_max_mhz": num(rows[0][3]),
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max((num(r[4]) or 0) for r in rows),
                "reasons": sorted(reasons)}


# -------------------------------------------------------------- reference

def oracle_rows_throughput(w, inputs, n_rows, seed=0, causal=False):
    """Time the fp64 oracle on n_rows random rows of the workload.
    Returns (TFLOP/s counted over allowed pairs of those rows, seconds, threads)."""
    import oracle
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = np.stack([rng.integers(0, w.B, n_rows), rng.integers(0, w.H, n_rows),
                     rng.integers(0, w.S_q, n_rows)], 1).astype(np.int64)
    lim = (lambda i: i + 1 + w.S_kv - w.S_q) if causal else (lambda i: w.S_kv)
    from video_diffusion_transformer_non_b200 import workloads as wl
    window = wl.window_of(w) if w.window is not None else None
    if window is not None:
        allowed = wl.window_row_counts(w, rows[:, 2])
    elif inputs["seg_q"] is not None:
        sq, sk = inputs["seg_q"], inputs["seg_kv"]
        allowed = np.array([int(np.count_nonzero(sk[b, :max(0, lim(i))] == sq[b, i]))
                            for b, _, i in rows])
    else:
        allowed = np.array([min(w.S_kv, max(0, lim(i))) for _, _, i in rows])
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.attn_rows(inputs["q"], inputs["k"], inputs["v"], rows, inputs["seg_q"],
                     inputs["seg_kv"], w.scale, nthreads=threads, causal=causal, window=window)
    dt = time.perf_counter() - t0
    flops = 4.0 * w.D * float(allowed.sum())
    return flops / dt / 1e12, dt, threads


def cpu_baseline(w, inputs, target_s=12.0, causal=False):
    """Oracle on a bounded sample sized to about target_s seconds of CPU work."""
    v, dt, thr = oracle_rows_throughput(w, inputs, 64, seed=1, causal=causal)
    n = int(max(64, min(200000, 64 * target_s / max(dt, 1e-3))))
    v, dt, thr = oracle_rows_throughput(w, inputs, n, seed=2, causal=causal)
    return {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{n} random (b,h,i) rows of {w.name} (all their allowed keys), "
                      f"fp64 oracle, {dt:.1f} s on {thr} threads"}


def run_reference(args, w, rank):
    if rank != 0:
        return 0
    from video_diffusion_transformer_non_b200 import workloads as wl
    inputs = wl.make_inputs(w)
    v, dt, thr = oracle_rows_throughput(w, inputs, 64, seed=1)
    # each step: a bounded sample, sized so warmup+steps take about
    # --ref-seconds (2 minutes by default)
    per_step_s = args.ref_seconds / max(1, args.steps + args.warmup)
    n = int(max(16, 64 * per_step_s / max(dt, 1e-3)))
    times, vals = [], []
    for s in range(args.warmup + args.steps):
        v, dt, thr = oracle_rows_throughput(w, inputs, n, seed=100 + s)
        if s >= args.warmup:
            times.append(dt)
            vals.append(v)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * float(np.mean(times)), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"each step {n} random rows of {w.name}, fp64 oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------- multi-rank logic

def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank_step: float, steps: int, world: int,
                       max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank ran `steps` steps of its own replica;
    the job took the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def rope_algorithmic_bytes(w) -> int:
    """q and k read once and written once, bf16."""
    return 2 * 2 * 2 * w.B * w.H * w.S_q * w.D


def workload_config(w, causal=False, rope=False):
    extra = {}
    if w.window is not None:
        extra = {"window": list(w.window), "volume": list(w.rope_grid),
                 "window_clamped": w.window_clamped, "token_order": "raster"}
    return {**extra, "workload": w.name + ("_causal" if causal else "") + ("_rope" if rope else ""),
            "B": w.B, "H": w.H, "S_q": w.S_q, "S_kv": w.S_kv, "D": w.D, "causal": causal,
            "segments": None if w.segments is None else [list(r) for r in w.segments],
            "description": w.description,
            "l2": "inputs larger than L2 (no flush)" if algorithmic_bytes(w) > 126e6
                  else "L2 flushed between steps",
            "parallelism": "replicas: one independent problem per GPU"}


# --------------------------------------------------------------------- ours

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=150)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="video_720p")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (smaller profiling cases)")
    ap.add_argument("--causal", action="store_true",
                    help="causal limit within segments (vidattn_fwd_ex, VIDATTN_CAUSAL)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: total oracle time budget")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rope", action="store_true",
                    help="each step rotates q and k (vidattn_rope3d, the workload's 3D RoPE "
                         "convention) before the attention")
    ap.add_argument("--split", type=int, default=0,
                    help="key splits per query block (VIDATTN_SPLIT_KV); 0: the library's choice")
    ap.add_argument("--rope-half-split", action="store_true",
                    help="with --rope: pair features k and k + d/2 instead of 2k and 2k+1")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from video_diffusion_transformer_non_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but {world} rank(s) were launched: for N > 1 run "
                 f"python -m torch.distributed.run --nproc-per-node N bench.py --gpus N")
    if args.impl == "reference":
        return run_reference(args, w, rank)

    import torch
    import torch.distributed as dist
    from video_diffusion_transformer_non_b200 import binding

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    lib = binding.load_library()
    inputs = wl.make_inputs(w, seed_offset=rank)
    up = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = up(inputs["q"]), up(inputs["k"]), up(inputs["v"])
    sq = None if inputs["seg_q"] is None else torch.from_numpy(inputs["seg_q"].copy()).to(dev)
    sk = None if inputs["seg_kv"] is None else torch.from_numpy(inputs["seg_kv"].copy()).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S_q), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    windowed = w.window is not None
    if windowed and (args.causal or args.rope):
        ap.error("window workloads run without --causal and --rope")
    if windowed:
        win = wl.window_of(w)
        cq = torch.from_numpy(win["coord_q"].copy()).to(dev)
        ck = torch.from_numpy(win["coord_kv"].copy()).to(dev)
        win_flags = binding.VIDATTN_WINDOW_CLAMPED if w.window_clamped else 0

    flags = (binding.VIDATTN_CAUSAL if args.causal else 0) | binding.VIDATTN_SPLIT_KV(args.split)
    use_rope = args.rope
    rope_interleaved = w.rope_interleaved and not args.rope_half_split
    # the attention reads the rotated q and k when the step includes the rotation
    qa, ka = (torch.empty_like(q), torch.empty_like(k)) if use_rope else (q, k)
    rope_ev = []     # (start, end) event pairs around each timed rotation launch

    def rope_launch():
        T, Hg, Wg = w.rope_grid
        d_t, d_h, d_w = w.rope_bands
        st = lib.vidattn_rope3d(q.data_ptr(), k.data_ptr(), qa.data_ptr(), ka.data_ptr(),
                                w.B, w.H, w.S_q, w.D, *q.stride()[:3], T, Hg, Wg, w.rope_offset,
                                d_t, d_h, d_w, w.rope_theta,
                                0 if rope_interleaved else binding.VIDATTN_ROPE_HALF_SPLIT, sh)
        if st != 0:
            raise RuntimeError(binding.status_string(st))

    def step(timed=False):
        if use_rope:
            if timed:
                e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                e[0].record(stream)
            rope_launch()
            if timed:
                e[1].record(stream)
                rope_ev.append(e)
        if windowed:
            st = lib.vidattn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), cq.data_ptr(),
                                        ck.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.H,
                                        w.S_q, w.S_kv, w.D, w.scale, *w.window, *w.rope_grid,
                                        win_flags, sh)
            if st != 0:
                raise RuntimeError(binding.status_string(st))
            return
        st = lib.vidattn_fwd_ex(qa.data_ptr(), ka.data_ptr(), v.data_ptr(),
                                None if sq is None else sq.data_ptr(),
                                None if sk is None else sk.data_ptr(),
                                out.data_ptr(), lse.data_ptr(), w.B, w.H, w.S_q, w.S_kv, w.D,
                                w.scale, flags, sh)
        if st != 0:
            raise RuntimeError(binding.status_string(st))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if binding.device_status() != 0:
        raise RuntimeError("device error during warm-up")

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier()
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for s in range(args.steps):
        step(timed=True)
        ev[s + 1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop() if sampler else None
    if binding.device_status() != 0:
        raise RuntimeError("device error during the timed region")
    per_step = [ev[s].elapsed_time(ev[s + 1]) for s in range(args.steps)]
    rope_ms = [a.elapsed_time(b) for a, b in rope_ev]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms_max = rank_max(total_ms)
    flops_step = wl.flops(w, causal=args.causal)
    value = weak_scaling_value(flops_step, args.steps, world, total_ms_max)
    ms_per_step = total_ms_max / args.steps

    # end to end through the host-buffer entry point: pinned inputs copied in,
    # forward, out and lse copied back, every step
    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(a if a.flags.writeable else a.copy()).pin_memory()
        hq, hk, hv = (pin(inputs[n].view(np.int16)) for n in ("q", "k", "v"))
        hsq = None if inputs["seg_q"] is None else pin(inputs["seg_q"])
        hsk = None if inputs["seg_kv"] is None else pin(inputs["seg_kv"])
        hout = torch.empty(out.shape, dtype=torch.int16).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        ptr = lambda t: None if t is None else t.data_ptr()

        hcq = pin(win["coord_q"]) if windowed else None
        hck = pin(win["coord_kv"]) if windowed else None

        def e2e_step_api():
            # pinned inputs in, the step's C-ABI calls, outputs back
            q.copy_(hq.view(torch.bfloat16), non_blocking=True)
            k.copy_(hk.view(torch.bfloat16), non_blocking=True)
            v.copy_(hv.view(torch.bfloat16), non_blocking=True)
            if hsq is not None:
                sq.copy_(hsq, non_blocking=True)
                sk.copy_(hsk, non_blocking=True)
            if windowed:
                cq.copy_(hcq, non_blocking=True)
                ck.copy_(hck, non_blocking=True)
            step()
            hout.copy_(out.view(torch.int16), non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        def e2e_step():
            if use_rope or windowed:
                return e2e_step_api()
            st = lib.vidattn_fwd_host(ptr(hq), ptr(hk), ptr(hv), ptr(hsq), ptr(hsk), ptr(hout),
                                      ptr(hlse), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      ptr(sq), ptr(sk), out.data_ptr(), lse.data_ptr(),
                                      w.B, w.H, w.S_q, w.S_kv, w.D, w.scale, sh)
            if st != 0:
                raise RuntimeError(binding.status_string(st))

        n_e2e = max(3, min(args.steps, 10))
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = rank_max(e0.elapsed_time(e1))
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsq, hsk, hcq, hck)
                  if t is not None)
        d2h = hout.numel() * 2 + hlse.numel() * 4
        e2e = {"value": weak_scaling_value(flops_step, n_e2e, world, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "ms_per_step": e_ms / n_e2e}

    peaks = load_peaks()
    # one attention launch (+ classify) per step, after the rotation when there is one
    kernel_ms = statistics.mean(per_step) - (statistics.mean(rope_ms) if rope_ms else 0.0)
    achieved = flops_step / (kernel_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"], "unit": UNIT,
                "frac": achieved / peaks["bf16"],
                "traffic": (measured_traffic(w, traffic_summary(w, args.causal))
                            if args.heads is None else None),
                "peak_source": f"{peaks['source']} bf16 dense (burst)",
                "frac_of_sustained": achieved / peaks["bf16_sustained"],
                "kernel": f"vidattn_fwd_kernel<{w.D}>",
                "algorithmic_flops_per_launch": flops_step,
                "algorithmic_bytes_per_launch": algorithmic_bytes(w)}

    rope = None
    if use_rope:
        r_ms = statistics.mean(rope_ms)
        r_bytes = rope_algorithmic_bytes(w)
        r_gbs = r_bytes / (r_ms * 1e-3) / 1e9
        rope = {"kernel": f"rope3d_kernel<{w.D}, {'interleaved' if rope_interleaved else 'half-split'}>",
                "ms_per_launch": r_ms, "ms_per_launch_min": min(rope_ms),
                "share_of_step": r_ms / statistics.mean(per_step),
                "convention": {"grid": list(w.rope_grid), "offset": w.rope_offset,
                               "bands": list(w.rope_bands), "theta": w.rope_theta,
                               "pairing": "interleaved" if rope_interleaved else "half-split"},
                "roofline": {"bound": "hbm", "achieved": r_gbs, "peak": peaks["hbm"],
                             "unit": "GB/s", "frac": r_gbs / peaks["hbm"],
                             "traffic": (measured_traffic(
                                 w, f"rope3d_kernel_d{w.D}__{w.name}.md", ROPE_SOURCES)
                                 if rope_interleaved and args.heads is None else None),
                             "peak_source": f"{peaks['source']} HBM copy",
                             "algorithmic_bytes_per_launch": r_bytes}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inputs, causal=args.causal)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, args.causal, rope=use_rope),
            "pct_of_bf16_peak": 100.0 * value / (world * peaks["bf16"]),
            "ms_per_step_min": min(per_step), "ms_per_step_median": statistics.median(per_step),
            "hbm_gbs": algorithmic_bytes(w) / (kernel_ms * 1e-3) / 1e9,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * (binding.kernels_per_call(
                sq, sk, w.B, w.H, w.S_q, w.S_kv, w.D, flags) + (1 if use_rope or windowed else 0)),
            "launch": (None if windowed else
                       binding.launch_plan(sq, w.B, w.H, w.S_q, w.S_kv, w.D, flags)),
            "rope3d": rope,
            "clocks": clocks,
        }
        if clocks and clocks.get("sm_mhz"):
            # the step's length in SM clock cycles at the median clock seen
            # under load: comparable across runs whose clocks differ
            clocks["mcycles_per_step"] = ms_per_step * 1e-3 * clocks["sm_mhz"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
