"""Host logic of bench.py on the CPU: the algorithmic byte counts behind the
roofline, the workload config of the JSON line, and the rule that a recorded
DRAM traffic figure is reported only while the kernel's code (comments
aside) is the code that was captured."""
import hashlib
import os

import pytest

import bench
from video_diffusion_transformer_non_b200 import workloads as wl


def test_algorithmic_bytes_of_the_480p_step():
    w = wl.WORKLOADS["video_480p"]
    # q, k, v read and out written (bf16), lse written (fp32), no ids
    assert bench.algorithmic_bytes(w) == 2 * 40 * 128 * (2 * 32760 + 2 * 32760) + 4 * 40 * 32760
    assert bench.algorithmic_bytes(w) == 1347091200
    # the rotary pass reads and writes q and k once
    assert bench.rope_algorithmic_bytes(w) == 2 * 2 * 2 * 40 * 32760 * 128


def test_ids_add_their_bytes():
    w = wl.WORKLOADS["joint_small"]
    base = 2 * w.B * w.H * w.D * 4 * w.S + 4 * w.B * w.H * w.S
    assert bench.algorithmic_bytes(w) == base + 4 * w.B * 2 * w.S


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_workload_config_names_the_workload(name):
    w = wl.WORKLOADS[name]
    cfg = bench.workload_config(w)
    assert cfg["workload"] == name
    for key in ("B", "H", "S_q", "S_kv", "D", "causal", "segments", "l2", "parallelism"):
        assert key in cfg
    assert not any(k in cfg for k in ("model", "global_batch"))
    if w.window is not None:
        assert cfg["window"] == list(w.window) and cfg["volume"] == list(w.rope_grid)
    assert bench.workload_config(w, causal=True)["workload"] == name + "_causal"
    assert bench.workload_config(w, rope=True)["workload"] == name + "_rope"


def test_code_only_drops_comments_and_blank_lines():
    src = "int a; // note\n\n/* block\n comment */ int b;  \n  // whole line\nint c;\n"
    assert bench.code_only(src) == "int a;\n int b;\nint c;"


def _fake_tree(tmp_path, code):
    csrc = tmp_path / "video_diffusion_transformer_non_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text(code)
    h = hashlib.sha256(bench.code_only(code).encode()).hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "summary.md").write_text(
        f"- kernel_sources_sha256: {h}\n- traffic_bytes_per_full_launch: 12345\n")
    return csrc / "k.cuh"


def test_recorded_traffic_follows_the_code(tmp_path, monkeypatch):
    src = _fake_tree(tmp_path, "__global__ void k() { int x = 1; }  // v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    w = wl.WORKLOADS["tiny"]
    get = lambda: bench.measured_traffic(w, "summary.md", ["k.cuh"])
    assert get() == 12345
    src.write_text("// a new comment\n__global__ void k() { int x = 1; }  // v2\n\n")
    assert get() == 12345                      # comments only: still the captured code
    src.write_text("__global__ void k() { int x = 2; }\n")
    assert get() is None                       # the code changed: no traffic claimed
    assert bench.measured_traffic(w, "absent.md", ["k.cuh"]) is None


def test_committed_summaries_parse():
    """The committed ncu summaries carry both fields bench.py reads."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for name in ("vidattn_fwd_kernel_d128__video_480p_h8.md", "rope3d_kernel_d128__video_480p.md",
                 "vidattn_fwd_kernel_d128__video_480p_causal_h8.md",
                 "vidattn_fwd_kernel_d64__cogvideox_joint_h8.md",
                 "vidattn_fwd_kernel_d128__window_480p_h8.md",
                 "vidattn_fwd_kernel_d128__video_720p_h8.md"):
        text = open(os.path.join(root, "profiles", name)).read()
        assert "kernel_sources_sha256:" in text and "traffic_bytes_per_full_launch:" in text


def test_causal_runs_read_the_causal_capture():
    """A causal bench line takes its traffic from the causal capture, never
    from the full-attention one of the same workload."""
    w = wl.WORKLOADS["video_480p"]
    assert bench.traffic_summary(w) == "vidattn_fwd_kernel_d128__video_480p_h8.md"
    assert bench.traffic_summary(w, causal=True) == \
        "vidattn_fwd_kernel_d128__video_480p_causal_h8.md"
    assert bench.traffic_summary(wl.WORKLOADS["video_720p"], causal=True) != \
        bench.traffic_summary(wl.WORKLOADS["video_720p"])


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root,
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    return [json.loads(l) for l in lines]


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference`: one JSON line with the contract's keys,
    the oracle timed on the host on the same workload and metric."""
    (line,) = _run_bench(["--impl", "reference", "--workload", "joint_small", "--steps", "3",
                          "--warmup", "3", "--ref-seconds", "3"])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert (line["steps"], line["warmup"], line["n_gpus"]) == (3, 3, 1)
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None and line["data"] == "synthetic"
    assert line["config"]["workload"] == "joint_small"
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1
    assert cpu["unit"] == bench.UNIT and "joint_small" in cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT,
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_bench_refuses_a_gpu_count_that_was_not_launched():
    """--gpus N must match the ranks torchrun started; a lone process asked
    for 2 GPUs stops with a message instead of timing one."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--impl", "reference"], cwd=root, env=env, capture_output=True,
                       text=True, timeout=120)
    assert p.returncode != 0 and "torch.distributed.run" in p.stderr
