"""Builds the vidattn shared library in-tree with nvcc for sm_100a.

    python -m video_diffusion_transformer_non_b200.build [--verbose-ptxas]

Output: video_diffusion_transformer_non_b200/csrc/libvidattn.so (C ABI of
include/vidattn.h).  The CUDA runtime is linked statically, so the library
needs only the NVIDIA driver at run time.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
OUT = os.path.join(CSRC, "libvidattn.so")
PROBES_OUT = os.path.join(CSRC, "libvidattn_probes.so")
# (output, sources, dependencies)
TARGETS = [
    (OUT, ["vidattn.cu"], ["vidattn.cu", "fwd_kernel.cuh", "classify.cuh", "ptx.cuh", "rope3d.cuh"]),
    # unit probes of the kernel's tensor-core steps, used only by the GPU tests
    (PROBES_OUT, ["probes.cu"], ["probes.cu", "fwd_kernel.cuh", "ptx.cuh"]),
]
# timeline-instrumented build of the library (-DVIDATTN_TRACE), for profiling
TRACE_OUT = os.path.join(CSRC, "libvidattn_trace.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(out, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    paths = [os.path.join(CSRC, d) for d in deps] + [os.path.join(ROOT, "include", "vidattn.h")]
    return any(os.path.getmtime(d) > t for d in paths)


def build(force: bool = False, ptxas_verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile every target that is missing or older than its sources."""
    for out, sources, deps in TARGETS:
        if not force and not needs_build(out, deps):
            continue
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
               "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static",
               "-I", os.path.join(ROOT, "include"), "-o", tmp]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        cmd += extra or []
        cmd += [os.path.join(CSRC, s) for s in sources]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return OUT


def build_trace() -> str:
    """libvidattn_trace.so: the library with per-event clock64 stamps
    (vidattn_trace_set); same kernels otherwise."""
    tmp = TRACE_OUT + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static", "-DVIDATTN_TRACE",
           "-I", os.path.join(ROOT, "include"), "-o", tmp, os.path.join(CSRC, "vidattn.cu")]
    subprocess.run(cmd, check=True)
    os.replace(tmp, TRACE_OUT)
    return TRACE_OUT


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--trace", action="store_true", help="also build libvidattn_trace.so")
    a = ap.parse_args(argv)
    print(build(force=a.force or a.verbose_ptxas, ptxas_verbose=a.verbose_ptxas))
    if a.trace:
        print(build_trace())


if __name__ == "__main__":
    sys.exit(main())
