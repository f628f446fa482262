"""The boundary from plain C: a C11 program includes include/vidattn.h, links
the built library and calls its host-side entry points (version, status
strings, kernels per call, argument errors, release).  Checks that the header
is valid C, not only C++, and that the exported symbols resolve from C.  No
kernel runs: every call that could launch fails its argument check first."""
import os
import shutil
import subprocess

import pytest

from video_diffusion_transformer_non_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "vidattn.h"

int main(void) {
  const char* v = vidattn_version();
  if (!v || !strstr(v, "sm_100a")) return 1;
  if (strcmp(vidattn_status_string(VIDATTN_OK), "ok") != 0) return 2;
  if (vidattn_kernels_per_call(NULL, NULL, 1, 2, 512, 512, 64, 0) != 1) return 3;
  if (vidattn_split_count(NULL, 1, 40, 32760, 32760, VIDATTN_SPLIT_KV(3)) != 3) return 3;
  /* argument errors, returned before anything touches a device */
  if (vidattn_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 2, 256, 256, 128, 0.1f, NULL)
      != VIDATTN_ERR_NULL) return 4;
  const void* p = (const void*)0x10000;
  if (vidattn_fwd_ex(p, p, p, NULL, NULL, (void*)p, (float*)p, 1, 2, 256, 256, 96, 0.1f,
                     VIDATTN_CAUSAL, NULL) != VIDATTN_ERR_UNSUPPORTED_D) return 5;
  if (vidattn_fwd_window(p, p, p, NULL, NULL, (void*)p, (float*)p, 1, 1, 8, 8, 128, 0.1f,
                         3, 3, 3, 2, 2, 2, VIDATTN_WINDOW_CLAMPED, NULL) != VIDATTN_ERR_NULL)
    return 6;
  if (vidattn_rope3d(p, NULL, (void*)p, NULL, 1, 1, 8, 64, 512, 512, 64, 2, 2, 2, 0,
                     16, 24, 24, 10000.0, VIDATTN_ROPE_HALF_SPLIT | 4, NULL)
      != VIDATTN_ERR_BAD_SHAPE) return 7;
  int32_t c = VIDATTN_COORD(3, 5, 7);
  if ((((uint32_t)c) >> 22) != 3u || ((((uint32_t)c) >> 11) & 2047u) != 5u ||
      (((uint32_t)c) & 2047u) != 7u) return 8;
  vidattn_release();
  printf("c abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    lib = binding.library_path()
    binding.load_library()            # builds nothing; fails loudly if the library is absent
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), lib,
                    "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "c abi ok"
