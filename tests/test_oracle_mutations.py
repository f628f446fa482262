"""The pins are sensitive: each plausible mistake, planted in a copy of the
oracle's C source (a dropped term, a wrong sign, a wrong index, a transposed or
swapped operand), makes at least one pin fail.  CPU only; the planted copies
live in a temporary directory and are never used for anything else."""
import ctypes
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from video_diffusion_transformer_non_b200 import workloads as wl

from test_oracle_pins import brute_force, rand_case

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTATIONS = {
    "mask_sign": ("if (seg_q != NULL && seg_kv[b * S_kv + j] != seg_q[b * S_q + i]) return 0;",
                  "if (seg_q != NULL && seg_kv[b * S_kv + j] == seg_q[b * S_q + i]) return 0;"),
    "causal_off_by_one": ("if (causal && j > i + (S_kv - S_q)) return 0;",
                          "if (causal && j >= i + (S_kv - S_q)) return 0;"),
    "causal_top_left": ("if (causal && j > i + (S_kv - S_q)) return 0;",
                        "if (causal && j > i) return 0;"),
    "causal_ignored": ("if (causal && j > i + (S_kv - S_q)) return 0;", ""),
    "dropped_normalisation": ("for (long d = 0; d < D; ++d) out_row[d] /= l;", ""),
    "dropped_scale": ("double s = scale * dot;", "double s = dot;"),
    "lse_sign": ("*lse_out = m + log(l);", "*lse_out = m - log(l);"),
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "k_for_v": ("bf16_bits_to_double(vb[j * D + d]);", "bf16_bits_to_double(kb[j * D + d]);"),
    "transposed_k": ("bf16_bits_to_double(kb[j * D + d]);\n    double s",
                     "bf16_bits_to_double(kb[d * S_kv + j]);\n    double s"),
    "seg_ignores_batch": ("!= seg_q[b * S_q + i]) return 0;", "!= seg_q[i]) return 0;"),
    "head_stride": ("const uint16_t* vb = v + (b * H + h) * S_kv * D;",
                    "const uint16_t* vb = v + (b * H) * S_kv * D;"),
    "max_not_subtracted_in_weights": ("double e = exp(s_scratch[j] - m);", "double e = exp(s_scratch[j]);"),
    "empty_rows_uniform": ("if (n_allowed == 0) {       /* nothing to attend to */",
                           "if (n_allowed < 0) {"),
}


def build_variant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation {name} does not match the oracle source exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", str(so),
                    str(path), "-lm"], check=True)
    lib = ctypes.CDLL(str(so))
    p, L = ctypes.c_void_p, ctypes.c_long
    lib.oracle_attn_fwd_f64.argtypes = [p, p, p, p, p, p, p, L, L, L, L, L, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_int]
    lib.oracle_attn_fwd_f64.restype = ctypes.c_int
    return lib


def call(lib, c, scale=None, causal=0):
    B, H, Sq, D = c["q"].shape
    Skv = c["k"].shape[2]
    out = np.zeros((B, H, Sq, D))
    lse = np.zeros((B, H, Sq))
    ptr = lambda a: None if a is None else a.ctypes.data
    with np.errstate(all="ignore"):
        lib.oracle_attn_fwd_f64(ptr(c["q"]), ptr(c["k"]), ptr(c["v"]), ptr(c["seg_q"]),
                                ptr(c["seg_kv"]), ptr(out), ptr(lse), B, H, Sq, Skv, D,
                                c["scale"] if scale is None else scale, causal, 1)
    return out, lse


def pins_pass(lib) -> bool:
    """A subset of the pins, run against an arbitrary oracle build."""
    for shape, n_ids, seed in [((2, 2, 6, 5, 3), 3, 3), ((1, 2, 5, 7, 3), 0, 1), ((2, 1, 8, 8, 4), 2, 2)]:
        c = rand_case(*shape, seed, n_ids)
        out, lse = call(lib, c)
        ro, rl = brute_force(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"])
        fin = np.isfinite(rl)
        if not np.array_equal(fin, np.isfinite(lse)):
            return False
        if not (np.max(np.abs(out - ro)) <= 1e-12):
            return False
        if fin.any() and not (np.max(np.abs(lse[fin] - rl[fin])) <= 1e-12):
            return False
        if not np.all(out[~fin] == 0):
            return False
    # causal brute force, S_q < S_kv and S_q > S_kv, with and without ids
    for shape, n_ids, seed in [((1, 2, 5, 8, 3), 0, 4), ((2, 1, 7, 4, 2), 2, 5)]:
        c = rand_case(*shape, seed, n_ids)
        out, lse = call(lib, c, causal=1)
        ro, rl = brute_force(c["q"], c["k"], c["v"], c["seg_q"], c["seg_kv"], c["scale"],
                             causal=True)
        fin = np.isfinite(rl)
        if not np.array_equal(fin, np.isfinite(lse)) or not np.max(np.abs(out - ro)) <= 1e-12:
            return False
    # closed form: weights 1/4 and 3/4
    c = dict(q=wl.f32_to_bf16_bits(np.ones((1, 1, 1, 1), np.float32)),
             k=wl.f32_to_bf16_bits(np.array([[[[0.0], [1.0]]]], np.float32)),
             v=wl.f32_to_bf16_bits(np.array([[[[2.0], [6.0]]]], np.float32)),
             seg_q=None, seg_kv=None, scale=math.log(3.0))
    out, lse = call(lib, c)
    return abs(out[0, 0, 0, 0] - 5.0) <= 1e-14 and abs(lse[0, 0, 0] - math.log(4.0)) <= 1e-15


def test_unmutated_copy_passes(tmp_path):
    lib = build_variant(tmp_path, "identity", "double s = scale * dot;", "double s = scale * dot;")
    assert pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = build_variant(tmp_path, name, old, new)
    assert not pins_pass(lib), f"planted mistake '{name}' was not caught by the pins"
