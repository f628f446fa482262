"""The C-ABI boundary, on the host: the library loads, exports every entry
point that include/vidattn.h declares, and rejects bad arguments with their
status before any CUDA call.  No kernel runs here (every call below fails its
argument check first, or has nothing to compute), so these pass without a GPU.
"""
import ctypes
import os
import re

import pytest

import video_diffusion_transformer_non_b200 as va
from video_diffusion_transformer_non_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# fake, never-dereferenced device addresses (16-byte aligned unless stated)
A = 0x10000
OK, NULL, BAD_D, BAD_SHAPE, MISALIGNED, CUDA, TIMEOUT, NO_DEVICE, SEG_PAIR = range(9)


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def header_names():
    with open(os.path.join(ROOT, "include", "vidattn.h")) as f:
        return re.findall(r"VIDATTN_API\s+[\w\s\*]+?\b(vidattn_\w+)\s*\(", f.read())


def test_header_declares_the_entry_points():
    names = set(header_names())
    assert {"vidattn_fwd", "vidattn_fwd_ex", "vidattn_fwd_host", "vidattn_status_string", "vidattn_device_status",
            "vidattn_rope3d", "vidattn_fwd_window",
            "vidattn_kernels_per_call", "vidattn_release", "vidattn_version",
            "vidattn_selftest_timeout", "vidattn_split_count", "vidattn_launch_plan",
            "vidattn_fwd_noalloc"} <= names
    assert set(binding.exported_symbols()) == names


def test_library_exports_every_declared_symbol(lib):
    cdll = ctypes.CDLL(binding.library_path())
    for name in header_names():
        assert hasattr(cdll, name), f"{name} declared in include/vidattn.h but not exported"


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.vidattn_version()
    for code in range(9):
        s = binding.status_string(code)
        assert s and s != "unknown status"
    assert binding.status_string(1234) == "unknown status"


def call(lib, q=A, k=A, v=A, sq=None, sk=None, out=A, lse=A, B=1, H=2, Sq=256, Skv=256, D=128,
         scale=0.125):
    return lib.vidattn_fwd(q, k, v, sq, sk, out, lse, B, H, Sq, Skv, D, scale, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), NULL), (dict(k=None), NULL), (dict(v=None), NULL),
    (dict(out=None), NULL), (dict(lse=None), NULL),
    (dict(sq=A), SEG_PAIR), (dict(sk=A), SEG_PAIR),
    (dict(D=96), BAD_D), (dict(D=256), BAD_D), (dict(D=0), BAD_D),
    (dict(B=0), BAD_SHAPE), (dict(H=0), BAD_SHAPE), (dict(B=70000), BAD_SHAPE),
    (dict(Sq=-1), BAD_SHAPE), (dict(Skv=-5), BAD_SHAPE),
    (dict(q=A + 8), MISALIGNED), (dict(k=A + 2), MISALIGNED), (dict(v=A + 4), MISALIGNED),
    (dict(out=A + 8), MISALIGNED), (dict(lse=A + 2), MISALIGNED),
    (dict(sq=A + 1, sk=A), MISALIGNED),
    (dict(scale=float("inf")), BAD_SHAPE), (dict(scale=float("nan")), BAD_SHAPE),
])
def test_argument_errors_return_before_any_launch(lib, kw, expect):
    assert call(lib, **kw) == expect


def test_unknown_flag_bits_are_rejected(lib):
    f = lib.vidattn_fwd_ex
    assert f(A, A, A, None, None, A, A, 1, 2, 256, 256, 128, 0.1, 2, None) == BAD_SHAPE
    assert f(A, A, A, None, None, A, A, 1, 2, 256, 256, 96, 0.1, 1, None) == BAD_D
    assert f(A, A, A, None, None, A, A, 1, 2, 0, 256, 128, 0.1, 1, None) == OK


def test_empty_query_is_a_no_op(lib):
    assert call(lib, Sq=0) == OK
    assert call(lib, Sq=0, sq=A, sk=A) == OK


def test_host_entry_point_argument_errors(lib):
    f = lib.vidattn_fwd_host
    args = [A] * 7 + [A] * 7 + [1, 2, 128, 128, 128, 0.1, None]
    a = list(args); a[0] = None
    assert f(*a) == NULL
    a = list(args)      # host seg set, device seg NULL
    a[10] = None; a[11] = None
    assert f(*a) == SEG_PAIR
    a = list(args); a[3] = None; a[4] = None     # host seg NULL, device seg set
    assert f(*a) == SEG_PAIR
    a = list(args); a[18] = 80
    assert f(*a) == BAD_D
    a = list(args); a[7] = A + 4
    assert f(*a) == MISALIGNED


def test_kernels_per_call(lib):
    # tiny: 4 units of 256 query rows, but only 4 key tiles: no split
    assert binding.kernels_per_call(None, None, 1, 2, 512, 512, 64) == 1
    assert binding.kernels_per_call(A, A, 2, 12, 4389, 4389, 128) == 2      # classify + attention
    assert binding.kernels_per_call(None, None, 1, 40, 32760, 32760, 128) == 1
    assert binding.kernels_per_call(A, A, 1, 2, 512, 8192, 64) == 3         # + classify + merge
    assert binding.kernels_per_call(None, None, 1, 40, 32760, 32760, 128,
                                    binding.VIDATTN_SPLIT_KV(2)) == 2
    assert binding.kernels_per_call(None, None, 1, 2, 0, 512, 64) == 0


def test_split_heuristic(lib):
    """The launch heuristic (pure host logic): key splits only when the
    256-row query blocks x heads x batch are fewer than 74 (half of 148 SMs),
    ceil(148 / units) of them, at most 16 and at least 8 key tiles each; the
    VIDATTN_SPLIT_KV request overrides it; nothing with ids beyond 2048 key
    tiles (the summaries are walked in global memory there)."""
    sc = binding.split_count
    S = binding.VIDATTN_SPLIT_KV
    assert sc(None, 1, 2, 512, 512) == 1              # tiny: 4 key tiles, too short to split
    assert sc(None, 1, 2, 512, 100000) == 16          # 4 units, many key tiles: capped at 16
    assert sc(None, 1, 1, 256, 128 * 15) == 1         # 15 key tiles: one range of 8+
    assert sc(None, 1, 1, 256, 128 * 16) == 2
    assert sc(None, 1, 2, 512, 128 * 40) == 5         # 4 units, 40 key tiles: 8 each
    assert sc(None, 1, 36, 512, 4096) == 3            # 72 units: ceil(148 / 72)
    assert sc(None, 1, 37, 512, 4096) == 1            # 74 units: enough
    assert sc(A, 2, 12, 4389, 4389) == 1              # joint_small: 432 units
    assert sc(None, 1, 40, 32760, 32760) == 1
    assert sc(None, 1, 1, 256, 300000) == 16          # no ids: any length splits
    assert sc(A, 1, 1, 256, 300000) == 1              # ids beyond 2048 key tiles: never
    assert sc(None, 1, 40, 32760, 32760, S(5)) == 5   # a request wins
    assert sc(None, 1, 2, 512, 512, S(64)) == 64
    assert sc(None, 1, 2, 512, 512, S(65)) == 0       # above 64: invalid
    assert sc(None, 1, 2, 0, 512) == 0 and sc(None, 1, 2, 512, 0) == 1


def test_launch_plan_argument_errors(lib):
    """Argument errors come back before the device is touched; on a host
    without an sm_100 GPU a valid query reports the missing device."""
    import ctypes
    g, k, pe = ctypes.c_int(-1), ctypes.c_int(-1), ctypes.c_int(-1)
    refs = (ctypes.byref(g), ctypes.byref(k), ctypes.byref(pe))
    assert lib.vidattn_launch_plan(None, 1, 2, 512, 512, 64, 0, None, refs[1], refs[2]) == NULL
    assert lib.vidattn_launch_plan(None, 1, 2, 512, 512, 96, 0, *refs) == BAD_D
    assert lib.vidattn_launch_plan(None, 1, 2, 512, 512, 64, 2, *refs) == BAD_SHAPE
    assert lib.vidattn_launch_plan(None, 1, 2, 0, 512, 64, 0, *refs) == BAD_SHAPE
    import torch
    if not torch.cuda.is_available():
        assert lib.vidattn_launch_plan(None, 1, 2, 512, 512, 64, 0, *refs) != 0
        assert (g.value, k.value, pe.value) == (-1, -1, -1)


def test_selftest_argument_range(lib):
    assert lib.vidattn_selftest_timeout(0, None) == BAD_SHAPE
    assert lib.vidattn_selftest_timeout(2000000, None) == BAD_SHAPE


def test_release_without_work_is_safe(lib):
    lib.vidattn_release()
    lib.vidattn_release()


def test_product_path_does_not_touch_the_oracle():
    """The product package never imports, loads or runs anything under
    oracle/; the oracle is test infrastructure."""
    pkg = os.path.dirname(va.__file__)
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"\bimport\s+oracle|from\s+oracle|attn_oracle|_attn_oracle",
                                     text), fn


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "library_path", lambda: str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        binding.load_library()


def rope(lib, q=A, k=A, qo=A + 0x100000, ko=A + 0x200000, B=1, H=2, S=128, D=128,
         sb=2 * 128 * 128, sh=128 * 128, ss=128, T=2, Hg=4, Wg=8, off=0, bands=(44, 42, 42),
         theta=10000.0, flags=0):
    return lib.vidattn_rope3d(q, k, qo, ko, B, H, S, D, sb, sh, ss, T, Hg, Wg, off, *bands,
                              theta, flags, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), NULL), (dict(qo=None), NULL), (dict(k=None), NULL), (dict(ko=None), NULL),
    (dict(D=96, bands=(32, 32, 32)), BAD_D),
    (dict(flags=2), BAD_SHAPE), (dict(B=0), BAD_SHAPE), (dict(H=0), BAD_SHAPE),
    (dict(S=0), BAD_SHAPE), (dict(S=63), BAD_SHAPE), (dict(off=65), BAD_SHAPE),
    (dict(off=-1, S=200), BAD_SHAPE), (dict(T=0), BAD_SHAPE), (dict(Wg=-8), BAD_SHAPE),
    (dict(bands=(43, 43, 42)), BAD_SHAPE), (dict(bands=(44, 42, 40)), BAD_SHAPE),
    (dict(bands=(-2, 66, 64)), BAD_SHAPE),
    (dict(theta=0.0), BAD_SHAPE), (dict(theta=-1.0), BAD_SHAPE),
    (dict(theta=float("inf")), BAD_SHAPE), (dict(theta=float("nan")), BAD_SHAPE),
    (dict(B=40000, H=40000), BAD_SHAPE),
    (dict(q=A + 8), MISALIGNED), (dict(ko=A + 2), MISALIGNED),
    (dict(ss=132), MISALIGNED), (dict(sh=4), MISALIGNED), (dict(sb=12), MISALIGNED),
])
def test_rope3d_argument_errors_return_before_any_launch(lib, kw, expect):
    assert rope(lib, **kw) == expect


def test_rope3d_q_only_is_accepted_by_the_checks(lib):
    """k_in and k_out both NULL passes the argument checks (then needs a GPU)."""
    st = rope(lib, k=None, ko=None)
    assert st in (OK, CUDA, NO_DEVICE)


def win(lib, q=A, k=A, v=A, cq=A + 0x1000, ck=A + 0x2000, out=A, lse=A, B=1, H=2, Sq=512, Skv=512,
        D=128, scale=0.125, size=(3, 5, 5), ext=(2, 16, 16), flags=0):
    return lib.vidattn_fwd_window(q, k, v, cq, ck, out, lse, B, H, Sq, Skv, D, scale, *size, *ext,
                                  flags, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(cq=None), NULL), (dict(ck=None), NULL), (dict(q=None), NULL),
    (dict(D=96), BAD_D), (dict(flags=2), BAD_SHAPE), (dict(flags=-1), BAD_SHAPE),
    (dict(size=(2, 5, 5)), BAD_SHAPE), (dict(size=(3, 0, 5)), BAD_SHAPE),
    (dict(size=(3, 5, -1)), BAD_SHAPE), (dict(ext=(0, 16, 16)), BAD_SHAPE),
    (dict(ext=(1025, 16, 16)), BAD_SHAPE), (dict(ext=(2, 2049, 16)), BAD_SHAPE),
    (dict(ext=(2, 16, 2049)), BAD_SHAPE), (dict(Skv=262145), BAD_SHAPE),
    (dict(scale=float("nan")), BAD_SHAPE), (dict(B=0), BAD_SHAPE),
    (dict(cq=A + 2), MISALIGNED), (dict(q=A + 8), MISALIGNED),
])
def test_window_argument_errors_return_before_any_launch(lib, kw, expect):
    assert win(lib, **kw) == expect


def test_window_empty_query_is_a_no_op(lib):
    assert win(lib, Sq=0) == OK


# --- the Python helpers' tensor checks ---------------------------------------
# The helpers (attention, attention_window, rope3d) check dtype, device,
# layout and shapes before a pointer reaches the library.  Here the device
# type the checks require is "cpu", and the library is replaced by one that
# fails the test when touched, so every case below must raise first.

@pytest.fixture
def host_checks(monkeypatch):
    torch = pytest.importorskip("torch")

    def no_library():
        raise AssertionError("an invalid call reached the library")
    monkeypatch.setattr(binding, "_DEVICE_TYPE", "cpu")
    monkeypatch.setattr(binding, "load_library", no_library)
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)
    return torch, bf, i32


def test_helpers_refuse_host_tensors_where_a_device_is_required():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        binding.rope3d(q, q, (1, 2, 4), (22, 22, 20))
    with pytest.raises(ValueError, match="CUDA"):
        binding.attention_window(q, q, q, torch.zeros(1, 8, dtype=torch.int32),
                                 torch.zeros(1, 8, dtype=torch.int32), (3, 3, 3), (1, 2, 4))


@pytest.mark.parametrize("case", [
    "dtype", "ndim", "strided", "kv_shape", "d_mismatch", "seg_one", "seg_dtype", "seg_shape",
    "not_tensor"])
def test_attention_helper_checks(host_checks, case):
    torch, bf, i32 = host_checks
    q, k, v = bf(1, 2, 8, 64), bf(1, 2, 16, 64), bf(1, 2, 16, 64)
    sq, sk = i32(1, 8), i32(1, 16)
    if case == "dtype":
        q = q.float()
    elif case == "ndim":
        q = q[0]
    elif case == "strided":
        q = bf(1, 8, 2, 64).transpose(1, 2)
    elif case == "kv_shape":
        v = bf(1, 2, 15, 64)
    elif case == "d_mismatch":
        k, v = bf(1, 2, 16, 128), bf(1, 2, 16, 128)
    elif case == "seg_one":
        sk = None
    elif case == "seg_dtype":
        sq = sq.long()
    elif case == "seg_shape":
        sk = i32(1, 8)
    elif case == "not_tensor":
        k = [0]
    with pytest.raises(ValueError):
        binding.attention(q, k, v, sq, sk)


@pytest.mark.parametrize("case", ["no_coords", "coord_dtype", "coord_shape"])
def test_window_helper_checks(host_checks, case):
    torch, bf, i32 = host_checks
    q = bf(1, 2, 8, 64)
    cq, ck = i32(1, 8), i32(1, 8)
    if case == "no_coords":
        cq = ck = None
    elif case == "coord_dtype":
        ck = ck.long()
    elif case == "coord_shape":
        cq = i32(2, 8)
    with pytest.raises(ValueError):
        binding.attention_window(q, q, q, cq, ck, (3, 3, 3), (1, 2, 4))


@pytest.mark.parametrize("case", ["dtype", "k_shape", "k_strides", "feature_stride", "out_shape",
                                  "out_k_alone"])
def test_rope_helper_checks(host_checks, case):
    torch, bf, i32 = host_checks
    q, k = bf(1, 2, 8, 64), bf(1, 2, 8, 64)
    kw = {}
    if case == "dtype":
        k = k.half()
    elif case == "k_shape":
        k = bf(1, 2, 9, 64)
    elif case == "k_strides":
        k = bf(1, 8, 2, 64).transpose(1, 2)
    elif case == "feature_stride":
        q = k = bf(1, 2, 64, 8).transpose(2, 3)
    elif case == "out_shape":
        kw["out_q"] = bf(1, 2, 8, 128)
    elif case == "out_k_alone":
        k = None
        kw["out_k"] = bf(1, 2, 8, 64)
    with pytest.raises(ValueError):
        binding.rope3d(q, k, (1, 2, 4), (22, 22, 20), **kw)
