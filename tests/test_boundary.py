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
            "vidattn_selftest_timeout"} <= names
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
    assert binding.kernels_per_call(None, None, 1, 2, 512, 512, 64) == 1
    assert binding.kernels_per_call(A, A, 2, 12, 4389, 4389, 128) == 2
    assert binding.kernels_per_call(None, None, 1, 2, 0, 512, 64) == 0


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
