"""The C ABI under random arguments, on the host: every entry point returns a
defined status for any combination of shapes, pointers (NULL, aligned,
misaligned), strides, windows and flag words, and never crashes.  Pointers
are fake and never dereferenced: calls that pass the argument checks stop at
the device check, because these tests run only where there is no GPU (with a
GPU present the module is skipped, so that no fake pointer can ever reach a
kernel)."""
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from video_diffusion_transformer_non_b200 import binding

STATUSES = set(range(10))
BASE = 0x10000

ptrs = st.sampled_from([None, BASE, BASE + 2, BASE + 4, BASE + 8, BASE + 16])
ints = st.integers(-3, 70000)
SETTINGS = dict(max_examples=300, deadline=None, derandomize=True,
                suppress_health_check=[HealthCheck.too_slow])


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def _gpu_present():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return True      # unknown: treat as present and skip


pytestmark = pytest.mark.skipif(_gpu_present(),
                                reason="host-only: fake pointers must never reach a GPU")


ARG_ERRORS = {1, 2, 3, 4, 8}      # NULL, D, shape, alignment, id pair
DEVICE = {5, 7}                    # no GPU here: the device check fails


def _expect(st_code, verdict):
    """verdict: "err" (an argument error), "ok" (nothing to compute) or
    "device" (the arguments pass; the call stops at the device check)."""
    assert st_code in STATUSES
    want = {"err": ARG_ERRORS, "ok": {0}, "device": DEVICE}[verdict]
    assert st_code in want, (st_code, verdict)


def _al(p, n):
    return p is None or p % n == 0


@settings(**SETTINGS)
@given(q=ptrs, k=ptrs, v=ptrs, sq=ptrs, sk=ptrs, out=ptrs, lse=ptrs, B=ints, H=ints,
       Sq=st.integers(-2, 300000), Skv=st.integers(-2, 300000), D=st.sampled_from([0, 32, 64, 96, 128, 256]),
       scale=st.sampled_from([0.0, -1.0, 0.125, float("inf"), float("nan")]),
       flags=st.sampled_from([0, 1, 2, 3, -1]))
def test_fwd_ex_returns_a_status(lib, q, k, v, sq, sk, out, lse, B, H, Sq, Skv, D, scale, flags):
    if flags not in (0, 1) or (Sq > 0 and not (q and out and lse)) or (Skv > 0 and not (k and v)) \
            or (sq is None) != (sk is None) or D not in (64, 128) \
            or not (1 <= B <= 65535 and 1 <= H <= 65535 and Sq >= 0 and Skv >= 0) \
            or not all(_al(p, 16) for p in (q, k, v, out)) or not _al(lse, 4) \
            or not (_al(sq, 4) and _al(sk, 4)) or not (scale == scale and abs(scale) < 1e38):
        verdict = "err"
    else:
        verdict = "ok" if Sq == 0 else "device"
    _expect(lib.vidattn_fwd_ex(q, k, v, sq, sk, out, lse, B, H, Sq, Skv, D, scale, flags, None),
            verdict)


@settings(**SETTINGS)
@given(q=ptrs, k=ptrs, qo=ptrs, ko=ptrs, B=ints, H=ints, S=st.integers(-2, 5000),
       D=st.sampled_from([0, 64, 96, 128]), sb=st.integers(-16, 4096), sh=st.integers(-16, 4096),
       ss=st.integers(-16, 4096), grid=st.tuples(st.integers(-1, 20), st.integers(-1, 20),
                                                st.integers(-1, 20)),
       off=st.integers(-2, 100), bands=st.tuples(st.integers(-2, 130), st.integers(-2, 130),
                                                 st.integers(-2, 130)),
       theta=st.sampled_from([0.0, -1.0, 1e4, float("nan")]), flags=st.sampled_from([0, 1, 2]))
def test_rope3d_returns_a_status(lib, q, k, qo, ko, B, H, S, D, sb, sh, ss, grid, off, bands,
                                 theta, flags):
    n_tensors = 1 if k is None else 2
    valid = (q and qo and (k is None) == (ko is None) and D in (64, 128) and flags in (0, 1)
             and B >= 1 and H >= 1 and S >= 1 and n_tensors * B * H < 2 ** 31
             and min(grid) >= 1 and off >= 0 and off + grid[0] * grid[1] * grid[2] <= S
             and min(bands) >= 0 and all(b % 2 == 0 for b in bands) and sum(bands) == D
             and theta == theta and theta > 0 and sb % 8 == 0 and sh % 8 == 0 and ss % 8 == 0
             and all(_al(p, 16) for p in (q, k, qo, ko)))
    _expect(lib.vidattn_rope3d(q, k, qo, ko, B, H, S, D, sb, sh, ss, *grid, off, *bands, theta,
                               flags, None), "device" if valid else "err")


@settings(**SETTINGS)
@given(q=ptrs, cq=ptrs, ck=ptrs, B=ints, H=ints, Sq=st.integers(-2, 300000),
       Skv=st.integers(-2, 300000), D=st.sampled_from([0, 64, 128]),
       size=st.tuples(st.integers(-1, 12), st.integers(-1, 12), st.integers(-1, 12)),
       ext=st.tuples(st.integers(-1, 3000), st.integers(-1, 3000), st.integers(-1, 3000)),
       flags=st.sampled_from([0, 1, 2]))
def test_fwd_window_returns_a_status(lib, q, cq, ck, B, H, Sq, Skv, D, size, ext, flags):
    ok_args = (cq and ck and flags in (0, 1) and (Sq <= 0 or q) and (Skv <= 0 or q)
               and D in (64, 128) and 1 <= B <= 65535 and 1 <= H <= 65535
               and Sq >= 0 and Skv >= 0 and _al(q, 16) and _al(cq, 4) and _al(ck, 4)
               and all(s >= 1 and s % 2 for s in size)
               and 1 <= ext[0] <= 1024 and 1 <= ext[1] <= 2048 and 1 <= ext[2] <= 2048
               and Skv <= 262144)
    verdict = "err" if not ok_args else ("ok" if Sq == 0 else "device")
    _expect(lib.vidattn_fwd_window(q, q, q, cq, ck, q, q, B, H, Sq, Skv, D, 0.1, *size, *ext,
                                   flags, None), verdict)
