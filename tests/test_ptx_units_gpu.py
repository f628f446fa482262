"""GPU unit tests of the forward kernel's tensor-core steps in isolation (one
CTA, one tile): TMA loads with 128-byte swizzle, S = Q K^T with both operands
in shared memory, and O = P V with P in tensor memory and V as an MN-major
operand.  Compared with plain fp64 matrix products of the same bf16 values."""
import ctypes
import os

import numpy as np
import pytest
import torch

from video_diffusion_transformer_non_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LIB = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "video_diffusion_transformer_non_b200", "csrc", "libvidattn_probes.so")


@pytest.fixture(scope="module")
def probes():
    lib = ctypes.CDLL(LIB)
    p = ctypes.c_void_p
    lib.probe_qk_pv.argtypes = [p, p, p, p, p, p, p, ctypes.c_int, p]
    lib.probe_qk_pv.restype = ctypes.c_int
    lib.probe_exp2_poly.argtypes = [p, p, ctypes.c_int, p]
    lib.probe_exp2_poly.restype = ctypes.c_int
    return lib


def test_fma_pipe_exp2_within_its_bound(probes):
    """The polynomial 2^x used for part of the softmax exponentials: relative
    error <= 7.5e-5 (the fitted cubic's bound) plus fp32 rounding, over
    x in [-125, 0]; below -125 it returns 2^-125."""
    rng = np.random.Generator(np.random.PCG64(5))
    x = np.concatenate([np.linspace(-125.0, 0.0, 500002), rng.uniform(-30, 0, 500000),
                        -rng.exponential(1.0, 100000), [0.0, -0.5, -1.0, -124.5, -125.0, -1e-7]])
    x = x.astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(-3.0))
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    assert probes.probe_exp2_poly(xd.data_ptr(), yd.data_ptr(), x.size,
                                  torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 7.5e-5 + 4e-7, rel.max()
    # below the clamp: 2^-125 times the cubic at 0
    lo = torch.tensor([-126.0, -200.0, -1e30, -130.0], dtype=torch.float32, device="cuda")
    lo_y = torch.empty_like(lo)
    assert probes.probe_exp2_poly(lo.data_ptr(), lo_y.data_ptr(), 4,
                                  torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert np.allclose(lo_y.cpu().numpy(), 2.0 ** -125, rtol=1e-4, atol=0)


@pytest.mark.parametrize("D", [64, 128])
def test_qk_and_pv_tiles(probes, D):
    rng = np.random.Generator(np.random.PCG64(D))
    bits = lambda shape: wl.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    q, k, v = bits((128, D)), bits((128, D)), bits((128, D))
    P = wl.f32_to_bf16_bits(rng.uniform(0, 1, (128, 128)).astype(np.float32))
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda()
    tq, tk, tv, tP = dev(q), dev(k), dev(v), dev(P)
    S = torch.full((128, 128), float("nan"), device="cuda")
    O = torch.full((128, D), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probes.probe_qk_pv(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), tP.data_ptr(),
                            S.data_ptr(), O.data_ptr(), status.data_ptr(), D,
                            torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "a probe wait timed out"
    f = lambda b: wl.bf16_bits_to_f32(b).astype(np.float64)
    S_ref = f(q) @ f(k).T
    O_ref = f(P) @ f(v)
    S_got, O_got = S.cpu().numpy(), O.cpu().numpy()
    # fp32 accumulation of exact bf16 products
    assert np.max(np.abs(S_got - S_ref)) <= 1e-3 * max(1.0, np.abs(S_ref).max()), "Q K^T tile wrong"
    assert np.max(np.abs(O_got - O_ref)) <= 1e-3 * max(1.0, np.abs(O_ref).max()), "P V tile wrong"
