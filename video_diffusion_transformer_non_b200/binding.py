"""ctypes binding to the vidattn C ABI (``include/vidattn.h``).

Argument marshalling only: tensors become raw pointers, streams become
``cudaStream_t`` handles.  Every step of the attention runs in the library's
CUDA kernels.  There is no fallback: if the library is missing or the call
fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libvidattn.so"
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "vidattn.h")

VIDATTN_OK = 0
_lib = None
# the device type the tensor helpers require (the library reads device memory)
_DEVICE_TYPE = "cuda"


def library_path() -> str:
    """The in-tree libvidattn.so, or the file named by VIDATTN_LIBRARY."""
    return os.environ.get("VIDATTN_LIBRARY") or os.path.join(_PKG, "csrc", _LIB_NAME)


def load_library():
    """Load libvidattn.so (built in-tree by ``build.py``); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m video_diffusion_transformer_non_b200.build` "
            "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(path)
    p, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.vidattn_fwd.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, f32, p]
    lib.vidattn_fwd.restype = i32
    lib.vidattn_fwd_ex.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, f32, i32, p]
    lib.vidattn_fwd_ex.restype = i32
    lib.vidattn_fwd_noalloc.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, f32, p]
    lib.vidattn_fwd_noalloc.restype = i32
    lib.vidattn_fwd_host.argtypes = [p, p, p, p, p, p, p,
                                     p, p, p, p, p, p, p,
                                     i32, i32, i32, i32, i32, f32, p]
    lib.vidattn_fwd_host.restype = i32
    lib.vidattn_status_string.argtypes = [i32]
    lib.vidattn_status_string.restype = ctypes.c_char_p
    lib.vidattn_release.argtypes = []
    lib.vidattn_release.restype = None
    lib.vidattn_device_status.argtypes = [p]
    lib.vidattn_device_status.restype = i32
    lib.vidattn_kernels_per_call.argtypes = [p, p, i32, i32, i32, i32, i32, i32]
    lib.vidattn_kernels_per_call.restype = i32
    lib.vidattn_split_count.argtypes = [p, i32, i32, i32, i32, i32]
    lib.vidattn_split_count.restype = i32
    ip = ctypes.POINTER(ctypes.c_int)
    lib.vidattn_launch_plan.argtypes = [p, i32, i32, i32, i32, i32, i32, ip, ip, ip]
    lib.vidattn_launch_plan.restype = i32
    lib.vidattn_selftest_timeout.argtypes = [i32, p]
    lib.vidattn_selftest_timeout.restype = i32
    lib.vidattn_fwd_window.argtypes = [p, p, p, p, p, p, p, i32, i32, i32, i32, i32, f32,
                                       i32, i32, i32, i32, i32, i32, i32, p]
    lib.vidattn_fwd_window.restype = i32
    i64, f64 = ctypes.c_longlong, ctypes.c_double
    lib.vidattn_rope3d.argtypes = [p, p, p, p, i32, i32, i32, i32, i64, i64, i64,
                                   i32, i32, i32, i32, i32, i32, i32, f64, i32, p]
    lib.vidattn_rope3d.restype = i32
    lib.vidattn_version.argtypes = []
    lib.vidattn_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def exported_symbols() -> list[str]:
    """Names of the functions declared in include/vidattn.h."""
    with open(_HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"VIDATTN_API\s+[\w\s\*]+?\b(vidattn_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return load_library().vidattn_status_string(int(status)).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):          # numpy array (host buffer)
        return x.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_tensors(named, dtype, ndim=None, contiguous=True):
    """Raise ValueError unless every tensor in ``named`` (name -> tensor or
    None) is a CUDA tensor of ``dtype`` on one device, ``ndim``-dimensional
    and (when asked) contiguous.  Runs before any pointer reaches the library,
    whose kernels read device memory in the documented layout only."""
    import torch
    device = None
    for name, t in named.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a torch tensor, not {type(t).__name__}")
        if t.device.type != _DEVICE_TYPE:
            raise ValueError(f"{name} must be on a CUDA device (is on {t.device})")
        if device is None:
            device = t.device
        elif t.device != device:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {device}")
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype} (is {t.dtype})")
        if ndim is not None and t.dim() != ndim:
            raise ValueError(f"{name} must have {ndim} dims (has shape {tuple(t.shape)})")
        if contiguous and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _check_qkv(q, k, v):
    """q bf16 [B,H,S_q,D], k and v bf16 [B,H,S_kv,D], contiguous, on one GPU."""
    import torch
    _check_tensors(dict(q=q, k=k, v=v), torch.bfloat16, ndim=4)
    if k.shape != v.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[3]:
        raise ValueError(f"shapes do not match: q {tuple(q.shape)}, k {tuple(k.shape)}, "
                         f"v {tuple(v.shape)}")


def _check_per_token(name_q, t_q, name_kv, t_kv, B, S_q, S_kv, device):
    """int32 [B,S_q] and [B,S_kv] per-token arrays (ids or coordinates), both
    or neither, contiguous, on the device of q."""
    import torch
    if (t_q is None) != (t_kv is None):
        raise ValueError(f"{name_q} and {name_kv} must both be given or both be None")
    if t_q is None:
        return
    _check_tensors({name_q: t_q, name_kv: t_kv}, torch.int32, ndim=2)
    if t_q.device != device:
        raise ValueError(f"{name_q} is on {t_q.device}, q on {device}")
    if tuple(t_q.shape) != (B, S_q) or tuple(t_kv.shape) != (B, S_kv):
        raise ValueError(f"{name_q} must be [B,S_q] = {(B, S_q)} and {name_kv} [B,S_kv] = "
                         f"{(B, S_kv)} (are {tuple(t_q.shape)}, {tuple(t_kv.shape)})")


def vidattn_fwd(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale, stream=None) -> int:
    """Enqueue the forward on ``stream`` (device pointers).  Returns the status."""
    return load_library().vidattn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seg_q), _ptr(seg_kv), _ptr(out), _ptr(lse),
        int(B), int(H), int(S_q), int(S_kv), int(D), float(scale), _stream(stream))


VIDATTN_CAUSAL = 1


def vidattn_fwd_ex(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale, flags,
                   stream=None) -> int:
    """vidattn_fwd with flags (VIDATTN_CAUSAL).  Returns the status."""
    return load_library().vidattn_fwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seg_q), _ptr(seg_kv), _ptr(out), _ptr(lse),
        int(B), int(H), int(S_q), int(S_kv), int(D), float(scale), int(flags), _stream(stream))


def vidattn_fwd_noalloc(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale,
                        stream=None) -> int:
    """vidattn_fwd without any device allocation (fixed library scratch, with a
    size limit); for callers that may not allocate.  Returns the status."""
    return load_library().vidattn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seg_q), _ptr(seg_kv), _ptr(out), _ptr(lse),
        int(B), int(H), int(S_q), int(S_kv), int(D), float(scale), _stream(stream))


def vidattn_fwd_host(h_q, h_k, h_v, h_seg_q, h_seg_kv, h_out, h_lse,
                     d_q, d_k, d_v, d_seg_q, d_seg_kv, d_out, d_lse,
                     B, H, S_q, S_kv, D, scale, stream=None) -> int:
    """Host buffers in and out, through caller-owned device staging buffers:
    copies in, forward, copies out, all enqueued on ``stream``."""
    return load_library().vidattn_fwd_host(
        _ptr(h_q), _ptr(h_k), _ptr(h_v), _ptr(h_seg_q), _ptr(h_seg_kv), _ptr(h_out), _ptr(h_lse),
        _ptr(d_q), _ptr(d_k), _ptr(d_v), _ptr(d_seg_q), _ptr(d_seg_kv), _ptr(d_out), _ptr(d_lse),
        int(B), int(H), int(S_q), int(S_kv), int(D), float(scale), _stream(stream))


def device_status(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the kernels' error word."""
    return load_library().vidattn_device_status(_stream(stream))


def selftest_timeout(timeout_us: int, stream=None) -> int:
    return load_library().vidattn_selftest_timeout(int(timeout_us), _stream(stream))


def kernels_per_call(seg_q, seg_kv, B, H, S_q, S_kv, D, flags=0) -> int:
    return load_library().vidattn_kernels_per_call(_ptr(seg_q), _ptr(seg_kv), int(B), int(H),
                                                   int(S_q), int(S_kv), int(D), int(flags))


def split_count(seg_q, B, H, S_q, S_kv, flags=0) -> int:
    """Key splits a vidattn_fwd_ex call with these arguments uses (the
    library's launch heuristic, or the VIDATTN_SPLIT_KV request in flags)."""
    return load_library().vidattn_split_count(_ptr(seg_q), int(B), int(H), int(S_q), int(S_kv),
                                              int(flags))


def launch_plan(seg_q, B, H, S_q, S_kv, D, flags=0) -> dict:
    """The launch a vidattn_fwd_ex call would make on the current device:
    dict(grid_ctas, key_splits, persistent).  Raises on an error status."""
    g, k, pe = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = load_library().vidattn_launch_plan(_ptr(seg_q), int(B), int(H), int(S_q), int(S_kv),
                                            int(D), int(flags), ctypes.byref(g), ctypes.byref(k),
                                            ctypes.byref(pe))
    if st != VIDATTN_OK:
        raise RuntimeError(f"vidattn_launch_plan: {status_string(st)}")
    return dict(grid_ctas=g.value, key_splits=k.value, persistent=bool(pe.value))


def VIDATTN_SPLIT_KV(n: int) -> int:
    """vidattn_fwd_ex flag: split every 256-row query block's keys into n ranges."""
    return (int(n) & 0xFF) << 8


def attention(q, k, v, seg_q=None, seg_kv=None, scale=None, stream=None, causal=False):
    """Allocate out/lse with torch and run ``vidattn_fwd``.
    q: bf16 [B,H,S_q,D]; k, v: bf16 [B,H,S_kv,D]; seg_*: int32 [B,S] or None.
    Returns (out bf16 [B,H,S_q,D], lse fp32 [B,H,S_q]); raises on error."""
    import torch
    _check_qkv(q, k, v)
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    _check_per_token("seg_q", seg_q, "seg_kv", seg_kv, B, S_q, S_kv, q.device)
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q.device)
    st = vidattn_fwd_ex(q, k, v, seg_q, seg_kv, out, lse, B, H, S_q, S_kv, D, scale,
                        VIDATTN_CAUSAL if causal else 0, stream)
    if st != VIDATTN_OK:
        raise RuntimeError(f"vidattn_fwd failed: {status_string(st)} ({st})")
    return out, lse


VIDATTN_ROPE_HALF_SPLIT = 1


def vidattn_rope3d(q_in, k_in, q_out, k_out, B, H, S, D, stride_b, stride_h, stride_s,
                   T, Hg, Wg, token_offset, d_t, d_h, d_w, theta, flags, stream=None) -> int:
    """Enqueue the 3D rotary embedding of q (and k) on ``stream``.  Returns the status."""
    return load_library().vidattn_rope3d(
        _ptr(q_in), _ptr(k_in), _ptr(q_out), _ptr(k_out), int(B), int(H), int(S), int(D),
        int(stride_b), int(stride_h), int(stride_s), int(T), int(Hg), int(Wg), int(token_offset),
        int(d_t), int(d_h), int(d_w), float(theta), int(flags), _stream(stream))


def rope3d(q, k=None, grid=None, bands=None, theta=10000.0, interleaved=True, token_offset=0,
           out_q=None, out_k=None, stream=None):
    """Rotate q (and k) by the 3D rotary embedding; returns (q_rot, k_rot or None),
    bf16 [B,H,S,D] contiguous.  q, k: bf16 [B,H,S,D] tensors whose last dim is
    contiguous, any other strides (a [B,S,H,D] tensor's ``transpose(1, 2)`` view
    works); grid = (T, Hg, Wg) of the video tokens; bands = (d_t, d_h, d_w).
    ``out_q=q`` (and ``out_k=k``) rotates a contiguous input in place."""
    import torch
    _check_tensors(dict(q=q, k=k, out_q=out_q, out_k=out_k), torch.bfloat16, ndim=4,
                   contiguous=False)
    if out_k is not None and k is None:
        raise ValueError("out_k without k")
    B, H, S, D = q.shape
    if k is not None and k.shape != q.shape:
        raise ValueError("q and k must have the same shape")
    if k is not None and k.stride() != q.stride():
        raise ValueError("q and k must have the same strides")
    if q.stride(3) != 1:
        raise ValueError("the feature dim must be contiguous")
    out_q = torch.empty((B, H, S, D), dtype=q.dtype, device=q.device) if out_q is None else out_q
    if k is not None and out_k is None:
        out_k = torch.empty((B, H, S, D), dtype=k.dtype, device=k.device)
    for o in (out_q, out_k):
        if o is not None and (tuple(o.shape) != (B, H, S, D) or not o.is_contiguous()):
            raise ValueError("outputs must be contiguous [B,H,S,D]")
    T, Hg, Wg = grid
    d_t, d_h, d_w = bands
    sb, sh, ss, _ = q.stride()
    st = vidattn_rope3d(q, k, out_q, out_k if k is not None else None, B, H, S, D, sb, sh, ss,
                        T, Hg, Wg, token_offset, d_t, d_h, d_w, theta,
                        0 if interleaved else VIDATTN_ROPE_HALF_SPLIT, stream)
    if st != VIDATTN_OK:
        raise RuntimeError(f"vidattn_rope3d failed: {status_string(st)} ({st})")
    return out_q, out_k


VIDATTN_WINDOW_CLAMPED = 1


def vidattn_fwd_window(q, k, v, coord_q, coord_kv, out, lse, B, H, S_q, S_kv, D, scale,
                       win_t, win_h, win_w, T, Hg, Wg, flags, stream=None) -> int:
    """Enqueue 3D neighbourhood attention on ``stream``.  Returns the status."""
    return load_library().vidattn_fwd_window(
        _ptr(q), _ptr(k), _ptr(v), _ptr(coord_q), _ptr(coord_kv), _ptr(out), _ptr(lse),
        int(B), int(H), int(S_q), int(S_kv), int(D), float(scale), int(win_t), int(win_h),
        int(win_w), int(T), int(Hg), int(Wg), int(flags), _stream(stream))


def attention_window(q, k, v, coord_q, coord_kv, size, extent, clamped=True, scale=None,
                     stream=None):
    """3D neighbourhood attention.  coord_*: int32 [B,S] packed t << 22 | h << 11 | w;
    size = (win_t, win_h, win_w), odd; extent = (T, Hg, Wg).  Returns (out, lse)."""
    import torch
    _check_qkv(q, k, v)
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    if coord_q is None or coord_kv is None:
        raise ValueError("a window needs coord_q and coord_kv")
    _check_per_token("coord_q", coord_q, "coord_kv", coord_kv, B, S_q, S_kv, q.device)
    if scale is None:
        scale = D ** -0.5
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q.device)
    st = vidattn_fwd_window(q, k, v, coord_q, coord_kv, out, lse, B, H, S_q, S_kv, D, scale,
                            *size, *extent, VIDATTN_WINDOW_CLAMPED if clamped else 0, stream)
    if st != VIDATTN_OK:
        raise RuntimeError(f"vidattn_fwd_window failed: {status_string(st)} ({st})")
    return out, lse
