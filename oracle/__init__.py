"""Test infrastructure only: the fp64 CPU oracle for segment-masked attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module compiles it with gcc and marshals numpy arrays through ctypes.
What it computes, with citations, is written at the top of ``attn_oracle.c``:
exact softmax(scale * Q K^T masked by segment-id equality) V, plus the natural
log-sum-exp of each row, with empty rows giving out = 0 and lse = -inf; with
causal=True a key is also limited to j <= i + (S_kv - S_q); with a ``window``
(a 3D neighbourhood: per-token packed coordinates t << 22 | h << 11 | w, an odd
window size and the volume extent per axis, centred or clamped) a key must
also lie in the query's window.

Inputs are bf16 bit patterns as ``numpy.uint16`` arrays in [B,H,S,D] order and
int32 segment ids in [B,S] order (or None for a single segment).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_attn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into _attn_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _declare(lib):
    """Argument and result types of the library's entry points."""
    p = ctypes.c_void_p
    L = ctypes.c_long
    lib.oracle_attn_fwd_f64.argtypes = [p, p, p, p, p, p, p, L, L, L, L, L,
                                        ctypes.c_double, ctypes.c_int, ctypes.c_int]
    lib.oracle_attn_fwd_f64.restype = ctypes.c_int
    lib.oracle_attn_rows_f64.argtypes = [p, p, p, p, p, p, L, p, p, L, L, L, L, L,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_int]
    lib.oracle_attn_rows_f64.restype = ctypes.c_int
    lib.oracle_attn_probs_f64.argtypes = [p, p, p, p, p, L, L, L, L, L, ctypes.c_double,
                                          ctypes.c_int]
    lib.oracle_attn_probs_f64.restype = ctypes.c_int
    W = [p, p, p, p, ctypes.c_int]     # coord_q, coord_kv, size[3], extent[3], clamped
    lib.oracle_attn_win_fwd_f64.argtypes = [p, p, p, p, p] + W + [
        p, p, L, L, L, L, L, ctypes.c_double, ctypes.c_int, ctypes.c_int]
    lib.oracle_attn_win_fwd_f64.restype = ctypes.c_int
    lib.oracle_attn_win_rows_f64.argtypes = [p, p, p, p, p] + W + [
        p, L, p, p, L, L, L, L, L, ctypes.c_double, ctypes.c_int, ctypes.c_int]
    lib.oracle_attn_win_rows_f64.restype = ctypes.c_int
    lib.oracle_attn_win_probs_f64.argtypes = [p, p, p, p] + W + [
        p, L, L, L, L, L, ctypes.c_double, ctypes.c_int]
    lib.oracle_attn_win_probs_f64.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check_inputs(q, k, v, seg_q, seg_kv):
    for name, a in (("q", q), ("k", k), ("v", v)):
        if a.dtype != np.uint16 or a.ndim != 4 or not a.flags.c_contiguous:
            raise TypeError(f"{name} must be a C-contiguous uint16 (bf16 bits) [B,H,S,D] array")
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    if k.shape != (B, H, S_kv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B,H,S_kv,D] with the batch, heads and D of q")
    if (seg_q is None) != (seg_kv is None):
        raise ValueError("seg_q and seg_kv must both be given or both be None")
    if seg_q is not None:
        for name, a, s in (("seg_q", seg_q, S_q), ("seg_kv", seg_kv, S_kv)):
            if a.dtype != np.int32 or a.shape != (B, s) or not a.flags.c_contiguous:
                raise TypeError(f"{name} must be a C-contiguous int32 [B,{s}] array")
    return B, H, S_q, S_kv, D


def _window_args(window, B, S_q, S_kv):
    """window: dict(coord_q int32 [B,S_q], coord_kv int32 [B,S_kv], size (kt,kh,kw),
    extent (T,Hg,Wg), clamped bool).  Returns the ctypes arguments and the
    arrays they point to (kept alive by the caller)."""
    cq = np.ascontiguousarray(window["coord_q"], dtype=np.int32)
    ck = np.ascontiguousarray(window["coord_kv"], dtype=np.int32)
    if cq.shape != (B, S_q) or ck.shape != (B, S_kv):
        raise ValueError("window coordinates must be int32 [B,S_q] and [B,S_kv]")
    size = np.ascontiguousarray(window["size"], dtype=np.int64)
    extent = np.ascontiguousarray(window["extent"], dtype=np.int64)
    if size.shape != (3,) or extent.shape != (3,):
        raise ValueError("window size and extent have one entry per axis (t, h, w)")
    keep = (cq, ck, size, extent)
    return [_ptr(cq), _ptr(ck), _ptr(size), _ptr(extent), int(bool(window["clamped"]))], keep


def attn_fwd(q, k, v, seg_q=None, seg_kv=None, scale=None, nthreads=0, causal=False,
             window=None):
    """All rows.  Returns (out float64 [B,H,S_q,D], lse float64 [B,H,S_q])."""
    B, H, S_q, S_kv, D = _check_inputs(q, k, v, seg_q, seg_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, H, S_q, D), np.float64)
    lse = np.empty((B, H, S_q), np.float64)
    if window is not None:
        wargs, _keep = _window_args(window, B, S_q, S_kv)
        rc = _load().oracle_attn_win_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(seg_q),
                                             _ptr(seg_kv), *wargs, _ptr(out), _ptr(lse),
                                             B, H, S_q, S_kv, D, float(scale),
                                             int(bool(causal)), int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_win_fwd_f64 failed with code {rc}")
        return out, lse
    rc = _load().oracle_attn_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(seg_q), _ptr(seg_kv),
                                     _ptr(out), _ptr(lse), B, H, S_q, S_kv, D,
                                     float(scale), int(bool(causal)), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_f64 failed with code {rc}")
    return out, lse


def attn_rows(q, k, v, rows, seg_q=None, seg_kv=None, scale=None, nthreads=0, causal=False,
              window=None):
    """Selected rows.  rows: int64 [n,3] of (b, h, i).
    Returns (out float64 [n,D], lse float64 [n])."""
    B, H, S_q, S_kv, D = _check_inputs(q, k, v, seg_q, seg_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    if window is not None:
        wargs, _keep = _window_args(window, B, S_q, S_kv)
        rc = _load().oracle_attn_win_rows_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(seg_q),
                                              _ptr(seg_kv), *wargs, _ptr(rows), n, _ptr(out),
                                              _ptr(lse), B, H, S_q, S_kv, D, float(scale),
                                              int(bool(causal)), int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_win_rows_f64 failed with code {rc}")
        return out, lse
    rc = _load().oracle_attn_rows_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(seg_q), _ptr(seg_kv),
                                      _ptr(rows), n, _ptr(out), _ptr(lse),
                                      B, H, S_q, S_kv, D, float(scale), int(bool(causal)),
                                      int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_rows_f64 failed with code {rc}")
    return out, lse


def attn_probs(q, k, seg_q=None, seg_kv=None, scale=None, causal=False, window=None):
    """Softmax weights [B,H,S_q,S_kv] (small inputs only); masked entries are 0."""
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    _check_inputs(q, k, k, seg_q, seg_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    probs = np.empty((B, H, S_q, S_kv), np.float64)
    if window is not None:
        wargs, _keep = _window_args(window, B, S_q, S_kv)
        rc = _load().oracle_attn_win_probs_f64(_ptr(q), _ptr(k), _ptr(seg_q), _ptr(seg_kv),
                                               *wargs, _ptr(probs), B, H, S_q, S_kv, D,
                                               float(scale), int(bool(causal)))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_win_probs_f64 failed with code {rc}")
        return probs
    rc = _load().oracle_attn_probs_f64(_ptr(q), _ptr(k), _ptr(seg_q), _ptr(seg_kv),
                                       _ptr(probs), B, H, S_q, S_kv, D, float(scale),
                                       int(bool(causal)))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_probs_f64 failed with code {rc}")
    return probs
