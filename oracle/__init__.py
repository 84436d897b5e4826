"""CPU oracle for the Mamba-3 SSM layer (fp64, plain C, loaded with ctypes).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline / reference legs of bench.py.  The library's product path never
imports it, and this package never imports the product library.

The C source (m3_oracle.c) holds the arithmetic and cites the paper passages
it follows.  This module only compiles it (gcc) and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None


class Dims(ctypes.Structure):
    # tgroups: theta groups (its third dimension: G like B and C, or H)
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "ngroups", "headdim", "dstate", "rank",
                 "tgroups")]


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/liboracle.so (gcc, -O2, C11)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall",
                        "-o", tmp, _SRC, "-lm", "-lpthread"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            vp, i64p, dp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.c_void_p
            L.m3o_scan.argtypes = [ctypes.POINTER(Dims), ctypes.c_int] + [vp] * 10 + \
                [dp, dp, vp, ctypes.c_int64, ctypes.c_int]
            L.m3o_scan.restype = ctypes.c_int
            L.m3o_decode_step.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, dp] + [vp] * 9 + [dp]
            L.m3o_decode_step.restype = ctypes.c_int
            for name in ("m3o_scan_mask", "m3o_scan_rope"):
                f = getattr(L, name)
                f.argtypes = [ctypes.POINTER(Dims)] + [vp] * 12
                f.restype = ctypes.c_int
            L.m3o_set_mutation.argtypes = [ctypes.c_int]
            L.m3o_set_mutation.restype = None
            L.m3o_get_mutation.restype = ctypes.c_int
            _lib = L
    return _lib


def _np(a, dtype):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> numpy (bf16 widened exactly)
        import torch
        a = a.detach().to("cpu")
        if a.dtype == torch.bfloat16:
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dims(x, B, theta):
    # x: [b][L][H][R][P], B: [b][L][G][R][N]
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    return Dims(b, L, H, G, P, N, R, theta.shape[2])


def scan(x, dt, A, lam, theta, B, C, h0=None, B_prev=None, x_prev=None,
         chains=None, nthreads=None, f64=False):
    """Token-by-token fp64 recurrence.  Returns (y, hL) as float64 arrays of the
    full shapes; only the listed chains (flat b*H + h) are filled when `chains`
    is given (the rest stay NaN).  Inputs may be numpy arrays or torch tensors;
    bf16 values are widened exactly.  With f64=True inputs are passed as fp64
    (for pins that need more than fp32 input precision)."""
    dt_ = np.float64 if f64 else np.float32
    arrs = [_np(v, dt_) for v in (x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)]
    d = _dims(arrs[0], arrs[5], arrs[4])
    y = np.full(arrs[0].shape, np.nan, dtype=np.float64)
    hL = np.full((d.batch, d.nheads, d.dstate, d.headdim), np.nan, dtype=np.float64)
    ch = None if chains is None else np.ascontiguousarray(chains, dtype=np.int64)
    if nthreads is None:
        nthreads = max(1, len(os.sched_getaffinity(0)))
    rc = lib().m3o_scan(ctypes.byref(d), 1 if f64 else 0, *[_ptr(a) for a in arrs],
                        y.ctypes.data_as(ctypes.c_void_p),
                        hL.ctypes.data_as(ctypes.c_void_p),
                        None if ch is None else ch.ctypes.data_as(ctypes.c_void_p),
                        0 if ch is None else len(ch), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"m3o_scan failed: {rc}")
    return y, hL


def scan_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, h0=None, B_prev=None, x_prev=None,
                nthreads=None):
    """Packed batch of independent sequences: sequence i is rows
    cu_seqlens[i]:cu_seqlens[i+1] of the token dimension of x [T][H][R][P],
    dt/A/lam [T][H], theta [T][G][N/2], B/C [T][G][R][N], with its own h0[i],
    B_prev[i], x_prev[i].  No state crosses a boundary, so this is `scan`
    (the token recurrence) applied to each sequence alone.  Returns y
    [T][H][R][P] (rows outside every sequence stay NaN) and the final states
    [S][H][N][P], float64."""
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    x, dt, A, lam, theta, B, C = (_np(v, np.float32) for v in (x, dt, A, lam, theta, B, C))
    h0, B_prev, x_prev = (_np(v, np.float32) for v in (h0, B_prev, x_prev))
    S = len(cu) - 1
    y = np.full(x.shape, np.nan, dtype=np.float64)
    hL = np.empty((S, x.shape[1], B.shape[3], x.shape[3]), dtype=np.float64)
    for i in range(S):
        a, e = cu[i], cu[i + 1]
        one = lambda v: None if v is None else v[i:i + 1]
        yi, hi = scan(x[None, a:e], dt[None, a:e], A[None, a:e], lam[None, a:e],
                      theta[None, a:e], B[None, a:e], C[None, a:e], h0=one(h0),
                      B_prev=one(B_prev), x_prev=one(x_prev), nthreads=nthreads)
        y[a:e] = yi[0]
        hL[i] = hi[0]
    return y, hL


def decode_step(state, x_t, dt, A, lam, theta, B_t, C_t, B_prev=None, x_prev=None,
                f64=False):
    """One decode step for every (b, h).  state [b][H][N][P] is copied and
    updated in fp64; returns (y_t [b][H][R][P], new_state)."""
    dt_ = np.float64 if f64 else np.float32
    st = np.array(_np(state, np.float64), dtype=np.float64, copy=True)
    arrs = [_np(v, dt_) for v in (x_t, dt, A, lam, theta, B_t, C_t, B_prev, x_prev)]
    b, H, R, P = arrs[0].shape
    G, N = arrs[5].shape[1], arrs[5].shape[3]
    d = Dims(b, 1, H, G, P, N, R, arrs[4].shape[1])
    y = np.zeros((b, H, R, P), dtype=np.float64)
    rc = lib().m3o_decode_step(ctypes.byref(d), 1 if f64 else 0,
                               st.ctypes.data_as(ctypes.c_void_p),
                               *[_ptr(a) for a in arrs], y.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise RuntimeError(f"m3o_decode_step failed: {rc}")
    return y, st


def _pin_form(name, x, dt, A, lam, theta, B, C, h0=None, B_prev=None, x_prev=None):
    arrs = [_np(v, np.float64) for v in (x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)]
    d = _dims(arrs[0], arrs[5], arrs[4])
    y = np.zeros(arrs[0].shape, dtype=np.float64)
    hL = np.zeros((d.batch, d.nheads, d.dstate, d.headdim), dtype=np.float64)
    rc = getattr(lib(), name)(ctypes.byref(d), *[_ptr(a) for a in arrs],
                              y.ctypes.data_as(ctypes.c_void_p),
                              hL.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise RuntimeError(f"{name} failed: {rc}")
    return y, hL


def scan_mask(*args, **kw):
    """Materialised structured-mask form (decay mask x width-2 convolution)."""
    return _pin_form("m3o_scan_mask", *args, **kw)


def scan_rope(*args, **kw):
    """Data-dependent RoPE form (real rotations + real quadratic form)."""
    return _pin_form("m3o_scan_rope", *args, **kw)


class mutation:
    """Context manager that plants a known mistake in the oracle (tests only)."""

    def __init__(self, m: int):
        self.m = m

    def __enter__(self):
        lib().m3o_set_mutation(self.m)
        return self

    def __exit__(self, *exc):
        lib().m3o_set_mutation(0)
        return False
