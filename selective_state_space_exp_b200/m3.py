"""Thin Python binding of libm3.so (the C ABI in include/m3.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch supplies device memory and the current stream.  There is no
fallback: if the library is missing or the tensors are not on a CUDA device,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# M3_LIBRARY=debug selects the bounds-checked build (lib/libm3_debug.so, see
# _build.build(debug=True)), whose kernels report M3_ERR_BOUNDS.
LIB_PATH = os.path.join(_PKG, "lib", "libm3_debug.so" if os.environ.get("M3_LIBRARY") == "debug"
                        else "libm3.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "m3.h")

M3_F32, M3_BF16 = 0, 1
M3_FLAG_SIMT = 1
M3_FLAG_TEST_TIMEOUT = 2
M3_FLAG_THETA_PER_HEAD = 4
M3_FLAG_DY_F32 = 8
M3_OK, M3_ERR_INVALID_ARGUMENT, M3_ERR_TIMEOUT = 0, -1, -6


def theta_flag(theta_groups: int, ngroups: int, nheads: int) -> int:
    """M3_FLAG_THETA_PER_HEAD when theta's group dimension is the head count
    (and differs from the B/C group count), 0 when it is the group count."""
    if theta_groups == ngroups:
        return 0
    if theta_groups == nheads:
        return M3_FLAG_THETA_PER_HEAD
    raise ValueError(f"theta has {theta_groups} groups: expected {ngroups} or {nheads}")


STATUS = {0: "M3_OK", -1: "M3_ERR_INVALID_ARGUMENT", -2: "M3_ERR_UNSUPPORTED",
          -3: "M3_ERR_ALIGNMENT", -4: "M3_ERR_WORKSPACE", -5: "M3_ERR_CUDA",
          -6: "M3_ERR_TIMEOUT", -7: "M3_ERR_BOUNDS"}


class M3Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, 'unknown')})")
        self.status = status


class Shape(ctypes.Structure):
    """m3_shape."""
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("rank", ctypes.c_int64), ("chunk", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_lib = None
_lock = threading.Lock()


def load() -> ctypes.CDLL:
    """Load libm3.so (built by __graft_entry__.build() or _build.py)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"library not built ({LIB_PATH}); run selective_state_space_exp_b200/_build.py")
            L = ctypes.CDLL(LIB_PATH)
            vp, sp = ctypes.c_void_p, ctypes.POINTER(Shape)
            L.m3_version.restype = ctypes.c_char_p
            L.m3_status_string.restype = ctypes.c_char_p
            L.m3_status_string.argtypes = [ctypes.c_int]
            L.m3_check_shape.argtypes = [sp]
            L.m3_check_shape.restype = ctypes.c_int
            L.m3_scan_workspace_size.argtypes = [sp, ctypes.POINTER(ctypes.c_size_t)]
            L.m3_scan_workspace_size.restype = ctypes.c_int
            L.m3_scan_workspace_bytes.argtypes = [sp]
            L.m3_scan_workspace_bytes.restype = ctypes.c_size_t
            L.m3_scan_plan.argtypes = [sp, ctypes.POINTER(ctypes.c_int),
                                       ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int)]
            L.m3_scan_plan.restype = ctypes.c_int
            L.m3_scan_fwd.argtypes = [sp] + [vp] * 13 + [ctypes.c_size_t, vp]
            L.m3_scan_fwd.restype = ctypes.c_int
            L.m3_scan_fwd_noalloc.argtypes = [sp] + [vp] * 13
            L.m3_scan_fwd_noalloc.restype = ctypes.c_int
            L.m3_decode_step.argtypes = [sp] + [vp] * 13
            L.m3_decode_step.restype = ctypes.c_int
            L.m3_stream_status.argtypes = [vp]
            L.m3_stream_status.restype = ctypes.c_int
            L.m3_scan_state_workspace_size.argtypes = [sp, ctypes.POINTER(ctypes.c_size_t)]
            L.m3_scan_state_workspace_size.restype = ctypes.c_int
            L.m3_scan_state.argtypes = [sp] + [vp] * 12 + [ctypes.c_size_t, vp]
            L.m3_scan_state.restype = ctypes.c_int
            L.m3_segment_totals.argtypes = [sp] + [vp] * 6
            L.m3_segment_totals.restype = ctypes.c_int
            L.m3_state_fold.argtypes = [sp, ctypes.c_int64] + [vp] * 6
            L.m3_state_fold.restype = ctypes.c_int
            L.m3_scan_fwd_varlen.argtypes = [sp, vp, ctypes.c_int64] + [vp] * 13 + \
                [ctypes.c_size_t, vp]
            L.m3_scan_fwd_varlen.restype = ctypes.c_int
            L.m3_scan_bwd_workspace_size.argtypes = [sp, ctypes.POINTER(ctypes.c_size_t)]
            L.m3_scan_bwd_workspace_size.restype = ctypes.c_int
            L.m3_scan_bwd.argtypes = [sp] + [vp] * 23 + [ctypes.c_size_t, vp]
            L.m3_scan_bwd.restype = ctypes.c_int
            L.m3_scan_bwd_varlen.argtypes = [sp, vp, ctypes.c_int64] + [vp] * 23 + \
                [ctypes.c_size_t, vp]
            L.m3_scan_bwd_varlen.restype = ctypes.c_int
            L.m3_bc_prep.argtypes = [sp] + [vp] * 6 + [ctypes.c_float, vp, vp, vp]
            L.m3_bc_prep.restype = ctypes.c_int
            L.m3_linear.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64] + [vp] * 4 + \
                [ctypes.c_int32, vp]
            L.m3_linear.restype = ctypes.c_int
            L.m3_mimo_up.argtypes = [sp] + [vp] * 4
            L.m3_mimo_up.restype = ctypes.c_int
            L.m3_mimo_down_gate.argtypes = [sp] + [vp] * 5
            L.m3_mimo_down_gate.restype = ctypes.c_int
            _lib = L
    return _lib


def _check(fn: str, st: int):
    if st != 0:
        raise M3Error(fn, st)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _io_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return M3_BF16
    if dtype == torch.float32:
        return M3_F32
    raise ValueError(f"unsupported io dtype {dtype}")


def make_shape(batch, seqlen, nheads, ngroups, headdim, dstate, rank, chunk, io_dtype,
               simt=False) -> Shape:
    return Shape(batch, seqlen, nheads, ngroups, headdim, dstate, rank, chunk,
                 _io_code(io_dtype) if isinstance(io_dtype, torch.dtype) else int(io_dtype),
                 M3_FLAG_SIMT if simt else 0)


def scan_shape(x: torch.Tensor, B: torch.Tensor, chunk: int, simt=False, theta=None) -> Shape:
    """Shape of a scan call; theta (if given) decides grouped or per-head rates."""
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    s = make_shape(b, L, H, G, P, N, R, chunk, x.dtype, simt)
    if theta is not None:
        s.flags |= theta_flag(theta.shape[2], G, H)
    return s


def workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check("m3_scan_workspace_size", load().m3_scan_workspace_size(ctypes.byref(shape),
                                                                   ctypes.byref(n)))
    return int(n.value)


def scan_plan(shape: Shape) -> dict:
    """How m3_scan_fwd runs `shape`: tensor_core (bool), segments, launches."""
    tc, seg, n = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int()
    _check("m3_scan_plan", load().m3_scan_plan(ctypes.byref(shape), ctypes.byref(tc),
                                               ctypes.byref(seg), ctypes.byref(n)))
    return {"tensor_core": bool(tc.value), "segments": int(seg.value), "launches": int(n.value)}


def m3_scan_fwd(x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None, B_prev=None,
                x_prev=None, *, y=None, final_state=None, want_final=True, workspace=None,
                simt=False, stream=None, extra_flags=0):
    """Chunked prefill scan.  x [b][L][H][R][P] (io dtype), dt/A/lam [b][L][H],
    theta [b][L][G][N/2] fp32, B/C [b][L][G][R][N] (io dtype).  R is x.shape[3].
    extra_flags: further M3_FLAG_* bits (diagnostics).  Returns (y, final_state)."""
    shape = scan_shape(x, B, chunk, simt, theta)
    shape.flags |= extra_flags
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((x.shape[0], x.shape[2], B.shape[4], x.shape[4]),
                                  dtype=torch.float32, device=x.device)
    need = workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    st = load().m3_scan_fwd(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam),
                            _ptr(theta), _ptr(B), _ptr(C), _ptr(h0), _ptr(B_prev),
                            _ptr(x_prev), _ptr(y), _ptr(final_state), _ptr(workspace),
                            ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("m3_scan_fwd", st)
    return y, final_state


def m3_scan_fwd_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None,
                       B_prev=None, x_prev=None, *, max_seqlen=None, y=None, final_state=None,
                       want_final=True, workspace=None, simt=False, stream=None):
    """Packed batch of S independent sequences: cu_seqlens [S+1] int32 on the
    device (sequence i is token rows cu_seqlens[i]:cu_seqlens[i+1]); x [T][H][R][P],
    dt/A/lam [T][H], theta [T][G][N/2], B/C [T][G][R][N]; h0 [S][H][N][P],
    B_prev [S][G][R][N], x_prev [S][H][R][P].  max_seqlen bounds every
    sequence's length (read from cu_seqlens, with a device sync, when None).
    Returns (y [T][H][R][P], final_state [S][H][N][P])."""
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    S = cu_seqlens.numel() - 1
    T, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    if max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if S > 0 else 0
    shape = make_shape(S, max_seqlen, H, G, P, N, R, chunk, x.dtype, simt)
    shape.flags |= theta_flag(theta.shape[1], G, H)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((S, H, N, P), dtype=torch.float32, device=x.device)
    need = workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    st = load().m3_scan_fwd_varlen(ctypes.byref(shape), _ptr(cu_seqlens), ctypes.c_int64(T),
                                   _ptr(x), _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(B),
                                   _ptr(C), _ptr(h0), _ptr(B_prev), _ptr(x_prev), _ptr(y),
                                   _ptr(final_state), _ptr(workspace),
                                   ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("m3_scan_fwd_varlen", st)
    return y, final_state


def m3_bc_prep(B_raw=None, C_raw=None, B_weight=None, B_bias=None, C_weight=None, C_bias=None,
               eps: float = 1e-6, *, B=None, C=None, stream=None):
    """QK-norm + per-channel scale + bias of raw B / C projections, either
    [b][L][G][R][N] (scan layout) or [b][G][R][N] (decode layout), io dtype.
    weight / bias [G][R][N] fp32 or None.  Returns (B, C) (None for a skipped one)."""
    ref = B_raw if B_raw is not None else C_raw
    if ref.dim() == 5:
        b, L, G, R, N = ref.shape
    else:
        (b, G, R, N), L = ref.shape, 1
    if B_raw is not None and B is None:
        B = torch.empty_like(B_raw)
    if C_raw is not None and C is None:
        C = torch.empty_like(C_raw)
    shape = make_shape(b, L, G, G, 16, N, R, 64, ref.dtype)
    st = load().m3_bc_prep(ctypes.byref(shape), _ptr(B_raw), _ptr(C_raw), _ptr(B_weight),
                           _ptr(B_bias), _ptr(C_weight), _ptr(C_bias), ctypes.c_float(eps),
                           _ptr(B), _ptr(C), _stream(stream))
    _check("m3_bc_prep", st)
    return B, C


def dy_flag(dy: torch.Tensor, x: torch.Tensor) -> int:
    """M3_FLAG_DY_F32 when dy is fp32 and the io dtype is not; otherwise dy
    must have x's dtype."""
    if dy.dtype == x.dtype:
        return 0
    if dy.dtype == torch.float32:
        return M3_FLAG_DY_F32
    raise TypeError(f"dy is {dy.dtype}: expected {x.dtype} or torch.float32")


def bwd_workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check("m3_scan_bwd_workspace_size",
           load().m3_scan_bwd_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return int(n.value)


def m3_scan_bwd(x, dt, A, lam, theta, B, C, dy, chunk: int = 64, h0=None, B_prev=None,
                x_prev=None, d_final=None, *, want_dh0=True, workspace=None, simt=False,
                stream=None):
    """Backward of m3_scan_fwd: gradients of sum(y * dy) + sum(final * d_final)
    with respect to every input.  dy has x's dtype, or fp32 (read unrounded).
    Returns a dict of fp32 tensors: x, dt, A, lam, theta, B, C, and h0 (when
    want_dh0), B_prev and x_prev (when B_prev is given), each in its input's
    layout.  bf16 io at N = 128, P = 64 runs on the tensor cores (bf16
    operands) unless simt is set (CUDA cores, fp32 throughout)."""
    shape = scan_shape(x, B, chunk, simt, theta)
    shape.flags |= dy_flag(dy, x)
    dev, f32 = x.device, torch.float32
    g = {"x": torch.empty(x.shape, dtype=f32, device=dev),
         "dt": torch.empty(dt.shape, dtype=f32, device=dev),
         "A": torch.empty(A.shape, dtype=f32, device=dev),
         "lam": torch.empty(lam.shape, dtype=f32, device=dev),
         "theta": torch.empty(theta.shape, dtype=f32, device=dev),
         "B": torch.empty(B.shape, dtype=f32, device=dev),
         "C": torch.empty(C.shape, dtype=f32, device=dev)}
    if want_dh0:
        g["h0"] = torch.empty((x.shape[0], x.shape[2], B.shape[4], x.shape[4]), dtype=f32,
                              device=dev)
    if B_prev is not None:
        g["B_prev"] = torch.empty(B_prev.shape, dtype=f32, device=dev)
        g["x_prev"] = torch.empty(x_prev.shape, dtype=f32, device=dev)
    need = bwd_workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = load().m3_scan_bwd(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam),
                            _ptr(theta), _ptr(B), _ptr(C), _ptr(h0), _ptr(B_prev), _ptr(x_prev),
                            _ptr(dy), _ptr(d_final), _ptr(g["x"]), _ptr(g["dt"]), _ptr(g["A"]),
                            _ptr(g["lam"]), _ptr(g["theta"]), _ptr(g["B"]), _ptr(g["C"]),
                            _ptr(g.get("h0")), _ptr(g.get("B_prev")), _ptr(g.get("x_prev")),
                            _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("m3_scan_bwd", st)
    return g


def m3_scan_bwd_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, dy, chunk: int = 64, h0=None,
                       B_prev=None, x_prev=None, d_final=None, *, max_seqlen=None,
                       want_dh0=True, workspace=None, simt=False, stream=None):
    """Backward of m3_scan_fwd_varlen (packed tensors without a batch
    dimension, as there).  Returns the gradient dict of m3_scan_bwd; simt as
    there."""
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    S = cu_seqlens.numel() - 1
    T, H, R, P = x.shape
    G, N = B.shape[1], B.shape[3]
    if max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if S > 0 else 0
    shape = make_shape(S, max_seqlen, H, G, P, N, R, chunk, x.dtype, simt)
    shape.flags |= theta_flag(theta.shape[1], G, H) | dy_flag(dy, x)
    dev, f32 = x.device, torch.float32
    g = {k: torch.empty(v.shape, dtype=f32, device=dev)
         for k, v in (("x", x), ("dt", dt), ("A", A), ("lam", lam), ("theta", theta), ("B", B),
                      ("C", C))}
    if want_dh0:
        g["h0"] = torch.empty((S, H, N, P), dtype=f32, device=dev)
    if B_prev is not None:
        g["B_prev"] = torch.empty(B_prev.shape, dtype=f32, device=dev)
        g["x_prev"] = torch.empty(x_prev.shape, dtype=f32, device=dev)
    need = bwd_workspace_size(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = load().m3_scan_bwd_varlen(
        ctypes.byref(shape), _ptr(cu_seqlens), ctypes.c_int64(T), _ptr(x), _ptr(dt), _ptr(A),
        _ptr(lam), _ptr(theta), _ptr(B), _ptr(C), _ptr(h0), _ptr(B_prev), _ptr(x_prev), _ptr(dy),
        _ptr(d_final), _ptr(g["x"]), _ptr(g["dt"]), _ptr(g["A"]), _ptr(g["lam"]),
        _ptr(g["theta"]), _ptr(g["B"]), _ptr(g["C"]), _ptr(g.get("h0")), _ptr(g.get("B_prev")),
        _ptr(g.get("x_prev")), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
        _stream(stream))
    _check("m3_scan_bwd_varlen", st)
    return g


def m3_scan_fwd_noalloc(x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None, B_prev=None,
                        x_prev=None, *, y=None, final_state=None, want_final=True, simt=False,
                        stream=None):
    """m3_scan_fwd without a workspace argument: the library's fixed device
    scratch (M3_NOALLOC_SCRATCH_BYTES) serves instead, for callers that cannot
    allocate device memory.  Returns (y, final_state)."""
    shape = scan_shape(x, B, chunk, simt, theta)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and want_final:
        final_state = torch.empty((x.shape[0], x.shape[2], B.shape[4], x.shape[4]),
                                  dtype=torch.float32, device=x.device)
    st = load().m3_scan_fwd_noalloc(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam),
                                    _ptr(theta), _ptr(B), _ptr(C), _ptr(h0), _ptr(B_prev),
                                    _ptr(x_prev), _ptr(y), _ptr(final_state), _stream(stream))
    _check("m3_scan_fwd_noalloc", st)
    return y, final_state


def m3_scan_state(x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None, B_prev=None,
                  x_prev=None, *, final_state=None, workspace=None, simt=False, stream=None):
    """The state after every sequence's last token, [b][H][N][P] fp32, without y."""
    shape = scan_shape(x, B, chunk, simt, theta)
    if final_state is None:
        final_state = torch.empty((x.shape[0], x.shape[2], B.shape[4], x.shape[4]),
                                  dtype=torch.float32, device=x.device)
    n = ctypes.c_size_t(0)
    _check("m3_scan_state_workspace_size",
           load().m3_scan_state_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(int(n.value), 1), dtype=torch.uint8, device=x.device)
    st = load().m3_scan_state(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(lam),
                              _ptr(theta), _ptr(B), _ptr(C), _ptr(h0), _ptr(B_prev),
                              _ptr(x_prev), _ptr(final_state), _ptr(workspace),
                              ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check("m3_scan_state", st)
    return final_state


def m3_segment_totals(x, dt, A, theta, B, chunk: int = 64, *, stream=None):
    """(lam_tot [b][H], phi_tot [b][H][N/2]): sum over the tokens of dt*A and
    of dt*theta for every (batch, head)."""
    shape = scan_shape(x, B, chunk, False, theta)
    b, _, H = dt.shape
    K = B.shape[4] // 2
    lam_tot = torch.empty((b, H), dtype=torch.float32, device=dt.device)
    phi_tot = torch.empty((b, H, K), dtype=torch.float32, device=dt.device)
    _check("m3_segment_totals", load().m3_segment_totals(
        ctypes.byref(shape), _ptr(dt), _ptr(A), _ptr(theta), _ptr(lam_tot), _ptr(phi_tot),
        _stream(stream)))
    return lam_tot, phi_tot


def m3_state_fold(h0, T, lam_tot, phi_tot, *, out=None, stream=None):
    """Fold segment summaries: h = h0 (None: zero); for each s:
    h = Rot(phi_tot[s]) exp(lam_tot[s]) h + T[s].  T [nseg][b][H][N][P]."""
    nseg, b, H, N, P = T.shape
    shape = make_shape(b, 1, H, 1, P, N, 1, 64, torch.float32)
    if out is None:
        out = torch.empty((b, H, N, P), dtype=torch.float32, device=T.device)
    _check("m3_state_fold", load().m3_state_fold(
        ctypes.byref(shape), ctypes.c_int64(nseg), _ptr(h0), _ptr(T) if nseg else None,
        _ptr(lam_tot) if nseg else None, _ptr(phi_tot) if nseg else None, _ptr(out),
        _stream(stream)))
    return out


def m3_decode_step(state, x_t, dt, A, lam, theta, B_t, C_t, B_prev=None, x_prev=None, *,
                   state_out=None, y=None, stream=None):
    """One decode step.  state [b][H][N][P] fp32; x_t [b][H][R][P]; dt/A/lam [b][H];
    theta [b][G][N/2] (or [b][H][N/2], per head); B_t/C_t [b][G][R][N].
    state_out defaults to `state` (in place).  Returns (y_t, state_out)."""
    b, H, R, P = x_t.shape
    G, N = B_t.shape[1], B_t.shape[3]
    shape = make_shape(b, 1, H, G, P, N, R, 64, x_t.dtype)
    shape.flags |= theta_flag(theta.shape[1], G, H)
    if state_out is None:
        state_out = state
    if y is None:
        y = torch.empty_like(x_t)
    st = load().m3_decode_step(ctypes.byref(shape), _ptr(state), _ptr(state_out), _ptr(x_t),
                               _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(B_t),
                               _ptr(C_t), _ptr(B_prev), _ptr(x_prev), _ptr(y),
                               _stream(stream))
    _check("m3_decode_step", st)
    return y, state_out


def m3_stream_status(stream=None) -> int:
    """Synchronise the stream and return the first device-side status."""
    return int(load().m3_stream_status(_stream(stream)))


def version() -> str:
    return load().m3_version().decode()


# ---- block projections around the layer ---------------------------------------

def m3_linear(A, W, bias=None, *, out=None, out_dtype=torch.bfloat16, stream=None):
    """out = A W^T (+ bias) on the tensor cores: A [..][K] bf16 (rows are
    tokens), W [N][K] bf16, bias [N] fp32; returns out [..][N] in out_dtype
    (bf16 or fp32)."""
    if A.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("m3_linear takes bf16 A and W")
    K = A.shape[-1]
    M = A.numel() // K if K else 0
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError(f"W is {tuple(W.shape)}, expected [N][{K}]")
    if out is None:
        out = torch.empty(A.shape[:-1] + (N,), dtype=out_dtype, device=A.device)
    code = M3_F32 if out.dtype == torch.float32 else M3_BF16
    st = load().m3_linear(ctypes.c_int64(M), ctypes.c_int64(N), ctypes.c_int64(K), _ptr(A),
                          _ptr(W), _ptr(bias), _ptr(out), ctypes.c_int32(code), _stream(stream))
    _check("m3_linear", st)
    return out


def _tokens_shape(T, H, R, P, dtype):
    """m3_shape of a block step over T tokens (one sequence of T tokens; the
    scan-only fields get admissible placeholders)."""
    return make_shape(1, T, H, 1, P, 16, R, 64, dtype, False)


def m3_mimo_up(x, w_up, *, X=None, stream=None):
    """X[..][h][r][p] = x[..][h][p] * w_up[h][r][p]: x [..][H][P] io dtype,
    w_up [H][R][P] fp32; returns X [..][H][R][P]."""
    H, R, P = w_up.shape
    T = x.numel() // (H * P)
    if X is None:
        X = torch.empty(x.shape[:-1] + (R, P), dtype=x.dtype, device=x.device)
    shape = _tokens_shape(T, H, R, P, x.dtype)
    st = load().m3_mimo_up(ctypes.byref(shape), _ptr(x), _ptr(w_up), _ptr(X), _stream(stream))
    _check("m3_mimo_up", st)
    return X


def m3_mimo_down_gate(Y, w_down, z=None, *, out=None, stream=None):
    """out[..][h][p] = (sum_r Y[..][h][r][p] w_down[h][r][p]) * silu(z[..][h][p]):
    Y [..][H][R][P] io dtype, w_down [H][R][P] fp32, z [..][H][P] io dtype or
    None (no gate); returns out [..][H][P]."""
    H, R, P = w_down.shape
    T = Y.numel() // (H * R * P)
    if out is None:
        out = torch.empty(Y.shape[:-2] + (P,), dtype=Y.dtype, device=Y.device)
    shape = _tokens_shape(T, H, R, P, Y.dtype)
    st = load().m3_mimo_down_gate(ctypes.byref(shape), _ptr(Y), _ptr(w_down), _ptr(z), _ptr(out),
                                  _stream(stream))
    _check("m3_mimo_down_gate", st)
    return out
