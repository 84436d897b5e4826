"""torch.autograd binding of the scan: the forward is m3_scan_fwd (or
m3_scan_fwd_varlen), the backward m3_scan_bwd (m3_scan_bwd_varlen), both
through the C ABI.  Argument marshalling only; every step runs in the
library's kernels.

    y, final_state = m3_scan(x, dt, A, lam, theta, B, C, chunk=64, h0=None,
                             B_prev=None, x_prev=None)

Layouts as m3_scan_fwd.  Gradients flow to every tensor argument that
requires them.  Precision: the incoming gradient of y is handed to the
backward as it arrives, never rounded here.  torch's engine delivers the
gradient of an output in that output's dtype, so for a bf16 layer dy is
already bf16 when it gets here; callers that hold fp32 output gradients and
want them used unrounded call m3.m3_scan_bwd directly with an fp32 dy (the
C ABI's M3_FLAG_DY_F32).  The final-state gradient is fp32.  The backward
computes every gradient in fp32; each is returned in its input's dtype, as
torch requires (bf16 x, B, C, B_prev, x_prev receive bf16 gradients, rounded
to nearest even once, at the end; dt, A, lam, theta, h0 are fp32).
"""
from __future__ import annotations

import torch

from . import m3

_NAMES = ("x", "dt", "A", "lam", "theta", "B", "C", "h0", "B_prev", "x_prev")


def _dy(dy, x):
    """dy as the backward reads it: x's dtype, or fp32 unrounded (anything else
    is converted to fp32 first, which is exact for every narrower float)."""
    if dy.dtype != x.dtype and dy.dtype != torch.float32:
        dy = dy.float()
    return dy.contiguous()


class M3Scan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, chunk, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev):
        y, fs = m3.m3_scan_fwd(x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev)
        ctx.chunk = chunk
        ctx.save_for_backward(x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)
        return y, fs

    @staticmethod
    def backward(ctx, dy, d_final):
        x, dt, A, lam, theta, B, C, h0, B_prev, x_prev = ctx.saved_tensors
        if dy is None:
            dy = torch.zeros_like(x)
        g = m3.m3_scan_bwd(x, dt, A, lam, theta, B, C, _dy(dy, x), ctx.chunk,
                           h0, B_prev, x_prev,
                           None if d_final is None else d_final.contiguous().float())
        inputs = dict(zip(_NAMES, (x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)))
        out = [None]  # chunk
        for i, name in enumerate(_NAMES):
            t = inputs[name]
            if t is None or not ctx.needs_input_grad[i + 1] or name not in g:
                out.append(None)
            else:
                out.append(g[name].to(t.dtype))
        return tuple(out)


def m3_scan(x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None, B_prev=None, x_prev=None):
    """Differentiable chunked scan: (y, final_state), gradients by m3_scan_bwd."""
    return M3Scan.apply(chunk, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)


class M3ScanVarlen(torch.autograd.Function):
    @staticmethod
    def forward(ctx, chunk, max_seqlen, cu_seqlens, x, dt, A, lam, theta, B, C, h0, B_prev,
                x_prev):
        y, fs = m3.m3_scan_fwd_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, chunk, h0, B_prev,
                                      x_prev, max_seqlen=max_seqlen)
        ctx.chunk, ctx.max_seqlen = chunk, max_seqlen
        ctx.save_for_backward(cu_seqlens, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)
        return y, fs

    @staticmethod
    def backward(ctx, dy, d_final):
        cu, x, dt, A, lam, theta, B, C, h0, B_prev, x_prev = ctx.saved_tensors
        if dy is None:
            dy = torch.zeros_like(x)
        g = m3.m3_scan_bwd_varlen(cu, x, dt, A, lam, theta, B, C, _dy(dy, x),
                                  ctx.chunk, h0, B_prev, x_prev,
                                  None if d_final is None else d_final.contiguous().float(),
                                  max_seqlen=ctx.max_seqlen)
        inputs = dict(zip(_NAMES, (x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)))
        out = [None, None, None]  # chunk, max_seqlen, cu_seqlens
        for i, name in enumerate(_NAMES):
            t = inputs[name]
            if t is None or not ctx.needs_input_grad[i + 3] or name not in g:
                out.append(None)
            else:
                out.append(g[name].to(t.dtype))
        return tuple(out)


def m3_scan_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, chunk: int = 64, h0=None,
                   B_prev=None, x_prev=None, *, max_seqlen=None):
    """Differentiable scan of a packed batch (layouts of m3_scan_fwd_varlen):
    (y, final states), gradients by m3_scan_bwd_varlen."""
    if max_seqlen is None:
        S = cu_seqlens.numel() - 1
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if S > 0 else 0
    return M3ScanVarlen.apply(chunk, max_seqlen, cu_seqlens, x, dt, A, lam, theta, B, C, h0,
                              B_prev, x_prev)
