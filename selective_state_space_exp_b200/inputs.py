"""Seeded synthetic inputs for the Mamba-3 SSM layer.

This module only draws random tensors with the workload's shapes and value
distributions; it holds none of the layer's arithmetic, so both the CUDA path
and the CPU oracle can consume its output.

Distributions (normal variances, not standard deviations):
  x       ~ N(0, 1)
  dt      = softplus(N(-2, 0.5))
  A       = -exp(U(0, ln 16))            ("fast" decay, the workload default)
          = -exp(U(ln 0.01, ln 0.1))     ("slow" decay: state survives chunks)
  lam     = sigmoid(N(0, 1))
  theta   ~ U(-pi, pi)                   angle rate; the step angle is dt*theta
  B, C    ~ N(0, 1/N)                    ("normal")
          or RMS-normalised N(0, 1) per (token, group, rank) over N, plus a
          bias ~ N(0, 0.1) drawn once per (group, rank, n)   ("rmsnorm")
  h0      ~ N(0, 1)
Values of the io dtype are rounded to it (bf16: round to nearest even) before
they are handed to either side, so both sides read identical numbers.

Tensor layouts are the library's (row-major):
  x: [b][L][H][R][P]   B, C: [b][L][G][R][N]   dt, A, lam: [b][L][H]
  theta: [b][L][G][N/2]   h0: [b][H][N][P]   B_prev: [b][G][R][N]
  x_prev: [b][H][R][P]
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Shape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int   # P
    dstate: int    # N
    rank: int = 1  # R
    ngroups: int = 1
    chunk: int = 64
    io: str = "bf16"  # "bf16" or "f32"

    @property
    def io_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.io == "bf16" else torch.float32


@dataclass
class Workload:
    shape: Shape
    bc: str = "rmsnorm"      # "rmsnorm" or "normal"
    decay: str = "fast"      # "fast" or "slow"
    with_h0: bool = False
    with_prev: bool = False
    theta_per_head: bool = False  # theta [..][H][N/2] instead of [..][G][N/2]


# The five workloads the layer is measured and checked on.
TINY_SISO_F32 = Workload(Shape(1, 256, 1, 16, 16, 1, 1, 64, "f32"), bc="normal")
SISO_PREFILL = Workload(Shape(8, 2048, 64, 64, 128, 1, 1, 64, "bf16"))
MIMO_PREFILL = Workload(Shape(8, 2048, 64, 64, 128, 4, 1, 64, "bf16"))
DECODE_SISO = Workload(Shape(128, 1, 64, 64, 128, 1, 1, 64, "bf16"), with_h0=True, with_prev=True)
DECODE_MIMO = Workload(Shape(128, 1, 64, 64, 128, 4, 1, 64, "bf16"), with_h0=True, with_prev=True)
LONG_MIMO_32K = Workload(Shape(1, 32768, 64, 64, 128, 4, 1, 64, "bf16"))
LONG_MIMO_16K = Workload(Shape(1, 16384, 64, 64, 128, 4, 1, 64, "bf16"))


def _gen(seed: int, device: str | torch.device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, mean, var, device):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(math.sqrt(var)).add_(mean)


def _uniform(g, shape, lo, hi, device):
    t = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    return t.mul_(hi - lo).add_(lo)


def _round_io(t: torch.Tensor, io: str) -> torch.Tensor:
    """Round to the io dtype and return it in that dtype."""
    return t.to(torch.bfloat16) if io == "bf16" else t.contiguous()


def _bc(g, s: Shape, lead: tuple, kind: str, device, bias=None):
    n = s.dstate
    shp = lead + (s.ngroups, s.rank, n)
    if kind == "normal":
        return _normal(g, shp, 0.0, 1.0 / n, device)
    v = _normal(g, shp, 0.0, 1.0, device)
    v = v / torch.sqrt(v.pow(2).mean(dim=-1, keepdim=True) + 1e-6)
    return v + bias


def draw_token_gates(g, s: Shape, lead: tuple, decay: str, device, theta_per_head=False):
    """dt, A, lam with shape lead + (H,), theta with shape lead + (G, N/2)
    (lead + (H, N/2) for per-head angle rates)."""
    H = s.nheads
    dt = torch.nn.functional.softplus(_normal(g, lead + (H,), -2.0, 0.5, device))
    if decay == "slow":
        A = -torch.exp(_uniform(g, lead + (H,), math.log(0.01), math.log(0.1), device))
    else:
        A = -torch.exp(_uniform(g, lead + (H,), 0.0, math.log(16.0), device))
    lam = torch.sigmoid(_normal(g, lead + (H,), 0.0, 1.0, device))
    tg = s.nheads if theta_per_head else s.ngroups
    theta = _uniform(g, lead + (tg, s.dstate // 2), -math.pi, math.pi, device)
    return dt.contiguous(), A.contiguous(), lam.contiguous(), theta.contiguous()


def make_scan_inputs(w: Workload, seed: int, device: str | torch.device = "cpu") -> dict:
    """Inputs of one prefill scan.  Returns a dict of tensors on `device`:
    x, B, C (io dtype), dt, A, lam, theta (fp32), optionally h0 (fp32) and
    B_prev, x_prev (io dtype)."""
    s = w.shape
    g = _gen(seed, device)
    lead = (s.batch, s.seqlen)
    bias = None
    if w.bc == "rmsnorm":
        bias = _normal(g, (s.ngroups, s.rank, s.dstate), 0.0, 0.1, device)
    x = _normal(g, lead + (s.nheads, s.rank, s.headdim), 0.0, 1.0, device)
    dt, A, lam, theta = draw_token_gates(g, s, lead, w.decay, device, w.theta_per_head)
    B = _bc(g, s, lead, w.bc, device, bias)
    C = _bc(g, s, lead, w.bc, device, bias)
    out = dict(x=_round_io(x, s.io), B=_round_io(B, s.io), C=_round_io(C, s.io),
               dt=dt, A=A, lam=lam, theta=theta)
    if w.with_h0:
        out["h0"] = _normal(g, (s.batch, s.nheads, s.dstate, s.headdim), 0.0, 1.0, device)
    if w.with_prev:
        out["B_prev"] = _round_io(_bc(g, s, (s.batch,), w.bc, device, bias), s.io)
        out["x_prev"] = _round_io(
            _normal(g, (s.batch, s.nheads, s.rank, s.headdim), 0.0, 1.0, device), s.io)
    return out


def make_decode_inputs(w: Workload, seed: int, steps: int,
                       device: str | torch.device = "cpu") -> dict:
    """Inputs of `steps` consecutive decode steps for batch*H chains:
    state0 [b][H][N][P] fp32, x [steps][b][H][R][P], B and C
    [steps][b][G][R][N] (io dtype), dt, A, lam [steps][b][H], theta
    [steps][b][G][N/2] (fp32), and B_prev [b][G][R][N], x_prev [b][H][R][P]
    for step 0 (drawn like any token).  Step t's previous token is step t-1."""
    s = w.shape
    g = _gen(seed, device)
    bias = None
    if w.bc == "rmsnorm":
        bias = _normal(g, (s.ngroups, s.rank, s.dstate), 0.0, 0.1, device)
    state0 = _normal(g, (s.batch, s.nheads, s.dstate, s.headdim), 0.0, 1.0, device)
    lead = (steps, s.batch)
    x = _normal(g, lead + (s.nheads, s.rank, s.headdim), 0.0, 1.0, device)
    dt, A, lam, theta = draw_token_gates(g, s, lead, w.decay, device, w.theta_per_head)
    B = _bc(g, s, lead, w.bc, device, bias)
    C = _bc(g, s, lead, w.bc, device, bias)
    B_prev = _bc(g, s, (s.batch,), w.bc, device, bias)
    x_prev = _normal(g, (s.batch, s.nheads, s.rank, s.headdim), 0.0, 1.0, device)
    return dict(state0=state0, x=_round_io(x, s.io), B=_round_io(B, s.io),
                C=_round_io(C, s.io), dt=dt, A=A, lam=lam, theta=theta,
                B_prev=_round_io(B_prev, s.io), x_prev=_round_io(x_prev, s.io))


def varlen_lengths(count: int, max_len: int, chunk: int, seed: int) -> list[int]:
    """A seeded length mix for a packed batch of `count` sequences: the edge
    lengths 0, 1, chunk - 1, chunk, chunk + 1 and max_len first (those that fit
    in `count`), the rest uniform in [1, max_len]."""
    edges = [v for v in (0, 1, chunk - 1, chunk, chunk + 1, max_len) if 0 <= v <= max_len]
    g = torch.Generator().manual_seed(int(seed))
    rest = torch.randint(1, max_len + 1, (max(0, count - len(edges)),), generator=g).tolist()
    return (edges + rest)[:count]


def make_varlen_inputs(w: Workload, lengths: list[int], seed: int,
                       device: str | torch.device = "cpu") -> dict:
    """Inputs of a packed batch of len(lengths) sequences stored back to back:
    the per-token tensors of make_scan_inputs without the batch dimension
    (x [T][H][R][P], dt [T][H], ...; T = sum(lengths)), drawn with the
    workload's distributions; cu_seqlens [S+1] int32; and, per sequence, h0
    [S][H][N][P] and B_prev, x_prev [S][..] when the workload asks for them.
    w.shape.batch and w.shape.seqlen are ignored."""
    s = w.shape
    T, S = int(sum(lengths)), len(lengths)
    packed = replace(w, shape=replace(s, batch=1, seqlen=T), with_h0=False, with_prev=False)
    out = {k: v[0].contiguous() for k, v in make_scan_inputs(packed, seed, device).items()}
    g = _gen(seed + 1, device)
    if w.with_h0:
        out["h0"] = _normal(g, (S, s.nheads, s.dstate, s.headdim), 0.0, 1.0, device)
    if w.with_prev:
        bias = _normal(g, (s.ngroups, s.rank, s.dstate), 0.0, 0.1, device)
        out["B_prev"] = _round_io(_bc(g, s, (S,), w.bc, device, bias), s.io)
        out["x_prev"] = _round_io(_normal(g, (S, s.nheads, s.rank, s.headdim), 0.0, 1.0, device),
                                  s.io)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    return out


def sample_chains(batch: int, nheads: int, count: int, seed: int = 7) -> list[int]:
    """A fixed, seeded set of flat chain indices b*H + h, always including the
    first and the last chain."""
    total = batch * nheads
    if count >= total:
        return list(range(total))
    g = torch.Generator().manual_seed(seed)
    mid = torch.randperm(total - 2, generator=g)[: max(count - 2, 0)] + 1
    return sorted({0, total - 1, *mid.tolist()})
