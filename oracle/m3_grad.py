"""Gradient oracle for the Mamba-3 SSM layer scan (fp64, plain PyTorch on the CPU).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: imported by tests/ and by
bench.py's CPU legs, never by the product library.

The forward pass is the token recurrence of the exponential-trapezoidal rule
with the complex (rotation) transition (PaperWeekly page sections 2.1-2.2;
rank-R inputs, section 2.3), written with real pairs:

  u_t   = sum_r B_{t,r} x_{t,r}^T                     (N x P, B's pairs (2k, 2k+1))
  w_t   = z_{t-1} + (1 - lam_t) dt_t u_{t-1}          (u_{-1} = B_prev x_prev^T, z_{-1} = h0)
  z_t   = exp(dt_t A_t) Rot(dt_t theta_t) w_t + lam_t dt_t u_t
  y_t,r = C_{t,r}^T z_t

and the gradients are those of the scalar  sum(y * dy) + sum(z_{L-1} * d_final)
taken by torch.autograd through that loop; nothing is blocked, chunked or
reordered.  The module's own pins (tests/test_grad_oracle.py) tie the forward
to the C oracle and every gradient to central finite differences of the C
oracle's forward, so autograd is checked from outside.
"""
from __future__ import annotations

import numpy as np
import torch

NAMES = ("x", "dt", "A", "lam", "theta", "B", "C", "h0", "B_prev", "x_prev")


def _t(v):
    if v is None:
        return None
    if isinstance(v, np.ndarray):
        v = torch.from_numpy(v)
    return v.detach().to("cpu").to(torch.float64).clone()


def forward(x, dt, A, lam, theta, B, C, h0=None, B_prev=None, x_prev=None):
    """y [b][L][H][R][P] and z_{L-1} [b][H][N][P] (fp64 tensors; autograd-able).
    Layouts as the library's: theta [b][L][Gt][N/2] with Gt = G or H."""
    b, L, H, R, P = x.shape
    G, N = B.shape[2], B.shape[4]
    Gt, K = theta.shape[2], N // 2
    grp = torch.arange(H) // (H // G)     # B / C group of each head
    tgrp = torch.arange(H) // (H // Gt)   # theta group of each head
    z = h0.clone() if h0 is not None else torch.zeros(b, H, N, P, dtype=torch.float64)
    z0, z1 = z[:, :, 0::2, :], z[:, :, 1::2, :]
    if B_prev is not None:
        u_prev = torch.einsum("bhrn,bhrp->bhnp", B_prev[:, grp], x_prev)
    else:
        u_prev = torch.zeros(b, H, N, P, dtype=torch.float64)
    ys = []
    for t in range(L):
        u = torch.einsum("bhrn,bhrp->bhnp", B[:, t][:, grp], x[:, t])
        eps = ((1.0 - lam[:, t]) * dt[:, t])[:, :, None, None]
        gam = (lam[:, t] * dt[:, t])[:, :, None, None]
        w0 = z0 + eps * u_prev[:, :, 0::2, :]
        w1 = z1 + eps * u_prev[:, :, 1::2, :]
        alpha = torch.exp(dt[:, t] * A[:, t])[:, :, None, None]
        phi = (dt[:, t][:, :, None] * theta[:, t][:, tgrp])[..., None]  # [b][H][K][1]
        cs, sn = torch.cos(phi), torch.sin(phi)
        z0 = alpha * (cs * w0 - sn * w1) + gam * u[:, :, 0::2, :]
        z1 = alpha * (sn * w0 + cs * w1) + gam * u[:, :, 1::2, :]
        Ct = C[:, t][:, grp]                                            # [b][H][R][N]
        ys.append(torch.einsum("bhrk,bhkp->bhrp", Ct[..., 0::2], z0)
                  + torch.einsum("bhrk,bhkp->bhrp", Ct[..., 1::2], z1))
        u_prev = u
    y = torch.stack(ys, dim=1) if L else torch.zeros(b, 0, H, R, P, dtype=torch.float64)
    zL = torch.stack([z0, z1], dim=3).reshape(b, H, N, P)  # re-interleave the pairs
    return y, zL


def scan_grads(x, dt, A, lam, theta, B, C, h0=None, B_prev=None, x_prev=None, dy=None,
               d_final=None):
    """Gradients of sum(y * dy) + sum(final * d_final) with respect to every
    input given (x, dt, A, lam, theta, B, C and, when passed, h0, B_prev,
    x_prev).  Returns (y, final, grads) with grads a dict of fp64 numpy arrays
    keyed by NAMES (absent inputs are left out)."""
    vals = [_t(v) for v in (x, dt, A, lam, theta, B, C, h0, B_prev, x_prev)]
    leaves = {}
    for name, v in zip(NAMES, vals):
        if v is not None:
            v.requires_grad_(True)
            leaves[name] = v
    y, zL = forward(*vals)
    loss = torch.zeros((), dtype=torch.float64)
    if dy is not None:
        loss = loss + (y * _t(dy)).sum()
    if d_final is not None:
        loss = loss + (zL * _t(d_final)).sum()
    names = list(leaves)
    gs = torch.autograd.grad(loss, [leaves[n] for n in names], allow_unused=True)
    grads = {n: (np.zeros(tuple(leaves[n].shape)) if g is None else g.numpy())
             for n, g in zip(names, gs)}
    return y.detach().numpy(), zL.detach().numpy(), grads


def scan_grads_varlen(cu_seqlens, x, dt, A, lam, theta, B, C, h0=None, B_prev=None,
                      x_prev=None, dy=None, d_final=None):
    """Gradients for a packed batch (layouts of the packed scan: token
    dimension first, no batch dimension; h0, B_prev, x_prev, d_final per
    sequence).  No state or input is shared between sequences, so each
    sequence's gradients are scan_grads of that sequence alone; they are
    written into packed arrays (rows outside every sequence stay zero)."""
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    packed = {"x": x, "dt": dt, "A": A, "lam": lam, "theta": theta, "B": B, "C": C}
    per_seq = {"h0": h0, "B_prev": B_prev, "x_prev": x_prev}
    out = {k: np.zeros(tuple(v.shape)) for k, v in packed.items()}
    for k, v in per_seq.items():
        if v is not None:
            out[k] = np.zeros(tuple(v.shape))
    for i in range(len(cu) - 1):
        a, e = cu[i], cu[i + 1]
        one = {k: v[None, a:e] for k, v in packed.items()}
        for k, v in per_seq.items():
            one[k] = None if v is None else v[i:i + 1]
        _, _, g = scan_grads(*[one[k] for k in NAMES],
                             dy=None if dy is None else dy[None, a:e],
                             d_final=None if d_final is None else d_final[i:i + 1])
        for k in packed:
            out[k][a:e] = g[k][0]
        for k in per_seq:
            if k in g:
                out[k][i] = g[k][0]
    return out
