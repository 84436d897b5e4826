"""fp64 oracle of the block projections around the Mamba-3 SSM layer.

TEST INFRASTRUCTURE ONLY: used by tests/ and bench.py's CPU legs; the
library never imports it and it never imports the library.

What it computes (PaperWeekly page section 2.4 and Figure 4 name these steps
-- the input projections, the data-dependent RoPE angles, the MIMO
projection, the output gate -- but print no formula; the readings below are
the plainest the rest supports):
  linear:          out = A W^T + bias          (a projection of each token's features;
                                               the angle rates theta are one, with no
                                               nonlinearity)
  mimo_up:         X[t][h][r][p] = x[t][h][p] w_up[h][r][p]
                   (each rank r of head h gets a learned copy of the head's input;
                   section 2.3: x_t becomes the P x R matrix X_t)
  mimo_down_gate:  out[t][h][p] = (sum_r Y[t][h][r][p] w_down[h][r][p]) silu(z[t][h][p]),
                   silu(v) = v / (1 + exp(-v))   (the block's output gate)
Inputs are widened exactly to fp64 (bf16 values included); everything is
computed in fp64 with numpy, whose matmul is the one library step.
"""
from __future__ import annotations

import numpy as np


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        import torch
        a = a.detach().to("cpu")
        if a.dtype == torch.bfloat16:
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def linear(A, W, bias=None):
    """A [..][K], W [N][K], bias [N] -> [..][N] (fp64)."""
    A, W, bias = _f64(A), _f64(W), _f64(bias)
    out = A @ W.T
    return out if bias is None else out + bias


def silu(v):
    v = _f64(v)
    return v / (1.0 + np.exp(-v))


def mimo_up(x, w_up):
    """x [..][H][P], w_up [H][R][P] -> X [..][H][R][P]."""
    x, w = _f64(x), _f64(w_up)
    return x[..., :, None, :] * w


def mimo_down_gate(Y, w_down, z=None):
    """Y [..][H][R][P], w_down [H][R][P], z [..][H][P] or None -> [..][H][P]."""
    Y, w = _f64(Y), _f64(w_down)
    y = (Y * w).sum(axis=-2)
    return y if z is None else y * silu(z)
