"""Oracle of the B / C projection prep of the Mamba-3 block (fp64, numpy).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: imported by tests/ and by
bench.py's CPU legs, never by the product library.

After the B and C projections the block applies a QK-norm and a learnable
bias (PaperWeekly page section 2.4, "normalisation and bias"; Figure 4): each
(token, group, rank) row of N values is divided by its root mean square, scaled
per channel and shifted per channel,

    out[n] = raw[n] / sqrt(mean_m raw[m]^2 + eps) * weight[n] + bias[n],

with weight and bias indexed by (group, rank, n).  The result is rounded to
the io dtype by the caller (round to nearest even for bf16).
"""
from __future__ import annotations

import numpy as np


def qk_norm_bias(raw, weight=None, bias=None, eps=1e-6):
    """raw [..., G, R, N] (any float array; bf16 tensors widen exactly),
    weight / bias [G, R, N] or None (1 / 0).  Returns fp64 [..., G, R, N]."""
    if hasattr(raw, "detach"):
        import torch
        raw = raw.detach().to("cpu").to(torch.float64).numpy()
    x = np.asarray(raw, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float64)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y
