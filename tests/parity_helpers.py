"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and measure the error as
max |gpu - ref| / max |ref| (separately for y and for the final state)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_exp_b200 import _build, m3
from selective_state_space_exp_b200.inputs import sample_chains

TOL = {"f32": 1e-4, "bf16": 2e-2}  # max|err| / max|ref| bars for the two io dtypes
# The tensor-core backward (bf16 io, N = 128, P = 64) rounds every MMA operand
# to bf16 (8 significant bits: a relative rounding error up to 2^-9, about
# 2e-3) and accumulates in fp32; each gradient is a sum of products of two or
# three such operands, so its error relative to max |ref| is a few 1e-3.  Its
# bar is the bf16 io bar of the forward.
BWD_TC_BAR = 2e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _build.build()
    m3.load()


def to_dev(d: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def gpu_scan(inp: dict, chunk: int, simt=False):
    g = to_dev(inp)
    y, fs = m3.m3_scan_fwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                           chunk, g.get("h0"), g.get("B_prev"), g.get("x_prev"), simt=simt)
    assert m3.m3_stream_status() == 0
    return y.float().cpu().numpy(), fs.cpu().numpy()


def oracle_scan(inp: dict, chains=None):
    return oracle.scan(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                       inp["C"], inp.get("h0"), inp.get("B_prev"), inp.get("x_prev"),
                       chains=chains)


def chain_rows(y, hL, chains, H):
    """Gather the outputs of the listed chains: y -> [n][L][R][P], hL -> [n][N][P]."""
    ys = np.stack([y[c // H, :, c % H] for c in chains])
    hs = np.stack([hL[c // H, c % H] for c in chains])
    return ys, hs


def rel_err(a, ref):
    denom = float(np.max(np.abs(ref))) if ref.size else 1.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(a - ref))) / max(denom, 1e-30)


def compare_scan(inp: dict, chunk: int, io: str, nsample=None, simt=False, seed=7):
    """Run both sides; return (err_y, err_state)."""
    b, L, H = inp["x"].shape[:3]
    chains = None if nsample is None else sample_chains(b, H, nsample, seed)
    yg, hg = gpu_scan(inp, chunk, simt)
    yo, ho = oracle_scan(inp, chains)
    if chains is None:
        chains = list(range(b * H))
    gy, gh = chain_rows(yg, hg, chains, H)
    oy, oh = chain_rows(yo, ho, chains, H)
    assert np.isfinite(gy).all() and np.isfinite(gh).all()
    return rel_err(gy, oy), rel_err(gh, oh)
