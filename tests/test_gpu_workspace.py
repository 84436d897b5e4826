"""Caller workspaces are scratch only: a workspace filled with NaN before the
call gives results identical, bit for bit, to a zero-filled one, and finite.
This shows that every scratch element a kernel reads was written earlier in
the same call (a read of stale scratch would carry the NaN into the result).

Covered: the prefill scan on both paths (the tensor-core path with several
segments per sequence, whose segment states live in the workspace; the
CUDA-core path, whose per-chunk states do), the packed-batch scan, and the
backward pass (per-chunk sums and states).  Several backward gradients are
float atomic sums whose order can differ between runs (those of the tensors
shared by a group's heads, B, C, theta, B_prev; dt, lam and x_prev, which also
take the next token's left-endpoint term; A through per-token sums in shared
memory), so those are compared to 1e-6 of their largest value; dx and dh0
must match exactly.
"""
import numpy as np
import pytest
import torch

from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import need_gpu, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def nan_bytes(n: int) -> torch.Tensor:
    """n bytes of fp32 NaN (0x7fc00000: also a bf16 NaN in either half)."""
    f = torch.full(((n + 3) // 4,), float("nan"), dtype=torch.float32, device="cuda")
    return f.view(torch.uint8)[:n]


def assert_same(a: torch.Tensor, b: torch.Tensor, what: str):
    assert torch.isfinite(a.float()).all(), what
    assert torch.equal(a, b), what


@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "cuda_core"])
def test_poisoned_workspace_scan(simt):
    w = I.Workload(I.Shape(1, 700, 4, 64, 128, 4, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    g = to_dev(I.make_scan_inputs(w, seed=9500 + int(simt)))
    shape = m3.scan_shape(g["x"], g["B"], 64, simt, g["theta"])
    if not simt:
        assert m3.scan_plan(shape)["segments"] > 1  # the workspace holds segment states
    n = m3.workspace_size(shape)
    assert n > 0
    args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], 64, g["h0"],
            g["B_prev"], g["x_prev"])
    y1, f1 = m3.m3_scan_fwd(*args, workspace=nan_bytes(n), simt=simt)
    y0, f0 = m3.m3_scan_fwd(*args, workspace=torch.zeros(n, dtype=torch.uint8, device="cuda"),
                            simt=simt)
    assert m3.m3_stream_status() == 0
    assert_same(y1, y0, "y")
    assert_same(f1, f0, "final state")


@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "cuda_core"])
def test_poisoned_workspace_varlen(simt):
    w = I.Workload(I.Shape(1, 1, 4, 64, 128, 2, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    lengths = [0, 1, 63, 64, 65, 900, 333]
    g = to_dev(I.make_varlen_inputs(w, lengths, seed=9510 + int(simt)))
    S, T, H, R, P = len(lengths), *g["x"].shape
    shape = m3.make_shape(S, max(lengths), H, 1, P, 128, R, 64, g["x"].dtype, simt)
    n = m3.workspace_size(shape)
    assert n > 0
    args = (g["cu_seqlens"], g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], 64,
            g["h0"], g["B_prev"], g["x_prev"])
    y1, f1 = m3.m3_scan_fwd_varlen(*args, max_seqlen=max(lengths), workspace=nan_bytes(n),
                                   simt=simt)
    y0, f0 = m3.m3_scan_fwd_varlen(*args, max_seqlen=max(lengths),
                                   workspace=torch.zeros(n, dtype=torch.uint8, device="cuda"),
                                   simt=simt)
    assert m3.m3_stream_status() == 0
    assert_same(y1, y0, "y")
    assert_same(f1, f0, "final states")


ATOMIC = ("dt", "A", "lam", "theta", "B", "C", "B_prev", "x_prev")


@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "cuda_core"])
def test_poisoned_workspace_bwd(simt):
    """Both backward forms (the tensor-core one also reads the state pass's
    bf16 operand blocks from the workspace)."""
    w = I.Workload(I.Shape(2, 300, 4, 64, 128, 2, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    g = to_dev(I.make_scan_inputs(w, seed=9520))
    gen = torch.Generator(device="cuda").manual_seed(9521)
    dy = torch.randn(g["x"].shape, generator=gen, device="cuda").to(torch.bfloat16)
    dfin = torch.randn(g["h0"].shape, generator=gen, device="cuda")
    n = m3.bwd_workspace_size(m3.scan_shape(g["x"], g["B"], 64, simt, g["theta"]))
    assert n > 0
    args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], dy, 64, g["h0"],
            g["B_prev"], g["x_prev"], dfin)
    r1 = m3.m3_scan_bwd(*args, workspace=nan_bytes(n), simt=simt)
    r0 = m3.m3_scan_bwd(*args, workspace=torch.zeros(n, dtype=torch.uint8, device="cuda"),
                        simt=simt)
    assert m3.m3_stream_status() == 0
    for k in r0:
        assert torch.isfinite(r1[k]).all(), k
        if k in ATOMIC:
            assert rel_err(r1[k].cpu().numpy(), r0[k].cpu().numpy()) <= 1e-6, k
        else:
            assert torch.equal(r1[k], r0[k]), k
    assert set(r0) >= {"x", "A", "h0", "x_prev"}
    assert np.isfinite(r0["x"].cpu().numpy()).all()
