"""The torch.autograd binding (selective_state_space_exp_b200.autograd.m3_scan):
loss.backward() through it gives the gradient oracle's gradients, for fp32 and
bf16 io, with and without h0 / previous token, and only for the inputs that
require them."""
import numpy as np
import pytest
import torch

from oracle import m3_grad
from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from selective_state_space_exp_b200.autograd import m3_scan
from parity_helpers import need_gpu, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def run(io, N, P, R, prev, seed, bar):
    w = I.Workload(I.Shape(2, 100, 4, P, N, R, 1, 64, io),
                   bc="rmsnorm" if io == "bf16" else "normal", decay="slow", with_h0=True,
                   with_prev=prev)
    inp = I.make_scan_inputs(w, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    dy = torch.randn(inp["x"].shape, generator=gen).to(inp["x"].dtype)
    dfin = torch.randn(inp["h0"].shape, generator=gen)
    leaves = {k: v.cuda().requires_grad_(True) for k, v in inp.items()}
    y, fs = m3_scan(leaves["x"], leaves["dt"], leaves["A"], leaves["lam"], leaves["theta"],
                    leaves["B"], leaves["C"], 64, leaves["h0"], leaves.get("B_prev"),
                    leaves.get("x_prev"))
    loss = (y.float() * dy.cuda().float()).sum() + (fs * dfin.cuda()).sum()
    loss.backward()
    assert m3.m3_stream_status() == 0
    _, _, ref = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES], dy=dy, d_final=dfin)
    errs = {}
    for k, t in leaves.items():
        assert t.grad is not None and t.grad.dtype == t.dtype, k
        errs[k] = rel_err(t.grad.float().cpu().numpy(), ref[k])
    bad = {k: v for k, v in errs.items() if not v <= bar}
    assert not bad, errs


def test_autograd_fp32_small():
    run("f32", 16, 16, 2, True, 1300, 1e-4)


def test_autograd_bf16_layer_shape():
    """bf16 inputs get bf16 gradients: the bar is the bf16 io bar."""
    run("bf16", 128, 64, 4, False, 1310, 2e-2)


def test_autograd_only_requested_gradients():
    w = I.Workload(I.Shape(1, 70, 2, 16, 16, 1, 1, 64, "f32"), bc="normal", with_h0=False)
    inp = {k: v.cuda() for k, v in I.make_scan_inputs(w, seed=1320).items()}
    x = inp["x"].clone().requires_grad_(True)
    y, fs = m3_scan(x, inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"], inp["C"])
    y.sum().backward()
    assert m3.m3_stream_status() == 0
    assert x.grad is not None and inp["dt"].grad is None
    _, _, ref = m3_grad.scan_grads(*[inp[k].cpu() for k in ("x", "dt", "A", "lam", "theta", "B",
                                                            "C")],
                                   dy=np.ones(tuple(inp["x"].shape)))
    assert rel_err(x.grad.cpu().numpy(), ref["x"]) <= 1e-4


def test_autograd_varlen():
    """The packed-batch binding against the gradient oracle run per sequence."""
    from selective_state_space_exp_b200.autograd import m3_scan_varlen
    w = I.Workload(I.Shape(1, 1, 2, 64, 128, 2, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    lengths = I.varlen_lengths(6, 150, 64, seed=1330)
    inp = I.make_varlen_inputs(w, lengths, seed=1331)
    gen = torch.Generator().manual_seed(1332)
    dy = torch.randn(inp["x"].shape, generator=gen).to(torch.bfloat16)
    dfin = torch.randn(inp["h0"].shape, generator=gen)
    leaves = {k: v.cuda().requires_grad_(k != "cu_seqlens") for k, v in inp.items()}
    y, fs = m3_scan_varlen(leaves["cu_seqlens"], leaves["x"], leaves["dt"], leaves["A"],
                           leaves["lam"], leaves["theta"], leaves["B"], leaves["C"], 64,
                           leaves["h0"], leaves["B_prev"], leaves["x_prev"])
    ((y.float() * dy.cuda().float()).sum() + (fs * dfin.cuda()).sum()).backward()
    assert m3.m3_stream_status() == 0
    ref = m3_grad.scan_grads_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"],
                                    inp["lam"], inp["theta"], inp["B"], inp["C"], inp["h0"],
                                    inp["B_prev"], inp["x_prev"], dy=dy, d_final=dfin)
    errs = {k: rel_err(leaves[k].grad.float().cpu().numpy(), ref[k]) for k in ref}
    bad = {k: v for k, v in errs.items() if not v <= 2e-2}
    assert not bad, errs
