"""Parity of the backward pass (m3_scan_bwd, through the C ABI) with the
gradient oracle (fp64 autograd through the token recurrence, pinned in
test_grad_oracle.py).

Bars, for every gradient tensor separately, as max |err| / max |ref|:
  - CUDA-core path (fp32 io, other shapes, or simt): 1e-4.  bf16 io shares the
    rounded inputs with the oracle and computes in fp32 as well, so it is held
    to the same 1e-4.
  - tensor-core path (bf16 io at N = 128, P = 64, the default there): its MMA
    operands are rounded to bf16, so BWD_TC_BAR (parity_helpers states why).
"""
import numpy as np
import pytest
import torch

from oracle import m3_grad
from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import BWD_TC_BAR, need_gpu, rel_err, to_dev

pytestmark = pytest.mark.gpu
BAR = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def case(batch=2, L=150, H=4, P=16, N=16, R=1, G=1, io="f32", decay="slow", h0=True,
         prev=True, tph=False, seed=0):
    w = I.Workload(I.Shape(batch, L, H, P, N, R, G, 64, io),
                   bc="rmsnorm" if io == "bf16" else "normal", decay=decay, with_h0=h0,
                   with_prev=prev, theta_per_head=tph)
    inp = I.make_scan_inputs(w, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    dy = torch.randn(inp["x"].shape, generator=gen)
    inp["dy"] = dy.to(inp["x"].dtype)
    inp["d_final"] = torch.randn((batch, H, N, P), generator=gen)
    return inp


def on_tc(inp, simt=False):
    """Whether m3_scan_bwd takes the tensor-core path for these inputs."""
    x, B = inp["x"], inp["B"]
    return not simt and x.dtype == torch.bfloat16 and B.shape[4] == 128 and x.shape[4] == 64


def compare(inp, chunk=64, with_final=True, simt=False):
    g = to_dev(inp)
    got = m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                         g["dy"], chunk, g.get("h0"), g.get("B_prev"), g.get("x_prev"),
                         g["d_final"] if with_final else None, simt=simt)
    assert m3.m3_stream_status() == 0
    _, _, ref = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES], dy=inp["dy"],
                                   d_final=inp["d_final"] if with_final else None)
    errs = {}
    for name, r in ref.items():
        if name == "h0" and "h0" not in inp:
            continue
        a = got[name].cpu().numpy()
        assert np.isfinite(a).all(), name
        errs[name] = rel_err(a, r)
    if "h0" not in inp:  # dh0 is the gradient with respect to a zero initial state
        _, _, r0 = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES[:7]],
                                      h0=np.zeros(tuple(got["h0"].shape)), dy=inp["dy"],
                                      d_final=inp["d_final"] if with_final else None)
        errs["h0"] = rel_err(got["h0"].cpu().numpy(), r0["h0"])
    bar = BWD_TC_BAR if on_tc(inp, simt) else BAR
    bad = {k: v for k, v in errs.items() if not v <= bar}
    assert not bad, f"errors above {bar}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_bwd_ranks(R):
    """Ragged length (150 is not a multiple of any backward chunk), h0, previous
    token, d_final; slow decay so that the adjoint crosses many chunks."""
    compare(case(R=R, seed=100 + R))


@pytest.mark.parametrize("G,tph", [(2, False), (4, False), (1, True), (2, True)])
def test_bwd_groups_and_angle_rates(G, tph):
    compare(case(R=2, G=G, tph=tph, seed=200 + G + 10 * tph))


@pytest.mark.parametrize("N,P", [(32, 32), (64, 16), (16, 128), (256, 32), (128, 64)])
def test_bwd_shapes(N, P):
    compare(case(batch=1, L=90, H=2, N=N, P=P, R=2, seed=300 + N + P))


def test_bwd_fast_decay_no_prev_no_final():
    compare(case(R=4, decay="fast", h0=False, prev=False, seed=400), with_final=False)


@pytest.mark.parametrize("L", [1, 2, 64, 65])
def test_bwd_edge_lengths(L):
    compare(case(batch=1, L=L, H=2, R=2, seed=500 + L))


@pytest.mark.parametrize("simt", [True, False], ids=["cuda_core", "tcgen05"])
def test_bwd_bf16_layer_shape(simt):
    """bf16 io at the layer's N = 128, P = 64 (a few chains), both paths."""
    compare(case(batch=1, L=200, H=2, N=128, P=64, R=4, io="bf16", seed=600), simt=simt)


def test_bwd_bf16_inputs_fp32_dy():
    """bf16 inputs with an fp32 output gradient (M3_FLAG_DY_F32), CUDA-core
    path: dy is read unrounded, so the gradients meet the 1e-4 bar against the
    oracle run with the same fp32 dy; the same dy rounded to bf16 first misses
    that bar, so the flag is what keeps the extra precision."""
    inp = case(batch=1, L=200, H=2, N=128, P=64, R=4, io="bf16", seed=610)
    gen = torch.Generator().manual_seed(611)
    inp["dy"] = torch.randn(inp["x"].shape, generator=gen)  # fp32, not rounded
    compare(inp, simt=True)
    g = to_dev(inp)
    rounded = m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                             g["dy"].to(torch.bfloat16), 64, g["h0"], g["B_prev"], g["x_prev"],
                             g["d_final"], simt=True)
    _, _, ref = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES], dy=inp["dy"],
                                   d_final=inp["d_final"])
    assert rel_err(rounded["x"].cpu().numpy(), ref["x"]) > BAR


def test_bwd_empty_sequence():
    inp = to_dev(case(batch=1, L=0, H=2, R=1, seed=700))
    got = m3.m3_scan_bwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                         inp["C"], inp["dy"], 64, inp["h0"], inp["B_prev"], inp["x_prev"],
                         inp["d_final"])
    assert m3.m3_stream_status() == 0
    assert torch.equal(got["h0"], inp["d_final"])
    assert float(got["B_prev"].abs().max()) == 0.0


def test_bwd_chunk_invariant():
    """The backward picks its own chunk; the caller's chunk changes nothing."""
    g = to_dev(case(R=2, seed=800))
    outs = [m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                           g["dy"], c, g["h0"], g["B_prev"], g["x_prev"], g["d_final"])
            for c in (16, 64)]
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]) or \
            rel_err(outs[0][k].cpu().numpy(), outs[1][k].cpu().numpy()) < 1e-6, k


@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "cuda_core"])
@pytest.mark.parametrize("R", [1, 4])
def test_bwd_full_size_sampled_chains(R, simt):
    """The bench's backward workload (b=8, L=2048, H=64, N=128, P=64, bf16 io,
    the workload's input recipe), gradients of a seeded sample of (batch, head)
    chains: everything a chain owns (dx, d dt, dA, d lam, dh0) against the
    gradient oracle run on that chain alone.  B, C and theta are shared by all
    64 heads (G = 1), so their gradients are sums over chains; they are covered
    by the small cases above."""
    w = I.Workload(I.Shape(8, 2048, 64, 64, 128, R, 1, 64, "bf16"), with_h0=True)
    inp = I.make_scan_inputs(w, seed=1001 + R)
    gen = torch.Generator().manual_seed(900 + R)
    dy = torch.randn(inp["x"].shape, generator=gen).to(torch.bfloat16)
    dfin = torch.randn(inp["h0"].shape, generator=gen)
    g = to_dev(inp)
    got = m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                         dy.cuda(), 64, g["h0"], None, None, dfin.cuda(), simt=simt)
    assert m3.m3_stream_status() == 0
    got = {k: v.cpu().numpy() for k, v in got.items()}
    bar = BAR if simt else BWD_TC_BAR
    for c in I.sample_chains(8, 64, 3, seed=11 + R):
        b, h = divmod(c, 64)
        one = {"x": inp["x"][b:b + 1, :, h:h + 1], "dt": inp["dt"][b:b + 1, :, h:h + 1],
               "A": inp["A"][b:b + 1, :, h:h + 1], "lam": inp["lam"][b:b + 1, :, h:h + 1],
               "theta": inp["theta"][b:b + 1], "B": inp["B"][b:b + 1], "C": inp["C"][b:b + 1],
               "h0": inp["h0"][b:b + 1, h:h + 1]}
        _, _, ref = m3_grad.scan_grads(*[one.get(k) for k in m3_grad.NAMES],
                                       dy=dy[b:b + 1, :, h:h + 1],
                                       d_final=dfin[b:b + 1, h:h + 1])
        errs = {"x": rel_err(got["x"][b, :, h], ref["x"][0, :, 0]),
                "dt": rel_err(got["dt"][b, :, h], ref["dt"][0, :, 0]),
                "A": rel_err(got["A"][b, :, h], ref["A"][0, :, 0]),
                "lam": rel_err(got["lam"][b, :, h], ref["lam"][0, :, 0]),
                "h0": rel_err(got["h0"][b, h], ref["h0"][0, 0])}
        bad = {k: v for k, v in errs.items() if not v <= bar}
        assert not bad, (c, errs)


@pytest.mark.parametrize("world,io", [(2, "f32"), (3, "bf16")])
def test_bwd_sequence_split_emulated_on_one_gpu(world, io):
    """The backward of the sequence split driven rank by rank with the
    library's kernels on one device: every input's gradient, in token order,
    against the gradient oracle on the whole sequence.  With bf16 io the
    segments' incoming states come from the tensor-core state-only pass
    (bf16 operands), so that case is held to the bf16 io bar."""
    from selective_state_space_exp_b200.parallel import (M3Ops, seq_boundary, seq_end_adjoint,
                                                         seq_incoming_state, seq_summary)
    N, P = (16, 16) if io == "f32" else (128, 64)
    inp = case(batch=1, L=60 * world, H=2, N=N, P=P, R=2, io=io, seed=1200 + world)
    g = to_dev(inp)
    L = inp["x"].shape[1]
    keys = ("x", "dt", "A", "lam", "theta", "B", "C", "dy")
    segs = [{k: g[k][:, r * L // world:(r + 1) * L // world].contiguous() for k in keys}
            for r in range(world)]
    ops = M3Ops()
    lasts = [seq_boundary(s["x"], s["B"]) for s in segs]
    prevs = [(g["B_prev"], g["x_prev"])] + [lasts[r - 1] for r in range(1, world)]
    sums = [seq_summary(ops, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                        *prevs[r]) for r, s in enumerate(segs)]
    Ts, lams, phis = [t[0] for t in sums], [t[1] for t in sums], [t[2] for t in sums]
    h_ins = [seq_incoming_state(ops, r, g["h0"], Ts, lams, phis) for r in range(world)]
    args = lambda r: (segs[r]["x"], segs[r]["dt"], segs[r]["A"], segs[r]["lam"],
                      segs[r]["theta"], segs[r]["B"], segs[r]["C"], 64, h_ins[r], *prevs[r])
    Ds = [ops.scan_bwd(*args(r), segs[r]["dy"], None)["h0"] for r in range(world)]
    parts = [ops.scan_bwd(*args(r), segs[r]["dy"],
                          seq_end_adjoint(ops, r, world, g["d_final"], Ds, lams, phis))
             for r in range(world)]
    for r in range(world - 1):
        parts[r]["B"][:, -1] += parts[r + 1]["B_prev"]
        parts[r]["x"][:, -1] += parts[r + 1]["x_prev"]
    assert m3.m3_stream_status() == 0
    _, _, ref = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES], dy=inp["dy"],
                                   d_final=inp["d_final"])
    errs = {k: rel_err(torch.cat([p[k] for p in parts], dim=1).cpu().numpy(), ref[k])
            for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    errs["h0"] = rel_err(parts[0]["h0"].cpu().numpy(), ref["h0"])
    errs["B_prev"] = rel_err(parts[0]["B_prev"].cpu().numpy(), ref["B_prev"])
    bar = BAR if io == "f32" else 2e-2
    bad = {k: v for k, v in errs.items() if not v <= bar}
    assert not bad, errs


# ---- the tensor-core path (bf16 io, N = 128, P = 64) ----------------------------
# Chunks of 64 rows: Q = 64 / R tokens.  Every case also runs the CUDA-core
# path on the same inputs, and the two must agree within the tensor-core bar.

def both_paths(inp, with_final=True):
    e_tc = compare(inp, with_final=with_final)
    e_sm = compare(inp, with_final=with_final, simt=True)
    g = to_dev(inp)
    outs = [m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                           g["dy"], 64, g.get("h0"), g.get("B_prev"), g.get("x_prev"),
                           g["d_final"] if with_final else None, simt=s) for s in (False, True)]
    for k in outs[1]:
        d = rel_err(outs[0][k].cpu().numpy(), outs[1][k].cpu().numpy())
        assert d <= BWD_TC_BAR, (k, d)
    return e_tc, e_sm


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_tc_bwd_ranks(R):
    """Ragged length (150 is not a multiple of 64 / R), h0, previous token,
    d_final, slow decay so that the adjoint crosses many chunks."""
    both_paths(case(batch=2, L=150, H=4, N=128, P=64, R=R, io="bf16", seed=1300 + R))


@pytest.mark.parametrize("G,tph", [(2, False), (4, False), (1, True), (2, True)])
def test_tc_bwd_groups_and_angle_rates(G, tph):
    both_paths(case(batch=1, L=100, H=4, N=128, P=64, R=2, G=G, io="bf16", tph=tph,
                    seed=1400 + G + 10 * tph))


def test_tc_bwd_fast_decay_no_prev_no_final():
    both_paths(case(batch=2, L=130, H=2, N=128, P=64, R=4, io="bf16", decay="fast", h0=False,
                    prev=False, seed=1500), with_final=False)


@pytest.mark.parametrize("R,L", [(1, 1), (1, 2), (1, 63), (1, 64), (1, 65), (4, 15), (4, 16),
                                 (4, 17), (8, 9)])
def test_tc_bwd_edge_lengths(R, L):
    """Lengths around the chunk (64 / R tokens): one token, a chunk less one,
    a chunk, a chunk and one."""
    both_paths(case(batch=1, L=L, H=2, N=128, P=64, R=R, io="bf16", seed=1600 + 100 * R + L))


def test_tc_bwd_fp32_dy():
    """An fp32 dy (M3_FLAG_DY_F32) on the tensor-core path."""
    inp = case(batch=1, L=120, H=2, N=128, P=64, R=4, io="bf16", seed=1700)
    gen = torch.Generator().manual_seed(1701)
    inp["dy"] = torch.randn(inp["x"].shape, generator=gen)
    compare(inp)
