"""Runs in a child process with M3_LIBRARY=debug (the bounds-checked build,
whose kernels test every index they form against their tensors' extents):
every call of the library on small valid inputs must leave the device status
word at 0 (no M3_ERR_BOUNDS), and the scans and the backward must still agree
with the oracle at the usual bars.  Prints one line per call and "ALL OK"."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import numpy as np  # noqa: E402
import torch  # noqa: E402

from oracle import m3_grad  # noqa: E402
from parity_helpers import BWD_TC_BAR, TOL, compare_scan, rel_err, to_dev  # noqa: E402
from selective_state_space_exp_b200 import inputs as I  # noqa: E402
from selective_state_space_exp_b200 import m3  # noqa: E402

assert m3.LIB_PATH.endswith("libm3_debug.so"), m3.LIB_PATH


def status_ok(what):
    st = m3.m3_stream_status()
    print(f"{what}: status {st}", flush=True)
    assert st == 0, (what, st)


def scans():
    cases = [  # (workload, chunk, io, simt)
        (I.Workload(I.Shape(1, 300, 4, 64, 128, 4, 1, 64, "bf16"), with_h0=True, with_prev=True), 64, "bf16", False),
        (I.Workload(I.Shape(2, 200, 4, 64, 128, 1, 2, 64, "bf16"), with_h0=True, with_prev=True), 64, "bf16", False),
        (I.Workload(I.Shape(1, 150, 2, 32, 64, 2, 1, 32, "f32"), bc="normal", with_h0=True, with_prev=True), 32, "f32", True),
        (I.Workload(I.Shape(1, 130, 2, 64, 128, 8, 1, 16, "bf16"), with_h0=True, with_prev=True), 16, "bf16", True),
    ]
    for i, (w, chunk, io, simt) in enumerate(cases):
        inp = I.make_scan_inputs(w, seed=8100 + i)
        ey, eh = compare_scan(inp, chunk, io, simt=simt)
        status_ok(f"scan {i} ({'cuda cores' if simt else 'tensor cores'}) err y {ey:.1e} state {eh:.1e}")
        assert ey <= TOL[io] and eh <= TOL[io]


def long_segments():
    """One chain cut into segments (the state-only pass and the combine)."""
    w = I.Workload(I.Shape(1, 4096, 2, 64, 128, 4, 1, 64, "bf16"), with_h0=True)
    inp = I.make_scan_inputs(w, seed=8200)
    g = to_dev(inp)
    plan = m3.scan_plan(m3.scan_shape(g["x"], g["B"], 64))
    ey, eh = compare_scan(inp, 64, "bf16")
    status_ok(f"segmented scan ({plan['segments']} segments) err y {ey:.1e} state {eh:.1e}")
    assert ey <= TOL["bf16"] and eh <= TOL["bf16"]


def varlen():
    w = I.Workload(I.Shape(1, 1, 2, 64, 128, 4, 1, 64, "bf16"), with_h0=True, with_prev=True)
    lengths = [0, 1, 63, 64, 65, 300]
    inp = to_dev(I.make_varlen_inputs(w, lengths, seed=8300))
    for simt in (False, True):
        y, h = m3.m3_scan_fwd_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"], inp["lam"],
                                     inp["theta"], inp["B"], inp["C"], 64, inp["h0"],
                                     inp["B_prev"], inp["x_prev"], max_seqlen=max(lengths),
                                     simt=simt)
        assert torch.isfinite(y.float()).all() and torch.isfinite(h).all()
        status_ok(f"varlen scan ({'cuda cores' if simt else 'tensor cores'})")
        g = m3.m3_scan_bwd_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"], inp["lam"],
                                  inp["theta"], inp["B"], inp["C"], inp["x"].clone(), 64,
                                  inp["h0"], inp["B_prev"], inp["x_prev"],
                                  max_seqlen=max(lengths), simt=simt)
        assert all(torch.isfinite(v).all() for v in g.values())
        status_ok(f"varlen backward ({'cuda cores' if simt else 'tensor cores'})")


def backward():
    for R, simt in ((1, False), (4, False), (2, True)):
        w = I.Workload(I.Shape(1, 150, 2, 64, 128, R, 1, 64, "bf16"), decay="slow", with_h0=True,
                       with_prev=True)
        inp = I.make_scan_inputs(w, seed=8400 + R)
        gen = torch.Generator().manual_seed(8401 + R)
        dy = torch.randn(inp["x"].shape, generator=gen).to(torch.bfloat16)
        dfin = torch.randn(inp["h0"].shape, generator=gen)
        g = to_dev(inp)
        got = m3.m3_scan_bwd(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"],
                             dy.cuda(), 64, g["h0"], g["B_prev"], g["x_prev"], dfin.cuda(),
                             simt=simt)
        _, _, ref = m3_grad.scan_grads(*[inp.get(k) for k in m3_grad.NAMES], dy=dy,
                                       d_final=dfin)
        err = max(rel_err(got[k].cpu().numpy(), ref[k]) for k in ref)
        status_ok(f"backward R={R} ({'cuda cores' if simt else 'tensor cores'}) max err {err:.1e}")
        assert err <= (1e-4 if simt else BWD_TC_BAR)


def decode():
    for R in (1, 4, 8):
        w = I.Workload(I.Shape(4, 1, 8, 64, 128, R, 2, 64, "bf16"), with_h0=True, with_prev=True)
        d = I.make_decode_inputs(w, seed=8500 + R, steps=3, device="cuda")
        state = d["state0"].clone()
        for t in range(3):  # step t's previous token is step t - 1
            Bp = d["B_prev"] if t == 0 else d["B"][t - 1]
            xp = d["x_prev"] if t == 0 else d["x"][t - 1]
            y, state = m3.m3_decode_step(state, d["x"][t], d["dt"][t], d["A"][t], d["lam"][t],
                                         d["theta"][t], d["B"][t], d["C"][t], Bp, xp)
        assert torch.isfinite(state).all()
        status_ok(f"decode R={R}")


def block_pieces():
    gen = torch.Generator(device="cuda").manual_seed(8600)
    A = torch.randn((300, 256), generator=gen, device="cuda").to(torch.bfloat16)
    W = torch.randn((192, 256), generator=gen, device="cuda").to(torch.bfloat16)
    out = m3.m3_linear(A, W)
    assert torch.isfinite(out.float()).all()
    status_ok("linear")
    T, H, R, P = 100, 4, 4, 64
    x = torch.randn((T, H, P), generator=gen, device="cuda").to(torch.bfloat16)
    w_up = torch.randn((H, R, P), generator=gen, device="cuda")
    X = m3.m3_mimo_up(x, w_up)
    Y = torch.randn((T, H, R, P), generator=gen, device="cuda").to(torch.bfloat16)
    z = torch.randn((T, H, P), generator=gen, device="cuda").to(torch.bfloat16)
    o = m3.m3_mimo_down_gate(Y, w_up, z)
    assert torch.isfinite(X.float()).all() and torch.isfinite(o.float()).all()
    status_ok("mimo up / down + gate")
    Braw = torch.randn((2, 50, 2, 4, 128), generator=gen, device="cuda").to(torch.bfloat16)
    prm = [torch.randn((2, 4, 128), generator=gen, device="cuda") for _ in range(4)]
    Bo, Co = m3.m3_bc_prep(Braw, Braw.clone(), *prm)
    assert torch.isfinite(Bo.float()).all()
    status_ok("bc prep")


def sequence_split():
    w = I.Workload(I.Shape(1, 256, 2, 64, 128, 2, 1, 64, "bf16"), with_h0=True, with_prev=True)
    g = to_dev(I.make_scan_inputs(w, seed=8700))
    T = m3.m3_scan_state(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], 64,
                         None, g["B_prev"], g["x_prev"])
    lam, phi = m3.m3_segment_totals(g["x"], g["dt"], g["A"], g["theta"], g["B"], 64)
    h = m3.m3_state_fold(g["h0"], T[None], lam[None], phi[None])
    assert torch.isfinite(h).all()
    status_ok("sequence split: state, totals, fold")


if __name__ == "__main__":
    m3.load()
    scans()
    long_segments()
    varlen()
    backward()
    decode()
    block_pieces()
    sequence_split()
    print("ALL OK", flush=True)
