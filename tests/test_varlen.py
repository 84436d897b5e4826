"""Packed variable-length batches (m3_scan_fwd_varlen).

CPU: the oracle's packed form is pinned to the batched scan and to the
continuation identity (a sequence split in two, the second part started from
the first part's final state and last token, gives the unsplit scan), so a
wrong slice, a state that leaks across a boundary or a misindexed h0 / B_prev
fails.  GPU: both CUDA paths against that oracle on length mixes with empty,
one-token, chunk-edge and long sequences, the segmented tensor-core plan, the
bit-exact agreement of a packed batch of equal lengths with the batched call,
and the kernels' check of the offsets.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import BWD_TC_BAR, TOL, need_gpu, rel_err, to_dev


def workload(H=2, P=16, N=16, R=1, G=1, chunk=64, io="f32", bc="normal", decay="slow",
             h0=True, prev=True):
    return I.Workload(I.Shape(1, 1, H, P, N, R, G, chunk, io), bc=bc, decay=decay,
                      with_h0=h0, with_prev=prev)


def oracle_varlen(inp):
    return oracle.scan_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"], inp["lam"],
                              inp["theta"], inp["B"], inp["C"], inp.get("h0"),
                              inp.get("B_prev"), inp.get("x_prev"))


# ---- oracle pins (CPU) ------------------------------------------------------

def test_oracle_varlen_equal_lengths_is_the_batched_scan():
    """S sequences of one length, packed, give the batched scan of [S][L]."""
    S, L = 3, 70
    w = workload(R=2)
    inp = I.make_varlen_inputs(w, [L] * S, seed=11)
    y, hL = oracle_varlen(inp)
    batched = {k: inp[k].reshape((S, L) + tuple(inp[k].shape[1:]))
               for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    yb, hb = oracle.scan(batched["x"], batched["dt"], batched["A"], batched["lam"],
                         batched["theta"], batched["B"], batched["C"], inp["h0"],
                         inp["B_prev"], inp["x_prev"])
    assert np.array_equal(y, yb.reshape(y.shape)) and np.array_equal(hL, hb)


def test_oracle_varlen_continuation():
    """Sequence 1 of the pack is the tail of a longer sequence, started from its
    head's final state with the head's last token as B_prev / x_prev: its y and
    final state are the long scan's (no state crosses into sequence 2, which
    gets a fresh h0)."""
    w = workload(R=2, h0=False, prev=False)
    full = I.make_varlen_inputs(w, [150], seed=12)
    yf, hf = oracle_varlen(full)
    cut = 90
    _, h_head = oracle.scan(*(full[k][None, :cut] for k in ("x", "dt", "A", "lam", "theta",
                                                             "B", "C")))
    other = I.make_varlen_inputs(workload(R=2), [40], seed=13)
    cat = lambda k: torch.cat([full[k][cut:], other[k]])
    packed = {k: cat(k) for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    packed["cu_seqlens"] = torch.tensor([0, 150 - cut, 150 - cut + 40], dtype=torch.int32)
    packed["h0"] = torch.cat([torch.from_numpy(h_head).float(), other["h0"]])
    packed["B_prev"] = torch.cat([full["B"][cut - 1:cut], other["B_prev"]])
    packed["x_prev"] = torch.cat([full["x"][cut - 1:cut], other["x_prev"]])
    y, hL = oracle_varlen(packed)
    # h_head went through fp32, so compare at fp32 rounding of the state
    assert rel_err(y[:150 - cut], yf[cut:]) < 1e-6
    assert rel_err(hL[0], hf[0]) < 1e-6
    y2, h2 = oracle_varlen(other)
    assert np.array_equal(y[150 - cut:], y2) and np.array_equal(hL[1], h2[0])


def test_oracle_varlen_empty_sequence_keeps_h0():
    """An empty sequence has no token for its left endpoint: its final state is h0."""
    w = workload()
    inp = I.make_varlen_inputs(w, [0, 5, 0], seed=14)
    y, hL = oracle_varlen(inp)
    assert y.shape[0] == 5
    assert np.array_equal(hL[0], inp["h0"][0].double().numpy())
    assert np.array_equal(hL[2], inp["h0"][2].double().numpy())


def test_varlen_lengths_mix():
    L = I.varlen_lengths(10, 300, 64, seed=3)
    assert L[:6] == [0, 1, 63, 64, 65, 300] and len(L) == 10
    assert all(1 <= v <= 300 for v in L[6:])


# ---- GPU parity -------------------------------------------------------------

def gpu_varlen(inp, chunk, simt=False, max_seqlen=None):
    g = to_dev(inp)
    y, fs = m3.m3_scan_fwd_varlen(g["cu_seqlens"], g["x"], g["dt"], g["A"], g["lam"],
                                  g["theta"], g["B"], g["C"], chunk, g.get("h0"),
                                  g.get("B_prev"), g.get("x_prev"), simt=simt,
                                  max_seqlen=max_seqlen)
    st = m3.m3_stream_status()
    return y.float().cpu().numpy(), fs.cpu().numpy(), st


def check_varlen(inp, chunk, io, simt=False):
    yg, hg, st = gpu_varlen(inp, chunk, simt)
    assert st == 0, st
    yo, ho = oracle_varlen(inp)
    assert np.isfinite(yg).all() and np.isfinite(hg).all()
    ey, eh = rel_err(yg, yo), rel_err(hg, ho)
    assert ey <= TOL[io] and eh <= TOL[io], f"err y {ey:.3e}, state {eh:.3e} (bar {TOL[io]})"


@pytest.mark.gpu
@pytest.mark.parametrize("R,chunk", [(1, 64), (2, 32), (2, 64), (4, 16), (4, 32), (4, 64)])
def test_varlen_tensor_core(R, chunk):
    """bf16 io, N = 128, P = 64 (tensor-core path): a mix of 0, 1, Q-1, Q, Q+1,
    300 and random lengths, each sequence with its own h0 and previous token."""
    need_gpu()
    w = workload(H=2, P=64, N=128, R=R, chunk=chunk, io="bf16", bc="rmsnorm", decay="slow")
    lengths = I.varlen_lengths(9, 300, chunk, seed=20 + R + chunk)
    inp = I.make_varlen_inputs(w, lengths, seed=5000 + 10 * R + chunk)
    x = to_dev(inp)["x"]
    shape = m3.make_shape(len(lengths), max(lengths), 2, 1, 64, 128, R, chunk, x.dtype)
    assert m3.scan_plan(shape)["tensor_core"]
    check_varlen(inp, chunk, "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_varlen_cuda_core(io, R):
    """The CUDA-core path (fp32 io, and bf16 io off the tensor-core shapes)."""
    need_gpu()
    w = workload(H=3, P=32, N=32, R=R, chunk=32, io=io,
                 bc="rmsnorm" if io == "bf16" else "normal")
    inp = I.make_varlen_inputs(w, I.varlen_lengths(8, 200, 32, seed=30 + R), seed=5100 + R)
    check_varlen(inp, 32, io, simt=True)


@pytest.mark.gpu
def test_varlen_segmented_plan():
    """Few long chains: the tensor-core plan cuts them into segments, and the
    short sequence's chain has segments with no chunk at all."""
    need_gpu()
    w = workload(H=2, P=64, N=128, R=4, chunk=64, io="bf16", bc="rmsnorm", decay="slow")
    lengths = [1500, 77]
    inp = I.make_varlen_inputs(w, lengths, seed=5200)
    shape = m3.make_shape(2, 1500, 2, 1, 64, 128, 4, 64, torch.bfloat16)
    assert m3.scan_plan(shape)["segments"] > 1
    check_varlen(inp, 64, "bf16")


@pytest.mark.gpu
@pytest.mark.parametrize("simt", [False, True])
def test_varlen_equal_lengths_bit_exact(simt):
    """A pack of equal lengths runs the batched call's arithmetic: same bits."""
    need_gpu()
    S, L = 3, 256
    w = workload(H=4, P=64, N=128, R=2, chunk=64, io="bf16", bc="rmsnorm")
    inp = to_dev(I.make_varlen_inputs(w, [L] * S, seed=5300))
    yv, hv = m3.m3_scan_fwd_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"],
                                   inp["lam"], inp["theta"], inp["B"], inp["C"], 64, inp["h0"],
                                   inp["B_prev"], inp["x_prev"], simt=simt)
    b = {k: inp[k].reshape((S, L) + tuple(inp[k].shape[1:]))
         for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    yb, hb = m3.m3_scan_fwd(b["x"], b["dt"], b["A"], b["lam"], b["theta"], b["B"], b["C"], 64,
                            inp["h0"], inp["B_prev"], inp["x_prev"], simt=simt)
    assert m3.m3_stream_status() == 0
    assert torch.equal(yv.view(torch.int16), yb.reshape(yv.shape).view(torch.int16))
    assert torch.equal(hv, hb)


@pytest.mark.gpu
@pytest.mark.parametrize("simt", [False, True])
def test_varlen_bad_offsets_reported(simt):
    """An offset past total_tokens and a decreasing pair are not read from:
    the call reports M3_ERR_INVALID_ARGUMENT and the valid sequences are exact."""
    need_gpu()
    w = workload(H=2, P=64, N=128, R=1, chunk=64, io="bf16", bc="rmsnorm")
    inp = I.make_varlen_inputs(w, [100, 120, 1, 1], seed=5400)  # T = 222
    ref = dict(inp)
    ref["cu_seqlens"] = torch.tensor([0, 100, 220], dtype=torch.int32)
    for k in ("h0", "B_prev", "x_prev"):
        ref[k] = inp[k][:2]
    # [0, 100) and [100, 220) valid; [220, 999) ends past T; [999, 500) decreases
    inp["cu_seqlens"] = torch.tensor([0, 100, 220, 999, 500], dtype=torch.int32)
    yg, hg, st = gpu_varlen(inp, 64, simt, max_seqlen=1000)
    assert st == m3.M3_ERR_INVALID_ARGUMENT
    yo, ho = oracle_varlen(ref)
    assert rel_err(yg[:220], yo[:220]) <= TOL["bf16"]
    assert rel_err(hg[:2], ho) <= TOL["bf16"]


@pytest.mark.gpu
@pytest.mark.parametrize("R", [1, 4])
def test_varlen_bench_workload(R):
    """The bench's packed-batch line exactly: 16 sequences of the seeded length
    mix up to 2048 tokens, the layer shape (H=64, N=128, P=64, bf16), every
    output against the oracle."""
    need_gpu()
    s = I.Shape(1, 1, 64, 64, 128, R, 1, 64, "bf16")
    lengths = I.varlen_lengths(16, 2048, 64, seed=1021)
    inp = I.make_varlen_inputs(I.Workload(s), lengths, seed=1021)
    yg, hg, st = gpu_varlen(inp, 64, max_seqlen=2048)
    assert st == 0
    yo, ho = oracle_varlen(inp)
    assert np.isfinite(yg).all()
    assert rel_err(yg, yo) <= TOL["bf16"] and rel_err(hg, ho) <= TOL["bf16"]


# ---- backward of packed batches ------------------------------------------------

@pytest.mark.gpu
@pytest.mark.parametrize("io,N,P,R,simt", [("f32", 16, 16, 2, False), ("bf16", 128, 64, 1, True),
                                           ("bf16", 128, 64, 4, True), ("bf16", 128, 64, 1, False),
                                           ("bf16", 128, 64, 4, False)])
def test_varlen_backward(io, N, P, R, simt):
    """m3_scan_bwd_varlen on a length mix (0, 1, Q-1, Q, Q+1, the maximum and
    random lengths) against the gradient oracle run sequence by sequence:
    every gradient within 1e-4 of max |ref| on the CUDA cores (fp32
    throughout), within the bf16-operand bar on the tensor cores (bf16 io at
    N = 128, P = 64 without simt)."""
    need_gpu()
    from oracle import m3_grad
    w = workload(H=2, P=P, N=N, R=R, chunk=64, io=io, bc="rmsnorm" if io == "bf16" else "normal")
    lengths = I.varlen_lengths(8, 150, 32, seed=70 + R)
    inp = I.make_varlen_inputs(w, lengths, seed=7000 + N + R)
    gen = torch.Generator().manual_seed(71 + R)
    dy = torch.randn(inp["x"].shape, generator=gen).to(inp["x"].dtype)
    dfin = torch.randn(inp["h0"].shape, generator=gen)
    g = to_dev(inp)
    got = m3.m3_scan_bwd_varlen(g["cu_seqlens"], g["x"], g["dt"], g["A"], g["lam"], g["theta"],
                                g["B"], g["C"], dy.cuda(), 64, g["h0"], g["B_prev"],
                                g["x_prev"], dfin.cuda(), max_seqlen=max(lengths), simt=simt)
    assert m3.m3_stream_status() == 0
    ref = m3_grad.scan_grads_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"],
                                    inp["lam"], inp["theta"], inp["B"], inp["C"], inp["h0"],
                                    inp["B_prev"], inp["x_prev"], dy=dy, d_final=dfin)
    errs = {k: rel_err(got[k].cpu().numpy(), ref[k]) for k in ref}
    bar = BWD_TC_BAR if (io == "bf16" and not simt) else 1e-4
    bad = {k: v for k, v in errs.items() if not v <= bar}
    assert not bad, errs
