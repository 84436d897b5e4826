"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Bars (max |err| / max |ref|, y and final state separately): 1e-4 for fp32 io,
2e-2 for bf16 io with fp32 accumulation and state.  Small cases compare every
output; full-size workloads compare a seeded sample of (batch, head) chains,
which the oracle computes independently of the others.
"""
import numpy as np
import pytest
import torch

from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import (TOL, chain_rows, compare_scan, gpu_scan, need_gpu, oracle_scan,
                            rel_err, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def small(batch=2, L=250, H=4, P=16, N=16, R=1, G=1, chunk=64, io="f32", bc="normal",
          decay="fast", h0=False, prev=False):
    return I.Workload(I.Shape(batch, L, H, P, N, R, G, chunk, io), bc=bc, decay=decay,
                      with_h0=h0, with_prev=prev)


def check(errs, io):
    ey, eh = errs
    assert ey <= TOL[io] and eh <= TOL[io], f"err y {ey:.3e}, state {eh:.3e} (bar {TOL[io]})"


# ---- prefill scan -----------------------------------------------------------

def test_tiny_siso_fp32_full():
    """The 256-token fp32 SISO case, every output against the oracle at 1e-4."""
    w = I.TINY_SISO_F32
    inp = I.make_scan_inputs(w, seed=1000)
    check(compare_scan(inp, w.shape.chunk, "f32"), "f32")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_ragged_small(io, R, chunk):
    """L = 250 (ragged last chunk), several tiles, initial state and previous token."""
    w = small(L=250, R=R, chunk=chunk, io=io, P=32, N=32, h0=True, prev=True,
              bc="rmsnorm" if io == "bf16" else "normal")
    inp = I.make_scan_inputs(w, seed=2000 + 10 * R + chunk)
    check(compare_scan(inp, chunk, io), io)


@pytest.mark.parametrize("N,P", [(16, 128), (256, 16), (64, 64), (128, 64)])
def test_shapes_grouped(N, P):
    """Groups G = H (per-head B, C, theta) and G = 2, slow decay so that every
    chunk's state reaches the next one."""
    for G in (2, 4):
        w = small(batch=2, L=200, H=4, G=G, N=N, P=P, R=2, io="f32", decay="slow", h0=True,
                  prev=True)
        inp = I.make_scan_inputs(w, seed=3000 + N + P + G)
        check(compare_scan(inp, 64, "f32"), "f32")


@pytest.mark.parametrize("L", [1, 63, 64, 65, 129])
def test_edge_lengths(L):
    w = small(L=L, R=2, io="f32", h0=True, prev=True, decay="slow")
    inp = I.make_scan_inputs(w, seed=4000 + L)
    check(compare_scan(inp, 64, "f32"), "f32")


def test_empty_sequence_returns_h0():
    w = small(L=0, h0=True)
    inp = to_dev(I.make_scan_inputs(w, seed=4100))
    y, fs = m3.m3_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                           inp["C"], 64, inp["h0"])
    assert y.numel() == 0
    assert torch.equal(fs, inp["h0"])
    _, fs0 = m3.m3_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                            inp["C"], 64)
    assert torch.count_nonzero(fs0) == 0


def test_chunk_invariance():
    """The chunk length is a performance parameter only (fp32 io, slow decay)."""
    w = small(L=300, R=4, P=32, N=64, io="f32", decay="slow", h0=True, prev=True)
    inp = I.make_scan_inputs(w, seed=4200)
    outs = [gpu_scan(inp, q) for q in (16, 32, 64)]
    for y, h in outs[1:]:
        assert rel_err(y, outs[0][0]) < 1e-5 and rel_err(h, outs[0][1]) < 1e-5


def test_split_continuation_on_gpu():
    """scan(L0) then scan(L1) seeded with (final state, last B, last x) equals
    scan(L0 + L1)."""
    w = small(L=200, R=2, P=32, N=32, io="f32", decay="slow", h0=True, prev=True)
    inp = I.make_scan_inputs(w, seed=4300)
    y, h = gpu_scan(inp, 64)
    L0 = 77
    seq = ("x", "dt", "A", "lam", "theta", "B", "C")
    a = {k: (v[:, :L0].contiguous() if k in seq else v) for k, v in inp.items()}
    ya, ha = gpu_scan(a, 64)
    b = {k: (v[:, L0:].contiguous() if k in seq else v) for k, v in inp.items()}
    b["h0"] = torch.from_numpy(ha)
    b["B_prev"] = inp["B"][:, L0 - 1].contiguous()
    b["x_prev"] = inp["x"][:, L0 - 1].contiguous()
    yb, hb = gpu_scan(b, 64)
    assert rel_err(np.concatenate([ya, yb], axis=1), y) < 1e-5
    assert rel_err(hb, h) < 1e-5


def test_slow_decay_siso_and_mimo():
    """Config-1 shapes (two sequences) with slow decay, so the inter-chunk state
    passing carries most of the output."""
    for R in (1, 4):
        w = I.Workload(I.Shape(2, 2048, 64, 64, 128, R, 1, 64, "bf16"), decay="slow",
                       with_h0=True, with_prev=True)
        inp = I.make_scan_inputs(w, seed=4400 + R)
        check(compare_scan(inp, 64, "bf16", nsample=6), "bf16")


@pytest.mark.parametrize("w,seed", [(I.SISO_PREFILL, 1001), (I.MIMO_PREFILL, 1002)],
                         ids=["siso_prefill_b8_L2048", "mimo_r4_prefill_b8_L2048"])
def test_full_size_prefill(w, seed):
    """The full workloads, every one of the 512 (batch, head) chains, on both
    GPU paths (tensor-core and CUDA-core) against one oracle run."""
    inp = I.make_scan_inputs(w, seed=seed)
    yo, ho = oracle_scan(inp)
    for simt in (False, True):
        yg, hg = gpu_scan(inp, w.shape.chunk, simt)
        assert np.isfinite(yg).all() and np.isfinite(hg).all()
        check((rel_err(yg, yo), rel_err(hg, ho)), "bf16")


# ---- tensor-core path: every tile shape, segments, ragged tails ----------------

@pytest.mark.parametrize("R,chunk", [(1, 64), (2, 64), (2, 32), (4, 64), (4, 32), (4, 16)])
@pytest.mark.parametrize("L,batch,H", [(250, 1, 4), (700, 2, 8)])
def test_tc_tiles_segments_ragged(R, chunk, L, batch, H):
    """N = 128, P = 64 bf16: M = chunk * R rows of 64, 128 or 256; few chains,
    so every chain is cut into several segments; ragged last chunk; initial
    state and previous token; slow decay so the carried state matters."""
    w = I.Workload(I.Shape(batch, L, H, 64, 128, R, 1, chunk, "bf16"), decay="slow",
                   with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=7000 + 10 * R + chunk + L)
    check(compare_scan(inp, chunk, "bf16"), "bf16")


@pytest.mark.parametrize("R,batch,H", [(4, 6, 75), (1, 8, 75)], ids=["r4_450_chains", "r1_600_chains"])
def test_tc_tail_split(R, batch, H):
    """Chains that fill a few waves and spill a handful into one more (450
    rank-4 chains on 148 one-CTA SMs, 600 rank-1 chains on 148 two-CTA SMs):
    the plan cuts only the last wave's chains in two (a state-only pass over
    their first halves, then the full pass as its dependent launch, whose
    second halves fold those summaries themselves).  Five chunks, the last
    ragged, so the halves are unequal; initial state and previous token, slow
    decay so the folded state matters; every chain against the oracle, and
    the last eight (the cut ones among them) on their own."""
    w = I.Workload(I.Shape(batch, 300, H, 64, 128, R, 1, 64, "bf16"), decay="slow",
                   with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=7700 + R)
    plan = m3.scan_plan(m3.scan_shape(inp["x"], inp["B"], 64))
    assert plan["tensor_core"] and plan["segments"] == 2 and plan["launches"] == 2, plan
    yg, hg = gpu_scan(inp, 64)
    yo, ho = oracle_scan(inp)
    assert np.isfinite(yg).all() and np.isfinite(hg).all()
    check((rel_err(yg, yo), rel_err(hg, ho)), "bf16")
    last = list(range(batch * H - 8, batch * H))
    gy, gh = chain_rows(yg, hg, last, H)
    oy, oh = chain_rows(yo, ho, last, H)
    check((rel_err(gy, oy), rel_err(gh, oh)), "bf16")


@pytest.mark.parametrize("R,chunk", [(1, 64), (2, 32), (2, 64), (4, 64), (4, 32)])
def test_tc_large_decay_chunks(R, chunk):
    """Every other chunk decays by hundreds of nats (dt ten times larger and
    A = -16 there), so the tensor-core path does those chunks in its plain
    form and the slow-decay chunks between in its factored form; few chains,
    so segments and the state-only pass are used too; ragged tail."""
    w = I.Workload(I.Shape(2, 700, 4, 64, 128, R, 1, chunk, "bf16"), decay="slow",
                   with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=7300 + 10 * R + chunk)
    odd = ((torch.arange(700) // chunk) % 2 == 1)[None, :, None]
    inp["dt"] = torch.where(odd, inp["dt"] * 10.0, inp["dt"]).contiguous()
    inp["A"] = torch.where(odd, torch.full_like(inp["A"], -16.0), inp["A"]).contiguous()
    lam_chunk = (inp["dt"] * inp["A"])[:, :chunk * (700 // chunk)].reshape(2, -1, chunk, 4).sum(2)
    assert float(lam_chunk.min()) < -300.0 and float(lam_chunk.max()) > -5.0
    check(compare_scan(inp, chunk, "bf16"), "bf16")


@pytest.mark.parametrize("nats", [95.0, 105.0])
@pytest.mark.parametrize("R", [1, 4])
def test_tc_decay_at_the_form_switch(nats, R):
    """Every chunk decays by the same total, just inside (95 nats: the
    factored form, factors up to e^47.5) or just outside (105 nats: the plain
    form) the switch between the two forms."""
    w = I.Workload(I.Shape(2, 640, 4, 64, 128, R, 1, 64, "bf16"), with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=7400 + R + int(nats))
    inp["dt"] = torch.ones_like(inp["dt"])
    inp["A"] = torch.full_like(inp["A"], -nats / 64.0)
    check(compare_scan(inp, 64, "bf16"), "bf16")


@pytest.mark.parametrize("R", [1, 4])
def test_tc_groups_and_fast_decay(R):
    """G = H (per-head B, C, theta) and the workload's fast decay."""
    w = I.Workload(I.Shape(2, 300, 4, 64, 128, R, 4, 64, "bf16"), with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=7100 + R)
    check(compare_scan(inp, 64, "bf16"), "bf16")


def test_tc_matches_cuda_core_path():
    """The two GPU paths agree with each other (bf16 io) to the bf16 bar."""
    w = I.Workload(I.Shape(2, 512, 8, 64, 128, 4, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = I.make_scan_inputs(w, seed=7200)
    y_tc, h_tc = gpu_scan(inp, 64, simt=False)
    y_sc, h_sc = gpu_scan(inp, 64, simt=True)
    assert rel_err(y_tc, y_sc) <= TOL["bf16"] and rel_err(h_tc, h_sc) <= TOL["bf16"]


@pytest.mark.parametrize("w,seed", [(I.LONG_MIMO_16K, 1014), (I.LONG_MIMO_32K, 1004)],
                         ids=["mimo_r4_L16384", "mimo_r4_L32768"])
def test_long_context_prefill(w, seed):
    """b = 1, H = 64 at L = 16384 and 32768: 16 of the 64 chains."""
    inp = I.make_scan_inputs(w, seed=seed)
    check(compare_scan(inp, w.shape.chunk, "bf16", nsample=16), "bf16")


def stressed_angles(inp, seed, dt_mean=1.0):
    """Replace dt by softplus(N(dt_mean, 0.5)) and theta by U(2.5, pi): the step
    angles all have one sign and are large, so the chunk-local cumulative
    angles reach hundreds of radians (64 tokens x ~1.3 x ~2.8 ~ 230 rad)."""
    g = torch.Generator().manual_seed(seed)
    dt = torch.nn.functional.softplus(torch.randn(inp["dt"].shape, generator=g)
                                      * 0.5 ** 0.5 + dt_mean)
    th = torch.rand(inp["theta"].shape, generator=g) * (np.pi - 2.5) + 2.5
    out = dict(inp)
    out["dt"], out["theta"] = dt.contiguous(), th.contiguous()
    return out


@pytest.mark.parametrize("R", [1, 4])
def test_angle_stress_large_chunk_angles(R):
    """Config-2 layer shape (two sequences, every chain) with slow decay and
    large one-signed step angles: the tensor-core path's fast sin/cos and
    exp2 see chunk-local angles of hundreds of radians; both paths against
    the oracle at the bf16 bar."""
    w = I.Workload(I.Shape(2, 2048, 64, 64, 128, R, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = stressed_angles(I.make_scan_inputs(w, seed=4500 + R), seed=4510 + R)
    phi = (inp["dt"][..., None] * inp["theta"][:, :, :1, :]).reshape(2, 32, 64, 64, 64)
    assert float(phi.sum(2).max()) > 150.0  # chunk-local angle at a chunk's end
    yo, ho = oracle_scan(inp)
    for simt in (False, True):
        yg, hg = gpu_scan(inp, 64, simt)
        check((rel_err(yg, yo), rel_err(hg, ho)), "bf16")


@pytest.mark.parametrize("R", [1, 4])
def test_one_signed_angles_many_segments(R):
    """Few chains (b = 1, H = 4, L = 4096), so each is cut into several
    segments whose summaries carry the total angle; one-signed angle rates
    and slow decay make that angle thousands of radians and let the state
    cross every segment boundary."""
    w = I.Workload(I.Shape(1, 4096, 4, 64, 128, R, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = stressed_angles(I.make_scan_inputs(w, seed=4600 + R), seed=4610 + R, dt_mean=-2.0)
    g = to_dev(inp)
    assert m3.scan_plan(m3.scan_shape(g["x"], g["B"], 64))["segments"] > 1
    check(compare_scan(inp, 64, "bf16"), "bf16")


# ---- decode step ------------------------------------------------------------

def gpu_decode(dec: dict, steps: int, in_place=True):
    g = to_dev(dec)
    state = g["state0"].clone()
    ys = []
    for t in range(steps):
        Bp = g["B_prev"] if t == 0 else g["B"][t - 1]
        xp = g["x_prev"] if t == 0 else g["x"][t - 1]
        out = None if in_place else torch.empty_like(state)
        y, state = m3.m3_decode_step(state, g["x"][t], g["dt"][t], g["A"][t], g["lam"][t],
                                     g["theta"][t], g["B"][t], g["C"][t], Bp, xp,
                                     state_out=out)
        ys.append(y)
    assert m3.m3_stream_status() == 0
    return torch.stack(ys, 1).float().cpu().numpy(), state.cpu().numpy()


def decode_as_scan(dec: dict) -> dict:
    """Decode inputs [steps][b]... rearranged into scan layout [b][steps]..."""
    out = {k: dec[k].transpose(0, 1).contiguous() for k in ("x", "dt", "A", "lam", "theta",
                                                            "B", "C")}
    out.update(h0=dec["state0"], B_prev=dec["B_prev"], x_prev=dec["x_prev"])
    return out


@pytest.mark.parametrize("w", [I.DECODE_SISO, I.DECODE_MIMO], ids=["R1", "R4"])
def test_decode_full_batch(w):
    """b = 128, H = 64: 32 decode steps, 64 of the 8192 chains against the
    oracle."""
    steps = 32
    dec = I.make_decode_inputs(w, seed=1003 if w.shape.rank == 1 else 1013, steps=steps)
    yg, hg = gpu_decode(dec, steps)
    sc = decode_as_scan(dec)
    b, H = w.shape.batch, w.shape.nheads
    chains = I.sample_chains(b, H, 64)
    yo, ho = oracle_scan(sc, chains)
    gy, gh = chain_rows(yg, hg, chains, H)
    oy, oh = chain_rows(yo, ho, chains, H)
    check((rel_err(gy, oy), rel_err(gh, oh)), "bf16")


def test_decode_1024_consecutive_steps():
    """1024 consecutive steps (R = 4, two sequences) against the oracle."""
    w = I.Workload(I.Shape(2, 1, 64, 64, 128, 4, 1, 64, "bf16"), with_h0=True, with_prev=True)
    steps = 1024
    dec = I.make_decode_inputs(w, seed=1023, steps=steps)
    yg, hg = gpu_decode(dec, steps)
    chains = I.sample_chains(2, 64, 6)
    yo, ho = oracle_scan(decode_as_scan(dec), chains)
    gy, gh = chain_rows(yg, hg, chains, 64)
    oy, oh = chain_rows(yo, ho, chains, 64)
    check((rel_err(gy, oy), rel_err(gh, oh)), "bf16")


def test_decode_fp32_small_every_output():
    w = I.Workload(I.Shape(3, 1, 4, 16, 32, 2, 2, 64, "f32"), bc="normal", with_h0=True,
                   with_prev=True)
    dec = I.make_decode_inputs(w, seed=5000, steps=40)
    yg, hg = gpu_decode(dec, 40)
    yo, ho = oracle_scan(decode_as_scan(dec))
    check((rel_err(yg, yo), rel_err(hg, ho)), "f32")


def test_decode_in_place_equals_out_of_place():
    w = I.Workload(I.Shape(4, 1, 8, 64, 128, 4, 1, 64, "bf16"), with_h0=True, with_prev=True)
    dec = I.make_decode_inputs(w, seed=5100, steps=3)
    y1, h1 = gpu_decode(dec, 3, in_place=True)
    y2, h2 = gpu_decode(dec, 3, in_place=False)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


@pytest.mark.parametrize("N,P,R,io,prev", [(256, 32, 8, "f32", True), (16, 128, 1, "bf16", False),
                                            (128, 128, 8, "f32", True), (64, 16, 4, "bf16", False),
                                            (256, 64, 8, "f32", True)])
def test_decode_shapes(N, P, R, io, prev):
    """Decode over other state shapes (the largest N * P with R = 8 included,
    one of them too large for two state buffers per CTA), two B/C groups,
    with and without the previous token at step 0."""
    w = I.Workload(I.Shape(3, 1, 4, P, N, R, 2, 64, io), bc="normal", with_h0=True,
                   with_prev=True)
    steps = 5
    dec = I.make_decode_inputs(w, seed=5400 + N + P + R, steps=steps)
    g = to_dev(dec)
    state = g["state0"].clone()
    ys = []
    for t in range(steps):
        Bp = (g["B_prev"] if prev else None) if t == 0 else g["B"][t - 1]
        xp = (g["x_prev"] if prev else None) if t == 0 else g["x"][t - 1]
        y, state = m3.m3_decode_step(state, g["x"][t], g["dt"][t], g["A"][t], g["lam"][t],
                                     g["theta"][t], g["B"][t], g["C"][t], Bp, xp)
        ys.append(y)
    assert m3.m3_stream_status() == 0
    yg = torch.stack(ys, 1).float().cpu().numpy()
    sc = decode_as_scan(dec)
    if not prev:
        sc.pop("B_prev")
        sc.pop("x_prev")
    yo, ho = oracle_scan(sc)
    check((rel_err(yg, yo), rel_err(state.cpu().numpy(), ho)), io)


def test_decode_equals_scan_on_gpu():
    """Driving the decode kernel token by token reproduces the scan kernels
    (fp32 io)."""
    w = I.Workload(I.Shape(2, 1, 4, 32, 64, 2, 1, 64, "f32"), bc="normal", decay="slow",
                   with_h0=True, with_prev=True)
    dec = I.make_decode_inputs(w, seed=5200, steps=150)
    yd, hd = gpu_decode(dec, 150)
    ys, hs = gpu_scan(decode_as_scan(dec), 32)
    assert rel_err(yd, ys) < 1e-5 and rel_err(hd, hs) < 1e-5


def test_bounded_wait_reports_timeout():
    """Failure path: with M3_FLAG_TEST_TIMEOUT every CTA of the tensor-core scan
    waits on an mbarrier that nothing completes; the wait gives up after its
    1 ms limit, the call reports M3_ERR_TIMEOUT through m3_stream_status, and
    the next call on the same context computes the right answer."""
    w = I.Workload(I.Shape(1, 200, 4, 64, 128, 1, 1, 64, "bf16"), with_h0=True)
    inp = I.make_scan_inputs(w, seed=5500)
    g = to_dev(inp)
    args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], 64, g["h0"])
    assert m3.scan_plan(m3.scan_shape(g["x"], g["B"], 64))["tensor_core"]
    m3.m3_scan_fwd(*args, extra_flags=m3.M3_FLAG_TEST_TIMEOUT)
    assert m3.m3_stream_status() == -6  # M3_ERR_TIMEOUT, and the word is cleared
    assert m3.m3_stream_status() == 0
    check(compare_scan(inp, 64, "bf16"), "bf16")


def test_gpu_rejects_bad_pointers():
    """Host-side checks with real device tensors: misaligned views and a small
    workspace return errors and launch nothing."""
    w = small(L=64, R=1, P=16, N=16, io="f32")
    inp = to_dev(I.make_scan_inputs(w, seed=5300))
    flat = torch.zeros(inp["x"].numel() + 4, device="cuda")
    x_mis = flat[1:1 + inp["x"].numel()].view_as(inp["x"])
    with pytest.raises(m3.M3Error) as e:
        m3.m3_scan_fwd(x_mis, inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                       inp["C"], 64)
    assert e.value.status == -3
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(m3.M3Error) as e:
        m3.m3_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                       inp["C"], 64, workspace=ws)
    assert e.value.status == -4
    assert m3.m3_stream_status() == 0


# ---- per-head angle rates (theta [b][L][H][N/2]) -----------------------------

@pytest.mark.parametrize("R,chunk,L,batch,H,G,simt", [
    (1, 64, 300, 2, 8, 1, False),    # tensor-core path, one tile per chunk
    (4, 64, 200, 1, 4, 1, False),    # tensor-core path, two tiles, several segments
    (2, 32, 130, 2, 4, 2, False),    # tensor-core path, two groups
    (2, 32, 130, 2, 4, 2, True),     # CUDA-core path
])
def test_per_head_theta_scan(R, chunk, L, batch, H, G, simt):
    """Per-head angle rates through both prefill paths against the oracle."""
    io = "bf16"
    w = I.Workload(I.Shape(batch, L, H, 64, 128, R, G, chunk, io), decay="slow", with_h0=True,
                   with_prev=True, theta_per_head=True)
    inp = I.make_scan_inputs(w, seed=8000 + 10 * R + L + (1 if simt else 0))
    assert inp["theta"].shape[2] == H
    check(compare_scan(inp, chunk, io, simt=simt), io)


def test_per_head_theta_scan_fp32_small():
    w = I.Workload(I.Shape(2, 150, 4, 16, 32, 2, 2, 32, "f32"), bc="normal", with_h0=True,
                   with_prev=True, theta_per_head=True)
    inp = I.make_scan_inputs(w, seed=8100)
    check(compare_scan(inp, 32, "f32"), "f32")


@pytest.mark.parametrize("R", [1, 4])
def test_per_head_theta_decode(R):
    """Both decode kernels (rank 1 streams, rank 4 pipelines) with per-head rates."""
    w = I.Workload(I.Shape(4, 1, 8, 64, 128, R, 2, 64, "bf16"), with_h0=True, with_prev=True,
                   theta_per_head=True)
    dec = I.make_decode_inputs(w, seed=8200 + R, steps=4)
    assert dec["theta"].shape[2] == 8
    yg, hg = gpu_decode(dec, 4)
    yo, ho = oracle_scan(decode_as_scan(dec))
    check((rel_err(yg, yo), rel_err(hg, ho)), "bf16")


# ---- sequence split across ranks: state-only scan, totals, fold ----------------

@pytest.mark.parametrize("R,chunk,L,batch,H,io,simt", [
    (1, 64, 700, 1, 8, "bf16", False),   # tensor-core path, several segments per chain
    (4, 64, 300, 2, 4, "bf16", False),   # two tiles per chunk
    (2, 32, 250, 2, 4, "f32", True),     # CUDA-core path
])
def test_scan_state_matches_oracle_final_state(R, chunk, L, batch, H, io, simt):
    N, P = (128, 64) if io == "bf16" else (32, 16)
    w = I.Workload(I.Shape(batch, L, H, P, N, R, 1, chunk, io), decay="slow", with_h0=True,
                   with_prev=True)
    inp = I.make_scan_inputs(w, seed=9000 + L)
    g = to_dev(inp)
    hs = m3.m3_scan_state(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], chunk,
                          g["h0"], g["B_prev"], g["x_prev"], simt=simt)
    assert m3.m3_stream_status() == 0
    _, ho = oracle_scan(inp)
    assert rel_err(hs.cpu().numpy(), ho) <= TOL[io]


def test_segment_totals_and_fold_match_numpy():
    w = I.Workload(I.Shape(2, 300, 4, 64, 128, 2, 2, 64, "bf16"), theta_per_head=True)
    inp = I.make_scan_inputs(w, seed=9100)
    g = to_dev(inp)
    lam, phi = m3.m3_segment_totals(g["x"], g["dt"], g["A"], g["theta"], g["B"], 64)
    dt, A, th = (inp[k].double().numpy() for k in ("dt", "A", "theta"))
    assert np.allclose(lam.cpu().numpy(), (dt * A).sum(1), rtol=1e-5, atol=1e-5)
    ref_phi = (dt[..., None] * th).sum(1)
    got_phi = phi.cpu().numpy().astype(np.float64)
    assert np.abs(got_phi).max() <= np.pi + 1e-6  # reduced to [-pi, pi]
    assert np.allclose(np.cos(got_phi), np.cos(ref_phi), atol=1e-5)
    assert np.allclose(np.sin(got_phi), np.sin(ref_phi), atol=1e-5)
    rng = np.random.default_rng(9101)
    nseg, b, H, N, P = 3, 2, 4, 128, 64
    T = rng.standard_normal((nseg, b, H, N, P)).astype(np.float32)
    lt = rng.uniform(-2.0, 0.0, (nseg, b, H)).astype(np.float32)
    pt = rng.uniform(-20.0, 20.0, (nseg, b, H, N // 2)).astype(np.float32)
    h0 = rng.standard_normal((b, H, N, P)).astype(np.float32)
    out = m3.m3_state_fold(*(torch.from_numpy(a).cuda() for a in (h0, T, lt, pt)))
    h = h0.astype(np.float64)
    for s in range(nseg):
        e = np.exp(lt[s].astype(np.float64))[:, :, None, None]
        c, sn = np.cos(pt[s].astype(np.float64))[..., None], np.sin(pt[s].astype(np.float64))[..., None]
        u0, u1 = e * h[:, :, 0::2], e * h[:, :, 1::2]
        n0, n1 = c * u0 - sn * u1 + T[s][:, :, 0::2], sn * u0 + c * u1 + T[s][:, :, 1::2]
        h = np.empty_like(h)
        h[:, :, 0::2], h[:, :, 1::2] = n0, n1
    assert rel_err(out.cpu().numpy(), h) <= 1e-5


@pytest.mark.parametrize("R,world", [(1, 4), (4, 3)])
def test_sequence_split_emulated_on_one_gpu(R, world):
    """The sequence split driven rank by rank with the library's kernels on one
    device; the ranks' y, in token order, and the last end state against one
    oracle scan of the whole sequence."""
    from selective_state_space_exp_b200.parallel import M3Ops, seq_boundary, seq_finish, seq_summary
    L = 192 * world
    w = I.Workload(I.Shape(1, L, 8, 64, 128, R, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = I.make_scan_inputs(w, seed=9200 + R)
    g = to_dev(inp)
    seq_keys = ("x", "dt", "A", "lam", "theta", "B", "C")
    segs = [{k: (g[k][:, r * L // world:(r + 1) * L // world].contiguous() if k in seq_keys
                 else g[k]) for k in g} for r in range(world)]
    ops = M3Ops()
    lasts = [seq_boundary(s["x"], s["B"]) for s in segs]
    prevs = [(g["B_prev"], g["x_prev"])] + [lasts[r - 1] for r in range(1, world)]
    sums = [seq_summary(ops, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                        *prevs[r]) for r, s in enumerate(segs)]
    Ts, lams, phis = [t[0] for t in sums], [t[1] for t in sums], [t[2] for t in sums]
    outs = [seq_finish(ops, r, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                       g["h0"], Ts, lams, phis, *prevs[r]) for r, s in enumerate(segs)]
    assert m3.m3_stream_status() == 0
    y = torch.cat([o[0] for o in outs], dim=1).float().cpu().numpy()
    yo, ho = oracle_scan(inp)
    check((rel_err(y, yo), rel_err(outs[-1][1].cpu().numpy(), ho)), "bf16")
