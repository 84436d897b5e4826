"""m3_scan_fwd_noalloc: the scan for callers that cannot allocate device memory
(for example a plugin inside a host framework that owns all device memory, or
a path where a cudaMalloc and the device synchronisation it may bring are not
acceptable).  Its scratch lives in a fixed library-owned device array, so the
caller passes inputs and outputs only.

It runs the very kernels of m3_scan_fwd on the same inputs, so its results
must equal m3_scan_fwd's (caller-provided workspace) bit for bit; any
difference would mean scratch left over from an earlier call was read.  The
tests therefore:
  - call it twice in a row on different shapes and inputs, each result equal
    bit for bit to m3_scan_fwd and within the parity bar of the oracle;
  - call it on inputs holding NaN (which fill the shared array with NaN
    partial states), then on clean inputs of the same shape: the clean result
    is finite and equal bit for bit to m3_scan_fwd;
  - call it on a shape whose workspace is exactly M3_NOALLOC_SCRATCH_BYTES,
    and check on the host that one chunk more is rejected;
  - repeat the comparison on every visible device (with one device this is
    the one above).
The file is named to be collected last.
"""
import ctypes

import pytest
import torch

from selective_state_space_exp_b200 import _build, m3
from selective_state_space_exp_b200 import inputs as I
from parity_helpers import TOL, need_gpu, oracle_scan, rel_err, to_dev

LIMIT = 16 * 1024 * 1024  # M3_NOALLOC_SCRATCH_BYTES


def run_both(inp: dict, chunk: int, simt: bool = False):
    g = to_dev(inp)
    args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], chunk,
            g.get("h0"), g.get("B_prev"), g.get("x_prev"))
    y_na, h_na = m3.m3_scan_fwd_noalloc(*args, simt=simt)
    assert m3.m3_stream_status() == 0
    y_ws, h_ws = m3.m3_scan_fwd(*args, simt=simt)
    assert m3.m3_stream_status() == 0
    return y_na, h_na, y_ws, h_ws


def assert_bitwise(y_na, h_na, y_ws, h_ws):
    assert torch.isfinite(y_na.float()).all() and torch.isfinite(h_na).all()
    assert torch.equal(y_na, y_ws)
    assert torch.equal(h_na, h_ws)


CASES = [
    (I.Workload(I.Shape(2, 250, 4, 32, 32, 2, 1, 64, "f32"), bc="normal", decay="slow",
                with_h0=True, with_prev=True), 6001, "f32"),
    (I.Workload(I.Shape(1, 300, 8, 64, 128, 4, 1, 64, "bf16"), with_h0=True,
                with_prev=True), 6002, "bf16"),
]


@pytest.mark.gpu
def test_noalloc_matches_workspace_scan_twice():
    """Two calls in a row, the second on other shapes and data: each equals
    m3_scan_fwd bit for bit and the oracle within the parity bar."""
    need_gpu()
    for w, seed, io in CASES:
        inp = I.make_scan_inputs(w, seed=seed)
        if io == "bf16":  # the tensor-core path's segment states live in the scratch
            g = to_dev(inp)
            assert m3.scan_plan(m3.scan_shape(g["x"], g["B"], w.shape.chunk))["segments"] > 1
        y_na, h_na, y_ws, h_ws = run_both(inp, w.shape.chunk)
        assert_bitwise(y_na, h_na, y_ws, h_ws)
        yo, ho = oracle_scan(inp)
        assert rel_err(y_na.float().cpu().numpy(), yo) <= TOL[io]
        assert rel_err(h_na.cpu().numpy(), ho) <= TOL[io]


@pytest.mark.gpu
@pytest.mark.parametrize("simt", [False, True], ids=["tcgen05", "cuda_core"])
def test_noalloc_clean_after_poisoned_call(simt):
    """A call whose inputs hold NaN leaves NaN in the shared array; the next,
    clean call on the same shape must not see it."""
    need_gpu()
    w = I.Workload(I.Shape(1, 700, 4, 64, 128, 4, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = I.make_scan_inputs(w, seed=6010 + int(simt))
    bad = dict(inp)
    bad["x"] = torch.full_like(inp["x"], float("nan"))
    bad["h0"] = torch.full_like(inp["h0"], float("nan"))
    g = to_dev(bad)
    y_bad, h_bad = m3.m3_scan_fwd_noalloc(g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"],
                                          g["C"], 64, g["h0"], g["B_prev"], g["x_prev"],
                                          simt=simt)
    assert m3.m3_stream_status() == 0
    assert torch.isnan(h_bad).all()  # the poison reached the scratch and the outputs
    assert_bitwise(*run_both(inp, 64, simt))


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit():
    """b = 1, H = 16, N = 128, P = 32, L = 4032 (63 chunks of 64), fp32: the
    CUDA-core path's workspace is exactly M3_NOALLOC_SCRATCH_BYTES; it runs and
    equals m3_scan_fwd bit for bit."""
    need_gpu()
    w = I.Workload(I.Shape(1, 4032, 16, 32, 128, 1, 1, 64, "f32"), bc="normal", decay="slow",
                   with_h0=True, with_prev=True)
    inp = I.make_scan_inputs(w, seed=6020)
    g = to_dev(inp)
    assert m3.workspace_size(m3.scan_shape(g["x"], g["B"], 64)) == LIMIT
    assert_bitwise(*run_both(inp, 64))


@pytest.mark.gpu
def test_noalloc_on_every_device():
    need_gpu()
    w, seed, _ = CASES[1]
    inp = I.make_scan_inputs(w, seed=seed + 100)
    for d in range(torch.cuda.device_count()):
        with torch.cuda.device(d):
            g = {k: v.to(f"cuda:{d}") for k, v in inp.items()}
            args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], 64,
                    g["h0"], g["B_prev"], g["x_prev"])
            y_na, h_na = m3.m3_scan_fwd_noalloc(*args)
            y_ws, h_ws = m3.m3_scan_fwd(*args)
            assert m3.m3_stream_status() == 0
            assert_bitwise(y_na, h_na, y_ws, h_ws)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """One chunk more than the exact-limit shape, and the SISO layer on the
    CUDA-core path: the workspace exceeds the fixed scratch, so the call returns
    M3_ERR_WORKSPACE on the host and launches nothing."""
    _build.build()
    lib = m3.load()
    fake = [ctypes.c_void_p(0x7f0000000000 + 0x100000 * i) for i in range(10)]
    for s, over in ((m3.Shape(1, 4033, 16, 1, 32, 128, 1, 64, m3.M3_F32, 0), 1),
                    (m3.Shape(1, 4032, 16, 1, 32, 128, 1, 64, m3.M3_F32, 0), 0),
                    (m3.Shape(8, 2048, 64, 1, 64, 128, 1, 64, m3.M3_BF16, m3.M3_FLAG_SIMT), 1)):
        n = ctypes.c_size_t()
        assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
        assert (n.value > LIMIT) == bool(over), n.value
        if over:
            st = lib.m3_scan_fwd_noalloc(ctypes.byref(s), fake[0], fake[1], fake[2], fake[3],
                                         fake[4], fake[5], fake[6], None, None, None, fake[7],
                                         fake[8], None)
            assert st == -4
