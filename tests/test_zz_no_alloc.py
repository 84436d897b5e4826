"""m3_scan_fwd_noalloc: the scan for callers that cannot allocate device memory
(for example a plugin inside a host framework that owns all device memory, or
a path where a cudaMalloc and the device synchronisation it may bring are not
acceptable).  Its scratch lives in a fixed library-owned device array, so the
caller passes inputs and outputs only.

These tests call it through the C ABI twice in a row, with different inputs,
and check each result against m3_scan_fwd (caller-provided workspace) within
the parity bars used everywhere else.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

from selective_state_space_exp_b200 import _build, m3
from selective_state_space_exp_b200 import inputs as I
from parity_helpers import TOL, need_gpu, rel_err, to_dev


def run_both(inp: dict, chunk: int):
    g = to_dev(inp)
    args = (g["x"], g["dt"], g["A"], g["lam"], g["theta"], g["B"], g["C"], chunk,
            g.get("h0"), g.get("B_prev"), g.get("x_prev"))
    y_na, h_na = m3.m3_scan_fwd_noalloc(*args)
    assert m3.m3_stream_status() == 0
    y_ws, h_ws = m3.m3_scan_fwd(*args)
    assert m3.m3_stream_status() == 0
    return (y_na.float().cpu().numpy(), h_na.cpu().numpy(),
            y_ws.float().cpu().numpy(), h_ws.cpu().numpy())


@pytest.mark.gpu
def test_noalloc_matches_workspace_scan_twice():
    need_gpu()
    cases = [
        (I.Workload(I.Shape(2, 250, 4, 32, 32, 2, 1, 64, "f32"), bc="normal", decay="slow",
                    with_h0=True, with_prev=True), 6001, "f32"),
        (I.Workload(I.Shape(1, 300, 8, 64, 128, 4, 1, 64, "bf16"), with_h0=True,
                    with_prev=True), 6002, "bf16"),
    ]
    for w, seed, io in cases:  # two calls in a row, the second after different data
        inp = I.make_scan_inputs(w, seed=seed)
        y_na, h_na, y_ws, h_ws = run_both(inp, w.shape.chunk)
        assert rel_err(y_na, y_ws) <= TOL[io] and rel_err(h_na, h_ws) <= TOL[io]
        assert np.isfinite(y_na).all() and np.isfinite(h_na).all()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """A shape whose workspace exceeds the fixed scratch returns
    M3_ERR_WORKSPACE on the host and launches nothing."""
    _build.build()
    lib = m3.load()
    s = m3.Shape(8, 2048, 64, 1, 64, 128, 1, 64, m3.M3_BF16, m3.M3_FLAG_SIMT)
    n = ctypes.c_size_t()
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value > 16 * 1024 * 1024
    fake = [ctypes.c_void_p(0x7f0000000000 + 0x100000 * i) for i in range(10)]
    st = lib.m3_scan_fwd_noalloc(ctypes.byref(s), fake[0], fake[1], fake[2], fake[3], fake[4],
                                 fake[5], fake[6], None, None, None, fake[7], fake[8], None)
    assert st == -4
