"""Parity of the block projections (m3_linear, m3_mimo_up, m3_mimo_down_gate,
through the C ABI) with their fp64 oracle (oracle/m3_block.py).

Bars (max |err| / max |ref|): bf16 outputs 2e-2 (one bf16 rounding of an
fp32 result); fp32 outputs of the bf16-operand projection 1e-4 (fp32
accumulation order only)."""
import numpy as np
import pytest
import torch

from oracle import m3_block as ob
from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import TOL, need_gpu, oracle_scan, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def bf16(t):
    return t.to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K,with_bias,f32", [
    (300, 256, 64, True, False),      # one N tile, M tail
    (1, 8, 8, False, False),          # smallest shapes
    (257, 64, 200, True, True),       # the narrow-N kernel, K tail, fp32 out (angle rates)
    (129, 200, 72, False, False),     # N tail inside a tile, K tail
    (1000, 1024, 512, True, False),   # several tiles per CTA in both directions
    (640, 520, 2048, False, True),    # long K, N tail past a full tile
])
def test_linear_matches_oracle(M, N, K, with_bias, f32):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A = bf16(torch.randn((M, K), generator=g))
    W = bf16(torch.randn((N, K), generator=g) / K ** 0.5)
    b = torch.randn((N,), generator=g) if with_bias else None
    out = m3.m3_linear(A.cuda(), W.cuda(), None if b is None else b.cuda(),
                       out_dtype=torch.float32 if f32 else torch.bfloat16)
    assert m3.m3_stream_status() == 0
    ref = ob.linear(A, W, b)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert rel_err(got, ref) <= (1e-4 if f32 else TOL["bf16"])


def test_linear_block_width():
    """A block input projection at the 1.5B-scale width (D = 2048 -> H*P =
    4096) on 2048 tokens: every output against the oracle."""
    g = torch.Generator().manual_seed(11)
    A = bf16(torch.randn((2048, 2048), generator=g))
    W = bf16(torch.randn((4096, 2048), generator=g) / 2048 ** 0.5)
    out = m3.m3_linear(A.cuda(), W.cuda())
    assert m3.m3_stream_status() == 0
    assert rel_err(out.float().cpu().numpy(), ob.linear(A, W)) <= TOL["bf16"]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_mimo_up_and_down_gate(io, R):
    g = torch.Generator().manual_seed(100 + R)
    T, H, P = 77, 4, 64
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    x = torch.randn((T, H, P), generator=g).to(dt)
    w_up = torch.randn((H, R, P), generator=g)
    w_dn = torch.randn((H, R, P), generator=g)
    z = torch.randn((T, H, P), generator=g).to(dt)
    X = m3.m3_mimo_up(x.cuda(), w_up.cuda())
    Xr = ob.mimo_up(x, w_up)
    bar = TOL["bf16"] if io == "bf16" else 1e-6
    assert rel_err(X.float().cpu().numpy(), Xr) <= bar
    Y = torch.randn((T, H, R, P), generator=g).to(dt)
    for zz in (None, z):
        out = m3.m3_mimo_down_gate(Y.cuda(), w_dn.cuda(), None if zz is None else zz.cuda())
        ref = ob.mimo_down_gate(Y, w_dn, zz)
        assert rel_err(out.float().cpu().numpy(), ref) <= (TOL["bf16"] if io == "bf16" else 1e-5)
    assert m3.m3_stream_status() == 0


def test_block_chain_up_scan_down_gate():
    """x -> MIMO up-projection -> the scan -> down-projection and gate, on the
    GPU through the C ABI, against the oracle chain on the same inputs (each
    GPU output is rounded to bf16 before the next step, on both sides)."""
    w = I.Workload(I.Shape(1, 300, 4, 64, 128, 4, 1, 64, "bf16"), decay="slow", with_h0=True,
                   with_prev=True)
    inp = I.make_scan_inputs(w, seed=9900)
    g = torch.Generator().manual_seed(9901)
    T, H, R, P = 300, 4, 4, 64
    x0 = bf16(torch.randn((1, T, H, P), generator=g))
    w_up = torch.randn((H, R, P), generator=g)
    w_dn = torch.randn((H, R, P), generator=g) / R
    z = bf16(torch.randn((1, T, H, P), generator=g))
    d = {k: v.cuda() for k, v in inp.items()}
    X = m3.m3_mimo_up(x0.cuda(), w_up.cuda())
    y, fs = m3.m3_scan_fwd(X, d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], 64,
                           d["h0"], d["B_prev"], d["x_prev"])
    out = m3.m3_mimo_down_gate(y, w_dn.cuda(), z.cuda())
    assert m3.m3_stream_status() == 0
    Xr = bf16(torch.from_numpy(ob.mimo_up(x0, w_up)).float())  # the oracle's own rounding
    assert rel_err(X.float().cpu().numpy(), Xr.float().numpy()) <= TOL["bf16"]
    ref_in = dict(inp, x=Xr)
    yo, ho = oracle_scan(ref_in)
    outr = ob.mimo_down_gate(bf16(torch.from_numpy(yo).float()), w_dn, z)
    assert rel_err(y.float().cpu().numpy(), yo) <= TOL["bf16"]
    assert rel_err(out.float().cpu().numpy(), outr) <= TOL["bf16"]


def test_block_ops_reject_bad_arguments():
    A = bf16(torch.randn((16, 12))).cuda()  # K = 12 is not a multiple of 8
    W = bf16(torch.randn((8, 12))).cuda()
    with pytest.raises(m3.M3Error) as e:
        m3.m3_linear(A, W)
    assert e.value.status == -2
    A = bf16(torch.randn((16, 16))).cuda()
    W = bf16(torch.randn((8, 16))).cuda()
    with pytest.raises(TypeError):
        m3.m3_linear(A.float(), W)
    assert m3.m3_stream_status() == 0
