"""Parity of m3_bc_prep (QK-norm + scale + bias of B and C, through the C ABI)
with its oracle, and of the prep followed by the scan with the oracle's prep
followed by the oracle's scan.

Bars: a bf16 output within one bf16 unit in the last place of the fp64 value
plus 2^-20 of the magnitude of its two terms |x_n w| + |b| (the kernel
evaluates x * rsqrt(ms + eps) * w + b in fp32, a few fp32 roundings of those
terms, then rounds to nearest even; where the terms cancel, the fp32 error can
exceed an ulp of the small result); fp32 outputs within 1e-6 of max |ref|; the
scan after the prep at the bf16 io bar (2e-2).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import m3_prep
from selective_state_space_exp_b200 import inputs as I
from selective_state_space_exp_b200 import m3
from parity_helpers import TOL, need_gpu, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def draw(shape, dtype, seed, G, R, N, scale=3.0):
    g = torch.Generator().manual_seed(seed)
    raw = (torch.randn(shape, generator=g) * scale).to(dtype)
    w = torch.randn((G, R, N), generator=g) * 0.5 + 1.0
    b = torch.randn((G, R, N), generator=g) * 0.3
    return raw, w, b


def ulp_check(got, ref, mag):
    """|got - ref| <= one bf16 ulp at |ref| (2^(e - 7) for |ref| in [2^e, 2^(e+1)))
    + 2^-20 * mag, mag = |x_n w| + |b|."""
    e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-30)))
    ulp = np.exp2(e - 7)
    bad = np.abs(got - ref) > ulp * (1 + 1e-9) + 2.0 ** -20 * mag + 1e-30
    return int(bad.sum())


def magnitude(raw, w=None, b=None, eps=1e-6):
    m = np.abs(m3_prep.qk_norm_bias(raw, None if w is None else w.double().numpy(), None, eps))
    return m if b is None else m + np.abs(b.double().numpy())


@pytest.mark.parametrize("N", [16, 64, 128, 256])
@pytest.mark.parametrize("G,R", [(1, 1), (4, 4), (2, 8)])
def test_prep_bf16(N, G, R):
    shape = (2, 37, G, R, N)
    Braw, wB, bB = draw(shape, torch.bfloat16, N + 10 * G + R, G, R, N)
    Craw, wC, bC = draw(shape, torch.bfloat16, N + 10 * G + R + 1, G, R, N)
    Bo, Co = m3.m3_bc_prep(Braw.cuda(), Craw.cuda(), wB.cuda(), bB.cuda(), wC.cuda(), bC.cuda(),
                           1e-6)
    assert m3.m3_stream_status() == 0
    for got, raw, w, b in ((Bo, Braw, wB, bB), (Co, Craw, wC, bC)):
        ref = m3_prep.qk_norm_bias(raw, w.double().numpy(), b.double().numpy(), 1e-6)
        assert ulp_check(got.float().cpu().numpy(), ref, magnitude(raw, w, b)) == 0


@pytest.mark.parametrize("N", [16, 128])
def test_prep_fp32_decode_layout_no_params(N):
    """fp32 io, the decode step's [b][G][R][N] layout, unit scale and no bias."""
    raw, _, _ = draw((5, 2, 4, N), torch.float32, 40 + N, 2, 4, N)
    Bo, Co = m3.m3_bc_prep(raw.cuda(), None, eps=1e-5)
    assert Co is None and m3.m3_stream_status() == 0
    ref = m3_prep.qk_norm_bias(raw, eps=1e-5)
    assert rel_err(Bo.cpu().numpy(), ref) <= 1e-6


def test_prep_in_place_and_one_tensor():
    shape = (3, 20, 1, 2, 128)
    raw, w, b = draw(shape, torch.bfloat16, 50, 1, 2, 128)
    d = raw.cuda()
    m3.m3_bc_prep(None, d, None, None, w.cuda(), b.cuda(), 1e-6, C=d)  # in place, C only
    assert m3.m3_stream_status() == 0
    ref = m3_prep.qk_norm_bias(raw, w.double().numpy(), b.double().numpy(), 1e-6)
    assert ulp_check(d.float().cpu().numpy(), ref, magnitude(raw, w, b)) == 0


def test_prep_then_scan_matches_oracle():
    """The layer from raw projections: prep then the tensor-core scan, against
    the oracle's prep rounded to bf16 then the oracle's scan."""
    w = I.Workload(I.Shape(2, 200, 4, 64, 128, 4, 1, 64, "bf16"), bc="normal", decay="slow",
                   with_h0=True, with_prev=False)
    inp = I.make_scan_inputs(w, seed=60)
    Braw, wB, bB = draw(inp["B"].shape, torch.bfloat16, 61, 1, 4, 128)
    Craw, wC, bC = draw(inp["C"].shape, torch.bfloat16, 62, 1, 4, 128)
    d = {k: v.cuda() for k, v in inp.items()}
    Bo, Co = m3.m3_bc_prep(Braw.cuda(), Craw.cuda(), wB.cuda(), bB.cuda(), wC.cuda(), bC.cuda())
    y, fs = m3.m3_scan_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], Bo, Co, 64, d["h0"])
    assert m3.m3_stream_status() == 0
    Bref = torch.from_numpy(m3_prep.qk_norm_bias(Braw, wB.double().numpy(), bB.double().numpy()))
    Cref = torch.from_numpy(m3_prep.qk_norm_bias(Craw, wC.double().numpy(), bC.double().numpy()))
    yo, ho = oracle.scan(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"],
                         Bref.float().bfloat16(), Cref.float().bfloat16(), inp["h0"])
    assert rel_err(y.float().cpu().numpy(), yo) <= TOL["bf16"]
    assert rel_err(fs.cpu().numpy(), ho) <= TOL["bf16"]


def test_prep_bench_workload_sampled_rows():
    """The bench's prep line (per-head B and C: [8][2048][64][1][128] bf16 each),
    a seeded sample of 4096 rows of each output against the oracle."""
    G, N = 64, 128
    gen = torch.Generator(device="cuda").manual_seed(1031)
    shp = (8, 2048, G, 1, N)
    Br = torch.randn(shp, generator=gen, device="cuda").to(torch.bfloat16)
    Cr = torch.randn(shp, generator=gen, device="cuda").to(torch.bfloat16)
    prm = [torch.randn((G, 1, N), generator=gen, device="cuda") for _ in range(4)]
    Bo, Co = m3.m3_bc_prep(Br, Cr, *prm)
    assert m3.m3_stream_status() == 0
    rows = np.random.default_rng(7).choice(8 * 2048 * G, size=4096, replace=False)
    for raw, out, w, b in ((Br, Bo, prm[0], prm[1]), (Cr, Co, prm[2], prm[3])):
        r2 = raw.reshape(-1, N)[torch.from_numpy(rows).cuda()].cpu()
        o2 = out.reshape(-1, N)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
        ch = torch.from_numpy(rows % G)
        wr, br = w.reshape(G, N).cpu()[ch], b.reshape(G, N).cpu()[ch]
        wr4 = wr.double().numpy()[:, None, None, :]
        br4 = br.double().numpy()[:, None, None, :]
        ref = m3_prep.qk_norm_bias(r2[:, None, None, :], wr4, br4)[:, 0, 0, :]
        mag = (np.abs(m3_prep.qk_norm_bias(r2[:, None, None, :], wr4, None))
               + np.abs(br4))[:, 0, 0, :]
        assert ulp_check(o2, ref, mag) == 0
