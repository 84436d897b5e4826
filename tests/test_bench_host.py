"""Host-side pieces of bench.py (no GPU): the algorithmic work formulas agree
with each other where they must, and the roofline arithmetic picks the bound
with the larger time."""
import dataclasses

import pytest

import bench
from selective_state_space_exp_b200 import inputs as I


def test_varlen_work_equals_batched_work_for_equal_lengths():
    s = I.SISO_PREFILL.shape
    f_b, b_b = bench.prefill_work(s)
    f_v, b_v = bench.varlen_work(s, [s.seqlen] * s.batch)
    assert f_v == pytest.approx(f_b, rel=1e-12)
    assert b_v == pytest.approx(b_b, rel=1e-12)


def test_prefill_work_matches_the_published_counts():
    """The SISO / MIMO prefill FLOPs and bytes quoted with the workloads:
    47.4 GFLOP / 310.4 MB and 346.8 GFLOP / 1140.9 MB."""
    f1, b1 = bench.prefill_work(I.SISO_PREFILL.shape)
    f2, b2 = bench.prefill_work(I.MIMO_PREFILL.shape)
    assert f1 == pytest.approx(47.45e9, rel=2e-3) and b1 == pytest.approx(310.4e6, rel=2e-3)
    assert f2 == pytest.approx(346.8e9, rel=2e-3) and b2 == pytest.approx(1140.9e6, rel=2e-3)


def test_backward_work_scales_with_tokens_and_rank():
    s = I.SISO_PREFILL.shape
    f, b = bench.bwd_work(s)
    f2, b2 = bench.bwd_work(dataclasses.replace(s, batch=2 * s.batch))
    assert f2 == pytest.approx(2 * f) and b2 == pytest.approx(2 * b)
    fm, _ = bench.bwd_work(I.MIMO_PREFILL.shape)
    assert fm > 2 * f


def test_roofline_picks_the_slower_bound():
    peaks = {"hbm_gbs": 6544.0, "bf16_tflops": 1653.3, "bf16_tflops_sustained": 1396.4}
    r = bench.roofline(1e12, 1e6, 1e-3, peaks, "measured")     # FLOP-heavy
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(1e12 / 1e-3 / 1e12 / 1653.3,
                                                                 rel=1e-3)
    r = bench.roofline(1e6, 1e9, 1e-3, peaks, "measured")      # byte-heavy
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(1e9 / 1e-3 / 1e9 / 6544.0, rel=1e-3)
    a = bench.alu_roofline(1e12, 1e6, 1.0, peaks)
    assert a["bound"] == "alu" and a["peak"] == pytest.approx(74.4, rel=1e-3)
