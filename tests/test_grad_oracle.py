"""Pins of the gradient oracle (oracle/m3_grad.py), CPU only.

Its forward loop is checked against the C oracle (an independent
implementation of the same recurrence), and every gradient it returns against
central finite differences of the C oracle's fp64 forward, so a dropped term,
a wrong sign or a misrouted index in either the loop or the use of autograd
fails here.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import m3_grad
from selective_state_space_exp_b200 import inputs as I


def tiny(L=6, H=2, G=1, R=2, N=4, P=3, theta_per_head=False, seed=0, decay="slow"):
    w = I.Workload(I.Shape(1, L, H, P, N, R, G, 64, "f32"), bc="normal", decay=decay,
                   with_h0=True, with_prev=True, theta_per_head=theta_per_head)
    inp = I.make_scan_inputs(w, seed=seed)
    return {k: v.double().numpy() for k, v in inp.items()}


@pytest.mark.parametrize("R,G,H,tph", [(1, 1, 1, False), (2, 1, 2, False), (3, 2, 4, False),
                                       (2, 1, 2, True)])
def test_forward_matches_c_oracle(R, G, H, tph):
    inp = tiny(L=40, H=H, G=G, R=R, N=8, P=5, theta_per_head=tph, seed=10 + R)
    args = [inp[k] for k in m3_grad.NAMES]
    y, zL = m3_grad.forward(*[torch.from_numpy(a) for a in args])
    yo, ho = oracle.scan(*args, f64=True)
    assert np.max(np.abs(y.numpy() - yo)) <= 1e-12 * np.max(np.abs(yo))
    assert np.max(np.abs(zL.numpy() - ho)) <= 1e-12 * np.max(np.abs(ho))


def _loss_c(inp, dy, dfin):
    yo, ho = oracle.scan(*[inp[k] for k in m3_grad.NAMES], f64=True)
    return float(np.sum(yo * dy) + np.sum(ho * dfin))


@pytest.mark.parametrize("G,H,tph", [(1, 2, False), (2, 2, False), (1, 2, True)])
def test_gradients_match_finite_differences(G, H, tph):
    """Every input, a seeded sample of coordinates each, central differences of
    the C oracle with step 1e-5: agreement to 1e-7 of the tensor's largest
    gradient (the difference's own error is ~1e-10)."""
    inp = tiny(L=6, H=H, G=G, R=2, N=4, P=3, theta_per_head=tph, seed=20 + G)
    rng = np.random.default_rng(5)
    dy = rng.standard_normal(inp["x"].shape)
    dfin = rng.standard_normal(inp["h0"].shape)
    _, _, grads = m3_grad.scan_grads(*[inp[k] for k in m3_grad.NAMES], dy=dy, d_final=dfin)
    h = 1e-5
    for name in m3_grad.NAMES:
        g = grads[name]
        flat = inp[name].reshape(-1)
        idx = rng.choice(flat.size, size=min(8, flat.size), replace=False)
        for i in idx:
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss_c(inp, dy, dfin)
            flat[i] = keep - h
            lm = _loss_c(inp, dy, dfin)
            flat[i] = keep
            fd = (lp - lm) / (2 * h)
            scale = max(np.max(np.abs(g)), 1e-12)
            assert abs(fd - g.reshape(-1)[i]) <= 1e-7 * scale, (name, int(i), fd, g.reshape(-1)[i])


def test_gradient_of_y_only_and_final_only_add_up():
    """The loss is linear in (dy, d_final): the two halves' gradients add up."""
    inp = tiny(L=9, seed=31)
    rng = np.random.default_rng(2)
    dy = rng.standard_normal(inp["x"].shape)
    dfin = rng.standard_normal(inp["h0"].shape)
    args = [inp[k] for k in m3_grad.NAMES]
    _, _, g_both = m3_grad.scan_grads(*args, dy=dy, d_final=dfin)
    _, _, g_y = m3_grad.scan_grads(*args, dy=dy)
    _, _, g_f = m3_grad.scan_grads(*args, d_final=dfin)
    for n in m3_grad.NAMES:
        assert np.allclose(g_both[n], g_y[n] + g_f[n], rtol=1e-12, atol=1e-12)


def test_varlen_gradients_are_the_batched_ones():
    """Packed sequences of one length: the per-sequence gradients placed back in
    the packed layout are the batched call's (a misplaced slice or a gradient
    leaking across a boundary fails)."""
    S, L = 3, 11
    inp = tiny(L=S * L, H=2, G=1, R=2, N=4, P=3, seed=41)
    rng = np.random.default_rng(8)
    flat = {k: inp[k][0] for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    per = {"h0": rng.standard_normal((S,) + inp["h0"].shape[1:]),
           "B_prev": rng.standard_normal((S,) + inp["B_prev"].shape[1:]),
           "x_prev": rng.standard_normal((S,) + inp["x_prev"].shape[1:])}
    dy = rng.standard_normal(flat["x"].shape)
    dfin = rng.standard_normal(per["h0"].shape)
    got = m3_grad.scan_grads_varlen([0, L, 2 * L, 3 * L], *[flat[k] for k in
                                    ("x", "dt", "A", "lam", "theta", "B", "C")],
                                    per["h0"], per["B_prev"], per["x_prev"], dy=dy,
                                    d_final=dfin)
    bat = {k: v.reshape((S, L) + v.shape[1:]) for k, v in flat.items()}
    _, _, ref = m3_grad.scan_grads(*[bat[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C")],
                                   per["h0"], per["B_prev"], per["x_prev"],
                                   dy=dy.reshape((S, L) + dy.shape[1:]), d_final=dfin)
    for k in ("x", "dt", "A", "lam", "theta", "B", "C"):
        assert np.allclose(got[k], ref[k].reshape(got[k].shape), rtol=1e-12, atol=1e-13), k
    for k in ("h0", "B_prev", "x_prev"):
        assert np.allclose(got[k], ref[k], rtol=1e-12, atol=1e-13), k
