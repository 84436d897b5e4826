"""Pins of the block-projection oracle (oracle/m3_block.py) to things other
than itself: a brute-force sum for the projection, closed forms of the gate,
and identities the readings imply (PaperWeekly page section 2.3-2.4)."""
import math

import numpy as np

from oracle import m3_block as ob


def test_linear_equals_brute_force_sum():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((5, 7))
    W = rng.standard_normal((3, 7))
    b = rng.standard_normal(3)
    out = ob.linear(A, W, b)
    for m in range(5):
        for n in range(3):
            s = b[n]
            for k in range(7):
                s += A[m, k] * W[n, k]
            assert abs(out[m, n] - s) < 1e-12


def test_linear_identity_and_linearity():
    rng = np.random.default_rng(2)
    A = rng.standard_normal((4, 6))
    assert np.array_equal(ob.linear(A, np.eye(6)), A)
    W = rng.standard_normal((5, 6))
    A2 = rng.standard_normal((4, 6))
    assert np.allclose(ob.linear(2.5 * A + A2, W), 2.5 * ob.linear(A, W) + ob.linear(A2, W),
                       atol=1e-12)


def test_silu_closed_forms():
    # silu(0) = 0, silu(1) = 1 / (1 + 1/e), silu(-1) = -1 / (1 + e); silu(v) -> v for large v
    assert ob.silu(np.array(0.0)) == 0.0
    assert abs(float(ob.silu(np.array(1.0))) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(float(ob.silu(np.array(-1.0))) + 1.0 / (1.0 + math.e)) < 1e-15
    assert abs(float(ob.silu(np.array(40.0))) - 40.0) < 1e-12
    assert abs(float(ob.silu(np.array(-40.0)))) < 1e-12


def test_mimo_up_broadcast_and_scaling():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 2, 4))           # [T][H][P]
    X = ob.mimo_up(x, np.ones((2, 3, 4)))        # every rank a copy of x
    assert X.shape == (6, 2, 3, 4)
    for r in range(3):
        assert np.array_equal(X[:, :, r], x)
    w = rng.standard_normal((2, 3, 4))
    X = ob.mimo_up(x, w)
    assert np.allclose(X[5, 1, 2], x[5, 1] * w[1, 2])


def test_mimo_down_gate_identities():
    rng = np.random.default_rng(4)
    Y = rng.standard_normal((5, 2, 1, 4))
    assert np.array_equal(ob.mimo_down_gate(Y, np.ones((2, 1, 4))), Y[:, :, 0])  # R = 1, w = 1
    Y = rng.standard_normal((5, 2, 3, 4))
    w = rng.standard_normal((2, 3, 4))
    y = ob.mimo_down_gate(Y, w)
    assert np.allclose(y[2, 1], sum(Y[2, 1, r] * w[1, r] for r in range(3)), atol=1e-12)
    z = np.zeros((5, 2, 4))
    assert np.array_equal(ob.mimo_down_gate(Y, w, z), np.zeros((5, 2, 4)))  # silu(0) = 0
    z = np.full((5, 2, 4), 60.0)
    assert np.allclose(ob.mimo_down_gate(Y, w, z), 60.0 * y, rtol=1e-12)


def test_up_then_down_recovers_the_input():
    """Ranks that copy the input and average it back give the input again."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 2, 8))
    R = 4
    X = ob.mimo_up(x, np.ones((2, R, 8)))
    assert np.allclose(ob.mimo_down_gate(X, np.full((2, R, 8), 1.0 / R)), x, atol=1e-14)
