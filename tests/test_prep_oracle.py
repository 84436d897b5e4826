"""Pins of the B / C prep oracle (oracle/m3_prep.py), CPU only: a library
routine (torch's RMS norm) for the normalisation, the closed form of the
output's mean square, scale invariance at eps = 0, and linearity in the
per-channel scale and bias."""
import numpy as np
import torch

from oracle import m3_prep


def raw(shape=(5, 7, 2, 3, 32), seed=0):
    return np.random.default_rng(seed).standard_normal(shape) * 3.0


def test_matches_library_rms_norm():
    x = raw()
    w = np.random.default_rng(1).standard_normal(x.shape[-3:])
    b = np.random.default_rng(2).standard_normal(x.shape[-3:])
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (x.shape[-1],), eps=1e-6).numpy()
    ref = ref * w + b
    assert np.max(np.abs(m3_prep.qk_norm_bias(x, w, b, 1e-6) - ref)) < 1e-12


def test_mean_square_closed_form():
    """With unit scale and no bias each row's mean square is ms / (ms + eps)."""
    x = raw(seed=3)
    eps = 0.25
    y = m3_prep.qk_norm_bias(x, eps=eps)
    ms = np.mean(x * x, axis=-1)
    assert np.allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12, atol=0)


def test_scale_invariance_without_eps():
    x = raw(seed=4)
    assert np.allclose(m3_prep.qk_norm_bias(7.5 * x, eps=0.0), m3_prep.qk_norm_bias(x, eps=0.0),
                       rtol=1e-12, atol=1e-12)


def test_linear_in_scale_and_bias():
    x = raw(seed=5)
    g = np.random.default_rng(6)
    w1, w2 = g.standard_normal(x.shape[-3:]), g.standard_normal(x.shape[-3:])
    b1 = g.standard_normal(x.shape[-3:])
    base = m3_prep.qk_norm_bias(x)
    assert np.allclose(m3_prep.qk_norm_bias(x, w1 + w2), m3_prep.qk_norm_bias(x, w1)
                       + m3_prep.qk_norm_bias(x, w2), rtol=1e-12, atol=1e-12)
    assert np.allclose(m3_prep.qk_norm_bias(x, None, b1), base + b1, rtol=1e-12, atol=1e-12)
