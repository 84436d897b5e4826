"""Randomised pins of the oracle (CPU, hypothesis): over random small shapes,
ranks, groups, angle-rate layouts and lengths, the token recurrence equals its
two independently written forms (the materialised decay x width-2
convolution mask, and the real RoPE quadratic form), y is linear in x, and a
scan split at any token and continued from the first part's final state and
last token equals the unsplit scan."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


def problem(seed, L, H, G, R, N, P, per_head):
    rng = np.random.default_rng(seed)
    b = 1
    Gt = H if per_head else G
    return dict(x=rng.standard_normal((b, L, H, R, P)),
                dt=np.log1p(np.exp(rng.normal(-1.0, 0.6, (b, L, H)))),
                A=-np.exp(rng.uniform(-1.0, 1.5, (b, L, H))),
                lam=1 / (1 + np.exp(-rng.standard_normal((b, L, H)))),
                theta=rng.uniform(-np.pi, np.pi, (b, L, Gt, N // 2)),
                B=rng.standard_normal((b, L, G, R, N)), C=rng.standard_normal((b, L, G, R, N)),
                h0=rng.standard_normal((b, H, N, P)), B_prev=rng.standard_normal((b, G, R, N)),
                x_prev=rng.standard_normal((b, H, R, P)))


ORDER = ("x", "dt", "A", "lam", "theta", "B", "C", "h0", "B_prev", "x_prev")
shapes = st.tuples(st.integers(0, 10 ** 6), st.integers(1, 24), st.sampled_from([(1, 1), (2, 1),
                   (2, 2), (4, 2)]), st.integers(1, 3), st.sampled_from([2, 4, 6]),
                   st.integers(1, 4), st.booleans())


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@settings(max_examples=40, deadline=None)
@given(shapes)
def test_three_forms_agree(sh):
    seed, L, (H, G), R, N, P, per_head = sh
    d = problem(seed, L, H, G, R, N, P, per_head)
    args = [d[k] for k in ORDER]
    y, h = oracle.scan(*args, f64=True)
    ym, hm = oracle.scan_mask(*args)
    yr, hr = oracle.scan_rope(*args)
    assert rel(ym, y) < 1e-10 and rel(hm, h) < 1e-10
    assert rel(yr, y) < 1e-10 and rel(hr, h) < 1e-10


@settings(max_examples=30, deadline=None)
@given(shapes, st.floats(-3.0, 3.0))
def test_linear_in_x(sh, a):
    seed, L, (H, G), R, N, P, per_head = sh
    d = problem(seed, L, H, G, R, N, P, per_head)
    x2 = np.random.default_rng(seed + 1).standard_normal(d["x"].shape)
    base = {**d, "h0": None, "B_prev": None, "x_prev": None}
    y1, _ = oracle.scan(*[base[k] for k in ORDER], f64=True)
    y2, _ = oracle.scan(*[{**base, "x": x2}[k] for k in ORDER], f64=True)
    y3, _ = oracle.scan(*[{**base, "x": a * d["x"] + x2}[k] for k in ORDER], f64=True)
    assert rel(y3, a * y1 + y2) < 1e-10 or np.max(np.abs(y3 - (a * y1 + y2))) < 1e-12


@settings(max_examples=30, deadline=None)
@given(shapes, st.floats(0.0, 1.0))
def test_split_continuation(sh, frac):
    seed, L, (H, G), R, N, P, per_head = sh
    d = problem(seed, L, H, G, R, N, P, per_head)
    cut = int(round(frac * L))
    y, h = oracle.scan(*[d[k] for k in ORDER], f64=True)
    seq = ("x", "dt", "A", "lam", "theta", "B", "C")
    first = {**{k: d[k][:, :cut] for k in seq}, "h0": d["h0"], "B_prev": d["B_prev"],
             "x_prev": d["x_prev"]}
    y1, h1 = oracle.scan(*[first[k] for k in ORDER], f64=True)
    if cut > 0:
        bp, xp = d["B"][:, cut - 1], d["x"][:, cut - 1]
    else:
        bp, xp = d["B_prev"], d["x_prev"]
    second = {**{k: d[k][:, cut:] for k in seq}, "h0": h1, "B_prev": bp, "x_prev": xp}
    y2, h2 = oracle.scan(*[second[k] for k in ORDER], f64=True)
    assert rel(np.concatenate([y1, y2], axis=1), y) < 1e-10
    assert rel(h2, h) < 1e-10


@settings(max_examples=12, deadline=None)
@given(st.integers(0, 10 ** 6), st.integers(1, 6), st.sampled_from([(1, 1), (2, 1), (2, 2)]),
       st.integers(1, 2), st.sampled_from([2, 4]), st.integers(1, 3), st.booleans())
def test_gradient_oracle_matches_finite_differences(seed, L, HG, R, N, P, per_head):
    """Random shapes: three random coordinates of every input, central
    differences of the C oracle against the autograd gradient oracle."""
    from oracle import m3_grad
    H, G = HG
    d = problem(seed, L, H, G, R, N, P, per_head)
    rng = np.random.default_rng(seed + 2)
    dy = rng.standard_normal(d["x"].shape)
    dfin = rng.standard_normal(d["h0"].shape)
    _, _, grads = m3_grad.scan_grads(*[d[k] for k in ORDER], dy=dy, d_final=dfin)

    def loss():
        yo, ho = oracle.scan(*[d[k] for k in ORDER], f64=True)
        return float(np.sum(yo * dy) + np.sum(ho * dfin))

    hstep = 1e-5
    for name in ORDER:
        flat = d[name].reshape(-1)
        g = grads[name].reshape(-1)
        scale = max(np.max(np.abs(g)), 1e-12)
        for i in rng.choice(flat.size, size=min(3, flat.size), replace=False):
            keep = flat[i]
            flat[i] = keep + hstep
            lp = loss()
            flat[i] = keep - hstep
            lm = loss()
            flat[i] = keep
            assert abs((lp - lm) / (2 * hstep) - g[i]) <= 1e-6 * scale, (name, int(i))
