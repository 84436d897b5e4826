"""Pins of the fp64 CPU oracle to facts fixed by the paper and by mathematics.

Every check compares the oracle's token-by-token recurrence with something
other than itself: hand-worked values, closed forms, textbook special cases,
the materialised structured mask, the data-dependent RoPE form, invariants.
The last test plants plausible mistakes in the oracle and shows that each one
fails at least one pin.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_problem(seed, b=2, L=11, H=4, G=2, P=3, N=6, R=2, h0=True, prev=True,
                 theta_scale=1.0, lam=None, A_range=(0.0, 1.5)):
    rng = np.random.default_rng(seed)
    d = dict(
        x=rng.standard_normal((b, L, H, R, P)),
        dt=np.log1p(np.exp(rng.normal(-1.0, 0.5, (b, L, H)))),
        A=-np.exp(rng.uniform(*A_range, (b, L, H))),
        lam=(1 / (1 + np.exp(-rng.standard_normal((b, L, H))))) if lam is None
        else np.full((b, L, H), float(lam)),
        theta=theta_scale * rng.uniform(-np.pi, np.pi, (b, L, G, N // 2)),
        B=rng.standard_normal((b, L, G, R, N)),
        C=rng.standard_normal((b, L, G, R, N)),
        h0=rng.standard_normal((b, H, N, P)) if h0 else None,
        B_prev=rng.standard_normal((b, G, R, N)) if prev else None,
        x_prev=rng.standard_normal((b, H, R, P)) if prev else None,
    )
    return d


def run(d, **kw):
    return oracle.scan(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                       d["h0"], d["B_prev"], d["x_prev"], f64=True, **kw)


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# --------------------------------------------------------------------------
# pin functions: each returns a relative error (0 when the oracle is right)

def pin_hand_examples():
    """Hand-worked examples (tests/golden/hand_examples.json)."""
    with open(os.path.join(HERE, "golden", "hand_examples.json")) as f:
        cases = json.load(f)["cases"]

    def num(v):
        if isinstance(v, str):
            return float(eval(v, {"ln2": math.log(2.0), "pi": math.pi}))
        return float(v)

    worst = 0.0
    for c in cases:
        dm = c["dims"]
        L, N, P, R = dm["seqlen"], dm["dstate"], dm["headdim"], dm["rank"]
        arr = lambda v, shp: np.array(
            [num(e) for e in np.array(v, dtype=object).ravel()], dtype=np.float64).reshape(shp)
        x = arr(c["x"], (1, L, 1, R, P))
        dt = arr(c["dt"], (1, L, 1))
        A = arr(c["A"], (1, L, 1))
        lam = arr(c["lam"], (1, L, 1))
        th = arr(c["theta"], (1, L, 1, N // 2))
        B = arr(c["B"], (1, L, 1, R, N))
        C = arr(c["C"], (1, L, 1, R, N))
        h0 = None if c["h0"] is None else arr(c["h0"], (1, 1, N, P))
        Bp = None if c["B_prev"] is None else arr(c["B_prev"], (1, 1, R, N))
        xp = None if c["x_prev"] is None else arr(c["x_prev"], (1, 1, R, P))
        y, hL = oracle.scan(x, dt, A, lam, th, B, C, h0, Bp, xp, f64=True)
        worst = max(worst, rel(y, arr(c["y"], y.shape)), rel(hL, arr(c["hL"], hL.shape)))
    return worst


def pin_mask_form(seed=1):
    """Recurrence == materialised (decay mask) x (width-2 convolution) form."""
    d = rand_problem(seed)
    y, hL = run(d)
    ym, hm = oracle.scan_mask(*[d[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C",
                                                 "h0", "B_prev", "x_prev")])
    return max(rel(y, ym), rel(hL, hm))


def pin_rope_form(seed=2):
    """Complex-state recurrence == real data-dependent-RoPE quadratic form."""
    d = rand_problem(seed, L=17, theta_scale=2.0)
    y, hL = run(d)
    yr, hr = oracle.scan_rope(*[d[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C",
                                                 "h0", "B_prev", "x_prev")])
    return max(rel(y, yr), rel(hL, hr))


def pin_mamba2(seed=3):
    """lam = 1 and theta = 0: the Mamba-2 recurrence h = alpha h + dt B x^T and its
    SSD quadratic form y_t = sum_{s<=t} exp(Lam_t - Lam_s) dt_s (C_t.B_s) x_s."""
    d = rand_problem(seed, lam=1.0, theta_scale=0.0, h0=False, prev=False)
    y, hL = run(d)
    b, L, H, R, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[4]
    y2 = np.zeros_like(y)
    y3 = np.zeros_like(y)
    h2 = np.zeros_like(hL)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            st = np.zeros((N, P))
            for t in range(L):
                a = math.exp(d["dt"][bi, t, h] * d["A"][bi, t, h])
                st = a * st + d["dt"][bi, t, h] * d["B"][bi, t, g].T @ d["x"][bi, t, h]
                y2[bi, t, h] = d["C"][bi, t, g] @ st
            h2[bi, h] = st
            lam_cum = np.cumsum(d["dt"][bi, :, h] * d["A"][bi, :, h])
            for t in range(L):
                acc = np.zeros((R, P))
                for s in range(t + 1):
                    w = math.exp(lam_cum[t] - lam_cum[s]) * d["dt"][bi, s, h]
                    acc += w * (d["C"][bi, t, g] @ d["B"][bi, s, g].T) @ d["x"][bi, s, h]
                y3[bi, t, h] = acc
    return max(rel(y, y2), rel(hL, h2), rel(y, y3))


def pin_real_when_theta_zero(seed=4):
    """theta = 0: the complex state carries two independent real recurrences
    h = alpha (h + (1-lam) dt B_{t-1} x_{t-1}^T) + lam dt B_t x_t^T."""
    d = rand_problem(seed, theta_scale=0.0)
    y, hL = run(d)
    b, L, H, R, P = d["x"].shape
    G = d["B"].shape[2]
    y2 = np.zeros_like(y)
    h2 = np.zeros_like(hL)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            st = d["h0"][bi, h].copy()
            for t in range(L):
                dt, lam = d["dt"][bi, t, h], d["lam"][bi, t, h]
                a = math.exp(dt * d["A"][bi, t, h])
                Bl = d["B_prev"][bi, g] if t == 0 else d["B"][bi, t - 1, g]
                xl = d["x_prev"][bi, h] if t == 0 else d["x"][bi, t - 1, h]
                st = a * (st + (1 - lam) * dt * Bl.T @ xl) + lam * dt * d["B"][bi, t, g].T @ d["x"][bi, t, h]
                y2[bi, t, h] = d["C"][bi, t, g] @ st
            h2[bi, h] = st
    return max(rel(y, y2), rel(hL, h2))


def pin_mimo_is_sum_of_siso(seed=5):
    """MIMO: the state is the sum over input ranks r of SISO states driven by
    (B_r, x_r); output rank r' reads it with C_r'.  R=1 runs of the same
    oracle reassemble the rank-R result."""
    d = rand_problem(seed, R=3)
    y, hL = run(d)
    R = d["x"].shape[3]
    ys = np.zeros_like(y)
    hs = np.zeros_like(hL)
    for r in range(R):
        for ro in range(R):
            e = dict(d)
            e["x"] = d["x"][:, :, :, r:r + 1]
            e["B"] = d["B"][:, :, :, r:r + 1]
            e["C"] = d["C"][:, :, :, ro:ro + 1]
            e["B_prev"] = d["B_prev"][:, :, r:r + 1]
            e["x_prev"] = d["x_prev"][:, :, r:r + 1]
            e["h0"] = d["h0"] if r == 0 else None
            yr, hr = run(e)
            ys[:, :, :, ro:ro + 1] += yr
            if ro == 0:
                hs += hr
    return max(rel(y, ys), rel(hL, hs))


def pin_norm_preserved(seed=6):
    """A = 0 and x = 0: the transition is a pure rotation by 2x2 blocks, so every
    pair's modulus |z_k| (and the Frobenius norm) is conserved."""
    d = rand_problem(seed, L=40, theta_scale=3.0)
    d["A"] = np.zeros_like(d["A"])
    d["x"] = np.zeros_like(d["x"])
    d["x_prev"] = np.zeros_like(d["x_prev"])
    _, hL = run(d)
    m0 = np.hypot(d["h0"][:, :, 0::2], d["h0"][:, :, 1::2])
    m1 = np.hypot(hL[:, :, 0::2], hL[:, :, 1::2])
    return rel(m1, m0)


def pin_steady_state(seed=7):
    """Constant inputs: z converges to (beta e^{i phi} + gamma) u / (1 - alpha e^{i phi}),
    beta = (1-lam) dt alpha, gamma = lam dt, u = sum_r b_r x_r (fixed point)."""
    rng = np.random.default_rng(seed)
    L, N, P, R = 3000, 4, 2, 2
    dt, A, lam = 0.3, -0.9, 0.35
    th = rng.uniform(-2, 2, N // 2)
    Bv = rng.standard_normal((R, N))
    xv = rng.standard_normal((R, P))
    Cv = rng.standard_normal((R, N))
    d = dict(x=np.broadcast_to(xv, (1, L, 1, R, P)).copy(),
             dt=np.full((1, L, 1), dt), A=np.full((1, L, 1), A), lam=np.full((1, L, 1), lam),
             theta=np.broadcast_to(th, (1, L, 1, N // 2)).copy(),
             B=np.broadcast_to(Bv, (1, L, 1, R, N)).copy(),
             C=np.broadcast_to(Cv, (1, L, 1, R, N)).copy(),
             h0=None, B_prev=Bv[None, None].copy(), x_prev=xv[None, None].copy())
    y, hL = run(d)
    alpha = math.exp(dt * A)
    beta, gamma = (1 - lam) * dt * alpha, lam * dt
    z = np.zeros((N // 2, P), dtype=complex)
    for k in range(N // 2):
        e = np.exp(1j * dt * th[k])
        u = (Bv[:, 2 * k] + 1j * Bv[:, 2 * k + 1]) @ xv
        z[k] = (beta * e + gamma) * u / (1 - alpha * e)
    h_ref = np.zeros((N, P))
    h_ref[0::2], h_ref[1::2] = z.real, z.imag
    y_ref = Cv @ h_ref
    return max(rel(hL[0, 0], h_ref), rel(y[0, -1, 0], y_ref))


def ode_error(lam, n, T=2.0, a=-0.7, omega=2.3, nu=1.7, b=(0.8 - 0.6j)):
    """|z_n - z(T)| for dz/dtau = (a + i omega) z + b sin(nu tau), z(0) = 0, with
    n steps of size T/n, against the closed-form solution."""
    h = T / n
    L = n + 1
    tau = np.arange(L) * h
    d = dict(x=np.sin(nu * tau).reshape(1, L, 1, 1, 1), dt=np.full((1, L, 1), h),
             A=np.full((1, L, 1), a), lam=np.full((1, L, 1), lam),
             theta=np.full((1, L, 1, 1), omega),
             B=np.broadcast_to(np.array([b.real, b.imag]), (1, L, 1, 1, 2)).copy(),
             C=np.broadcast_to(np.array([1.0, 0.0]), (1, L, 1, 1, 2)).copy(),
             h0=None, B_prev=None, x_prev=None)
    _, hL = run(d)
    zn = hL[0, 0, 0, 0] + 1j * hL[0, 0, 1, 0]
    mu = a + 1j * omega
    zT = b / 2j * ((np.exp(1j * nu * T) - np.exp(mu * T)) / (1j * nu - mu)
                   - (np.exp(-1j * nu * T) - np.exp(mu * T)) / (-1j * nu - mu))
    return abs(zn - zT), abs(zT)


def pin_second_order():
    """lam = 1/2 (trapezoid) converges at order 2; lam = 1 and lam = 0 (the two
    Euler ends) at order 1.  Returns how far the observed orders are off."""
    orders = {}
    for lam in (0.5, 1.0, 0.0):
        e1, _ = ode_error(lam, 200)
        e2, _ = ode_error(lam, 400)
        orders[lam] = math.log2(e1 / e2)
    return max(abs(orders[0.5] - 2.0), abs(orders[1.0] - 1.0), abs(orders[0.0] - 1.0)) / 10.0


def pin_split_continuation(seed=8):
    """scan(L0 + L1) == scan of the second part seeded with the first part's
    final state and its last token's (B, x) as the previous token."""
    d = rand_problem(seed, L=14)
    y, hL = run(d)
    L0 = 5
    a = {k: (v[:, :L0] if k in ("x", "dt", "A", "lam", "theta", "B", "C") else v)
         for k, v in d.items()}
    ya, ha = run(a)
    b2 = {k: (v[:, L0:] if k in ("x", "dt", "A", "lam", "theta", "B", "C") else v)
          for k, v in d.items()}
    b2["h0"] = ha
    b2["B_prev"] = d["B"][:, L0 - 1]
    b2["x_prev"] = d["x"][:, L0 - 1]
    yb, hb = run(b2)
    return max(rel(np.concatenate([ya, yb], axis=1), y), rel(hb, hL))


def pin_linearity(seed=9):
    """For fixed gates, y and the final state are linear in (x, x_prev, h0)."""
    d1 = rand_problem(seed)
    d2 = rand_problem(seed + 100)
    for k in ("dt", "A", "lam", "theta", "B", "C", "B_prev"):
        d2[k] = d1[k]
    s = -1.7
    d3 = dict(d1)
    for k in ("x", "x_prev", "h0"):
        d3[k] = s * d1[k] + d2[k]
    y1, h1 = run(d1)
    y2, h2 = run(d2)
    y3, h3 = run(d3)
    return max(rel(y3, s * y1 + y2), rel(h3, s * h1 + h2))


PINS = {
    "hand_examples": (pin_hand_examples, 1e-12),
    "mask_form": (pin_mask_form, 1e-11),
    "rope_form": (pin_rope_form, 1e-11),
    "mamba2": (pin_mamba2, 1e-11),
    "real_when_theta_zero": (pin_real_when_theta_zero, 1e-11),
    "mimo_sum_of_siso": (pin_mimo_is_sum_of_siso, 1e-11),
    "norm_preserved": (pin_norm_preserved, 1e-12),
    "steady_state": (pin_steady_state, 1e-10),
    "second_order": (pin_second_order, 0.01),
    "split_continuation": (pin_split_continuation, 1e-12),
    "linearity": (pin_linearity, 1e-11),
}


@pytest.mark.parametrize("name", list(PINS))
def test_pin(name):
    fn, tol = PINS[name]
    err = fn()
    assert err <= tol, f"{name}: {err:.3e} > {tol:.1e}"


def test_rotation_blocks_are_orthogonal():
    """The 2x2 rotation blocks used by the RoPE form keep vector norms."""
    rng = np.random.default_rng(10)
    for _ in range(100):
        phi = rng.uniform(-50, 50)
        v = rng.standard_normal(2)
        Rm = np.array([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]])
        assert abs(np.linalg.norm(Rm @ v) - np.linalg.norm(v)) < 1e-12


def test_decode_driver_equals_scan():
    """The decode step, driven token by token, reproduces the scan."""
    d = rand_problem(11, L=9)
    y, hL = run(d)
    st = d["h0"]
    for t in range(d["x"].shape[1]):
        Bp = d["B_prev"] if t == 0 else d["B"][:, t - 1]
        xp = d["x_prev"] if t == 0 else d["x"][:, t - 1]
        yt, st = oracle.decode_step(st, d["x"][:, t], d["dt"][:, t], d["A"][:, t],
                                    d["lam"][:, t], d["theta"][:, t], d["B"][:, t],
                                    d["C"][:, t], Bp, xp, f64=True)
        assert rel(yt, y[:, t]) < 1e-13
    assert rel(st, hL) < 1e-13


def test_chain_subset_and_threads():
    """Computing a subset of chains, with any thread count, gives the same
    numbers for those chains and leaves the others untouched."""
    d = rand_problem(12, b=3, H=4)
    y, hL = run(d, nthreads=1)
    ys, hs = run(d, chains=[1, 6, 11], nthreads=3)
    for c in (1, 6, 11):
        bi, h = divmod(c, 4)
        assert np.array_equal(ys[bi, :, h], y[bi, :, h])
        assert np.array_equal(hs[bi, h], hL[bi, h])
    assert np.isnan(ys[0, :, 0]).all()


def test_empty_sequence():
    d = rand_problem(13, L=0)
    y, hL = run(d)
    assert y.shape[1] == 0
    assert np.array_equal(hL, d["h0"])


def test_fp32_inputs_widen_exactly():
    """fp32 inputs are widened to fp64 before any arithmetic."""
    d = rand_problem(14)
    d32 = {k: (None if v is None else v.astype(np.float32)) for k, v in d.items()}
    d64 = {k: (None if v is None else v.astype(np.float64)) for k, v in d32.items()}
    y32, h32 = oracle.scan(*[d32[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C",
                                              "h0", "B_prev", "x_prev")])
    y64, h64 = run(d64)
    assert np.array_equal(y32, y64) and np.array_equal(h32, h64)


MUTATIONS = {
    1: "left-endpoint term dropped",
    2: "rotation sign flipped",
    3: "left term reads B_t, x_t",
    4: "lam and 1-lam swapped",
    5: "output not conjugated",
    6: "left term not decayed",
    7: "step angle not scaled by dt",
    8: "decay exponent not scaled by dt",
}


@pytest.mark.parametrize("m", list(MUTATIONS))
def test_pins_catch_planted_mistake(m):
    failed = []
    with oracle.mutation(m):
        for name, (fn, tol) in PINS.items():
            try:
                err = fn()
            except Exception:  # a crash also counts as caught
                err = float("inf")
            if not err <= tol:
                failed.append(name)
    assert failed, f"mutation {m} ({MUTATIONS[m]}) passed every pin"


# ---- per-head angle rates (theta [b][L][H][N/2], a layout variant) ----------

def test_per_head_theta_equal_across_group_matches_grouped():
    """theta given per head, but equal for the heads of each group, gives the
    grouped result exactly (the two layouts index the same rates)."""
    d = rand_problem(901, H=4, G=2)
    y0, h0 = run(d)
    per_head = dict(d, theta=np.repeat(d["theta"], 2, axis=2))  # head h -> group h // 2
    y1, h1 = run(per_head)
    assert np.array_equal(y0, y1) and np.array_equal(h0, h1)


def test_per_head_theta_each_head_matches_its_own_problem():
    """With distinct per-head rates, every head equals an independent one-head
    problem that takes that head's rates as its (shared) theta."""
    d = rand_problem(902, H=4, G=1)
    rng = np.random.default_rng(903)
    d["theta"] = rng.uniform(-np.pi, np.pi, (2, 11, 4, 3))
    y, hL = run(d)
    for h in range(4):
        one = dict(x=d["x"][:, :, h:h + 1], dt=d["dt"][:, :, h:h + 1],
                   A=d["A"][:, :, h:h + 1], lam=d["lam"][:, :, h:h + 1],
                   theta=d["theta"][:, :, h:h + 1], B=d["B"], C=d["C"],
                   h0=d["h0"][:, h:h + 1], B_prev=d["B_prev"], x_prev=d["x_prev"][:, h:h + 1])
        y1, h1 = run(one)
        assert rel(y[:, :, h:h + 1], y1) < 1e-13 and rel(hL[:, h:h + 1], h1) < 1e-13


def test_per_head_theta_forms_agree():
    """The mask form and the RoPE form read per-head rates the same way."""
    d = rand_problem(904, H=4, G=2, L=9)
    rng = np.random.default_rng(905)
    d["theta"] = rng.uniform(-np.pi, np.pi, (2, 9, 4, 3))
    y, hL = run(d)
    for name in ("scan_mask", "scan_rope"):
        yf, hf = getattr(oracle, name)(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"],
                                       d["C"], d["h0"], d["B_prev"], d["x_prev"])
        assert rel(yf, y) < 1e-11 and rel(hf, hL) < 1e-11, name


def test_per_head_theta_decode_matches_scan():
    d = rand_problem(906, H=4, G=2, L=5)
    rng = np.random.default_rng(907)
    d["theta"] = rng.uniform(-np.pi, np.pi, (2, 5, 4, 3))
    y, hL = run(d)
    st = d["h0"]
    for t in range(5):
        Bp = d["B_prev"] if t == 0 else d["B"][:, t - 1]
        xp = d["x_prev"] if t == 0 else d["x"][:, t - 1]
        yt, st = oracle.decode_step(st, d["x"][:, t], d["dt"][:, t], d["A"][:, t],
                                    d["lam"][:, t], d["theta"][:, t], d["B"][:, t],
                                    d["C"][:, t], Bp, xp, f64=True)
        assert rel(yt, y[:, t]) < 1e-12
    assert rel(st, hL) < 1e-12
