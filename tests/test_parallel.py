"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding covers
every (batch, head) chain exactly once, and the timing reductions take the
slowest rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_exp_b200.parallel import max_over_ranks, shard_range, sum_over_ranks


@pytest.mark.parametrize("n,world", [(8, 2), (7, 2), (1, 2), (64, 8), (5, 3)])
def test_shard_range_partitions(n, world):
    seen = []
    for r in range(world):
        a, b = shard_range(n, world, r)
        assert 0 <= a <= b <= n
        seen.extend(range(a, b))
    assert seen == list(range(n))


def test_shard_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a, b = shard_range(8, world, rank)
        local_chains = (b - a) * 64
        t = 1.0 + rank  # this rank's step time
        out[rank] = torch.tensor([max_over_ranks(t), sum_over_ranks(local_chains)])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        mx, total = out[r].tolist()
        assert mx == 2.0          # the slowest rank
        assert total == 8 * 64    # every chain exactly once


def test_single_process_reductions_are_identity():
    assert max_over_ranks(3.5) == 3.5 and sum_over_ranks(2.0) == 2.0


# ---- sequence split across ranks (context parallel) ---------------------------
# The host orchestration with the oracle standing in for the per-rank kernels:
# the ranks' y, concatenated in token order, and the last rank's end state
# must equal one oracle scan over the whole sequence.

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from oracle import m3_grad  # noqa: E402
from selective_state_space_exp_b200.parallel import (seq_boundary, seq_finish,  # noqa: E402
                                                     seq_parallel_scan, seq_summary)


class OracleOps:
    """Per-rank steps computed by the fp64 oracle and numpy (test stand-in)."""

    def scan_state(self, x, dt, A, lam, theta, B, C, chunk, B_prev, x_prev):
        _, hL = oracle.scan(x, dt, A, lam, theta, B, C, None, B_prev, x_prev, f64=True)
        return torch.from_numpy(hL)

    def segment_totals(self, x, dt, A, theta, B, chunk):
        dtn, An, thn = dt.numpy(), A.numpy(), theta.numpy()
        H, Gt = dtn.shape[2], thn.shape[2]
        th_h = thn[:, :, np.arange(H) // (H // Gt)]
        return (torch.from_numpy((dtn * An).sum(axis=1)),
                torch.from_numpy((dtn[..., None] * th_h).sum(axis=1)))

    def state_fold(self, h0, T, lam, phi):
        h = np.zeros(T.shape[1:]) if h0 is None else h0.numpy().copy()
        for s in range(T.shape[0]):
            e = np.exp(lam[s].numpy())[:, :, None, None]
            c = np.cos(phi[s].numpy())[..., None]
            sn = np.sin(phi[s].numpy())[..., None]
            u0, u1 = e * h[:, :, 0::2], e * h[:, :, 1::2]
            n0 = c * u0 - sn * u1 + T[s].numpy()[:, :, 0::2]
            n1 = sn * u0 + c * u1 + T[s].numpy()[:, :, 1::2]
            h = np.empty_like(h)
            h[:, :, 0::2], h[:, :, 1::2] = n0, n1
        return torch.from_numpy(h)

    def scan_fwd(self, x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev):
        y, hL = oracle.scan(x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, f64=True)
        return torch.from_numpy(y), torch.from_numpy(hL)

    def scan_bwd(self, x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev, dy, d_final):
        _, _, g = m3_grad.scan_grads(x, dt, A, lam, theta, B, C, h0, B_prev, x_prev, dy=dy,
                                     d_final=d_final)
        return {k: torch.from_numpy(v) for k, v in g.items()}


def _seq_problem(L=24, theta_per_head=False):
    rng = np.random.default_rng(77)
    b, H, G, P, N, R = 2, 4, 2, 3, 6, 2
    Gt = H if theta_per_head else G
    d = dict(x=rng.standard_normal((b, L, H, R, P)),
             dt=np.log1p(np.exp(rng.normal(-1.0, 0.5, (b, L, H)))),
             A=-np.exp(rng.uniform(0.0, 1.0, (b, L, H))),
             lam=1 / (1 + np.exp(-rng.standard_normal((b, L, H)))),
             theta=rng.uniform(-np.pi, np.pi, (b, L, Gt, N // 2)),
             B=rng.standard_normal((b, L, G, R, N)), C=rng.standard_normal((b, L, G, R, N)),
             h0=rng.standard_normal((b, H, N, P)), B_prev=rng.standard_normal((b, G, R, N)),
             x_prev=rng.standard_normal((b, H, R, P)))
    return {k: torch.from_numpy(v) for k, v in d.items()}


def _segment(d, rank, world):
    L = d["x"].shape[1]
    a, b = rank * L // world, (rank + 1) * L // world
    return {k: (v[:, a:b].contiguous() if k in ("x", "dt", "A", "lam", "theta", "B", "C") else v)
            for k, v in d.items()}


def _seq_worker(rank, world, port, out, theta_per_head):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = _segment(_seq_problem(theta_per_head=theta_per_head), rank, world)
        y, hL = seq_parallel_scan(s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"],
                                  64, s["h0"], s["B_prev"], s["x_prev"], ops=OracleOps())
        out[rank] = (y, hL)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,theta_per_head", [(2, False), (3, True)])
def test_gloo_sequence_split_matches_one_scan(world, theta_per_head):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_seq_worker, args=(world, port, out, theta_per_head), nprocs=world, join=True)
    d = _seq_problem(theta_per_head=theta_per_head)
    y_ref, h_ref = oracle.scan(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                               d["h0"], d["B_prev"], d["x_prev"], f64=True)
    y = np.concatenate([out[r][0].numpy() for r in range(world)], axis=1)
    assert np.max(np.abs(y - y_ref)) <= 1e-10 * np.max(np.abs(y_ref))
    hL = out[world - 1][1].numpy()
    assert np.max(np.abs(hL - h_ref)) <= 1e-10 * np.max(np.abs(h_ref))


def test_sequence_split_phases_in_one_process():
    """The same phases driven rank by rank in one process (the exchange is a
    list), as a one-device emulation does."""
    world = 4
    d = _seq_problem(L=20)
    segs = [_segment(d, r, world) for r in range(world)]
    ops = OracleOps()
    lasts = [seq_boundary(s["x"], s["B"]) for s in segs]
    prevs = [(d["B_prev"], d["x_prev"])] + [(lasts[r - 1][0], lasts[r - 1][1]) for r in range(1, world)]
    sums = [seq_summary(ops, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                        *prevs[r]) for r, s in enumerate(segs)]
    Ts, lams, phis = [t[0] for t in sums], [t[1] for t in sums], [t[2] for t in sums]
    ys = [seq_finish(ops, r, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                     d["h0"], Ts, lams, phis, *prevs[r])[0] for r, s in enumerate(segs)]
    y_ref, _ = oracle.scan(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                           d["h0"], d["B_prev"], d["x_prev"], f64=True)
    y = np.concatenate([t.numpy() for t in ys], axis=1)
    assert np.max(np.abs(y - y_ref)) <= 1e-10 * np.max(np.abs(y_ref))


# ---- backward of the sequence split ----------------------------------------------

def _seq_bwd_problem(L=24, theta_per_head=False):
    d = _seq_problem(L=L, theta_per_head=theta_per_head)
    rng = np.random.default_rng(78)
    d["dy"] = torch.from_numpy(rng.standard_normal(tuple(d["x"].shape)))
    d["d_final"] = torch.from_numpy(rng.standard_normal(tuple(d["h0"].shape)))
    return d


def _bwd_reference(d):
    _, _, g = m3_grad.scan_grads(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                                 d["h0"], d["B_prev"], d["x_prev"], dy=d["dy"],
                                 d_final=d["d_final"])
    return g


def _check_split_grads(parts, ref, world):
    for k in ("x", "dt", "A", "lam", "theta", "B", "C"):
        got = np.concatenate([parts[r][k].numpy() for r in range(world)], axis=1)
        assert np.max(np.abs(got - ref[k])) <= 1e-10 * np.max(np.abs(ref[k])), k
    for k_got, k_ref in (("h_in", "h0"), ("B_prev", "B_prev"), ("x_prev", "x_prev")):
        got = parts[0][k_got].numpy()
        assert np.max(np.abs(got - ref[k_ref])) <= 1e-10 * np.max(np.abs(ref[k_ref])), k_got


def _seq_bwd_worker(rank, world, port, out, theta_per_head):
    from selective_state_space_exp_b200.parallel import seq_parallel_scan_bwd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = _seq_bwd_problem(theta_per_head=theta_per_head)
        s = _segment(d, rank, world)
        L = d["x"].shape[1]
        dy = d["dy"][:, rank * L // world:(rank + 1) * L // world].contiguous()
        g = seq_parallel_scan_bwd(s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"],
                                  dy, 64, s["h0"], s["B_prev"], s["x_prev"], d["d_final"],
                                  ops=OracleOps())
        out[rank] = g
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,theta_per_head", [(2, False), (3, True)])
def test_gloo_sequence_split_backward_matches_one_backward(world, theta_per_head):
    """Gradients of the split scan, ranks as gloo processes with the oracle
    standing in for the kernels: every input's gradient, in token order, equals
    the gradient oracle's on the whole sequence (the last token of each
    segment carries the next segment's left-endpoint terms)."""
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_seq_bwd_worker, args=(world, port, out, theta_per_head), nprocs=world, join=True)
    _check_split_grads(out, _bwd_reference(_seq_bwd_problem(theta_per_head=theta_per_head)), world)


def test_sequence_split_backward_phases_in_one_process():
    """The backward's phases rank by rank in one process (4 ranks)."""
    from selective_state_space_exp_b200.parallel import seq_end_adjoint, seq_incoming_state
    world = 4
    d = _seq_bwd_problem(L=20)
    L = d["x"].shape[1]
    segs = [_segment(d, r, world) for r in range(world)]
    dys = [d["dy"][:, r * L // world:(r + 1) * L // world] for r in range(world)]
    ops = OracleOps()
    lasts = [seq_boundary(s["x"], s["B"]) for s in segs]
    prevs = [(d["B_prev"], d["x_prev"])] + [lasts[r - 1] for r in range(1, world)]
    sums = [seq_summary(ops, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                        *prevs[r]) for r, s in enumerate(segs)]
    Ts, lams, phis = [t[0] for t in sums], [t[1] for t in sums], [t[2] for t in sums]
    h_ins = [seq_incoming_state(ops, r, d["h0"], Ts, lams, phis) for r in range(world)]
    args = lambda r: (segs[r]["x"], segs[r]["dt"], segs[r]["A"], segs[r]["lam"],
                      segs[r]["theta"], segs[r]["B"], segs[r]["C"], 64, h_ins[r], *prevs[r])
    Ds = [ops.scan_bwd(*args(r), dys[r], None)["h0"] for r in range(world)]
    parts = []
    for r in range(world):
        d_end = seq_end_adjoint(ops, r, world, d["d_final"], Ds, lams, phis)
        g = ops.scan_bwd(*args(r), dys[r], d_end)
        parts.append({k: v.clone() for k, v in g.items()})
    for r in range(world - 1):  # the next segment's left-endpoint gradients
        parts[r]["B"][:, -1] += parts[r + 1]["B_prev"]
        parts[r]["x"][:, -1] += parts[r + 1]["x_prev"]
    parts[0]["h_in"] = parts[0]["h0"]
    _check_split_grads(parts, _bwd_reference(d), world)


def test_sequence_split_backward_without_h0_or_previous_token():
    """The zero paths: no initial state, no previous token, no final-state
    gradient (4 ranks in one process, oracle stand-ins)."""
    from selective_state_space_exp_b200.parallel import seq_end_adjoint, seq_incoming_state
    world = 4
    d = _seq_bwd_problem(L=16)
    for k in ("h0", "B_prev", "x_prev", "d_final"):
        d[k] = None
    L = d["x"].shape[1]
    segs = [_segment(d, r, world) for r in range(world)]
    dys = [d["dy"][:, r * L // world:(r + 1) * L // world] for r in range(world)]
    ops = OracleOps()
    lasts = [seq_boundary(s["x"], s["B"]) for s in segs]
    prevs = [(None, None)] + [lasts[r - 1] for r in range(1, world)]
    sums = [seq_summary(ops, s["x"], s["dt"], s["A"], s["lam"], s["theta"], s["B"], s["C"], 64,
                        *prevs[r]) for r, s in enumerate(segs)]
    Ts, lams, phis = [t[0] for t in sums], [t[1] for t in sums], [t[2] for t in sums]
    h_ins = [seq_incoming_state(ops, r, None, Ts, lams, phis) for r in range(world)]
    h_ins[0] = torch.zeros_like(Ts[0])
    args = lambda r: (segs[r]["x"], segs[r]["dt"], segs[r]["A"], segs[r]["lam"],
                      segs[r]["theta"], segs[r]["B"], segs[r]["C"], 64, h_ins[r], *prevs[r])
    Ds = [ops.scan_bwd(*args(r), dys[r], None)["h0"] for r in range(world)]
    assert seq_end_adjoint(ops, world - 1, world, None, Ds, lams, phis) is None
    parts = [{k: v.clone() for k, v in
              ops.scan_bwd(*args(r), dys[r], seq_end_adjoint(ops, r, world, None, Ds, lams,
                                                               phis)).items()}
             for r in range(world)]
    for r in range(world - 1):
        parts[r]["B"][:, -1] += parts[r + 1]["B_prev"]
        parts[r]["x"][:, -1] += parts[r + 1]["x_prev"]
    _, _, ref = m3_grad.scan_grads(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"],
                                   np.zeros(tuple(Ts[0].shape)), dy=d["dy"])
    for k in ("x", "dt", "A", "lam", "theta", "B", "C"):
        got = np.concatenate([parts[r][k].numpy() for r in range(world)], axis=1)
        assert np.max(np.abs(got - ref[k])) <= 1e-10 * np.max(np.abs(ref[k])), k
    assert np.max(np.abs(parts[0]["h0"].numpy() - ref["h0"])) <= 1e-10 * np.max(np.abs(ref["h0"]))


# ---- batch sharding, assembled ------------------------------------------------
# Each rank scans its shard_range share of one seeded batch (the oracle standing
# in for the rank's kernels); batch_gather assembles the shares, which must
# equal one oracle scan of the whole batch.

from selective_state_space_exp_b200.parallel import batch_gather, batch_shard  # noqa: E402


def _batch_problem(b=5):
    rng = np.random.default_rng(91)
    L, H, G, P, N, R = 12, 2, 1, 3, 4, 2
    d = dict(x=rng.standard_normal((b, L, H, R, P)),
             dt=np.log1p(np.exp(rng.normal(-1.0, 0.5, (b, L, H)))),
             A=-np.exp(rng.uniform(0.0, 1.0, (b, L, H))),
             lam=1 / (1 + np.exp(-rng.standard_normal((b, L, H)))),
             theta=rng.uniform(-np.pi, np.pi, (b, L, G, N // 2)),
             B=rng.standard_normal((b, L, G, R, N)), C=rng.standard_normal((b, L, G, R, N)),
             h0=rng.standard_normal((b, H, N, P)), B_prev=rng.standard_normal((b, G, R, N)),
             x_prev=rng.standard_normal((b, H, R, P)))
    return {k: torch.from_numpy(v) for k, v in d.items()}


def _batch_worker(rank, world, port, out, b):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = batch_shard(_batch_problem(b), world, rank)
        if d["x"].shape[0]:
            y, hL = OracleOps().scan_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"],
                                         d["C"], 4, d["h0"], d["B_prev"], d["x_prev"])
        else:  # more ranks than rows: this rank launches nothing (batch 0 is not a shape)
            y = torch.zeros(d["x"].shape, dtype=torch.float64)
            hL = torch.zeros(d["h0"].shape, dtype=torch.float64)
        out[rank] = (batch_gather(y, b).numpy(), batch_gather(hL, b).numpy(), y.shape[0])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,b", [(2, 5), (3, 5), (2, 1)])
def test_gloo_batch_shards_assemble_to_the_whole_batch(world, b):
    out = mp.Manager().dict()
    mp.spawn(_batch_worker, args=(world, _free_port(), out, b), nprocs=world, join=True)
    d = _batch_problem(b)
    y_ref, h_ref = OracleOps().scan_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"],
                                        d["C"], 4, d["h0"], d["B_prev"], d["x_prev"])
    assert sum(out[r][2] for r in range(world)) == b  # every batch row scanned once
    for r in range(world):
        y, hL, _ = out[r]
        assert y.shape == tuple(y_ref.shape) and hL.shape == tuple(h_ref.shape)
        np.testing.assert_allclose(y, y_ref.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(hL, h_ref.numpy(), rtol=0, atol=1e-12)


def test_batch_gather_rejects_a_wrong_share():
    out = mp.Manager().dict()
    mp.spawn(_bad_share_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    assert out[0] == "ValueError" and out[1] == "ValueError"


def _bad_share_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        try:
            batch_gather(torch.zeros(4, 3), 5)  # shares of 5 rows are 3 and 2
            out[rank] = "ok"
        except ValueError:
            out[rank] = "ValueError"
    finally:
        dist.destroy_process_group()
