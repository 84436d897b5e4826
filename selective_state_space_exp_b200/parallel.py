"""Multi-GPU plumbing for the layer (one process per GPU, torch.distributed).

Batch sharding: the (batch, head) chains of the recurrence are independent,
so the layer shards by batch with no collective on the data path; a
collective appears only in measurement (the slowest rank's time).

Sequence split (context parallel): each rank holds the same number of
consecutive tokens of every sequence.  Over a segment the recurrence unrolls
(PaperWeekly page section 2.2, exponential-trapezoidal step) to
h_end = exp(Lam_seg) Rot(Phi_seg) h_start + T, so one exchange suffices: the
ranks all-gather each segment's last token (the next segment's trapezoid left
endpoint), then their summaries (T from a zero start, Lam_seg, Phi_seg); each
rank folds the earlier segments' summaries into its incoming state and scans
its segment from it.  The steps run in the library's kernels (m3_scan_state,
m3_segment_totals, m3_state_fold, m3_scan_fwd); the per-rank phases are plain
functions so that one process can also drive every rank in turn.

The backward of the split needs one more exchange.  The adjoint of segment r's
end state is dG_end(r) = d_final for the last segment, else
dG_end(r) = exp(Lam_{r+1}) Rot(-Phi_{r+1}) dG_end(r+1) + D_{r+1}, the transpose
of segment r+1's state transition applied to its own end adjoint plus D_{r+1},
the adjoint that segment r+1's outputs send to its incoming state (the dh0 of
its backward with no final-state gradient).  So each rank computes D_r, the
ranks all-gather them, each folds the later segments' (D, Lam, -Phi) into its
end adjoint with the forward's fold, and runs its backward from it; the
gradients of a segment's first-token left endpoint (its B_prev, x_prev: the
previous segment's last token) go back to the previous rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, stop) share of n independent items for `rank`; the
    first n % world ranks take one extra item."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """Maximum of a per-rank scalar over the default process group (the value
    itself when no group is initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def batch_shard(tensors: dict, world: int, rank: int) -> dict:
    """This rank's contiguous share (shard_range over dim 0) of every batched
    tensor of a layer call; None entries pass through."""
    n = next(v.shape[0] for v in tensors.values() if v is not None)
    a, b = shard_range(n, world, rank)
    return {k: (None if v is None else v[a:b]) for k, v in tensors.items()}


def batch_gather(local: torch.Tensor, n: int, group=None) -> torch.Tensor:
    """Assemble the ranks' batch shards (in rank order, as batch_shard cut
    them) into the whole batch of n rows on every rank.  Not part of the
    layer's data path, which needs no exchange; a caller that wants one rank
    to hold every output uses it after the step."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    rows = max(b - a for a, b in (shard_range(n, world, r) for r in range(world)))
    a, b = shard_range(n, world, rank)
    if local.shape[0] != b - a:
        raise ValueError(f"rank {rank} holds {local.shape[0]} rows, its share is {b - a}")
    pad = local.new_zeros((rows,) + tuple(local.shape[1:]))
    pad[: b - a] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([parts[r][: e - s] for r, (s, e) in
                      enumerate(shard_range(n, world, r) for r in range(world))])


# ---- sequence split across ranks (context parallel) ---------------------------

class M3Ops:
    """The library's calls for the per-rank steps of the sequence split."""

    def scan_state(self, x, dt, A, lam, theta, B, C, chunk, B_prev, x_prev):
        from . import m3
        return m3.m3_scan_state(x, dt, A, lam, theta, B, C, chunk, None, B_prev, x_prev)

    def segment_totals(self, x, dt, A, theta, B, chunk):
        from . import m3
        return m3.m3_segment_totals(x, dt, A, theta, B, chunk)

    def state_fold(self, h0, T, lam_tot, phi_tot):
        from . import m3
        return m3.m3_state_fold(h0, T, lam_tot, phi_tot)

    def scan_fwd(self, x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev):
        from . import m3
        return m3.m3_scan_fwd(x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev)

    def scan_bwd(self, x, dt, A, lam, theta, B, C, chunk, h0, B_prev, x_prev, dy, d_final):
        """Gradient dict of m3_scan_bwd (keys x, dt, A, lam, theta, B, C, h0 and,
        with a previous token, B_prev, x_prev)."""
        from . import m3
        return m3.m3_scan_bwd(x, dt, A, lam, theta, B, C, dy, chunk, h0, B_prev, x_prev, d_final)


def seq_boundary(x: torch.Tensor, B: torch.Tensor):
    """This segment's last token: (B [b][G][R][N], x [b][H][R][P]), the next
    segment's left endpoint."""
    return B[:, -1].contiguous(), x[:, -1].contiguous()


def seq_summary(ops, x, dt, A, lam, theta, B, C, chunk, B_prev, x_prev):
    """(T, lam_tot, phi_tot) of this segment: its end state from a zero start
    (its own left endpoint included) and its log-decay and angle totals."""
    T = ops.scan_state(x, dt, A, lam, theta, B, C, chunk, B_prev, x_prev)
    lam_tot, phi_tot = ops.segment_totals(x, dt, A, theta, B, chunk)
    return T, lam_tot, phi_tot


def seq_finish(ops, rank, x, dt, A, lam, theta, B, C, chunk, h0, Ts, lams, phis, B_prev, x_prev):
    """Fold segments 0..rank-1 into this segment's incoming state (from the
    sequence's h0) and scan the segment from it.  Returns (y, end state)."""
    if rank == 0:
        h_in = h0
    else:
        h_in = ops.state_fold(h0, torch.stack(Ts[:rank]), torch.stack(lams[:rank]),
                              torch.stack(phis[:rank]))
    return ops.scan_fwd(x, dt, A, lam, theta, B, C, chunk, h_in, B_prev, x_prev)


def _all_gather(t: torch.Tensor, group=None) -> list[torch.Tensor]:
    t = t.contiguous()
    out = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, t, group=group)
    return out


def seq_parallel_scan(x, dt, A, lam, theta, B, C, chunk=64, h0=None, B_prev=None, x_prev=None,
                      *, group=None, ops=None):
    """The scan of sequences split across the ranks of `group` in token order:
    rank r holds tokens [r*Ls, (r+1)*Ls) of every sequence (the same Ls on
    every rank).  h0 is the sequences' initial state and B_prev / x_prev their
    previous token: pass the same values (or None) on every rank; only rank 0
    uses them.  Returns this rank's (y, end state of its segment); the last
    rank's end state is the sequences' final state."""
    ops = ops or M3Ops()
    r = dist.get_rank(group)
    B_last, x_last = seq_boundary(x, B)
    gB, gx = _all_gather(B_last, group), _all_gather(x_last, group)
    Bp, xp = (B_prev, x_prev) if r == 0 else (gB[r - 1], gx[r - 1])
    T, lam_tot, phi_tot = seq_summary(ops, x, dt, A, lam, theta, B, C, chunk, Bp, xp)
    Ts, lams, phis = _all_gather(T, group), _all_gather(lam_tot, group), _all_gather(phi_tot, group)
    return seq_finish(ops, r, x, dt, A, lam, theta, B, C, chunk, h0, Ts, lams, phis, Bp, xp)


# ---- backward of the sequence split --------------------------------------------

def seq_incoming_state(ops, rank, h0, Ts, lams, phis):
    """The state entering segment `rank`: segments 0..rank-1 folded from h0."""
    if rank == 0:
        return h0
    return ops.state_fold(h0, torch.stack(Ts[:rank]), torch.stack(lams[:rank]),
                          torch.stack(phis[:rank]))


def seq_end_adjoint(ops, rank, world, d_final, Ds, lams, phis):
    """The adjoint of segment `rank`'s end state: d_final (None: zero) carried
    back through segments world-1 .. rank+1, each step
    d <- exp(Lam_s) Rot(-Phi_s) d + D_s (the forward's fold with the angles
    negated).  Returns None for a zero adjoint."""
    later = list(range(world - 1, rank, -1))
    if not later:
        return d_final
    return ops.state_fold(d_final, torch.stack([Ds[s] for s in later]),
                          torch.stack([lams[s] for s in later]),
                          torch.stack([-phis[s] for s in later]))


def seq_parallel_scan_bwd(x, dt, A, lam, theta, B, C, dy, chunk=64, h0=None, B_prev=None,
                          x_prev=None, d_final=None, *, group=None, ops=None):
    """Gradients of the split scan (the layout of seq_parallel_scan): this
    rank's dy [b][Ls][H][R][P]; d_final, h0, B_prev, x_prev the same on every
    rank (only the last rank uses d_final, only rank 0 h0 and the previous
    token).  The forward's exchange is repeated to get each segment's incoming
    state.  Returns this rank's gradient dict: x, dt, A, lam, theta, B, C of
    its segment (its last token's B and x including the next segment's
    left-endpoint terms), "h_in" (the adjoint of its incoming state: the
    sequences' dh0 on rank 0) and, on rank 0 with a previous token, B_prev and
    x_prev."""
    ops = ops or M3Ops()
    r, world = dist.get_rank(group), dist.get_world_size(group)
    B_last, x_last = seq_boundary(x, B)
    gB, gx = _all_gather(B_last, group), _all_gather(x_last, group)
    Bp, xp = (B_prev, x_prev) if r == 0 else (gB[r - 1], gx[r - 1])
    T, lam_tot, phi_tot = seq_summary(ops, x, dt, A, lam, theta, B, C, chunk, Bp, xp)
    Ts, lams, phis = _all_gather(T, group), _all_gather(lam_tot, group), _all_gather(phi_tot, group)
    h_in = seq_incoming_state(ops, r, h0, Ts, lams, phis)
    if h_in is None:
        h_in = torch.zeros_like(T)
    D = ops.scan_bwd(x, dt, A, lam, theta, B, C, chunk, h_in, Bp, xp, dy, None)["h0"]
    Ds = _all_gather(D, group)
    d_end = seq_end_adjoint(ops, r, world, d_final, Ds, lams, phis)
    g = ops.scan_bwd(x, dt, A, lam, theta, B, C, chunk, h_in, Bp, xp, dy, d_end)
    # the next segment's first token used this segment's last B and x
    zB = torch.zeros_like(B_last, dtype=g["B"].dtype)
    zx = torch.zeros_like(x_last, dtype=g["x"].dtype)
    gBp = _all_gather(g["B_prev"] if Bp is not None else zB, group)
    gxp = _all_gather(g["x_prev"] if Bp is not None else zx, group)
    out = {k: g[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C")}
    if r + 1 < world:
        out["B"] = out["B"].clone()
        out["x"] = out["x"].clone()
        out["B"][:, -1] += gBp[r + 1]
        out["x"][:, -1] += gxp[r + 1]
    out["h_in"] = g["h0"]
    if r == 0 and B_prev is not None:
        out["B_prev"], out["x_prev"] = g["B_prev"], g["x_prev"]
    return out
