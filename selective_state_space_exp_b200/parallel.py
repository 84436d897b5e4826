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
