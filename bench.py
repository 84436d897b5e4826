"""Benchmark of the Mamba-3 SSM layer on B200: prefill tokens/s (headline: the
MIMO rank-4 layer, b = 8, L = 2048, H = 64, P = 64, N = 128, chunk 64) and, as
lines of their own, the SISO layer, the long-context MIMO layer at L = 32768
and 16384, and decode tokens/s at rank 1 and rank 4 (b = 128, 1024 consecutive
steps), each with its roofline fraction and the fp64 CPU oracle timed on a
bounded sample as a baseline; an end-to-end number through host buffers for
the headline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl m3|reference]

One step = one m3_scan_fwd over the workload's whole batch (all chunks,
heads and sequences) with inputs already resident in HBM.  Under torchrun each
rank runs its own batch (weak scaling, no collective on the data path); the
reported value is all ranks' tokens over the slowest rank's device time.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_exp_b200 import inputs as I  # noqa: E402
from selective_state_space_exp_b200 import m3  # noqa: E402
from selective_state_space_exp_b200.parallel import max_over_ranks as _max_ranks  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "siso_prefill": I.SISO_PREFILL,
    "mimo_prefill": I.MIMO_PREFILL,
    "long_mimo_16k": I.LONG_MIMO_16K,
    "long_mimo_32k": I.LONG_MIMO_32K,
}
DECODE = {"decode_siso": I.DECODE_SISO, "decode_mimo": I.DECODE_MIMO}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---- algorithmic work (FLOPs at chunk Q with the causal count, bytes read
# once + written once) -----------------------------------------------------

def prefill_work(s: I.Shape):
    """Algorithmic FLOPs and bytes of one scan.

    Per chunk-head with M = Q*R rows: S = C~ B~^T over the causal (t >= s)
    token blocks, K = N; (M o S) X, K = Q*R, N = P; chunk state B~^T X (N x P,
    K = Q*R); chunk output C~ h (Q*R x P, K = N).  Causal token-block count:
    Q(Q+1)/2 * R^2 entries."""
    Q, R, N, P = s.chunk, s.rank, s.dstate, s.headdim
    nc = math.ceil(s.seqlen / Q)
    causal = Q * (Q + 1) // 2 * R * R
    per_ch = 2 * causal * N + 2 * causal * P + 2 * (Q * R) * N * P + 2 * (Q * R) * N * P
    flops = per_ch * nc * s.batch * s.nheads
    io = 2 if s.io == "bf16" else 4
    tok = s.batch * s.seqlen
    byt = (2 * tok * s.nheads * R * P * io                 # x in, y out
           + 2 * tok * s.ngroups * R * N * io              # B, C
           + 3 * tok * s.nheads * 4                        # dt, A, lam
           + tok * s.ngroups * (N // 2) * 4                # theta
           + s.batch * s.nheads * N * P * 4)               # final state
    return float(flops), float(byt)


def varlen_work(s: I.Shape, lengths):
    """Algorithmic FLOPs and bytes of a packed batch: the sum over its
    sequences of one-sequence scans (each sequence's last chunk counted like a
    whole causal chunk, as for a ragged batch row)."""
    f = b = 0.0
    for n in lengths:
        fi, bi = prefill_work(dataclasses.replace(s, batch=1, seqlen=int(n)))
        f, b = f + fi, b + bi
    return f, b


VARLEN_SEQS = 16   # sequences in the packed-batch line: the length mix of
VARLEN_MAX = 2048  # inputs.varlen_lengths (edges 0, 1, Q-1, Q, Q+1, max; rest uniform)


def time_varlen(inp, s, max_len, steps, warmup, flush):
    shape = m3.make_shape(len(inp["cu_seqlens"]) - 1, max_len, s.nheads, s.ngroups, s.headdim,
                          s.dstate, s.rank, s.chunk, inp["x"].dtype)
    ws = torch.empty(max(m3.workspace_size(shape), 1), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(inp["x"])
    fs = torch.empty((len(inp["cu_seqlens"]) - 1, s.nheads, s.dstate, s.headdim),
                     dtype=torch.float32, device="cuda")

    def step():
        m3.m3_scan_fwd_varlen(inp["cu_seqlens"], inp["x"], inp["dt"], inp["A"], inp["lam"],
                              inp["theta"], inp["B"], inp["C"], s.chunk, max_seqlen=max_len,
                              y=y, final_state=fs, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    st = m3.m3_stream_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    return [a.elapsed_time(b) * 1e-3 for a, b in ev]


def varlen_line(s, rank, world, steps, warmup, flush, peaks, psrc):
    """The packed variable-length batch of the workload's layer shape."""
    lengths = I.varlen_lengths(VARLEN_SEQS, VARLEN_MAX, s.chunk, seed=1021)
    inp = I.make_varlen_inputs(I.Workload(s), lengths, seed=1021 + 7919 * rank, device="cuda")
    barrier(world)
    t = max_over_ranks(sum(time_varlen(inp, s, VARLEN_MAX, steps, warmup, flush)),
                       world) / steps
    f, b = varlen_work(s, lengths)
    return {"workload": f"packed batch of {len(lengths)} sequences, lengths 0..{VARLEN_MAX} "
                        f"({sum(lengths)} tokens), layer shape as the main line",
            "value": round(world * sum(lengths) / t, 1), "unit": "tokens/s",
            "ms_per_step": round(t * 1e3, 4), "lengths": lengths,
            "roofline": roofline(f, b, t, peaks, psrc)}


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
# (the nominal unit count and maximum SM clock; nothing here measures it)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_tc(s: I.Shape) -> bool:
    """Whether m3_scan_bwd runs on the tensor cores (bf16 io at N = 128, P = 64)."""
    return s.io == "bf16" and s.dstate == 128 and s.headdim == 64


def bwd_rows(s: I.Shape, simt=False):
    """Rows per chunk the backward picks (the library's rule: 64 on the
    tensor cores, else 32 rows, two CTAs per SM)."""
    return 64 if bwd_tc(s) and not simt else 32


def bwd_work(s: I.Shape, simt=False):
    """Algorithmic FLOPs and bytes of one m3_scan_bwd.

    Per chunk-head of the backward's chunking (M = Qb * R rows, causal token
    blocks Qb(Qb+1)/2 * R^2): the score and dY X^T products (2 * causal * (N + P)),
    dCt and dBt (2 * causal * N each), dX (2 * causal * P), and five N x P x M
    state products (the forward chunk state it recomputes, D_c, dY G^T,
    dGhat x, dGhat^T Bt): 10 * M * N * P.  Bytes: every input and dy read
    once, every gradient (fp32) and the final-state adjoint written once."""
    R, N, P = s.rank, s.dstate, s.headdim
    M = bwd_rows(s, simt)
    Qb = M // R
    causal = Qb * (Qb + 1) // 2 * R * R
    nc = math.ceil(s.seqlen / Qb)
    flops = (causal * (2 * (N + P) + 4 * N + 2 * P) + 10 * M * N * P) * nc * s.batch * s.nheads
    io = 2 if s.io == "bf16" else 4
    tok = s.batch * s.seqlen
    byt = (3 * tok * s.nheads * R * P * io                 # x, dy in; (y is not read)
           + tok * s.nheads * R * P * 4 - tok * s.nheads * R * P * io  # dx out (fp32)
           + 2 * tok * s.ngroups * R * N * (io + 4)        # B, C in; dB, dC out
           + 3 * tok * s.nheads * 4 * 2                    # dt, A, lam in; their grads out
           + tok * s.ngroups * (N // 2) * 4 * 2            # theta in, dtheta out
           + 2 * s.batch * s.nheads * N * P * 4)           # d_final in, dh0 out
    return float(flops), float(byt)


def alu_roofline(flops, byt, seconds, peaks):
    t_alu = flops / (FP32_ALU_TFLOPS * 1e12)
    t_hbm = byt / (peaks["hbm_gbs"] * 1e9)
    if t_alu >= t_hbm:
        ach = flops / seconds / 1e12
        return {"bound": "alu", "achieved": round(ach, 2), "peak": round(FP32_ALU_TFLOPS, 1),
                "unit": "TFLOP/s", "frac": round(ach / FP32_ALU_TFLOPS, 4),
                "roofline_time_us": round(t_alu * 1e6, 2),
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 x 1.965 GHz (nominal)"}
    ach = byt / seconds / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "roofline_time_us": round(t_hbm * 1e6, 2)}


def time_bwd(inp, s, steps, warmup, flush, simt=False):
    gen = torch.Generator(device="cuda").manual_seed(77)
    dy = torch.randn(inp["x"].shape, generator=gen, device="cuda").to(inp["x"].dtype)
    dfin = torch.randn((s.batch, s.nheads, s.dstate, s.headdim), generator=gen, device="cuda")
    ws = torch.empty(max(m3.bwd_workspace_size(m3.scan_shape(inp["x"], inp["B"], s.chunk, simt)),
                         1),
                     dtype=torch.uint8, device="cuda")

    def step():
        m3.m3_scan_bwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                       inp["C"], dy, s.chunk, d_final=dfin, workspace=ws, simt=simt)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    st = m3.m3_stream_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    return [a.elapsed_time(b) * 1e-3 for a, b in ev]


def bwd_line(inp, s, world, steps, warmup, flush, peaks, psrc, simt=False):
    barrier(world)
    t = max_over_ranks(sum(time_bwd(inp, s, steps, warmup, flush, simt)), world) / steps
    f, b = bwd_work(s, simt)
    line = {"metric": "backward tokens/s", "value": round(world * s.batch * s.seqlen / t, 1),
            "unit": "tokens/s", "ms_per_step": round(t * 1e3, 4)}
    if bwd_tc(s) and not simt:
        line["path"] = ("m3_scan_bwd: 3 launches (per-chunk sums and per-chunk gradients on the "
                        "tensor cores, tcgen05 bf16 operands, fp32 accumulators; both state "
                        f"passes on the CUDA cores), chunks of {bwd_rows(s)} rows")
        line["roofline"] = roofline(f, b, t, peaks, psrc)
    else:
        line["path"] = ("m3_scan_bwd: 3 launches (per-chunk sums, both state passes, "
                        "per-chunk gradients), CUDA cores fp32")
        line["roofline"] = alu_roofline(f, b, t, peaks)
    return line


def prep_line(s, world, steps, warmup, flush, peaks, psrc):
    """m3_bc_prep (QK-norm + scale + bias of B and C) on the layer's tokens
    with B and C per head (G = H): HBM-bound, every raw value read once and
    every output written once."""
    G, R, N = s.nheads, s.rank, s.dstate
    gen = torch.Generator(device="cuda").manual_seed(1031)
    shp = (s.batch, s.seqlen, G, R, N)
    Br = torch.randn(shp, generator=gen, device="cuda").to(torch.bfloat16)
    Cr = torch.randn(shp, generator=gen, device="cuda").to(torch.bfloat16)
    prm = [torch.randn((G, R, N), generator=gen, device="cuda") for _ in range(4)]
    Bo, Co = torch.empty_like(Br), torch.empty_like(Cr)

    def step():
        m3.m3_bc_prep(Br, Cr, *prm, B=Bo, C=Co)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    if m3.m3_stream_status() != 0:
        raise RuntimeError("device status")
    barrier(world)
    t = max_over_ranks(sum(a.elapsed_time(b) * 1e-3 for a, b in ev), world) / steps
    byt = 4.0 * Br.numel() * 2 + 4 * G * R * N * 4
    return {"workload": f"B and C per head: [{s.batch}][{s.seqlen}][{G}][{R}][{N}] bf16 each",
            "value": round(world * s.batch * s.seqlen / t, 1), "unit": "tokens/s",
            "us_per_step": round(t * 1e6, 2),
            "roofline": roofline(0.0, byt, t, peaks, psrc)}


def time_calls(fn, steps, warmup, flush):
    """Mean device time of fn() over `steps` calls (CUDA events on the current
    stream, L2 flushed before each timed call)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        fn()
        ev[i][1].record()
    torch.cuda.synchronize()
    if m3.m3_stream_status() != 0:
        raise RuntimeError("device status")
    return sum(a.elapsed_time(b) * 1e-3 for a, b in ev) / steps


def block_line(world, steps, warmup, flush, peaks, psrc):
    """The block projections around the layer at the 1.5B-scale width
    (D = 2048, H * P = 4096, G * N / 2 = 64 angle rates) on the SISO workload's
    16384 tokens: the gate projection z = u W_z (m3_linear, tcgen05), the angle
    projection theta = u W_theta (fp32 out), and the rank-4 MIMO up- and
    down-projections with the output gate (HBM-bound)."""
    T, D, HP, NTH, H, P, R = 8 * 2048, 2048, 4096, 64, 64, 64, 4
    gen = torch.Generator(device="cuda").manual_seed(1041)
    u = torch.randn((T, D), generator=gen, device="cuda").to(torch.bfloat16)
    Wz = (torch.randn((HP, D), generator=gen, device="cuda") / D ** 0.5).to(torch.bfloat16)
    Wt = (torch.randn((NTH, D), generator=gen, device="cuda") / D ** 0.5).to(torch.bfloat16)
    z = torch.empty((T, HP), dtype=torch.bfloat16, device="cuda")
    th = torch.empty((T, NTH), dtype=torch.float32, device="cuda")
    x = torch.randn((T, H, P), generator=gen, device="cuda").to(torch.bfloat16)
    w_up = torch.randn((H, R, P), generator=gen, device="cuda")
    w_dn = torch.randn((H, R, P), generator=gen, device="cuda")
    X = torch.empty((T, H, R, P), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((T, H, P), dtype=torch.bfloat16, device="cuda")
    zz = z.view(T, H, P)
    t_z = time_calls(lambda: m3.m3_linear(u, Wz, out=z), steps, warmup, flush)
    t_t = time_calls(lambda: m3.m3_linear(u, Wt, out=th), steps, warmup, flush)
    t_u = time_calls(lambda: m3.m3_mimo_up(x, w_up, X=X), steps, warmup, flush)
    t_d = time_calls(lambda: m3.m3_mimo_down_gate(X, w_dn, zz, out=out), steps, warmup, flush)
    barrier(world)
    t_z, t_t, t_u, t_d = (max_over_ranks(v, world) for v in (t_z, t_t, t_u, t_d))
    fz, bz = 2.0 * T * HP * D, 2.0 * (T * D + HP * D + T * HP)
    ft, bt = 2.0 * T * NTH * D, 2.0 * (T * D + NTH * D) + 4.0 * T * NTH
    bu = 2.0 * T * H * P * (1 + R) + 4.0 * H * R * P
    bd = 2.0 * T * H * P * (R + 2) + 4.0 * H * R * P
    return {
        "workload": f"{T} tokens, D = {D}, H * P = {HP}, angle rates {NTH}, rank {R}, bf16",
        "gate_projection": {"kernel": "gemm_tc_kernel (tcgen05, 128 x 256 tiles)",
                            "us_per_call": round(t_z * 1e6, 2),
                            "roofline": roofline(fz, bz, t_z, peaks, psrc)},
        "angle_projection": {"kernel": "gemm_tc_kernel (tcgen05, 128 x 64 tiles), fp32 out",
                             "us_per_call": round(t_t * 1e6, 2),
                             "roofline": roofline(ft, bt, t_t, peaks, psrc)},
        "mimo_up": {"us_per_call": round(t_u * 1e6, 2),
                    "roofline": roofline(0.0, bu, t_u, peaks, psrc)},
        "mimo_down_gate": {"us_per_call": round(t_d * 1e6, 2),
                           "roofline": roofline(0.0, bd, t_d, peaks, psrc)},
    }


def decode_work(s: I.Shape):
    R, N, P = s.rank, s.dstate, s.headdim
    bh = s.batch * s.nheads
    io = 2 if s.io == "bf16" else 4
    flops = bh * N * P * (6 * R + 4)
    byt = (2 * bh * N * P * 4 + 3 * bh * R * P * io + 3 * s.batch * s.ngroups * R * N * io
           + 3 * bh * 4 + s.batch * s.ngroups * (N // 2) * 4)
    return float(flops), float(byt)


def profile_traffic(summary: str, key: str = "traffic_bytes_per_launch"):
    """DRAM bytes per launch recorded in a committed ncu summary under profiles/,
    or None when the kernel's sources changed since the counters were taken
    (the summary names its source files and their combined sha256)."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith(("|", " ", "#")):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    try:
        h = hashlib.sha256()
        for rel in fields["source_files"].split():
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != fields["source_sha256"]:
            return None
        return int(fields[key])
    except (KeyError, OSError, ValueError):
        return None


def roofline(flops, byt, seconds, peaks, src, sustained=False):
    tf = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_tensor = flops / (tf * 1e12)
    t_hbm = byt / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / seconds / 1e12
        ts = peaks.get("bf16_tflops_sustained")
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": tf, "unit": "TFLOP/s",
                "frac": round(ach / tf, 4), "roofline_time_us": round(t_tensor * 1e6, 2),
                "peak_source": f"{src} bf16 {'sustained' if sustained else 'burst'}",
                "frac_of_sustained": round(ach / ts, 4) if ts and not sustained else None}
    ach = byt / seconds / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "roofline_time_us": round(t_hbm * 1e6, 2),
            "peak_source": f"{src} HBM copy"}


# ---- clocks ---------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- distributed plumbing --------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    return _max_ranks(v, device="cuda") if world > 1 else v


# ---- device timing ---------------------------------------------------------

L2_FLUSH_BYTES = 256 << 20


def time_prefill(inp, s, steps, warmup, flush):
    ws = torch.empty(max(m3.workspace_size(m3.scan_shape(inp["x"], inp["B"], s.chunk)), 1),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty_like(inp["x"])
    fs = torch.empty((s.batch, s.nheads, s.dstate, s.headdim), dtype=torch.float32,
                     device="cuda")

    def step():
        m3.m3_scan_fwd(inp["x"], inp["dt"], inp["A"], inp["lam"], inp["theta"], inp["B"],
                       inp["C"], s.chunk, y=y, final_state=fs, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    st = m3.m3_stream_status()
    if st != 0:
        raise RuntimeError(f"device status {st}")
    return [a.elapsed_time(b) * 1e-3 for a, b in ev]


def time_decode(dec, s, steps, warmup):
    state = dec["state0"].clone()
    y = torch.empty_like(dec["x"][0])

    def step(t):
        Bp = dec["B_prev"] if t == 0 else dec["B"][t - 1]
        xp = dec["x_prev"] if t == 0 else dec["x"][t - 1]
        m3.m3_decode_step(state, dec["x"][t], dec["dt"][t], dec["A"][t], dec["lam"][t],
                          dec["theta"][t], dec["B"][t], dec["C"][t], Bp, xp, y=y)

    for t in range(warmup):
        step(t)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for t in range(warmup, warmup + steps):
        step(t)
    b.record()
    torch.cuda.synchronize()
    if m3.m3_stream_status() != 0:
        raise RuntimeError("device status")
    return a.elapsed_time(b) * 1e-3


def time_e2e_prefill(inp_host, s, steps):
    """Through host buffers: every step copies its inputs from pinned host
    memory to the device, runs the scan, and copies y and the final state back
    to pinned host memory.  Steps are pipelined as a serving loop would run
    them: copies in on one stream, the scan on a second, copies out on a
    third, two device / host buffer sets, events ordering every reuse, so step
    i's copy out overlaps step i+1's copy in and scan (PCIe is full duplex).
    Timed with CUDA events from the first copy in to the last copy out."""
    names = ("x", "dt", "A", "lam", "theta", "B", "C")
    nb = 2
    pin = {k: inp_host[k].pin_memory() for k in names}
    dev = [{k: torch.empty_like(pin[k], device="cuda") for k in names} for _ in range(nb)]
    ys = [torch.empty(pin["x"].shape, dtype=pin["x"].dtype, device="cuda") for _ in range(nb)]
    fss = [torch.empty((s.batch, s.nheads, s.dstate, s.headdim), dtype=torch.float32,
                       device="cuda") for _ in range(nb)]
    y_h = [torch.empty(pin["x"].shape, dtype=pin["x"].dtype).pin_memory() for _ in range(nb)]
    fs_h = [torch.empty(fss[0].shape, dtype=torch.float32).pin_memory() for _ in range(nb)]
    ws = torch.empty(max(m3.workspace_size(m3.scan_shape(dev[0]["x"], dev[0]["B"], s.chunk)), 1),
                     dtype=torch.uint8, device="cuda")
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = y_h[0].numel() * y_h[0].element_size() + fs_h[0].numel() * 4
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        done_cmp, done_out = [None] * nb, [None] * nb
        for i in range(n):
            j = i % nb
            e_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if done_cmp[j] is not None:  # the scan that read buffer j is done
                    s_in.wait_event(done_cmp[j])
                for k in names:
                    dev[j][k].copy_(pin[k], non_blocking=True)
                e_in.record(s_in)
            e_c = torch.cuda.Event()
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in)
                if done_out[j] is not None:  # y / final state of buffer j copied out
                    s_cmp.wait_event(done_out[j])
                m3.m3_scan_fwd(dev[j]["x"], dev[j]["dt"], dev[j]["A"], dev[j]["lam"],
                               dev[j]["theta"], dev[j]["B"], dev[j]["C"], s.chunk, y=ys[j],
                               final_state=fss[j], workspace=ws, stream=s_cmp)
                e_c.record(s_cmp)
            done_cmp[j] = e_c
            e_o = torch.cuda.Event()
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                y_h[j].copy_(ys[j], non_blocking=True)
                fs_h[j].copy_(fss[j], non_blocking=True)
                e_o.record(s_out)
            done_out[j] = e_o

    run(2)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    run(steps)
    b.record(s_out)
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e-3 / steps, h2d, d2h


# ---- CPU oracle baseline ----------------------------------------------------

def cpu_oracle_prefill(inp_host, s, budget_s=10.0, single_thread=False):
    """Time the oracle (as it stands) on whole (batch, head) chains of the same
    workload until about `budget_s` seconds of CPU work; tokens/s counts the
    tokens those chains cover (chains / nheads * seqlen).  With single_thread,
    also the same oracle on one thread on a smaller sample."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    total = s.batch * s.nheads
    done, elapsed = 0, 0.0
    step = max(cores, 1)
    while done < total and elapsed < budget_s:
        chains = list(range(done, min(done + step, total)))
        t0 = time.perf_counter()
        oracle.scan(inp_host["x"], inp_host["dt"], inp_host["A"], inp_host["lam"],
                    inp_host["theta"], inp_host["B"], inp_host["C"], chains=chains,
                    nthreads=cores)
        elapsed += time.perf_counter() - t0
        done += len(chains)
    tokens = done / s.nheads * s.seqlen
    res = {"value": round(tokens / elapsed, 1), "unit": "tokens/s", "cores": cores,
           "kind": "oracle",
           "sample": f"{done} of {total} (batch, head) chains, all {s.seqlen} tokens each, "
                     f"{elapsed:.1f} s on {cores} threads"}
    if not single_thread:
        return res
    # the same oracle on one thread, on a smaller sample of the same chains
    one = min(max(1, done // max(cores, 1)), total)
    t0 = time.perf_counter()
    oracle.scan(inp_host["x"], inp_host["dt"], inp_host["A"], inp_host["lam"],
                inp_host["theta"], inp_host["B"], inp_host["C"], chains=list(range(one)),
                nthreads=1)
    t1 = time.perf_counter() - t0
    res["single_thread"] = {"value": round(one / s.nheads * s.seqlen / t1, 1),
                            "unit": "tokens/s", "cores": 1, "sample": f"{one} chains, {t1:.1f} s"}
    return res


DECODE_CPU_STEPS = 64


def cpu_oracle_decode(dec, s, budget_s=10.0, steps=DECODE_CPU_STEPS):
    """The oracle's decode driver (m3o_decode_step as it stands, one thread) on
    the first `steps` decode steps of whole batch rows (every head), one row
    after another until about `budget_s` seconds.  tokens/s = rows x steps /
    time.  A step's cost does not depend on its index, so this is also the
    rate of the full 1024-step run: the figure is extrapolated from the first
    `steps` steps, and the sample says so."""
    import oracle
    rows, elapsed = 0, 0.0
    host = {k: v.cpu() for k, v in dec.items()}
    while rows < s.batch and elapsed < budget_s:
        i = rows
        st = host["state0"][i:i + 1].double().numpy()
        t0 = time.perf_counter()
        for t in range(steps):
            Bp = host["B_prev"][i:i + 1] if t == 0 else host["B"][t - 1, i:i + 1]
            xp = host["x_prev"][i:i + 1] if t == 0 else host["x"][t - 1, i:i + 1]
            _, st = oracle.decode_step(st, host["x"][t, i:i + 1], host["dt"][t, i:i + 1],
                                       host["A"][t, i:i + 1], host["lam"][t, i:i + 1],
                                       host["theta"][t, i:i + 1], host["B"][t, i:i + 1],
                                       host["C"][t, i:i + 1], Bp, xp)
        elapsed += time.perf_counter() - t0
        rows += 1
    return {"value": round(rows * steps / elapsed, 1), "unit": "tokens/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{rows} of {s.batch} sequences (all {s.nheads} heads), the first "
                      f"{steps} of the workload's steps, {elapsed:.1f} s on one thread; "
                      f"tokens/s extrapolated to the full run (constant cost per step)"}


# ---- one bench line per workload ---------------------------------------------

SEEDS = {"siso_prefill": 1001, "mimo_prefill": 1002, "long_mimo_32k": 1004,
         "long_mimo_16k": 1014, "decode_r1": 1003, "decode_r4": 1013}
PROFILE = {"siso_prefill": "tc_scan_kernel_siso_prefill.md",
           "mimo_prefill": "tc_scan_kernel_mimo_prefill.md"}


def prefill_traffic(name, plan):
    """DRAM bytes per launch of the scan kernel's full pass from its committed
    ncu summary, and where it came from: one-launch calls, and calls that cut
    only a last wave's chains in two (their full pass covers every token once;
    its state-only and combine launches are not counted)."""
    summary = PROFILE.get(name)
    if not summary or not plan["tensor_core"] or plan["segments"] > 2:
        return None, None
    t = profile_traffic(summary)
    return t, (f"profiles/{summary}" if t is not None else None)


def prefill_line(name, rank, world, steps, warmup, flush, peaks, psrc, cpu=True):
    """Device throughput of m3_scan_fwd on one workload (inputs resident in HBM,
    L2 flushed between timed steps), its roofline and the oracle baseline.
    Returns (line, device inputs)."""
    w = WORKLOADS[name]
    s = w.shape
    inp = I.make_scan_inputs(w, seed=SEEDS[name] + 7919 * rank, device="cuda")
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = time_prefill(inp, s, steps, warmup, flush)
    barrier(world)
    per_step = max_over_ranks(sum(times), world) / steps
    flops, byt = prefill_work(s)
    plan = m3.scan_plan(m3.scan_shape(inp["x"], inp["B"], s.chunk))
    kern = "tc_scan_kernel (tcgen05)" if plan["tensor_core"] else "CUDA-core scan kernels"
    traffic, traffic_src = prefill_traffic(name, plan)
    line = {
        "metric": "prefill tokens/s",
        "value": round(world * s.batch * s.seqlen / per_step, 1),
        "unit": "tokens/s", "steps": steps, "warmup": warmup,
        "ms_per_step": round(per_step * 1e3, 4),
        "config": {"workload": name, **shape_cfg(s),
                   "l2": "flushed between timed steps (256 MiB write)",
                   "path": f"{kern}, {plan['launches']} launch(es) per call, "
                           f"at most {plan['segments']} segment(s) per sequence"},
        "roofline": {**roofline(flops, byt, per_step, peaks, psrc),
                     "scope": ("the one kernel launch of each m3_scan_fwd call, CUDA events on "
                               "the launching stream" if plan["launches"] == 1 else
                               "whole m3_scan_fwd call (all its launches), CUDA events on the "
                               "launching stream"),
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_flops": flops, "algorithmic_bytes": byt},
        "gpu_launches": steps * plan["launches"],
        "clocks": clk.summary(),
    }
    if cpu and rank == 0 and world == 1:
        host = {k: v.cpu() for k, v in inp.items()}
        line["cpu_baseline"] = cpu_oracle_prefill(host, s)
    return line, inp


def decode_line(name, rank, world, dsteps, warmup, peaks, psrc, cpu=True):
    """1024 consecutive decode steps (b = 128, H = 64), state updated in place."""
    dw = I.DECODE_SISO if name == "decode_r1" else I.DECODE_MIMO
    ds = dw.shape
    dec = I.make_decode_inputs(dw, seed=SEEDS[name] + 7919 * rank, steps=dsteps + warmup,
                               device="cuda")
    barrier(world)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t = time_decode(dec, ds, dsteps, warmup)
    dt_total = max_over_ranks(t, world)
    dflops, dbyt = decode_work(ds)
    dkey = "traffic_bytes_per_launch_r1" if ds.rank == 1 else "traffic_bytes_per_launch_r4"
    dtraffic = profile_traffic("decode_kernels_b128_h64_n128_p64.md", dkey)
    line = {
        "metric": "decode tokens/s", "value": round(world * ds.batch * dsteps / dt_total, 1),
        "unit": "tokens/s", "steps": dsteps, "us_per_step": round(dt_total / dsteps * 1e6, 2),
        "config": {"workload": name, **shape_cfg(ds),
                   "l2": "not flushed: each step streams the 268 MB state, twice L2"},
        "roofline": {**roofline(dflops, dbyt, dt_total / dsteps, peaks, psrc),
                     "scope": "one m3_decode_step launch, averaged over the consecutive steps",
                     "traffic": dtraffic,
                     "traffic_source": ("profiles/decode_kernels_b128_h64_n128_p64.md"
                                        if dtraffic is not None else None)},
        "gpu_launches": dsteps,
        "clocks": clk.summary(),
    }
    if cpu and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_oracle_decode(dec, ds)
    return line


# ---- main -------------------------------------------------------------------

def run_reference(args, s, wname):
    """The reference arm: the fp64 CPU oracle on the host cores, same workload
    and metric, one bounded sample per step."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = I.make_scan_inputs(WORKLOADS[wname], seed=SEEDS[wname])
    vals = []
    budget = max(2.0, 120.0 / max(args.steps + args.warmup, 1))
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_prefill(inp, s, budget_s=budget, single_thread=False)
        if i >= args.warmup:
            vals.append(r)
    v = statistics.mean(r["value"] for r in vals)
    line = {"impl": "reference", "metric": "prefill tokens/s", "value": round(v, 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wname, **shape_cfg(s)},
            "cpu_baseline": {"value": round(v, 1), "unit": "tokens/s", "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": round(v, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def shape_cfg(s: I.Shape):
    return {"batch": s.batch, "seqlen": s.seqlen, "nheads": s.nheads, "headdim": s.headdim,
            "dstate": s.dstate, "rank": s.rank, "ngroups": s.ngroups, "chunk": s.chunk,
            "io": s.io}


HEADLINE = "mimo_prefill"
SUBLINES = ("siso_prefill", "long_mimo_32k", "long_mimo_16k")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="m3", choices=["m3", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1024,
                    help="consecutive decode steps timed (each with its own token's inputs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode", "varlen", "bwd", "prep", "block"],
                    default=None,
                    help="run one part only (for profiling); prints its own line")
    ap.add_argument("--batch", type=int, default=None,
                    help="with --only: override the workload's batch (small profiling cases)")
    ap.add_argument("--simt", action="store_true",
                    help="with --only bwd: the CUDA-core backward (profiling)")
    ap.add_argument("--chunk", type=int, default=None,
                    help="with --only: override the workload's chunk length")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    s = WORKLOADS[args.workload].shape
    if args.batch is not None or args.chunk is not None:
        if args.only is None:
            raise SystemExit("--batch and --chunk are for the --only profiling modes")
        if args.batch is not None:
            s = dataclasses.replace(s, batch=args.batch)
        if args.chunk is not None:
            s = dataclasses.replace(s, chunk=args.chunk)

    if args.impl == "reference":
        run_reference(args, s, args.workload)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    m3.load()
    world, rank, local = dist_setup(args.gpus)
    peaks, psrc = load_peaks()

    if args.only == "decode":
        dw = I.DECODE_MIMO if s.rank > 1 else I.DECODE_SISO
        if args.batch is not None:
            dw = dataclasses.replace(dw, shape=dataclasses.replace(dw.shape, batch=args.batch))
        dec = I.make_decode_inputs(dw, seed=1003, steps=args.decode_steps + args.warmup,
                                   device="cuda")
        t = time_decode(dec, dw.shape, args.decode_steps, args.warmup)
        dflops, dbyt = decode_work(dw.shape)
        print(json.dumps({"only": "decode", "us_per_step": round(t / args.decode_steps * 1e6, 2),
                          "roofline": roofline(dflops, dbyt, t / args.decode_steps, peaks, psrc)}))
        return
    if args.only == "prep":
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        print(json.dumps({"only": "prep", **prep_line(s, 1, args.steps, args.warmup, flush, peaks,
                                                      psrc)}))
        return
    if args.only == "block":
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        print(json.dumps({"only": "block", **block_line(1, args.steps, args.warmup, flush, peaks,
                                                        psrc)}))
        return
    if args.only == "bwd":
        inp = I.make_scan_inputs(I.Workload(s), seed=1001, device="cuda")
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        print(json.dumps({"only": "bwd", **bwd_line(inp, s, 1, args.steps, args.warmup, flush,
                                                    peaks, psrc, args.simt)}))
        return
    if args.only == "varlen":
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        line = varlen_line(s, 0, 1, args.steps, args.warmup, flush, peaks, psrc)
        print(json.dumps({"only": "varlen", **line}))
        return
    if args.only == "prefill":
        inp = I.make_scan_inputs(I.Workload(s), seed=1001, device="cuda")
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        times = time_prefill(inp, s, args.steps, args.warmup, flush)
        flops, byt = prefill_work(s)
        per = sum(times) / len(times)
        print(json.dumps({"only": "prefill", "ms_per_step": round(per * 1e3, 4),
                          "roofline": roofline(flops, byt, per, peaks, psrc)}))
        return

    cpu = not args.no_cpu_baseline
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    # the headline workload (inputs drawn on the device, seeded per rank)
    head, inp = prefill_line(args.workload, rank, world, args.steps, args.warmup, flush, peaks,
                             psrc, cpu=False)
    inp_host = {k: v.cpu() for k, v in inp.items()}
    del inp
    # end to end through host buffers (the same inputs, copied from pinned host memory)
    e2e_step, h2d, d2h = time_e2e_prefill(inp_host, s, max(3, args.steps // 4))
    e2e_step = max_over_ranks(e2e_step, world)
    tokens = s.batch * s.seqlen
    line = {
        "metric": "prefill tokens/s",
        "value": head["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": s.io, "data": "synthetic",
        "config": {**head["config"], "parallelism": f"dp{world} (independent batches per rank)"},
        "roofline": head["roofline"],
        "e2e": {"value": round(world * tokens / e2e_step, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_step * 1e3, 3),
                "mode": "pinned host buffers; copies in, scan, copies out on three streams "
                        "with two buffer sets (step i's copy out overlaps step i+1)"},
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if cpu and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_oracle_prefill(inp_host, s, single_thread=True)
    del inp_host

    # the other prefill workloads and both decode ranks, each a line of its own
    siso_inp = None
    for name in SUBLINES:
        if name == args.workload:
            continue
        sub, sub_inp = prefill_line(name, rank, world, args.steps, args.warmup, flush, peaks,
                                    psrc, cpu=cpu)
        line[name] = sub
        if name == "siso_prefill":
            siso_inp = sub_inp
        del sub_inp
    for name in ("decode_r1", "decode_r4"):
        line[name] = decode_line(name, rank, world, args.decode_steps, args.warmup, peaks, psrc,
                                 cpu=cpu)

    # the SISO layer with B and C per head (G = H), which moves 0.5 GB more
    # through HBM per call
    ss = I.SISO_PREFILL.shape
    s2 = dataclasses.replace(ss, ngroups=ss.nheads)
    inp2 = I.make_scan_inputs(I.Workload(s2), seed=1011 + 7919 * rank, device="cuda")
    barrier(world)
    t2 = max_over_ranks(sum(time_prefill(inp2, s2, max(3, args.steps // 2), args.warmup,
                                         flush)), world) / max(3, args.steps // 2)
    f2, b2 = prefill_work(s2)
    line["siso_per_head_bc"] = {
        "workload": "siso_prefill, B and C per head (ngroups = nheads = 64)",
        "value": round(world * s2.batch * s2.seqlen / t2, 1), "unit": "tokens/s",
        "ms_per_step": round(t2 * 1e3, 4), "roofline": roofline(f2, b2, t2, peaks, psrc)}
    del inp2

    # a packed batch of mixed lengths with the SISO layer shape
    line["varlen"] = varlen_line(ss, rank, world, max(3, args.steps // 2), args.warmup, flush,
                                 peaks, psrc)
    # QK-norm + bias prep of B and C (block-level step before the scan)
    line["bc_prep"] = prep_line(ss, world, 10, args.warmup, flush, peaks, psrc)
    # backward of the SISO and MIMO scans (gradients of every input)
    if siso_inp is None:
        siso_inp = I.make_scan_inputs(I.SISO_PREFILL, seed=SEEDS["siso_prefill"] + 7919 * rank,
                                      device="cuda")
    line["backward"] = bwd_line(siso_inp, ss, world, 3, args.warmup, flush, peaks, psrc)
    del siso_inp
    # the block projections around the layer (tensor-core GEMMs, MIMO up / down, gate)
    line["block"] = block_line(world, 10, args.warmup, flush, peaks, psrc)
    ms = I.MIMO_PREFILL.shape
    mimo_inp = I.make_scan_inputs(I.MIMO_PREFILL, seed=SEEDS["mimo_prefill"] + 7919 * rank,
                                  device="cuda")
    line["backward_mimo"] = bwd_line(mimo_inp, ms, world, 3, args.warmup, flush, peaks, psrc)
    del mimo_inp
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
