"""The C ABI library: it builds, loads, exports every symbol include/m3.h
declares, and rejects bad arguments on the host before touching the GPU.
No test here launches a kernel."""
import ctypes
import re

import pytest

from selective_state_space_exp_b200 import _build, m3


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return m3.load()


def declared_functions():
    src = open(m3.HEADER).read()
    return re.findall(r"M3_API\s+[\w\s\*]+?\b(m3_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"m3_scan_fwd", "m3_decode_step", "m3_scan_workspace_size", "m3_scan_workspace_bytes",
            "m3_stream_status", "m3_check_shape", "m3_status_string", "m3_version"} <= names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.m3_version()
    for code, name in m3.STATUS.items():
        assert lib.m3_status_string(code).decode() == name


def shape(**kw):
    d = dict(batch=2, seqlen=100, nheads=4, ngroups=1, headdim=64, dstate=128, rank=1,
             chunk=64, io_dtype=m3.M3_BF16, flags=0)
    d.update(kw)
    return m3.Shape(**d)


@pytest.mark.parametrize("kw,expect", [
    ({}, 0),
    (dict(rank=4), 0), (dict(rank=8, headdim=16, dstate=16), 0),
    (dict(dstate=16, headdim=16, io_dtype=m3.M3_F32), 0),
    (dict(seqlen=0), 0),
    (dict(batch=0), -1), (dict(nheads=0), -1), (dict(seqlen=-1), -1),
    (dict(dstate=127), -1), (dict(nheads=6, ngroups=4), -1), (dict(io_dtype=7), -1),
    (dict(flags=8), 0), (dict(flags=16), -1), (dict(chunk=0), -1),
    (dict(rank=3), -2), (dict(dstate=96), -2), (dict(headdim=48), -2),
    (dict(headdim=256), -2), (dict(dstate=256, headdim=128), -2), (dict(chunk=48), -2),
    (dict(chunk=128), -2), (dict(batch=70000), -2),
])
def test_check_shape(lib, kw, expect):
    s = shape(**kw)
    assert lib.m3_check_shape(ctypes.byref(s)) == expect


def test_workspace_size(lib):
    n = ctypes.c_size_t()
    s = shape(seqlen=0)
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0 and n.value == 0
    # CUDA-core path: one N x P fp32 state per chunk-head (3 chunks, the last ragged)
    s = shape(seqlen=130, flags=m3.M3_FLAG_SIMT)
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value >= 2 * 4 * 3 * 128 * 64 * 4
    # tensor-core path: 8 chains are cut into 3 segments -> 2 carried states per chain
    s = shape(seqlen=130)
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert 2 * 4 * 2 * 128 * 64 * 4 <= n.value < 2 * 4 * 3 * 128 * 64 * 4
    # many chains: one segment per chain, no workspace at all
    s = shape(batch=8, nheads=64, seqlen=2048)
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0 and n.value == 0
    # rank 4 (one CTA per SM on 148 SMs): 512 chains leave a fourth wave of 68,
    # which are cut in two -> one N x P state and 1 + N/2 totals per cut chain
    s = shape(batch=8, nheads=64, seqlen=2048, rank=4)
    assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value == 68 * 128 * 64 * 4 + (68 * 65 * 4 + 255) // 256 * 256  # parts 256-byte aligned
    assert lib.m3_scan_workspace_size(ctypes.byref(s), None) == -1
    assert lib.m3_scan_workspace_size(None, ctypes.byref(n)) == -1


def test_workspace_bytes_matches_the_status_form(lib):
    """m3_scan_workspace_bytes returns the value m3_scan_workspace_size writes,
    and SIZE_MAX where the status form returns an error."""
    size_max = ctypes.c_size_t(-1).value
    for kw in (dict(seqlen=0), dict(seqlen=130, flags=m3.M3_FLAG_SIMT), dict(seqlen=130),
               dict(batch=8, nheads=64, seqlen=2048), dict(seqlen=4096, flags=m3.M3_FLAG_SIMT)):
        s = shape(**kw)
        n = ctypes.c_size_t()
        assert lib.m3_scan_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
        assert lib.m3_scan_workspace_bytes(ctypes.byref(s)) == n.value
    for kw in (dict(nheads=0), dict(headdim=0), dict(chunk=48), dict(io_dtype=7)):
        s = shape(**kw)
        assert lib.m3_check_shape(ctypes.byref(s)) != 0
        assert lib.m3_scan_workspace_bytes(ctypes.byref(s)) == size_max
    assert lib.m3_scan_workspace_bytes(None) == size_max


# Fake, never dereferenced device addresses: every case below fails a host
# check before any CUDA call is made.
A16 = 0x7f0000000000
P = [ctypes.c_void_p(A16 + 0x100000 * i) for i in range(16)]


def scan_call(lib, s, **over):
    args = dict(x=P[0], dt=P[1], A=P[2], lam=P[3], theta=P[4], B=P[5], C=P[6], h0=None,
                B_prev=None, x_prev=None, y=P[7], fs=P[8], ws=P[9], wsb=0, stream=None)
    args.update(over)
    return lib.m3_scan_fwd(None if s is None else ctypes.byref(s), args["x"], args["dt"], args["A"], args["lam"],
                           args["theta"], args["B"], args["C"], args["h0"], args["B_prev"],
                           args["x_prev"], args["y"], args["fs"], args["ws"],
                           ctypes.c_size_t(args["wsb"]), args["stream"])


def test_scan_rejects_bad_arguments(lib):
    s = shape()
    assert scan_call(lib, s, x=None) == -1
    assert scan_call(lib, s, y=None) == -1
    assert scan_call(lib, s, theta=None) == -1
    assert scan_call(lib, s, B_prev=P[10]) == -1           # B_prev without x_prev
    assert scan_call(lib, s, x=ctypes.c_void_p(A16 + 8)) == -3
    assert scan_call(lib, s, y=ctypes.c_void_p(A16 + 2)) == -3
    assert scan_call(lib, s, dt=ctypes.c_void_p(A16 + 2)) == -3
    assert scan_call(lib, s, theta=ctypes.c_void_p(A16 + 4)) == -3
    assert scan_call(lib, s, ws=None) == -4
    assert scan_call(lib, s, wsb=16) == -4
    assert scan_call(lib, s, ws=ctypes.c_void_p(A16 + 16), wsb=1 << 40) == -4
    assert scan_call(lib, shape(rank=3)) == -2
    assert scan_call(lib, None) == -1


def decode_call(lib, s, **over):
    args = dict(si=P[0], so=P[0], x=P[1], dt=P[2], A=P[3], lam=P[4], theta=P[5], B=P[6],
                C=P[7], Bp=None, xp=None, y=P[8], stream=None)
    args.update(over)
    return lib.m3_decode_step(ctypes.byref(s), args["si"], args["so"], args["x"], args["dt"],
                              args["A"], args["lam"], args["theta"], args["B"], args["C"],
                              args["Bp"], args["xp"], args["y"], args["stream"])


def test_decode_rejects_bad_arguments(lib):
    s = shape()
    assert decode_call(lib, s, si=None) == -1
    assert decode_call(lib, s, y=None) == -1
    assert decode_call(lib, s, xp=P[9]) == -1                       # x_prev without B_prev
    assert decode_call(lib, s, so=ctypes.c_void_p(A16 + 64)) == -1  # partial overlap
    assert decode_call(lib, s, x=ctypes.c_void_p(A16 + 0x100000 + 4)) == -3
    assert decode_call(lib, s, lam=ctypes.c_void_p(A16 + 1)) == -3
    assert decode_call(lib, shape(headdim=24)) == -2


@pytest.mark.parametrize("kw,tc,seg,launches", [
    (dict(batch=8, nheads=64, seqlen=2048), 1, 1, 1),            # many chains: one segment
    (dict(batch=8, nheads=64, seqlen=2048, rank=4), 1, 2, 2),    # last wave's chains cut in two
    (dict(batch=1, nheads=64, seqlen=32768, rank=4), 1, None, 3),  # few chains: segments
    (dict(batch=8, nheads=64, seqlen=2048, flags=1), 0, 1, 3),     # forced CUDA-core path
    (dict(io_dtype=0, dstate=16, headdim=16), 0, 1, 3),            # fp32 io
    (dict(seqlen=0), 1, 1, 0),
    (dict(rank=8), 0, 1, 3),                                       # R = 8: CUDA-core path
])
def test_scan_plan(lib, kw, tc, seg, launches):
    s = shape(**kw)
    t, g, n = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int()
    assert lib.m3_scan_plan(ctypes.byref(s), ctypes.byref(t), ctypes.byref(g), ctypes.byref(n)) == 0
    assert t.value == tc and n.value == launches
    if seg is None:
        assert g.value > 1
    else:
        assert g.value == seg
    assert lib.m3_scan_plan(ctypes.byref(s), None, None, None) == 0
    assert lib.m3_scan_plan(None, None, None, None) == -1


def prep_call(lib, s, **over):
    args = dict(Br=P[0], Cr=P[1], wB=None, bB=None, wC=None, bC=None, eps=1e-6, B=P[2], C=P[3])
    args.update(over)
    return lib.m3_bc_prep(ctypes.byref(s), args["Br"], args["Cr"], args["wB"], args["bB"],
                          args["wC"], args["bC"], ctypes.c_float(args["eps"]), args["B"],
                          args["C"], None)


def test_bc_prep_rejects_bad_arguments(lib):
    s = shape()  # 200 tokens x 128 bf16: 51200 bytes per tensor
    assert prep_call(lib, s, B=None) == -1                         # raw B without output
    assert prep_call(lib, s, Cr=None) == -1                        # C output without raw C
    assert prep_call(lib, s, eps=-1.0) == -1
    assert prep_call(lib, s, eps=float("nan")) == -1
    assert prep_call(lib, s, B=ctypes.c_void_p(A16 + 0x100000 + 4096)) == -1   # B overlaps raw C
    assert prep_call(lib, s, B=P[3], C=P[3]) == -1                 # one output for both
    assert prep_call(lib, s, B=ctypes.c_void_p(A16 + 0x200000 + 8)) == -3
    assert prep_call(lib, s, wB=ctypes.c_void_p(A16 + 0x500000 + 4)) == -3
    assert prep_call(lib, shape(rank=3)) == -2


def varlen_call(lib, s, **over):
    args = dict(cu=P[11], T=200, x=P[0], dt=P[1], A=P[2], lam=P[3], theta=P[4], B=P[5], C=P[6],
                h0=None, Bp=None, xp=None, y=P[7], fs=None, ws=P[9], wsb=1 << 30, stream=None)
    args.update(over)
    return lib.m3_scan_fwd_varlen(ctypes.byref(s), args["cu"], ctypes.c_int64(args["T"]),
                                  args["x"], args["dt"], args["A"], args["lam"], args["theta"],
                                  args["B"], args["C"], args["h0"], args["Bp"], args["xp"],
                                  args["y"], args["fs"], args["ws"], ctypes.c_size_t(args["wsb"]),
                                  args["stream"])


def test_varlen_rejects_bad_arguments(lib):
    s = shape()
    assert varlen_call(lib, s, cu=None) == -1
    assert varlen_call(lib, s, T=-1) == -1
    assert varlen_call(lib, s, cu=ctypes.c_void_p(A16 + 0xB00000 + 2)) == -1  # not 4-byte aligned
    assert varlen_call(lib, s, x=None) == -1
    assert varlen_call(lib, s, Bp=P[10]) == -1                               # B_prev alone
    assert varlen_call(lib, s, y=ctypes.c_void_p(A16 + 0x700000 + 8)) == -3
    need = ctypes.c_size_t()
    s_long = shape(batch=1, nheads=1, seqlen=4096)  # one chain: cut into segments
    assert lib.m3_scan_workspace_size(ctypes.byref(s_long), ctypes.byref(need)) == 0
    assert need.value > 0 and varlen_call(lib, s_long, T=4096, ws=None, wsb=0) == -4
    assert varlen_call(lib, shape(rank=3)) == -2


def bwd_call(lib, s, varlen=False, **over):
    args = dict(x=P[0], dt=P[1], A=P[2], lam=P[3], theta=P[4], B=P[5], C=P[6], h0=None, Bp=None,
                xp=None, dy=P[7], dfin=None, dx=P[8], ddt=P[9], dA=P[10], dlam=P[11], dth=P[12],
                dB=P[13], dC=P[14], dh0=None, dBp=None, dxp=None, ws=P[15], wsb=1 << 40,
                stream=None, cu=P[11], T=200)
    args.update(over)
    rest = [args[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C", "h0", "Bp", "xp", "dy",
                              "dfin", "dx", "ddt", "dA", "dlam", "dth", "dB", "dC", "dh0",
                              "dBp", "dxp", "ws")] + [ctypes.c_size_t(args["wsb"]), args["stream"]]
    if varlen:
        return lib.m3_scan_bwd_varlen(ctypes.byref(s), args["cu"], ctypes.c_int64(args["T"]),
                                      *rest)
    return lib.m3_scan_bwd(ctypes.byref(s), *rest)


def test_bwd_workspace_and_bad_arguments(lib):
    n = ctypes.c_size_t()
    s = shape(batch=2, seqlen=130, io_dtype=m3.M3_F32, dstate=16, headdim=16)
    assert lib.m3_scan_bwd_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    # 32-row chunks (R = 1): 5 per sequence; chunk states and adjoints, totals, final states
    assert n.value >= 2 * (2 * 4 * 5 * 16 * 16 * 4) + 2 * 4 * 16 * 16 * 4
    assert lib.m3_scan_bwd_workspace_size(None, ctypes.byref(n)) == -1
    for varlen in (False, True):
        assert bwd_call(lib, s, varlen, dy=None) == -1
        assert bwd_call(lib, s, varlen, dth=None) == -1
        assert bwd_call(lib, s, varlen, dC=None) == -1
        assert bwd_call(lib, s, varlen, Bp=P[10]) == -1                  # B_prev without x_prev
        assert bwd_call(lib, s, varlen, dBp=P[10]) == -1                 # dB_prev without dx_prev
        assert bwd_call(lib, s, varlen, dx=ctypes.c_void_p(A16 + 0x800000 + 4)) == -3
        assert bwd_call(lib, s, varlen, ddt=ctypes.c_void_p(A16 + 0x900000 + 2)) == -3
        assert bwd_call(lib, s, varlen, ws=None) == -4
        assert bwd_call(lib, s, varlen, wsb=16) == -4
        assert bwd_call(lib, shape(rank=3), varlen) == -2
    assert bwd_call(lib, s, True, cu=None) == -1
    assert bwd_call(lib, s, True, T=-5) == -1
