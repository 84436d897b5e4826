"""The bounds-checked build (M3_DEBUG_BOUNDS): a sanitizer substitute.  Its
kernels test the indices they form (chains, chunks, token ranges, segments,
output elements, heads) against the extents of the call's tensors and report
M3_ERR_BOUNDS instead of touching memory outside them.  Every call of the
library on small valid inputs (both scan paths, segments, packed batches,
both backward forms, decode at R = 1, 4, 8, the block pieces and the
sequence-split calls) must leave the status word at 0 and, where compared,
agree with the oracle.  The calls run in a child process that loads
lib/libm3_debug.so (M3_LIBRARY=debug)."""
import os
import subprocess
import sys

import pytest

from selective_state_space_exp_b200 import _build
from parity_helpers import need_gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_every_call_in_bounds():
    need_gpu()
    _build.build(debug=True)
    env = dict(os.environ, M3_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_child.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "ALL OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


def test_bounds_status_code():
    """M3_ERR_BOUNDS has its name in the status table and the header."""
    from selective_state_space_exp_b200 import m3
    assert m3.STATUS[-7] == "M3_ERR_BOUNDS"
    assert "M3_ERR_BOUNDS = -7" in open(m3.HEADER).read()
