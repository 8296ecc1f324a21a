"""The index-checking debug build (libfa_debug.so) on the GPU.

That build compiles every raw-pointer global access of every kernel with a
range check against its buffer; a failed check skips the access and records
FA_ERR_BOUNDS in the device status word (nothing traps).  It stands in for
a memory checker: a small forward + backward per mask kind, the cross,
variable-length and deterministic forms and a decode step run through it in
a child process (the library is chosen at import time), and each must leave
the status word at FA_OK and still match the oracle."""
import os
import subprocess
import sys

import pytest

from helpers import has_gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "exact_io_aware_65_b200", "libfa_debug.so")

CHILD = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import to_dev, f64, assert_o, assert_lse, assert_grad

assert fa.LIB_PATH.endswith("libfa_debug.so"), fa.LIB_PATH

def check(name, x, m, scale, O, L, g):
    st = fa.device_status()
    assert st == 0, f"{name}: device status {st}"
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], m, x["mask"], scale)
    assert_o(f64(O), ref["O"], name)
    assert_lse(f64(L), ref["LSE"], name)
    for nm, t in zip(("dQ", "dK", "dV"), g):
        assert_grad(f64(t), ref[nm], nm, name)

for B, H, N, d, m in [(2, 3, 300, 64, "none"), (2, 3, 300, 64, "causal"), (1, 2, 383, 128, "block"),
                      (1, 2, 257, 128, "causal"), (3, 1, 1, 64, "none")]:
    sc = float(np.float32(d ** -0.5))
    x = workloads.make_inputs(workloads.Workload("t", B, H, N, d, m, sc), 4)
    dv = to_dev(x)
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], sc)
    g = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], sc)
    check(f"{B}x{H}x{N}x{d}-{m}", x, m, sc, O, L, g)
    g2 = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], sc, deterministic=True)
    check(f"{B}x{H}x{N}x{d}-{m} deterministic", x, m, sc, O, L, g2)

for Nq, Nk, d, m in [(300, 700, 128, "causal"), (700, 300, 64, "causal"), (129, 1000, 64, "block")]:
    sc = float(np.float32(d ** -0.5))
    x = workloads.make_cross_inputs(1, 2, Nq, Nk, d, m, seed=5)
    dv = to_dev(x)
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], sc)
    g = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], sc)
    check(f"cross {Nq}x{Nk}x{d}-{m}", x, m, sc, O, L, g)

# decode: a few queries against a longer cache
x = workloads.make_cross_inputs(2, 4, 4, 3000, 128, "causal", seed=6)
dv = to_dev(x)
sc = float(np.float32(128 ** -0.5))
O, L = fa.decode(dv["Q"], dv["K"], dv["V"], "causal", sc)
st = fa.device_status()
assert st == 0, f"decode: device status {st}"
rO, rL = oracle.fwd(x["Q"], x["K"], x["V"], "causal", None, sc)
assert_o(f64(O), rO, "decode")
assert_lse(f64(L), rL, "decode")
print("debug build: every case ran with status FA_OK")
"""


@pytest.mark.gpu
@pytest.mark.skipif(not has_gpu(), reason="needs a B200")
def test_debug_build_reports_no_out_of_range_access():
    assert os.path.exists(DEBUG_LIB), "build it with python -m exact_io_aware_65_b200.build --debug-bounds"
    env = dict(os.environ, FA_LIBRARY=DEBUG_LIB)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "status FA_OK" in r.stdout
