"""The standard (materialising) attention baseline, fa_standard_fwd, against
the fp64 oracle and against the fused forward: it computes the same
attention, only through an N x N grid in HBM."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_lse, max_abs, rel_l2, O_REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

# The baseline rounds the normalised probabilities P to bf16 and then O:
# |err(O_i)| <= 2^-9 sum_j P_ij |V_j| + 2^-9 |O_i| <= 2^-8 max|V|, about
# 1.8e-2 for the N(0,1) inputs here (max |V| about 4.5).  Its rel-L2 bound is
# the fused forward's.
STD_MAX_ABS = 2e-2

CASES = [(1, 2, 128, 64, "none"), (2, 2, 300, 128, "causal"), (1, 3, 640, 64, "block"),
         (1, 1, 1, 128, "causal"), (2, 1, 1000, 128, "none")]


@pytest.mark.parametrize("case", CASES, ids=[f"{b}x{h}x{n}x{d}-{m}" for b, h, n, d, m in CASES])
def test_standard_matches_oracle_and_fused(case):
    B, H, N, d, m = case
    w = workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5)))
    x = workloads.make_inputs(w, 21, grad=False)
    dv = to_dev(x)
    O, L = fa.standard_fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], w.scale)
    O2, L2 = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], w.scale)
    assert fa.device_status() == 0
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], m, x["mask"], w.scale)
    assert max_abs(f64(O), Or) <= STD_MAX_ABS and rel_l2(f64(O), Or) <= O_REL_L2, case
    assert_lse(f64(L), Lr, str(case))
    assert (O.float() - O2.float()).abs().max().item() <= STD_MAX_ABS


def test_standard_workspace_is_quadratic():
    a = fa.standard_fwd_workspace_size(1, 1, 1024, 64)
    b = fa.standard_fwd_workspace_size(1, 1, 2048, 64)
    assert a >= 6 * 1024 * 1024 and 3.9 < b / a < 4.1
    assert fa.standard_fwd_workspace_size(1, 1, 16385, 64) == 0
