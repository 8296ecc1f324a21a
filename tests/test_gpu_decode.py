"""Decode against a KV cache (fa_decode): a few queries per head against a
long key/value history, split over the keys and merged by log-sum-exp.
Element by element against the fp64 oracle, and against the tensor-core
forward (fa_fwd_qk) on the same inputs."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_o, assert_lse

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

CASES = [
    (1, 1, 1, 1, 128, "none"),
    (1, 2, 1, 129, 64, "causal"),
    (2, 4, 1, 1000, 128, "causal"),
    (1, 3, 3, 300, 64, "none"),
    (1, 8, 4, 5000, 128, "causal"),
    (2, 2, 16, 3000, 64, "causal"),
    (1, 2, 16, 10, 128, "causal"),       # more queries than keys: leading rows see nothing
    (1, 2, 7, 777, 128, "none"),
    (4, 8, 1, 33000, 128, "none"),
    (1, 32, 2, 8192, 128, "causal"),
]
IDS = [f"{b}x{h}x{nq}x{nk}x{d}-{m}" for b, h, nq, nk, d, m in CASES]


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_decode_matches_oracle(case):
    B, H, Nq, Nk, d, m = case
    scale = float(np.float32(d ** -0.5))
    x = workloads.make_cross_inputs(B, H, Nq, Nk, d, m, seed=3 * Nq + Nk)
    dv = to_dev(x)
    O, L = fa.decode(dv["Q"], dv["K"], dv["V"], m, scale)
    assert fa.device_status() == 0
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], m, None, scale)
    assert_o(f64(O), Or, str(case))
    assert_lse(f64(L), Lr, str(case))


@pytest.mark.parametrize("case", [(2, 4, 1, 2048, 128, "causal"), (1, 4, 8, 1500, 64, "none")])
def test_decode_agrees_with_tensor_core_forward(case):
    B, H, Nq, Nk, d, m = case
    x = to_dev(workloads.make_cross_inputs(B, H, Nq, Nk, d, m, seed=9))
    O1, L1 = fa.decode(x["Q"], x["K"], x["V"], m)
    O2, L2 = fa.fwd(x["Q"], x["K"], x["V"], m)
    assert (O1.float() - O2.float()).abs().max().item() <= 1e-2
    assert (L1 - L2).abs().max().item() <= 1e-3


@pytest.mark.parametrize("case", [(4, 40, 8, 2048, 128, "causal"), (2, 80, 16, 1000, 64, "none"),
                                  (1, 160, 4, 300, 64, "causal")])
def test_decode_with_a_head_per_sm_matches_oracle(case):
    # four or more queries and at least one head per SM (148): the call runs
    # the tensor-core forward; the result must be the same attention
    B, H, Nq, Nk, d, m = case
    scale = float(np.float32(d ** -0.5))
    x = workloads.make_cross_inputs(B, H, Nq, Nk, d, m, seed=Nq + Nk)
    dv = to_dev(x)
    O, L = fa.decode(dv["Q"], dv["K"], dv["V"], m, scale)
    assert fa.device_status() == 0
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], m, None, scale)
    assert_o(f64(O), Or, str(case))
    assert_lse(f64(L), Lr, str(case))


def test_decode_refuses_what_it_does_not_do():
    q = torch.zeros((1, 1, 17, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 100, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 17), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    lib = fa.lib()
    args = (q.data_ptr(), k.data_ptr(), k.data_ptr(), 1, 1, 17, 100, 64)
    assert lib.fa_decode(*args, 0, 0.125, o.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(), None) == 2
    assert lib.fa_decode_workspace_size(1, 1, 17, 100, 64) == 0
    args = (q.data_ptr(), k.data_ptr(), k.data_ptr(), 1, 1, 4, 100, 64)
    assert lib.fa_decode(*args, 2, 0.125, o.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(), None) == 2
    need = lib.fa_decode_workspace_size(1, 1, 4, 100, 64)
    assert need > 0
    assert lib.fa_decode(*args, 0, 0.125, o.data_ptr(), lse.data_ptr(), ws.data_ptr(), need - 1, None) == 4
