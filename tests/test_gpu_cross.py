"""Queries and keys of different counts (fa_fwd_qk, fa_bwd_qk) against the
fp64 oracle on the same seeded bf16 inputs: cross-attention without a mask,
bottom-right causal (including more queries than keys, and a single query
against a long history), and block masks over a non-square tile grid."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_o, assert_lse, assert_grad

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

CASES = [
    (1, 2, 128, 384, 64, "none"),
    (2, 2, 64, 1100, 128, "none"),
    (1, 3, 513, 200, 128, "none"),
    (1, 2, 300, 700, 128, "causal"),
    (2, 1, 700, 300, 64, "causal"),      # more queries than keys: leading rows see nothing
    (1, 2, 1, 1000, 128, "causal"),      # one new query against a long history
    (2, 2, 77, 1536, 64, "causal"),
    (1, 1, 257, 129, 64, "block"),
    (1, 2, 400, 900, 128, "block"),
]
IDS = [f"{b}x{h}x{nq}x{nk}x{d}-{m}" for b, h, nq, nk, d, m in CASES]


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_cross_forward_and_backward(case):
    B, H, Nq, Nk, d, m = case
    scale = float(np.float32(d ** -0.5))
    x = workloads.make_cross_inputs(B, H, Nq, Nk, d, m, seed=Nq + Nk)
    dv = to_dev(x)
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], scale)
    dQ, dK, dV = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], scale)
    assert fa.device_status() == 0
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], m, x["mask"], scale)
    assert_o(f64(O), ref["O"], str(case))
    assert_lse(f64(L), ref["LSE"], str(case))
    for name, g in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert_grad(f64(g), ref[name], name, str(case))


def test_cross_square_call_matches_square_api():
    """fa_fwd_qk / fa_bwd_qk with Nq = Nk give the same bits as fa_fwd / fa_bwd."""
    B, H, N, d = 1, 2, 640, 128
    x = workloads.make_cross_inputs(B, H, N, N, d, "causal", seed=5)
    dv = to_dev(x)
    lib = fa.lib()
    O1 = torch.empty_like(dv["Q"])
    L1 = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    assert lib.fa_fwd_qk(dv["Q"].data_ptr(), dv["K"].data_ptr(), dv["V"].data_ptr(), B, H, N, N, d, 1, None,
                         float(d ** -0.5), O1.data_ptr(), L1.data_ptr(), None) == 0
    O2, L2 = fa.fwd(dv["Q"], dv["K"], dv["V"], "causal", None, float(d ** -0.5))
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    assert fa.bwd_workspace_size(B, H, N, d, Nk=3 * N) == fa.bwd_workspace_size(B, H, N, d)


def test_cross_rejects_bad_key_count():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    rc = fa.lib().fa_fwd_qk(q.data_ptr(), q.data_ptr(), q.data_ptr(), 1, 1, 128, 0, 64, 0, None, 0.125,
                            o.data_ptr(), lse.data_ptr(), None)
    assert rc == 1
    assert fa.lib().fa_bwd_workspace_size_qk(1, 1, 128, 0, 64) == 0
