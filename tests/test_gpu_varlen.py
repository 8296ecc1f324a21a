"""Variable-length batches in padded storage (fa_fwd_varlen, fa_bwd_varlen):
each batch element is its own attention problem over its first seqlens_q[b]
query rows and seqlens_k[b] keys.  Checked sequence by sequence against the
oracle on the unpadded slices; padding rows must come out exactly zero (O,
gradients) and -inf (LSE)."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_o, assert_lse, assert_grad

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

CASES = [
    # (H, Nq, Nk, d, mask, seqlens_q, seqlens_k)
    (2, 640, 640, 128, "causal", [640, 300, 0, 1], [640, 300, 0, 1]),
    (2, 640, 640, 64, "none", [640, 129, 513, 1], [200, 640, 1, 77]),
    (2, 384, 900, 128, "causal", [384, 100, 250], [900, 700, 1]),
    (3, 512, 512, 64, "block", [512, 257, 130], [512, 400, 512]),
]
IDS = [f"{m}-d{d}-{nq}x{nk}" for h, nq, nk, d, m, lq, lk in CASES]


@pytest.mark.parametrize("case", CASES, ids=IDS)
@pytest.mark.parametrize("deterministic", [False, True], ids=["default", "deterministic"])
def test_varlen_forward_and_backward(case, deterministic):
    H, Nq, Nk, d, m, lq, lk = case
    B = len(lq)
    scale = float(np.float32(d ** -0.5))
    x = workloads.make_cross_inputs(B, H, Nq, Nk, d, m, seed=Nq + Nk + B)
    dv = to_dev(x)
    sq = torch.tensor(lq, dtype=torch.int32, device="cuda")
    sk = torch.tensor(lk, dtype=torch.int32, device="cuda")
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], scale, seqlens_q=sq, seqlens_k=sk)
    dQ, dK, dV = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], scale,
                        seqlens_q=sq, seqlens_k=sk, deterministic=deterministic)
    assert fa.device_status() == 0
    O, L, dQ, dK, dV = (f64(t) for t in (O, L, dQ, dK, dV))
    for b in range(B):
        Lq, Lk = lq[b], lk[b]
        # padding comes out exactly zero / -inf
        assert np.all(O[b, :, Lq:] == 0) and np.all(np.isneginf(L[b, :, Lq:]))
        assert np.all(dQ[b, :, Lq:] == 0) and np.all(dK[b, :, Lk:] == 0) and np.all(dV[b, :, Lk:] == 0)
        if Lq == 0 or Lk == 0:
            assert np.all(O[b] == 0) and np.all(dK[b] == 0) and np.all(dV[b] == 0)
            continue
        bm = None
        if m == "block":
            bm = x["mask"][: (Lq + 127) // 128, : (Lk + 127) // 128].contiguous()
        sl = lambda t, n: t[b:b + 1, :, :n]
        ref = oracle.bwd(sl(x["Q"], Lq), sl(x["K"], Lk), sl(x["V"], Lk), sl(x["dO"], Lq), m, bm, scale)
        what = f"{case} b={b}"
        assert_o(O[b:b + 1, :, :Lq], ref["O"], what)
        assert_lse(L[b:b + 1, :, :Lq], ref["LSE"], what)
        assert_grad(dQ[b:b + 1, :, :Lq], ref["dQ"], "dQ", what)
        assert_grad(dK[b:b + 1, :, :Lk], ref["dK"], "dK", what)
        assert_grad(dV[b:b + 1, :, :Lk], ref["dV"], "dV", what)


def test_varlen_with_full_lengths_equals_plain_calls():
    B, H, N, d = 2, 2, 700, 128
    x = to_dev(workloads.make_cross_inputs(B, H, N, N, d, "causal", seed=4))
    full = torch.full((B,), N, dtype=torch.int32, device="cuda")
    O1, L1 = fa.fwd(x["Q"], x["K"], x["V"], "causal", seqlens_q=full, seqlens_k=full)
    O2, L2 = fa.fwd(x["Q"], x["K"], x["V"], "causal")
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
