"""Backward parity: fa_bwd through the C ABI against the fp64 oracle's
gradients on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_grad, GRAD_REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

SMALL = [
    (1, 1, 128, 64, "none"),
    (1, 1, 1, 64, "none"),
    (1, 1, 1, 128, "causal"),
    (2, 3, 300, 64, "none"),
    (2, 3, 300, 64, "causal"),
    (2, 3, 300, 64, "block"),
    (1, 2, 640, 128, "causal"),
    (1, 2, 257, 128, "none"),
    (1, 2, 383, 128, "block"),
    (3, 1, 127, 64, "causal"),
    (1, 1, 129, 128, "causal"),
    (2, 2, 1024, 64, "causal"),
    (1, 2, 1024, 128, "none"),
]


def run(w, x, O=None, L=None):
    d = to_dev(x)
    if O is None:
        O, L = fa.fwd(d["Q"], d["K"], d["V"], w.mask, d["mask"], w.scale)
    g = fa.bwd(d["Q"], d["K"], d["V"], O, d["dO"], L, w.mask, d["mask"], w.scale)
    assert fa.device_status() == 0
    return g


@pytest.mark.parametrize("shape", SMALL, ids=[f"{b}x{h}x{n}x{d}-{m}" for b, h, n, d, m in SMALL])
@pytest.mark.parametrize("seed", [0, 1])
def test_bwd_small(shape, seed):
    B, H, N, d, m = shape
    w = workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5)))
    x = workloads.make_inputs(w, seed)
    dQ, dK, dV = run(w, x)
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], m, x["mask"], w.scale)
    for name, g in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert_grad(f64(g), ref[name], name, str(shape))


@pytest.mark.parametrize("shape", [(2, 3, 300, 64, "causal"), (1, 2, 383, 128, "block")])
def test_bwd_from_oracle_statistics(shape):
    """Feed the oracle's O (rounded to bf16) and LSE (fp32) to isolate the
    backward's own error from the forward's."""
    B, H, N, d, m = shape
    w = workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5)))
    x = workloads.make_inputs(w, 5)
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], m, x["mask"], w.scale)
    O = torch.from_numpy(ref["O"]).to(torch.bfloat16).cuda()
    L = torch.from_numpy(ref["LSE"]).to(torch.float32).cuda()
    dQ, dK, dV = run(w, x, O, L)
    for name, g in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert_grad(f64(g), ref[name], name, str(shape))


def test_bwd_block_mask_with_empty_rows_and_columns():
    w = workloads.Workload("t", 1, 2, 384, 64, "block", 0.125)
    x = workloads.make_inputs(w, 6)
    x["mask"] = torch.tensor([[1, 0, 1], [0, 0, 0], [0, 0, 1]], dtype=torch.uint8)
    dQ, dK, dV = run(w, x)
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], "block", x["mask"], w.scale)
    assert (f64(dQ)[:, :, 128:256] == 0).all()      # query block that sees nothing
    assert (f64(dK)[:, :, 128:256] == 0).all()      # key block nobody sees
    assert (f64(dV)[:, :, 128:256] == 0).all()
    for name, g in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert_grad(f64(g), ref[name], name)


@pytest.mark.parametrize("mask", ["none", "causal", "block"])
def test_bwd_gradient_identities(mask):
    """Properties that hold at any size: rows of dS sum to zero, so sum_j dK_j
    = 0; rows of P sum to one, so sum_j dV_j = sum_i dO_i."""
    w = workloads.Workload("t", 2, 2, 1024, 128, mask, float(np.float32(128 ** -0.5)))
    x = workloads.make_inputs(w, 7)
    dQ, dK, dV = run(w, x)
    dk, dv, do = f64(dK), f64(dV), f64(x["dO"])
    scale_k = np.abs(dk).sum(axis=2).max()
    assert np.abs(dk.sum(axis=2)).max() <= 2e-2 * scale_k
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=2e-2 * np.abs(do).sum(axis=2).max())


@pytest.mark.parametrize("name", workloads.ORDER)
def test_bwd_workloads_one_head(name):
    """Full-size workloads in the benchmark's launch configuration; the
    oracle recomputes one whole head (heads are independent)."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, 0)
    dQ, dK, dV = run(w, x)
    h = w.B * w.H - 1
    sl = lambda t: t.reshape(w.B * w.H, w.N, w.d)[h:h + 1]
    ref = oracle.bwd(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(x["dO"]), w.mask, x["mask"], w.scale)
    for nm, g in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert_grad(f64(sl(g)), ref[nm][0:1], nm, name)


@pytest.mark.parametrize("name", workloads.ORDER)
def test_bwd_workloads_every_head(name):
    """Full-size workloads in the benchmark's launch configuration, checked
    element by element in every head: sampled dQ rows against the oracle's
    per-row gradient, and sampled dK, dV key rows against its per-key-column
    gradient (first, last and tile-boundary rows and keys among them); plus
    the identities sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i over every key
    (rows of dS sum to zero, rows of P to one; every query row of these
    workloads sees a key)."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, 3)
    dQ, dK, dV = run(w, x)
    BH = w.B * w.H
    rng = np.random.default_rng(11)
    per = 6
    rows = rng.integers(0, w.N, (BH, per))
    rows[:, 0], rows[:, 1] = 0, w.N - 1
    rows[:, 2], rows[:, 3] = min(127, w.N - 1), min(128, w.N - 1)
    heads = np.repeat(np.arange(BH), per)
    rows = rows.reshape(-1)
    _, _, dQs = oracle.rows(x["Q"], x["K"], x["V"], heads, rows, dO=x["dO"], mask_kind=w.mask,
                            block_mask=x["mask"], scale=w.scale)
    g = f64(dQ).reshape(BH, w.N, w.d)[heads, rows].reshape(BH, per, w.d)
    ref = dQs.reshape(BH, per, w.d)
    for h in range(BH):
        assert_grad(g[h], ref[h], "dQ", f"{name} head {h}")
    keys = rng.integers(0, w.N, (BH, per))
    keys[:, 0], keys[:, 1] = 0, w.N - 1
    keys[:, 2], keys[:, 3] = min(127, w.N - 1), min(128, w.N - 1)
    keys = keys.reshape(-1)
    dKs, dVs = oracle.cols(x["Q"], x["K"], x["V"], x["dO"], heads, keys, mask_kind=w.mask,
                           block_mask=x["mask"], scale=w.scale)
    for nm, gt, rf in (("dK", dK, dKs), ("dV", dV, dVs)):
        got = f64(gt).reshape(BH, w.N, w.d)[heads, keys].reshape(BH, per, w.d)
        rf = rf.reshape(BH, per, w.d)
        for h in range(BH):
            assert_grad(got[h], rf[h], nm, f"{name} head {h}")
    dk = f64(dK).reshape(BH, w.N, w.d)
    dv = f64(dV).reshape(BH, w.N, w.d)
    do = f64(x["dO"]).reshape(BH, w.N, w.d)
    kscale = np.abs(dk).sum(axis=1).max(axis=1)
    assert (np.abs(dk.sum(axis=1)).max(axis=1) <= 2e-2 * kscale + 1e-6).all()
    vscale = np.abs(do).sum(axis=1).max(axis=1)
    assert (np.abs(dv.sum(axis=1) - do.sum(axis=1)).max(axis=1) <= 2e-2 * vscale).all()


@pytest.mark.parametrize("shape", [(1, 2, 1000, 128, "causal"), (2, 2, 640, 64, "none"),
                                   (1, 2, 900, 64, "block"), (1, 2, 300, 700, 128, "causal")],
                         ids=["1x2x1000x128-causal", "2x2x640x64-none", "1x2x900x64-block", "cross-300x700-causal"])
def test_bwd_deterministic_reproducible_and_exact(shape):
    """fa_bwd_qk_deterministic: the same bits on every run, and the oracle's
    gradients within the usual tolerance."""
    if len(shape) == 5:
        B, H, N, d, m = shape
        x = workloads.make_inputs(workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5))), 8)
    else:
        B, H, N, Nk, d, m = shape
        x = workloads.make_cross_inputs(B, H, N, Nk, d, m, seed=8)
    scale = float(np.float32(d ** -0.5))
    dv = to_dev(x)
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], m, dv["mask"], scale)
    runs = [fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, m, dv["mask"], scale, deterministic=True)
            for _ in range(3)]
    assert fa.device_status() == 0
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], m, x["mask"], scale)
    for name, g in zip(("dQ", "dK", "dV"), runs[0]):
        assert_grad(f64(g), ref[name], name, str(shape))


@pytest.mark.parametrize("name", ["gpt2_s1k_causal", "long_s8k_d128_causal"])
def test_bwd_deterministic_full_size(name):
    """Full-size workloads: the ordered dQ additions complete (no wait runs
    out), repeat bit for bit, and agree with the unordered backward."""
    w = workloads.WORKLOADS[name]
    dv = to_dev(workloads.make_inputs(w, 0))
    O, L = fa.fwd(dv["Q"], dv["K"], dv["V"], w.mask, dv["mask"], w.scale)
    a = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, w.mask, dv["mask"], w.scale, deterministic=True)
    b = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, w.mask, dv["mask"], w.scale, deterministic=True)
    c = fa.bwd(dv["Q"], dv["K"], dv["V"], O, dv["dO"], L, w.mask, dv["mask"], w.scale)
    assert fa.device_status() == 0
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y)
        err = (x.float() - z.float()).norm() / z.float().norm()
        assert err.item() <= 1e-3
