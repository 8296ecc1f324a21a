"""Forward parity: the CUDA path through the C ABI against the fp64 oracle on
the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, to_dev, f64, assert_o, assert_lse, rel_l2, O_REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

SMALL = [
    # (B, H, N, d, mask)
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
]


def run_fwd(w, x):
    d = to_dev(x)
    O, L = fa.fwd(d["Q"], d["K"], d["V"], w.mask, d["mask"], w.scale)
    assert fa.device_status() == 0
    return O, L


@pytest.mark.parametrize("shape", SMALL, ids=[f"{b}x{h}x{n}x{d}-{m}" for b, h, n, d, m in SMALL])
@pytest.mark.parametrize("seed", [0, 1])
def test_fwd_small(shape, seed):
    B, H, N, d, m = shape
    w = workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5)))
    x = workloads.make_inputs(w, seed, grad=False)
    O, L = run_fwd(w, x)
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], m, x["mask"], w.scale)
    assert_o(f64(O), Or, str(shape))
    assert_lse(f64(L), Lr, str(shape))


def test_fwd_block_mask_with_empty_rows():
    # a custom mask whose second block row keeps nothing: those queries see no key
    w = workloads.Workload("t", 1, 2, 384, 64, "block", 0.125)
    x = workloads.make_inputs(w, 3, grad=False)
    x["mask"] = torch.tensor([[1, 0, 1], [0, 0, 0], [0, 1, 1]], dtype=torch.uint8)
    O, L = run_fwd(w, x)
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], "block", x["mask"], w.scale)
    assert (f64(O)[:, :, 128:256] == 0).all()
    assert np.isneginf(f64(L)[:, :, 128:256]).all()
    assert_o(f64(O), Or)
    assert_lse(f64(L), Lr)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask", ["none", "causal", "block"])
@pytest.mark.parametrize("growth", [2.0, 0.5])
def test_fwd_scores_growing_or_shrinking_along_the_keys(d, mask, growth):
    # K's key tile j is scaled by growth**j.  Growing: from the third key tile
    # on, each tile's exponentials outgrow the row's reference maximum by far
    # more than 2^16, so every such tile is redone on a new reference and O and
    # l are rescaled.  Shrinking: later tiles fall far below the reference.
    # (The block mask at d = 64 runs the two-pipeline forward.)
    B, H, N = 1, 2, 768
    w = workloads.Workload("t", B, H, N, d, mask, float(np.float32(d ** -0.5)))
    x = workloads.make_inputs(w, 5, grad=False)
    f = torch.tensor([growth ** (j // 128) for j in range(N)], dtype=torch.float32)
    x["K"] = (x["K"].float() * f[None, None, :, None]).to(torch.bfloat16).contiguous()
    O, L = run_fwd(w, x)
    Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], mask, x["mask"], w.scale)
    # Growing scores make each output row nearly one row of V (|O| up to ~4),
    # so the fixed absolute bound does not fit.  The bound here follows the
    # arithmetic: each weight of P is rounded to bf16 (relative error at most
    # 2^-8) while l sums the unrounded weights, which moves O_i by at most
    # 2^-8 sum_j w_ij |v_j| (w the exact softmax weights: the oracle's output
    # with |V| in place of V); rounding O to bf16 adds at most 2^-8 |O_i|; the
    # fp32 scores and the approximate exponential add far less than 1e-3.
    Wabs, _ = oracle.fwd(x["Q"], x["K"], x["V"].abs(), mask, x["mask"], w.scale)
    err = np.abs(f64(O) - Or)
    bound = 2.0 ** -8 * (Wabs + np.abs(Or)) + 1e-3
    assert (err <= bound).all(), f"growth {growth}: worst excess {(err - bound).max():.3e}"
    assert rel_l2(f64(O), Or) <= O_REL_L2
    assert_lse(f64(L), Lr, f"growth {growth}")


def test_fwd_constant_scores_closed_form():
    # Q = 0: every visible key gets the same weight, O_i = mean of visible V rows
    w = workloads.Workload("t", 1, 2, 512, 128, "causal", 0.088)
    x = workloads.make_inputs(w, 4, grad=False)
    x["Q"].zero_()
    O, L = run_fwd(w, x)
    v = f64(x["V"])
    want = np.cumsum(v, axis=2) / np.arange(1, 513)[None, None, :, None]
    assert_o(f64(O), want)
    assert_lse(f64(L), np.broadcast_to(np.log(np.arange(1, 513)), (1, 2, 512)))


@pytest.mark.parametrize("name", workloads.ORDER)
def test_fwd_workloads_sampled(name):
    """Full-size workloads in the launch configuration the benchmark uses:
    one whole head and 64 sampled rows from the others against the oracle."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, 0, grad=False)
    O, L = run_fwd(w, x)
    O, L = f64(O).reshape(w.B * w.H, w.N, w.d), f64(L).reshape(w.B * w.H, w.N)
    q, k, v = (x[n].reshape(w.B * w.H, w.N, w.d) for n in ("Q", "K", "V"))
    h = w.B * w.H - 1
    Or, Lr = oracle.fwd(q[h:h + 1], k[h:h + 1], v[h:h + 1], w.mask, x["mask"], w.scale)
    assert_o(O[h:h + 1], Or, name)
    assert_lse(L[h:h + 1], Lr, name)
    rng = np.random.default_rng(0)
    heads = rng.integers(0, w.B * w.H, 64)
    rows = rng.integers(0, w.N, 64)
    rows[:4] = [0, w.N - 1, min(127, w.N - 1), min(128, w.N - 1)]
    Os, Ls = oracle.rows(q, k, v, heads, rows, mask_kind=w.mask, block_mask=x["mask"], scale=w.scale)
    assert_o(O[heads, rows], Os, name)
    assert_lse(L[heads, rows], Ls, name)
