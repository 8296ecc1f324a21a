"""The seeded input recipe and the work accounting both sides of every
parity check and the benchmark rest on, on CPU: the five workloads' shapes
and scales, reproducible draws in the stated order, the block mask's
density and diagonal, kept-entry counts against brute force over the
visibility rule, and the FLOP convention (4d per kept score entry forward,
10d backward)."""
import math
import os
import sys

import numpy as np
import pytest
import torch

import workloads

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_the_five_workloads():
    want = {
        "tiny": (1, 1, 128, 64, "none", 1 / 8),
        "bert_large_s512": (16, 16, 512, 64, "none", 1 / 8),
        "gpt2_s1k_causal": (8, 12, 1024, 64, "causal", 1 / 8),
        "long_s8k_d128_causal": (2, 16, 8192, 128, "causal", 1 / math.sqrt(128)),
        "block_sparse_s16k": (1, 8, 16384, 64, "block", 1 / 8),
    }
    assert list(workloads.WORKLOADS) == list(want)
    for name, (B, H, N, d, m, scale) in want.items():
        w = workloads.WORKLOADS[name]
        assert (w.B, w.H, w.N, w.d, w.mask) == (B, H, N, d, m)
        assert w.scale == float(np.float32(scale))      # the fp32 value the kernels get


def test_draws_are_seeded_in_the_stated_order():
    w = workloads.Workload("t", 2, 3, 200, 64, "none", 0.125)
    a = workloads.make_inputs(w, seed=7)
    b = workloads.make_inputs(w, seed=7)
    c = workloads.make_inputs(w, seed=8)
    g = torch.Generator("cpu").manual_seed(7)
    for name in ("Q", "K", "V", "dO"):
        assert a[name].dtype == torch.bfloat16 and a[name].shape == (2, 3, 200, 64) and a[name].is_contiguous()
        assert torch.equal(a[name], b[name]) and not torch.equal(a[name], c[name])
        ref = torch.randn((2, 3, 200, 64), generator=g, dtype=torch.float32).to(torch.bfloat16)
        assert torch.equal(a[name], ref), name
    assert a["mask"] is None
    assert "dO" not in workloads.make_inputs(w, seed=7, grad=False)


def test_block_mask_keeps_the_diagonal_at_the_stated_density():
    nb = workloads.WORKLOADS["block_sparse_s16k"].nb
    assert nb == 128
    dens = []
    for seed in range(4):
        m = workloads.block_mask(nb, seed)
        assert m.dtype == torch.uint8 and m.shape == (nb, nb)
        assert bool(m.diagonal().all())
        assert torch.equal(m, workloads.block_mask(nb, seed))
        off = m.sum().item() - nb
        dens.append(off / (nb * nb - nb))
    assert abs(np.mean(dens) - workloads.P_KEEP) < 0.01   # 4 x 16256 Bernoulli(0.25) draws


@pytest.mark.parametrize("N", [1, 100, 128, 129, 300, 383])
@pytest.mark.parametrize("kind", ["none", "causal", "block"])
def test_kept_entries_match_brute_force(N, kind):
    w = workloads.Workload("t", 1, 1, N, 64, kind, 0.125)
    mask = workloads.block_mask(w.nb, 3) if kind == "block" else None
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    if kind == "none":
        allow = np.ones((N, N), bool)
    elif kind == "causal":
        allow = j <= i
    else:
        allow = mask.numpy().astype(bool)[i // 128, j // 128]
    assert workloads.kept_entries(w, mask) == int(allow.sum())
    tiles = {(a // 128, b // 128) for a, b in zip(*np.nonzero(allow))}
    assert workloads.kept_blocks(w, mask) == len(tiles)


def test_flop_convention():
    w = workloads.WORKLOADS["long_s8k_d128_causal"]
    f = bench.flops(w, None)
    E = 8192 * 8193 // 2
    assert f["E"] == E
    assert f["fwd"] == 4 * 2 * 16 * E * 128 and f["bwd"] == 10 * 2 * 16 * E * 128
    assert abs((f["fwd"] + f["bwd"]) / 1e9 - 1924.4) < 0.1   # GFLOP per fwd+bwd step
