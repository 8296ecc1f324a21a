"""One problem split by heads (bench.py --split heads): each rank's part, run
on its own, gives the same outputs as the whole problem in those heads.  The
ranks are simulated one after the other on one GPU (they never wait on one
another: the split has no collective).  O, LSE, dK and dV are computed in a
fixed order and must match bit for bit; dQ's reduce-adds land in no fixed
order, so it is held to the gradient tolerance."""
import numpy as np
import pytest
import torch

import bench
import exact_io_aware_65_b200 as fa
import workloads
from helpers import has_gpu, to_dev, f64, rel_l2, GRAD_REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]


@pytest.mark.parametrize("name,world", [("gpt2_s1k_causal", 3), ("block_sparse_s16k", 2),
                                        ("long_s8k_d128_causal", 4)])
def test_head_split_matches_whole_problem(name, world):
    w = workloads.WORKLOADS[name]
    x = workloads.make_inputs(w, 0)
    d = to_dev(x)
    O, L = fa.fwd(d["Q"], d["K"], d["V"], w.mask, d["mask"], w.scale)
    g = fa.bwd(d["Q"], d["K"], d["V"], O, d["dO"], L, w.mask, d["mask"], w.scale)
    heads = w.B * w.H
    for r in range(world):
        h0, h1 = bench.head_range(heads, world, r)
        part = to_dev(bench.slice_heads(x, w, h0, h1))
        o, l = fa.fwd(part["Q"], part["K"], part["V"], w.mask, part["mask"], w.scale)
        gp = fa.bwd(part["Q"], part["K"], part["V"], o, part["dO"], l, w.mask, part["mask"], w.scale)
        assert fa.device_status() == 0
        sl = lambda t: t.reshape(heads, w.N, -1)[h0:h1] if t.dim() == 4 else t.reshape(heads, w.N)[h0:h1]
        assert torch.equal(o.reshape(h1 - h0, w.N, w.d), sl(O))
        assert torch.equal(l.reshape(h1 - h0, w.N), sl(L))
        assert torch.equal(gp[1].reshape(h1 - h0, w.N, w.d), sl(g[1]))
        assert torch.equal(gp[2].reshape(h1 - h0, w.N, w.d), sl(g[2]))
        err = rel_l2(f64(gp[0]).reshape(h1 - h0, w.N, w.d), f64(sl(g[0])))
        assert err <= GRAD_REL_L2 * 0.1, f"rank {r} dQ rel-L2 {err:.3e} against the whole problem"
