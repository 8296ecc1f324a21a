"""fa_bwd_static_workspace: the backward for callers that cannot allocate
device memory (say, a runtime whose device memory is all handed out up front
by its own pool, or a latency-critical loop that must not stall on the
implicit synchronisation of cudaMalloc/cudaFree).  It runs the same kernels
as fa_bwd with their scratch in a fixed array inside the library.

The GPU test calls it through the C ABI twice in a row -- the second call
finds the first call's leftovers in the shared array -- and checks both
results against fa_bwd with a caller-allocated workspace.  This file is
named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import workloads
from helpers import has_gpu, to_dev, f64, rel_l2, GRAD_REL_L2

MAX_BYTES = 64 * 1024 * 1024


def call_static(d, O, L, w, dQ, dK, dV):
    mptr = d["mask"].data_ptr() if d["mask"] is not None else None
    return fa.lib().fa_bwd_static_workspace(
        d["Q"].data_ptr(), d["K"].data_ptr(), d["V"].data_ptr(), O.data_ptr(), d["dO"].data_ptr(),
        L.data_ptr(), w.B, w.H, w.N, w.d, fa.MASKS[w.mask], mptr, w.scale,
        dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), None)


def test_static_workspace_refuses_problems_that_do_not_fit():
    # checked on the host before any device work: runs without a GPU too
    B, H, N, d = 2, 16, 8192, 128
    assert fa.bwd_workspace_size(B, H, N, d) > MAX_BYTES
    L = fa.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = L.fa_bwd_static_workspace(fake, fake, fake, fake, fake, fake, B, H, N, d, 1, None, 0.088,
                                   fake, fake, fake, None)
    assert rc == 4  # FA_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.skipif(not has_gpu(), reason="needs a B200")
@pytest.mark.parametrize("shape", [(2, 3, 300, 64, "causal"), (1, 4, 1024, 128, "none"),
                                   (1, 8, 2048, 64, "block")])
def test_static_workspace_matches_fa_bwd_twice(shape):
    """Two calls in a row against fa_bwd with a caller-allocated workspace.
    dK and dV are sums in a fixed order (no atomics), so they must be equal
    bit for bit; dQ's bulk reduce-adds land in no fixed order, so it is held
    to the gradient tolerance.  The device's free memory must not move across
    the second call: the array was reserved by the first one."""
    B, H, N, d, m = shape
    w = workloads.Workload("t", B, H, N, d, m, float(np.float32(d ** -0.5)))
    assert fa.bwd_workspace_size(B, H, N, d) <= MAX_BYTES
    x = workloads.make_inputs(w, 11)
    dev = to_dev(x)
    O, L = fa.fwd(dev["Q"], dev["K"], dev["V"], m, dev["mask"], w.scale)
    want = fa.bwd(dev["Q"], dev["K"], dev["V"], O, dev["dO"], L, m, dev["mask"], w.scale)
    torch.cuda.synchronize()
    for call in range(2):
        got = [torch.full_like(t, float("nan")) for t in want]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert call_static(dev, O, L, w, *got) == 0
        assert fa.device_status() == 0
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before, "the second call changed free device memory"
        err = rel_l2(f64(got[0]), f64(want[0]))
        assert err <= GRAD_REL_L2, f"call {call} dQ rel-L2 {err:.3e}"
        for name, g, r in zip(("dK", "dV"), got[1:], want[1:]):
            assert torch.equal(g, r), f"call {call} {name} differs from fa_bwd"
