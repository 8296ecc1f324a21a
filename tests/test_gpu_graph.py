"""The calls inside a CUDA graph: a forward + backward step and a decode step
are captured once, then replayed on new inputs copied into the same buffers.
Every replay must equal an eager call on those inputs bit for bit (the
forward, decode and the deterministic backward fix their arithmetic order;
the ordinary backward fixes it for dK and dV, and dQ is checked against the
oracle's tolerance).  Replaying several times also checks that the
forward's work counter is back at zero at the end of every launch, since a
graph bakes the counter's slot into the launch."""
import numpy as np
import pytest
import torch

import exact_io_aware_65_b200 as fa
import oracle
import workloads
from helpers import has_gpu, f64, assert_o, assert_lse, assert_grad

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not has_gpu(), reason="needs a B200")]

REPLAYS = 3


def _inputs(B, H, N, d, mask, seed):
    w = workloads.Workload("graph", B, H, N, d, mask, float(np.float32(d ** -0.5)))
    return w, workloads.make_inputs(w, seed=seed)


def _step(st, w, deterministic):
    m = st.get("mask")
    O, L = fa.fwd(st["Q"], st["K"], st["V"], w.mask, m, w.scale, O=st["O"], LSE=st["LSE"])
    fa.bwd(st["Q"], st["K"], st["V"], O, st["dO"], L, w.mask, m, w.scale, dQ=st["dQ"], dK=st["dK"],
           dV=st["dV"], workspace=st["ws"], deterministic=deterministic)


@pytest.mark.parametrize("deterministic", [False, True], ids=["atomic-dq", "ordered-dq"])
# (the block-mask case runs the d = 64 forward's two-pipeline kernel, whose
# work counter is reset by the last of its 2 x grid pipelines)
@pytest.mark.parametrize("shape", [(2, 3, 700, 64, "causal"), (1, 4, 1100, 128, "none"), (2, 3, 900, 64, "block")],
                         ids=lambda s: "x".join(map(str, s)))
def test_fwd_bwd_graph_replays_equal_eager(shape, deterministic):
    B, H, N, d, mask = shape
    w, x0 = _inputs(B, H, N, d, mask, seed=11)
    st = {k: x0[k].cuda() for k in ("Q", "K", "V", "dO")}
    if x0["mask"] is not None:
        st["mask"] = x0["mask"].cuda()
    st["O"] = torch.empty_like(st["Q"])
    st["LSE"] = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    st["dQ"], st["dK"], st["dV"] = (torch.empty_like(st["Q"]) for _ in range(3))
    st["ws"] = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):          # first calls set up per-device state outside the capture
        _step(st, w, deterministic)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(st, w, deterministic)
    torch.cuda.synchronize()

    outs = ("O", "LSE", "dQ", "dK", "dV")
    for r in range(REPLAYS):
        _, x = _inputs(B, H, N, d, mask, seed=100 + r)
        for k in ("Q", "K", "V", "dO"):
            st[k].copy_(x[k])
        if x["mask"] is not None:
            st["mask"].copy_(x["mask"])  # a new mask in the same buffer: read when the graph runs
        g.replay()
        got = {k: st[k].clone() for k in outs}
        assert fa.device_status() == 0
        _step(st, w, deterministic)      # eager, same buffers and inputs
        torch.cuda.synchronize()
        exact = outs if deterministic else ("O", "LSE", "dK", "dV")
        for k in exact:
            assert torch.equal(got[k], st[k]), f"replay {r}: {k} differs from the eager call"
        ref = oracle.bwd(x["Q"], x["K"], x["V"], x["dO"], mask, x["mask"], w.scale)
        assert_o(f64(got["O"]), ref["O"], f"replay {r}")
        assert_lse(f64(got["LSE"]), ref["LSE"], f"replay {r}")
        for k in ("dQ", "dK", "dV"):
            assert_grad(f64(got[k]), ref[k], k, f"replay {r}")
    del g


def test_decode_graph_replays_equal_eager():
    B, H, Nq, Nk, d, mask = 2, 8, 1, 6000, 128, "causal"
    scale = float(np.float32(d ** -0.5))
    x0 = workloads.make_cross_inputs(B, H, Nq, Nk, d, mask, seed=5)
    st = {k: x0[k].cuda() for k in ("Q", "K", "V")}
    st["O"] = torch.empty_like(st["Q"])
    st["LSE"] = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    st["ws"] = torch.empty(fa.decode_workspace_size(B, H, Nq, Nk, d), dtype=torch.uint8, device="cuda")

    def step():
        fa.decode(st["Q"], st["K"], st["V"], mask, scale, O=st["O"], LSE=st["LSE"], workspace=st["ws"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()

    for r in range(REPLAYS):
        x = workloads.make_cross_inputs(B, H, Nq, Nk, d, mask, seed=50 + r)
        for k in ("Q", "K", "V"):
            st[k].copy_(x[k])
        g.replay()
        O_g, L_g = st["O"].clone(), st["LSE"].clone()
        assert fa.device_status() == 0
        step()
        torch.cuda.synchronize()
        assert torch.equal(O_g, st["O"]) and torch.equal(L_g, st["LSE"]), f"replay {r} differs from eager"
        Or, Lr = oracle.fwd(x["Q"], x["K"], x["V"], mask, None, scale)
        assert_o(f64(O_g), Or, f"replay {r}")
        assert_lse(f64(L_g), Lr, f"replay {r}")
    del g
