"""Randomised pins of the fp64 oracle against PyTorch's fp64 attention and
autograd (an independent library routine): query and key counts drawn
independently (ragged, N_q != N_k), small head dimensions, the three mask
kinds with random tile sizes, and block masks that may leave a row or a
column with nothing visible.  The visibility rule is built here straight
from its definition: every key for no mask; key j for query i iff
j <= i + (N_k - N_q) for causal (bottom-right aligned); tile (i // block,
j // block) kept for the block mask.  CPU only."""
import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle


def visible(Nq, Nk, kind, bm, block):
    if kind == "none":
        return torch.ones(Nq, Nk, dtype=torch.bool)
    if kind == "causal":
        i = torch.arange(Nq)[:, None]
        j = torch.arange(Nk)[None, :]
        return j <= i + (Nk - Nq)
    t = torch.from_numpy(bm).bool()
    return t.repeat_interleave(block, 0)[:Nq].repeat_interleave(block, 1)[:, :Nk]


problems = st.fixed_dictionaries({
    "B": st.integers(1, 2), "H": st.integers(1, 2),
    "Nq": st.integers(1, 160), "Nk": st.integers(1, 160),
    "d": st.sampled_from([4, 8, 16]),
    "kind": st.sampled_from(["none", "causal", "block"]),
    "block": st.sampled_from([16, 32, 64]),
    "scale": st.floats(0.05, 1.0),
    "seed": st.integers(0, 2**31 - 1),
})


@settings(max_examples=40, deadline=None)
@given(problems)
def test_oracle_matches_torch_attention_and_autograd(p):
    B, H, Nq, Nk, d, kind, block = p["B"], p["H"], p["Nq"], p["Nk"], p["d"], p["kind"], p["block"]
    scale = p["scale"]
    g = torch.Generator().manual_seed(p["seed"])
    q, do = (torch.randn((B, H, Nq, d), generator=g, dtype=torch.float64) for _ in range(2))
    k, v = (torch.randn((B, H, Nk, d), generator=g, dtype=torch.float64) for _ in range(2))
    bm = None
    if kind == "block":
        nbq, nbk = -(-Nq // block), -(-Nk // block)
        bm = (torch.rand((nbq, nbk), generator=g) < 0.5).to(torch.uint8).numpy()
    allow = visible(Nq, Nk, kind, bm, block)
    live = allow.any(dim=1)                       # rows that see at least one key

    O, L = oracle.fwd(q, k, v, kind, bm, scale, block=block)
    gr = oracle.bwd(q, k, v, do, kind, bm, scale, block=block)
    lv = live.numpy()

    # rows that see nothing: O = 0, LSE = -inf, and no gradient flows from them
    assert np.all(O[:, :, ~lv] == 0) and np.all(np.isneginf(L[:, :, ~lv]))
    assert np.all(gr["dQ"][:, :, ~lv] == 0)
    dead_cols = ~allow.any(dim=0).numpy()         # keys nobody sees
    assert np.all(gr["dK"][:, :, dead_cols] == 0) and np.all(gr["dV"][:, :, dead_cols] == 0)
    if not lv.any():
        return

    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allow, scale=scale)
    (out[:, :, live] * do[:, :, live]).sum().backward()
    np.testing.assert_allclose(O[:, :, lv], out.detach()[:, :, live].numpy(), atol=1e-10)
    s = scale * torch.einsum("bhid,bhjd->bhij", q, k)
    lse = torch.logsumexp(s.masked_fill(~allow, float("-inf")), dim=-1)
    np.testing.assert_allclose(L[:, :, lv], lse[:, :, live].numpy(), atol=1e-11)
    # gradients of sum(dO * O) over the live rows; the oracle's dead rows add nothing
    np.testing.assert_allclose(gr["dQ"][:, :, lv], qt.grad[:, :, live].numpy(), atol=1e-9, err_msg="dQ")
    np.testing.assert_allclose(gr["dK"], kt.grad.numpy(), atol=1e-9, err_msg="dK")
    np.testing.assert_allclose(gr["dV"], vt.grad.numpy(), atol=1e-9, err_msg="dV")
