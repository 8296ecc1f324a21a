"""Pins for the fp64 CPU oracle, each against something other than the oracle
itself: hand-derived closed forms, invariants of softmax attention, finite
differences, the blocked online-softmax restatement of the exactness claim,
and an independent library routine (PyTorch's CPU fp64 attention + autograd).
CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle.online import attention_online, allowed_matrix


KINDS = ("none", "causal", "block")
KIND_ID = {"none": 0, "causal": 1, "block": 2}


def rnd(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


def small_mask(N, block, seed):
    nb = (N + block - 1) // block
    m = (np.random.default_rng(seed).random((nb, nb)) < 0.4).astype(np.uint8)
    np.fill_diagonal(m, 1)
    return m


# ---------------------------------------------------------------- golden ----

def _ev(x):
    return eval(x, {"__builtins__": {}}, {"e": math.e, "ln": math.log})


@pytest.mark.parametrize("case", ["none", "causal"])
def test_worked_example_closed_form(golden_dir, case):
    fx = json.load(open(os.path.join(golden_dir, "worked_example_n3.json")))
    Q, K, V, dO = (np.array(fx[n], dtype=np.float64)[None] for n in ("Q", "K", "V", "dO"))
    want = {k: np.vectorize(_ev, otypes=[float])(np.array(v, dtype=object)).astype(np.float64)
            for k, v in fx["cases"][case].items()}
    O, L = oracle.fwd(Q, K, V, case, scale=fx["scale"])
    np.testing.assert_allclose(O[0], want["O"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(L[0], want["LSE"], rtol=0, atol=1e-14)
    g = oracle.bwd(Q, K, V, dO, case, scale=fx["scale"])
    for n in ("dQ", "dK", "dV"):
        np.testing.assert_allclose(g[n][0], want[n], rtol=0, atol=1e-14, err_msg=n)
    np.testing.assert_allclose(g["D"][0], want["D"], rtol=0, atol=1e-14)


def test_score_grid_size(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "score_grid_8000.json")))
    w = workloads.Workload("grid", 1, 1, fx["N"], 64, "none", 0.125)
    assert workloads.kept_entries(w, None) == fx["entries"]


# ------------------------------------------------ exactness of tiling ------

@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("tiles", [(1, 1), (7, 7), (64, 64), (128, 128), (200, 200), (64, 7)])
def test_online_blocked_equals_two_pass(kind, tiles):
    N, d, scale, block = 200, 16, 0.3, 64
    q, k, v = rnd((N, d), 1), rnd((N, d), 2), rnd((N, d), 3)
    bm = small_mask(N, block, 4) if kind == "block" else None
    O, L = oracle.fwd(q[None], k[None], v[None], kind, bm, scale, block=block)
    tm, tn = tiles
    n_kt = (N + tn - 1) // tn
    for order in (None, np.random.default_rng(5).permutation(n_kt)):
        O2, L2 = attention_online(q, k, v, scale, KIND_ID[kind], bm, block, tm, tn, order)
        np.testing.assert_allclose(O2, O[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L2, L[0], rtol=0, atol=1e-12)


# ------------------------------------------------------ softmax rows -------

@pytest.mark.parametrize("kind", KINDS)
def test_probability_rows(kind):
    N, d, block = 150, 8, 32
    q, k = rnd((2, N, d), 6), rnd((2, N, d), 7)
    bm = small_mask(N, block, 8) if kind == "block" else None
    P = oracle.probs(q, k, kind, bm, 0.5, block=block)
    allow = allowed_matrix(N, KIND_ID[kind], bm, block)
    assert (P >= 0).all()
    assert (P[:, ~allow] == 0).all()
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)


# ------------------------------------------------------ closed forms -------

@pytest.mark.parametrize("kind", KINDS)
def test_constant_scores_give_mean_of_visible_values(kind):
    N, d, block = 300, 8, 64
    q = np.zeros((1, N, d))
    k, v = rnd((1, N, d), 9), rnd((1, N, d), 10)
    bm = small_mask(N, block, 11) if kind == "block" else None
    O, L = oracle.fwd(q, k, v, kind, bm, 0.125, block=block)
    allow = allowed_matrix(N, KIND_ID[kind], bm, block)
    cnt = allow.sum(1)
    want = (allow.astype(np.float64) @ v[0]) / cnt[:, None]
    np.testing.assert_allclose(O[0], want, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L[0], np.log(cnt), rtol=0, atol=1e-13)
    if kind == "none":
        np.testing.assert_allclose(L[0], math.log(N), atol=1e-13)
    if kind == "causal":
        np.testing.assert_allclose(L[0], np.log(np.arange(1, N + 1)), atol=1e-13)


def test_single_key():
    d, scale = 16, 0.37
    q, k, v = rnd((3, 1, d), 12), rnd((3, 1, d), 13), rnd((3, 1, d), 14)
    O, L = oracle.fwd(q, k, v, "none", scale=scale)
    np.testing.assert_array_equal(O, v)
    np.testing.assert_allclose(L[:, 0], scale * (q[:, 0] * k[:, 0]).sum(-1), atol=1e-14)


def test_causal_row_zero():
    N, d, scale = 50, 16, 0.2
    q, k, v = rnd((1, N, d), 15), rnd((1, N, d), 16), rnd((1, N, d), 17)
    O, L = oracle.fwd(q, k, v, "causal", scale=scale)
    np.testing.assert_array_equal(O[0, 0], v[0, 0])
    assert abs(L[0, 0] - scale * q[0, 0] @ k[0, 0]) < 1e-14


def test_empty_row_convention():
    # a block mask with an empty block row: those queries see nothing
    N, d, block = 8, 4, 4
    bm = np.array([[0, 0], [1, 1]], dtype=np.uint8)
    q, k, v, do = (rnd((1, N, d), s) for s in (18, 19, 20, 21))
    O, L = oracle.fwd(q, k, v, "block", bm, 0.5, block=block)
    assert (O[0, :4] == 0).all() and np.isneginf(L[0, :4]).all()
    g = oracle.bwd(q, k, v, do, "block", bm, 0.5, block=block)
    assert (g["dQ"][0, :4] == 0).all()
    assert np.isfinite(g["dK"]).all() and np.isfinite(g["dV"]).all()


# -------------------------------------------------------- invariants -------

def test_key_permutation_and_query_permutation():
    N, d, scale = 120, 12, 0.25
    q, k, v = rnd((1, N, d), 22), rnd((1, N, d), 23), rnd((1, N, d), 24)
    O, L = oracle.fwd(q, k, v, "none", scale=scale)
    p = np.random.default_rng(25).permutation(N)
    O2, L2 = oracle.fwd(q, k[:, p], v[:, p], "none", scale=scale)
    np.testing.assert_allclose(O2, O, atol=1e-13)
    np.testing.assert_allclose(L2, L, atol=1e-13)
    O3, L3 = oracle.fwd(q[:, p], k, v, "none", scale=scale)
    np.testing.assert_allclose(O3, O[:, p], atol=1e-13)
    np.testing.assert_allclose(L3, L[:, p], atol=1e-13)


@pytest.mark.parametrize("kind", KINDS)
def test_key_shift_invariance(kind):
    N, d, scale, block = 96, 8, 0.4, 32
    q, k, v = rnd((1, N, d), 26), rnd((1, N, d), 27), rnd((1, N, d), 28)
    bm = small_mask(N, block, 29) if kind == "block" else None
    c = rnd((d,), 30)
    O, L = oracle.fwd(q, k, v, kind, bm, scale, block=block)
    O2, L2 = oracle.fwd(q, k + c, v, kind, bm, scale, block=block)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L + scale * (q[0] @ c), atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_value_affine_equivariance(kind):
    N, d, scale, block = 96, 8, 0.4, 32
    q, k, v = rnd((1, N, d), 31), rnd((1, N, d), 32), rnd((1, N, d), 33)
    bm = small_mask(N, block, 34) if kind == "block" else None
    A, b = rnd((d, d), 35), rnd((d,), 36)
    O, _ = oracle.fwd(q, k, v, kind, bm, scale, block=block)
    O2, _ = oracle.fwd(q, k, v @ A + b, kind, bm, scale, block=block)
    np.testing.assert_allclose(O2[0], O[0] @ A + b, atol=1e-12)


# ---------------------------------------------------------- gradients ------

@pytest.mark.parametrize("kind", KINDS)
def test_gradients_by_finite_differences(kind):
    N, d, scale, block, h = 12, 6, 0.7, 4, 1e-6
    q, k, v, do = (rnd((1, N, d), s) for s in (37, 38, 39, 40))
    bm = small_mask(N, block, 41) if kind == "block" else None

    def loss(q_, k_, v_):
        O, _ = oracle.fwd(q_, k_, v_, kind, bm, scale, block=block)
        return float((O * do).sum())

    g = oracle.bwd(q, k, v, do, kind, bm, scale, block=block)
    for name, idx in (("dQ", 0), ("dK", 1), ("dV", 2)):
        fd = np.zeros((N, d))
        for i in range(N):
            for c in range(d):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[idx][0, i, c] += h
                args_m[idx][0, i, c] -= h
                fd[i, c] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        ref = g[name][0]
        err = np.abs(fd - ref).max() / max(1e-30, np.abs(ref).max())
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("kind", KINDS)
def test_gradient_identities(kind):
    N, d, scale, block = 160, 16, 0.3, 64
    q, k, v, do = (rnd((2, N, d), s) for s in (42, 43, 44, 45))
    bm = small_mask(N, block, 46) if kind == "block" else None
    g = oracle.bwd(q, k, v, do, kind, bm, scale, block=block)
    # rows of dS sum to zero => sum_j dK_j = 0
    np.testing.assert_allclose(g["dK"].sum(1), 0.0, atol=1e-12)
    # rows of P sum to one => sum_j dV_j = sum_i dO_i
    np.testing.assert_allclose(g["dV"].sum(1), do.sum(1), atol=1e-11)
    # D_i = dO_i . O_i
    np.testing.assert_allclose(g["D"], (do * g["O"]).sum(-1), atol=1e-12)
    O, L = oracle.fwd(q, k, v, kind, bm, scale, block=block)
    np.testing.assert_allclose(g["O"], O, atol=1e-13)
    np.testing.assert_allclose(g["LSE"], L, atol=1e-13)


# -------------------------------------------- independent library check ----

@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("shape", [(1, 3, 128, 64), (2, 2, 200, 32)])
def test_against_torch_sdpa_fp64(kind, shape):
    B, H, N, d = shape
    block = 64
    scale = 0.125
    g = torch.Generator().manual_seed(47)
    q, k, v, do = (torch.randn(shape, generator=g, dtype=torch.float64) for _ in range(4))
    bm = small_mask(N, block, 48) if kind == "block" else None
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    if kind == "none":
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    elif kind == "causal":
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    else:
        am = torch.from_numpy(allowed_matrix(N, 2, bm, block))
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    out.backward(do)
    O, L = oracle.fwd(q, k, v, kind, bm, scale, block=block)
    np.testing.assert_allclose(O, out.detach().numpy(), atol=1e-10)
    gr = oracle.bwd(q, k, v, do, kind, bm, scale, block=block)
    for name, t in (("dQ", qt), ("dK", kt), ("dV", vt)):
        np.testing.assert_allclose(gr[name], t.grad.numpy(), atol=1e-10, err_msg=name)
    # LSE against a direct logsumexp of the masked scores
    s = scale * torch.einsum("bhid,bhjd->bhij", q, k)
    allow = torch.from_numpy(allowed_matrix(N, KIND_ID[kind], bm, block))
    lse = torch.logsumexp(s.masked_fill(~allow, float("-inf")), dim=-1)
    np.testing.assert_allclose(L, lse.numpy(), atol=1e-12)


# ---------------------------------------------------------- row path -------

@pytest.mark.parametrize("kind", KINDS)
def test_row_path_matches_full_path(kind):
    B, H, N, d, block = 2, 2, 260, 32, 128
    q, k, v, do = (rnd((B, H, N, d), s) for s in (49, 50, 51, 52))
    bm = small_mask(N, block, 53) if kind == "block" else None
    g = oracle.bwd(q, k, v, do, kind, bm, 0.2, block=block)
    heads = [0, 1, 3, 2, 3]
    rows = [0, 259, 128, 77, 129]
    O, L, dQ = oracle.rows(q, k, v, heads, rows, dO=do, mask_kind=kind, block_mask=bm,
                           scale=0.2, block=block)
    fO = g["O"].reshape(B * H, N, d)
    fL = g["LSE"].reshape(B * H, N)
    fdQ = g["dQ"].reshape(B * H, N, d)
    for r, (h, i) in enumerate(zip(heads, rows)):
        np.testing.assert_allclose(O[r], fO[h, i], atol=1e-13)
        np.testing.assert_allclose(L[r], fL[h, i], atol=1e-13)
        np.testing.assert_allclose(dQ[r], fdQ[h, i], atol=1e-13)


@pytest.mark.parametrize("kind", KINDS)
def test_col_path_matches_full_path(kind):
    """The key-column sampler (used for sampled dK, dV parity at full size)
    against the full backward: first, last and tile-boundary keys, repeated
    heads and keys in any order."""
    B, H, N, d, block = 2, 2, 260, 32, 128
    q, k, v, do = (rnd((B, H, N, d), s) for s in (54, 55, 56, 57))
    bm = small_mask(N, block, 58) if kind == "block" else None
    g = oracle.bwd(q, k, v, do, kind, bm, 0.2, block=block)
    heads = [0, 1, 3, 2, 3, 0, 3]
    keys = [0, 259, 128, 77, 127, 259, 0]
    dK, dV = oracle.cols(q, k, v, do, heads, keys, mask_kind=kind, block_mask=bm, scale=0.2, block=block)
    fdK = g["dK"].reshape(B * H, N, d)
    fdV = g["dV"].reshape(B * H, N, d)
    for c, (h, j) in enumerate(zip(heads, keys)):
        np.testing.assert_allclose(dK[c], fdK[h, j], atol=1e-13)
        np.testing.assert_allclose(dV[c], fdV[h, j], atol=1e-13)


@pytest.mark.parametrize("Nq,Nk", [(77, 160), (160, 77)])
def test_col_path_against_torch_sdpa_fp64(Nq, Nk):
    """The key-column sampler against PyTorch's fp64 attention + autograd
    (bottom-right causal through torch.tril, queries and keys of different
    counts), independently of the oracle's full backward."""
    d, scale = 16, 0.3
    g = torch.Generator().manual_seed(80)
    q, do = (torch.randn((1, 2, Nq, d), generator=g, dtype=torch.float64) for _ in range(2))
    k, v = (torch.randn((1, 2, Nk, d), generator=g, dtype=torch.float64) for _ in range(2))
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    am = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
    live = am.any(dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    (out[:, :, live] * do[:, :, live]).sum().backward()
    heads = [0, 1, 1, 0]
    keys = [0, Nk - 1, Nk // 2, 63]
    dK, dV = oracle.cols(q, k, v, do * live[None, None, :, None], heads, keys, mask_kind="causal", scale=scale)
    for c, (h, j) in enumerate(zip(heads, keys)):
        np.testing.assert_allclose(dK[c], kt.grad[0, h, j].numpy(), atol=1e-10)
        np.testing.assert_allclose(dV[c], vt.grad[0, h, j].numpy(), atol=1e-10)


def test_bf16_inputs_are_widened_exactly():
    w = workloads.WORKLOADS["tiny"]
    x = workloads.make_inputs(w, seed=0)
    a = oracle._f64(x["Q"])
    np.testing.assert_array_equal(a, x["Q"].float().double().numpy())
    assert x["Q"].dtype == torch.bfloat16


# ------------------------------------ queries and keys of different counts --
# Causal with Nq != Nk is aligned at the bottom right: query i sees key j iff
# j <= i + (Nk - Nq) (the last query sees every key).

def test_cross_causal_suffix_equals_square_problem():
    """The last Nq queries of a square causal problem over Nk keys see exactly
    what Nq queries see against those Nk keys: O, LSE and dQ agree, and with
    dO zero on the other rows so do dK and dV."""
    Nk, Nq, d, scale = 40, 13, 8, 0.4
    q, k, v, do = (rnd((2, Nk, d), s) for s in (60, 61, 62, 63))
    do_sq = do.copy()
    do_sq[:, : Nk - Nq] = 0.0
    sq = oracle.bwd(q, k, v, do_sq, "causal", None, scale)
    cr = oracle.bwd(q[:, Nk - Nq:], k, v, do[:, Nk - Nq:], "causal", None, scale)
    for name in ("O", "dQ"):
        np.testing.assert_allclose(cr[name], sq[name][:, Nk - Nq:], atol=1e-13, err_msg=name)
    np.testing.assert_allclose(cr["LSE"], sq["LSE"][:, Nk - Nq:], atol=1e-13)
    for name in ("dK", "dV"):
        np.testing.assert_allclose(cr[name], sq[name], atol=1e-13, err_msg=name)


def test_cross_causal_more_queries_than_keys():
    """Nq > Nk: the first Nq - Nk queries see no key (O = 0, LSE = -inf, no
    gradient); the last Nk form the square causal problem over the keys."""
    Nk, Nq, d, scale = 9, 20, 6, 0.5
    q, do = rnd((1, Nq, d), 64), rnd((1, Nq, d), 65)
    k, v = rnd((1, Nk, d), 66), rnd((1, Nk, d), 67)
    cr = oracle.bwd(q, k, v, do, "causal", None, scale)
    sq = oracle.bwd(q[:, Nq - Nk:], k, v, do[:, Nq - Nk:], "causal", None, scale)
    e = Nq - Nk
    assert np.all(cr["O"][:, :e] == 0.0) and np.all(cr["dQ"][:, :e] == 0.0)
    assert np.all(np.isneginf(cr["LSE"][:, :e]))
    for name in ("O", "dQ"):
        np.testing.assert_allclose(cr[name][:, e:], sq[name], atol=1e-13, err_msg=name)
    for name in ("dK", "dV"):
        np.testing.assert_allclose(cr[name], sq[name], atol=1e-13, err_msg=name)


@pytest.mark.parametrize("Nk", [1, 5, 300])
def test_single_query_sees_every_key(Nk):
    """Decode shape: one query against Nk keys; under bottom-right causal it
    sees every key, so causal equals no mask."""
    d, scale = 16, 0.25
    q, do = rnd((3, 1, d), 68), rnd((3, 1, d), 69)
    k, v = rnd((3, Nk, d), 70), rnd((3, Nk, d), 71)
    a = oracle.bwd(q, k, v, do, "causal", None, scale)
    b = oracle.bwd(q, k, v, do, "none", None, scale)
    for name in ("O", "LSE", "dQ", "dK", "dV"):
        np.testing.assert_allclose(a[name], b[name], atol=0, err_msg=name)


@pytest.mark.parametrize("kind", ["none", "causal"])
@pytest.mark.parametrize("Nq,Nk", [(1, 300), (77, 160), (160, 77)])
def test_cross_against_torch_sdpa_fp64(kind, Nq, Nk):
    """PyTorch's fp64 attention with autograd; causal through a boolean mask
    from torch.tril with the diagonal shifted by Nk - Nq."""
    d, scale = 32, 0.2
    g = torch.Generator().manual_seed(72)
    q, do = (torch.randn((1, 2, Nq, d), generator=g, dtype=torch.float64) for _ in range(2))
    k, v = (torch.randn((1, 2, Nk, d), generator=g, dtype=torch.float64) for _ in range(2))
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    am = None
    if kind == "causal":
        am = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
    if am is not None and not am.any(dim=1).all():
        # PyTorch returns NaN for a row with no visible key; compare the rest
        live = am.any(dim=1)
    else:
        live = torch.ones(Nq, dtype=torch.bool)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale)
    (out[:, :, live] * do[:, :, live]).sum().backward()
    gr = oracle.bwd(q, k, v, do * live[None, None, :, None], kind, None, scale)
    np.testing.assert_allclose(gr["O"][:, :, live.numpy()], out.detach()[:, :, live].numpy(), atol=1e-10)
    for name, t in (("dQ", qt), ("dK", kt), ("dV", vt)):
        ref = t.grad.numpy()
        got = gr[name]
        if name == "dQ":
            ref, got = ref[:, :, live.numpy()], got[:, :, live.numpy()]
        np.testing.assert_allclose(got, ref, atol=1e-10, err_msg=name)


def test_cross_block_mask_is_query_blocks_by_key_blocks():
    """A block mask over Nq != Nk is ceil(Nq/b) x ceil(Nk/b): all ones equals
    no mask, and a mask keeping key block 2 only equals attention over the
    keys of that block."""
    Nq, Nk, d, b, scale = 200, 330, 8, 64, 0.3
    q, k, v = rnd((2, Nq, d), 73), rnd((2, Nk, d), 74), rnd((2, Nk, d), 75)
    nbq, nbk = -(-Nq // b), -(-Nk // b)
    ones = np.ones((nbq, nbk), np.uint8)
    O1, L1 = oracle.fwd(q, k, v, "block", ones, scale, block=b)
    O0, L0 = oracle.fwd(q, k, v, "none", None, scale)
    np.testing.assert_allclose(O1, O0, atol=0)
    np.testing.assert_allclose(L1, L0, atol=0)
    col = np.zeros((nbq, nbk), np.uint8)
    col[:, 2] = 1
    O2, L2 = oracle.fwd(q, k, v, "block", col, scale, block=b)
    O3, L3 = oracle.fwd(q, k[:, 2 * b:3 * b], v[:, 2 * b:3 * b], "none", None, scale)
    np.testing.assert_allclose(O2, O3, atol=1e-14)
    np.testing.assert_allclose(L2, L3, atol=1e-14)


def test_cross_gradients_by_finite_differences():
    Nq, Nk, d, scale, h = 5, 9, 4, 0.6, 1e-6
    q, do = rnd((1, Nq, d), 76), rnd((1, Nq, d), 77)
    k, v = rnd((1, Nk, d), 78), rnd((1, Nk, d), 79)

    def loss(q_, k_, v_):
        O, _ = oracle.fwd(q_, k_, v_, "causal", None, scale)
        return float((O * do).sum())

    g = oracle.bwd(q, k, v, do, "causal", None, scale)
    for name, idx, n in (("dQ", 0, Nq), ("dK", 1, Nk), ("dV", 2, Nk)):
        fd = np.zeros((n, d))
        for i in range(n):
            for c in range(d):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[idx][0, i, c] += h
                args_m[idx][0, i, c] -= h
                fd[i, c] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        ref = g[name][0]
        err = np.abs(fd - ref).max() / max(1e-30, np.abs(ref).max())
        assert err < 1e-6, (name, err)
