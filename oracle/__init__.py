"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It is independent of the CUDA library:
no shared code, headers, helpers or constants.

The arithmetic lives in ``oracle.c`` (naive attention and its gradient, fp64,
see that file's header for the definition and the passages it follows).  This
module only marshals arrays: any tensor is widened to fp64 (bf16 -> fp64 is
exact, so the oracle sees the very bits the GPU sees) and laid out
[B*H, N, d].

``online.py`` holds the blocked online-softmax restatement used to pin the
exactness claim against this two-pass definition.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import build as _build

MASK_NONE, MASK_CAUSAL, MASK_BLOCK = 0, 1, 2
_KINDS = {"none": MASK_NONE, "causal": MASK_CAUSAL, "block": MASK_BLOCK}

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_ip = ctypes.POINTER(ctypes.c_int)


def load(path: str):
    """Open an oracle shared library and declare its C signatures."""
    L = ctypes.CDLL(path)
    i, d = ctypes.c_int, ctypes.c_double
    L.oracle_num_threads.restype = i
    L.oracle_fwd.argtypes = [_dp, _dp, _dp, i, i, i, i, _u8p, i, d, _dp, _dp]
    L.oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, _u8p, i, d,
                             _dp, _dp, _dp, _dp, _dp, _dp]
    L.oracle_rows.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, _u8p, i, d,
                              _ip, _ip, i, _dp, _dp, _dp]
    L.oracle_probs.argtypes = [_dp, _dp, i, i, i, i, _u8p, i, d, _dp]
    # the same four with separate query and key counts (Nq, Nk)
    L.oracle_fwd_qk.argtypes = [_dp, _dp, _dp, i, i, i, i, i, _u8p, i, d, _dp, _dp]
    L.oracle_bwd_qk.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, i, _u8p, i, d,
                                _dp, _dp, _dp, _dp, _dp, _dp]
    L.oracle_rows_qk.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, i, _u8p, i, d,
                                 _ip, _ip, i, _dp, _dp, _dp]
    L.oracle_probs_qk.argtypes = [_dp, _dp, i, i, i, i, i, _u8p, i, d, _dp]
    L.oracle_cols_qk.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, i, _u8p, i, d,
                                 _ip, _ip, i, _dp, _dp]
    for f in (L.oracle_fwd, L.oracle_bwd, L.oracle_rows, L.oracle_probs,
              L.oracle_fwd_qk, L.oracle_bwd_qk, L.oracle_rows_qk, L.oracle_probs_qk,
              L.oracle_cols_qk):
        f.restype = i
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


class using:
    """Context manager that routes every call of this module to another
    build of the oracle (the mutation tests plant mistakes that way)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _f64(x) -> np.ndarray:
    """Widen to a C-contiguous fp64 numpy array (exact for bf16/fp32 input)."""
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _mask_args(mask, kind):
    kind = _KINDS.get(kind, kind)
    if kind == MASK_BLOCK:
        if isinstance(mask, torch.Tensor):
            mask = mask.detach().cpu().numpy()
        m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
        return kind, m, m.ctypes.data_as(_u8p)
    return kind, None, None


def _shape(Q):
    *lead, N, d = Q.shape
    BH = int(np.prod(lead)) if lead else 1
    return tuple(lead), BH, N, d


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"oracle call failed with code {rc}")


def _nk(K, BH, d):
    _, bh, Nk, dk = _shape(K)
    if bh != BH or dk != d:
        raise ValueError("K must have the same heads and head dimension as Q")
    return Nk


def fwd(Q, K, V, mask_kind="none", block_mask=None, scale=None, block=128):
    """O [..., Nq, d] and LSE [..., Nq] in fp64 (K, V [..., Nk, d])."""
    q, k, v = _f64(Q), _f64(K), _f64(V)
    lead, BH, N, d = _shape(q)
    Nk = _nk(k, BH, d)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    kind, m, mp = _mask_args(block_mask, mask_kind)
    O = np.empty((BH, N, d))
    L = np.empty((BH, N))
    _check(lib().oracle_fwd_qk(_ptr(q), _ptr(k), _ptr(v), BH, N, Nk, d, kind, mp, block, scale,
                               _ptr(O), _ptr(L)))
    return O.reshape(*lead, N, d), L.reshape(*lead, N)


def bwd(Q, K, V, dO, mask_kind="none", block_mask=None, scale=None, block=128):
    """dict with dQ, O [..., Nq, d], dK, dV [..., Nk, d] and LSE, D [..., Nq]
    (fp64), all recomputed."""
    q, k, v, do = _f64(Q), _f64(K), _f64(V), _f64(dO)
    lead, BH, N, d = _shape(q)
    Nk = _nk(k, BH, d)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    kind, m, mp = _mask_args(block_mask, mask_kind)
    out = {n: np.empty((BH, N if n in ("dQ", "O") else Nk, d)) for n in ("dQ", "dK", "dV", "O")}
    L = np.empty((BH, N))
    D = np.empty((BH, N))
    _check(lib().oracle_bwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(do), BH, N, Nk, d, kind, mp, block,
                               scale, _ptr(out["dQ"]), _ptr(out["dK"]), _ptr(out["dV"]),
                               _ptr(out["O"]), _ptr(L), _ptr(D)))
    res = {n: a.reshape(*lead, a.shape[1], d) for n, a in out.items()}
    res["LSE"] = L.reshape(*lead, N)
    res["D"] = D.reshape(*lead, N)
    return res


def rows(Q, K, V, heads, rws, dO=None, mask_kind="none", block_mask=None, scale=None,
         block=128):
    """O [R, d], LSE [R] (and dQ [R, d] when dO is given) for the query rows
    ``(heads[r], rws[r])``; ``heads`` index the flattened B*H axis."""
    q, k, v = _f64(Q), _f64(K), _f64(V)
    do = _f64(dO) if dO is not None else None
    lead, BH, N, d = _shape(q)
    Nk = _nk(k, BH, d)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    kind, m, mp = _mask_args(block_mask, mask_kind)
    hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    rs = np.ascontiguousarray(np.asarray(rws, dtype=np.int32))
    R = len(hs)
    O = np.empty((R, d))
    L = np.empty((R,))
    dQ = np.empty((R, d)) if do is not None else None
    _check(lib().oracle_rows_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(do), BH, N, Nk, d, kind, mp, block,
                                scale, hs.ctypes.data_as(_ip), rs.ctypes.data_as(_ip), R,
                                _ptr(O), _ptr(L), _ptr(dQ)))
    return (O, L, dQ) if do is not None else (O, L)


def cols(Q, K, V, dO, heads, keys, mask_kind="none", block_mask=None, scale=None, block=128):
    """dK [C, d] and dV [C, d] for the key rows ``(heads[c], keys[c])``;
    ``heads`` index the flattened B*H axis.  Costs one forward over the
    heads named, plus O(Nq d) per key."""
    q, k, v, do = _f64(Q), _f64(K), _f64(V), _f64(dO)
    lead, BH, N, d = _shape(q)
    Nk = _nk(k, BH, d)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    kind, m, mp = _mask_args(block_mask, mask_kind)
    hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    ks = np.ascontiguousarray(np.asarray(keys, dtype=np.int32))
    C = len(hs)
    dK = np.empty((C, d))
    dV = np.empty((C, d))
    _check(lib().oracle_cols_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(do), BH, N, Nk, d, kind, mp, block,
                                scale, hs.ctypes.data_as(_ip), ks.ctypes.data_as(_ip), C,
                                _ptr(dK), _ptr(dV)))
    return dK, dV


def probs(Q, K, mask_kind="none", block_mask=None, scale=None, block=128):
    """Softmax probabilities P [..., Nq, Nk] (small sizes only)."""
    q, k = _f64(Q), _f64(K)
    lead, BH, N, d = _shape(q)
    Nk = _nk(k, BH, d)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    kind, m, mp = _mask_args(block_mask, mask_kind)
    P = np.empty((BH, N, Nk))
    _check(lib().oracle_probs_qk(_ptr(q), _ptr(k), BH, N, Nk, d, kind, mp, block, scale, _ptr(P)))
    return P.reshape(*lead, N, Nk)
