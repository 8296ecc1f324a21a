"""Blocked online-softmax attention in fp64 -- TEST INFRASTRUCTURE ONLY.

A restatement of the tiling + online-softmax idea in plain numpy, used to pin
the oracle's two-pass definition against the exactness claim: "FlashAttention:
making attention fast by respecting the memory hierarchy" (tiling paragraph
and the running-total analogy) and the Dao et al. summary page, section
"Softmax / tiling", say that visiting key/value blocks one at a time while
keeping a running normaliser yields the same softmax as seeing the whole row.

Per query row the state is (m, l, acc): the running max of the scaled
scores, the running sum of exp(score - m) and the running un-normalised
output.  A new block with scores s and values v updates it as
    m' = max(m, max s);  c = exp(m - m')
    l' = c l + sum exp(s - m');  acc' = c acc + exp(s - m') v
and at the end O = acc / l, LSE = m + ln l.  Blocks may come in any order.
"""
from __future__ import annotations

import numpy as np


def allowed_matrix(N: int, kind: int, block_mask=None, block: int = 128) -> np.ndarray:
    """Boolean [N, N] visibility: none / causal (j <= i) / block grid."""
    if kind == 0:
        return np.ones((N, N), dtype=bool)
    if kind == 1:
        return np.tril(np.ones((N, N), dtype=bool))
    bm = np.asarray(block_mask, dtype=bool)
    idx = np.arange(N) // block
    return bm[idx[:, None], idx[None, :]]


def attention_online(q, k, v, scale, kind=0, block_mask=None, block=128,
                     tile_m=64, tile_n=64, order=None):
    """One head: q, k, v fp64 [N, d].  Returns O [N, d], LSE [N].

    ``tile_m`` / ``tile_n`` are the query / key tile sizes; ``order`` is an
    optional permutation of the key-tile indices (visiting order)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, d = q.shape
    allow = allowed_matrix(N, kind, block_mask, block)
    n_kt = (N + tile_n - 1) // tile_n
    order = range(n_kt) if order is None else order
    O = np.zeros((N, d))
    LSE = np.full(N, -np.inf)
    for i0 in range(0, N, tile_m):
        i1 = min(N, i0 + tile_m)
        m = np.full(i1 - i0, -np.inf)
        l = np.zeros(i1 - i0)
        acc = np.zeros((i1 - i0, d))
        for t in order:
            j0, j1 = t * tile_n, min(N, (t + 1) * tile_n)
            s = scale * (q[i0:i1] @ k[j0:j1].T)
            s = np.where(allow[i0:i1, j0:j1], s, -np.inf)
            m_new = np.maximum(m, s.max(axis=1))
            live = m_new > -np.inf                      # rows that have seen a key
            safe = np.where(live, m_new, 0.0)
            c = np.where(live, np.exp(np.where(live, m - safe, 0.0)), 1.0)
            p = np.where(np.isfinite(s), np.exp(s - safe[:, None]), 0.0)
            l = c * l + p.sum(axis=1)
            acc = c[:, None] * acc + p @ v[j0:j1]
            m = m_new
        live = l > 0
        O[i0:i1] = np.where(live[:, None], acc / np.where(live, l, 1.0)[:, None], 0.0)
        LSE[i0:i1] = np.where(live, m + np.log(np.where(live, l, 1.0)), -np.inf)
    return O, LSE
