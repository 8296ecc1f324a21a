"""Seeded synthetic workloads for exact attention.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic.  Both sides of every parity check (the CUDA library and
the fp64 oracle) take their inputs from here, so the two see the same bits.

Shapes follow the workloads the FlashAttention pages quote: BERT-large at
sequence 512 and GPT-2 at sequence 1K ("Paper Abstract" of the Dao et al.
summary page), a long causal context, and a long block-sparse sequence in the
spirit of Path-X (sequence 16K, same abstract).  No dataset is used: Q, K, V
and dO are i.i.d. N(0, 1) draws rounded to bf16.

Recipe (fixed, so results are reproducible):
  * ``torch.Generator('cpu').manual_seed(seed)``; fp32 ``randn`` of shape
    [B, H, N, d] drawn in the order Q, K, V, dO; each cast to bf16 with
    round-to-nearest-even.
  * Block mask (kind ``"block"``): a second generator seeded with
    ``seed + 1``; ``rand(nb, nb) < p_keep`` with ``nb = ceil(N / 128)``; the
    diagonal blocks are then forced to 1 so that no query row is empty.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BLOCK = 128          # block-mask granularity on both axes
P_KEEP = 0.25        # probability that an off-diagonal block is kept

MASK_NONE, MASK_CAUSAL, MASK_BLOCK = 0, 1, 2
MASK_KINDS = {"none": MASK_NONE, "causal": MASK_CAUSAL, "block": MASK_BLOCK}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    mask: str          # "none" | "causal" | "block"
    scale: float       # the fp32 value handed to the kernels

    @property
    def mask_kind(self) -> int:
        return MASK_KINDS[self.mask]

    @property
    def nb(self) -> int:
        return (self.N + BLOCK - 1) // BLOCK

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _f32(x: float) -> float:
    return float(torch.tensor(x, dtype=torch.float32).item())


# The five workloads, smallest first.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 64, "none", _f32(1 / math.sqrt(64))),
    "bert_large_s512": Workload("bert_large_s512", 16, 16, 512, 64, "none", _f32(1 / 8)),
    "gpt2_s1k_causal": Workload("gpt2_s1k_causal", 8, 12, 1024, 64, "causal", _f32(1 / 8)),
    "long_s8k_d128_causal": Workload("long_s8k_d128_causal", 2, 16, 8192, 128, "causal",
                                     _f32(1 / math.sqrt(128))),
    # The scale is not given for this shape; 1/sqrt(d) = 1/8 is the plain reading.
    "block_sparse_s16k": Workload("block_sparse_s16k", 1, 8, 16384, 64, "block", _f32(1 / 8)),
}
ORDER = list(WORKLOADS)


def block_mask(nb: int, seed: int, p_keep: float = P_KEEP) -> torch.Tensor:
    """uint8 [nb, nb] block mask, 1 = keep; diagonal always kept."""
    g = torch.Generator("cpu").manual_seed(seed + 1)
    m = (torch.rand(nb, nb, generator=g) < p_keep).to(torch.uint8)
    m.fill_diagonal_(1)
    return m.contiguous()


def make_inputs(w: Workload, seed: int = 0, grad: bool = True) -> dict:
    """Q, K, V (and dO when ``grad``) as contiguous bf16 CPU tensors [B,H,N,d],
    plus ``mask`` (uint8 [nb, nb] or None)."""
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    for name in ("Q", "K", "V", "dO") if grad else ("Q", "K", "V"):
        out[name] = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()
    out["mask"] = block_mask(w.nb, seed) if w.mask == "block" else None
    return out


def make_cross_inputs(B: int, H: int, Nq: int, Nk: int, d: int, mask: str, seed: int = 0) -> dict:
    """Queries and keys of different counts: Q, dO [B,H,Nq,d] and K, V
    [B,H,Nk,d], bf16 CPU, drawn like ``make_inputs`` in the order Q, K, V, dO;
    ``mask`` a uint8 [ceil(Nq/128), ceil(Nk/128)] grid for kind "block"
    (generator seed + 1, keep probability P_KEEP, no forced blocks), else
    None."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = {}
    for name, n in (("Q", Nq), ("K", Nk), ("V", Nk), ("dO", Nq)):
        out[name] = torch.randn((B, H, n, d), generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()
    if mask == "block":
        gm = torch.Generator("cpu").manual_seed(seed + 1)
        nbq, nbk = (Nq + BLOCK - 1) // BLOCK, (Nk + BLOCK - 1) // BLOCK
        out["mask"] = (torch.rand(nbq, nbk, generator=gm) < P_KEEP).to(torch.uint8).contiguous()
    else:
        out["mask"] = None
    return out


def kept_blocks(w: Workload, mask: torch.Tensor | None) -> int:
    """Number of 128x128 (or ragged-edge) score tiles a query attends to, summed
    over query tiles.  Pure counting, used for FLOP accounting."""
    nb = w.nb
    if w.mask == "none":
        return nb * nb
    if w.mask == "causal":
        return nb * (nb + 1) // 2
    return int(mask.sum().item())


def kept_entries(w: Workload, mask: torch.Tensor | None) -> int:
    """E: kept score entries per head (the algorithmic work unit).
    none: N^2; causal: N(N+1)/2; block: entries inside kept blocks."""
    N = w.N
    if w.mask == "none":
        return N * N
    if w.mask == "causal":
        return N * (N + 1) // 2
    nb = w.nb
    sizes = torch.full((nb,), BLOCK, dtype=torch.int64)
    sizes[-1] = N - BLOCK * (nb - 1)
    m = mask.to(torch.int64)
    return int((sizes[:, None] * sizes[None, :] * m).sum().item())
