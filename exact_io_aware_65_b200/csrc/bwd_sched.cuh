// bwd_sched.cuh -- the backward main kernel's launch parameters and its
// work schedule: which (head, key tile) a work item is, which query tiles it
// visits, and, for the deterministic dQ, the place of each (key tile, query
// tile) addition in the fixed order.  The kernel in fa_bwd.cu runs these
// functions in every role; they are host-callable too, so that a host test
// can walk the schedule of any problem and compare it with the visibility
// rule.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fa.h"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int BK = 128;  // keys per work item
constexpr int BQ = 128;  // queries per step

struct Params {
  int BH, N, Npad, nq, n_items, mask_kind;  // N, Npad, nq: query rows, padded rows, tiles
  int Nk, nk, off;  // key rows and tiles; causal: query i sees keys j <= i + off
  const uint8_t* block_mask;
  float scale, scale_log2;
  const float* Dw;
  const float* L2w;
  float* dq_acc;
  int H;             // heads per batch element
  const int* seqlens_q;  // optional per-batch-element lengths (device int [B])
  const int* seqlens_k;
  uint32_t* sched;
  uint32_t* turn;     // [BH, nq] dQ addition counters (deterministic mode)
  int deterministic;  // add each query tile's dQ parts in key-tile order
  int group;  // heads per scheduling group
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  uint64_t timeout_ns;
  uint32_t* status;
};

// Heads per scheduling group.  The group's Q and dO tiles (bf16) and fp32
// dQ accumulator rows are the backward's working set in L2, kept to about
// 64 MiB; at least 8 heads, or all of them (short sequences: one group,
// whose longest-first order then evens out the CTAs' work).
__host__ __device__ inline int sched_group(int BH, int N, int d) {
  const long long per_head = 8LL * (N > 0 ? N : 1) * d;  // Q, dO bf16 and the fp32 dQ rows
  const long long fit = (64LL << 20) / per_head;
  const long long g = fit > 8 ? fit : 8;
  return (int)(g < BH ? g : BH);
}

struct Item {
  int bh, j;
  int Lq, Lk, off, nqb;  // this sequence's query rows and keys, causal offset, query tiles
};

// Work item idx -> (head, key tile).  Heads are taken in groups of
// p.group, so the query-side tiles and dQ rows in flight at any time belong
// to a few heads and stay in L2; within a group low key tiles come first
// (under a causal mask they meet the most query tiles and run longest).

template <bool VARLEN>
__host__ __device__ __forceinline__ Item item_at(const Params& p, int idx) {
  const int per_group = p.group * p.nk;
  const int g = idx / per_group, r = idx % per_group;
  const int gsize = min(p.group, p.BH - g * p.group);
  Item it;
  it.j = r / gsize;
  it.bh = g * p.group + r % gsize;
  if (VARLEN) {
    const int b = it.bh / p.H;
    const bool bok = FA_IN_BOUNDS(p.status, b, 1, p.BH / p.H);
    it.Lq = p.seqlens_q ? (bok ? min(max(ld_ro(p.seqlens_q + b), 0), p.N) : 0) : p.N;
    it.Lk = p.seqlens_k ? (bok ? min(max(ld_ro(p.seqlens_k + b), 0), p.Nk) : 0) : p.Nk;
    it.off = it.Lk - it.Lq;
    it.nqb = (it.Lq + BQ - 1) / BQ;
  } else {  // every sequence fills its slice: the launch's own sizes
    it.Lq = p.N;
    it.Lk = p.Nk;
    it.off = p.off;
    it.nqb = p.nq;
  }
  return it;
}

// Deterministic dQ: the part of key tile j for query tile i is added only
// once the key tiles before it that see query tile i have added theirs, so
// every dQ element is summed in ascending key-tile order.  Its position in
// that order:
__host__ __device__ __forceinline__ uint32_t add_rank(const Params& p, int j, int i) {
  if (p.mask_kind == FA_MASK_BLOCK) {
    uint32_t r = 0;
    for (int k = 0; k < j; ++k)
      r += FA_IN_BOUNDS(p.status, (size_t)i * p.nk + k, 1, (size_t)p.nq * p.nk) &&
           ld_ro(p.block_mask + (size_t)i * p.nk + k) != 0;
    return r;
  }
  // no mask, or causal: a lower key tile is visible to every query row that
  // sees a higher one, so all j tiles before this one see query tile i
  return (uint32_t)j;
}

// Next query tile >= i of the sequence that attends to key tile j (p.nq if
// none; a key tile past the sequence's keys has none).  Causal: the rows
// that see some key of tile j are those >= j * BK - off.
template <bool VARLEN>
__host__ __device__ __forceinline__ int next_q(const Params& p, const Item& it, int i) {
  const int j = it.j;
  if (VARLEN && j * BK >= it.Lk) return p.nq;
  if (p.mask_kind == FA_MASK_CAUSAL) {
    const int first = max(0, j * BK - it.off) / BQ;
    if (i < first) i = first;
  } else if (p.mask_kind == FA_MASK_BLOCK) {
    for (; i < it.nqb; ++i)
      if (FA_IN_BOUNDS(p.status, (size_t)i * p.nk + j, 1, (size_t)p.nq * p.nk) &&
          ld_ro(p.block_mask + (size_t)i * p.nk + j))
        break;
  }
  return (!VARLEN || i < it.nqb) ? i : p.nq;
}

}  // namespace bwd
}  // namespace fa
