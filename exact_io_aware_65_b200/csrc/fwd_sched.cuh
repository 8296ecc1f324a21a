// fwd_sched.cuh -- the forward's launch parameters and its work schedule:
// which (head, query-tile pair) a work item is, and which key tiles each
// query tile of it visits.  The kernel in fa_fwd.cu runs these functions in
// every role; they are host-callable too, so that a host test can walk the
// schedule of any problem and compare it with the visibility rule.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fa.h"
#include "sm100.cuh"

namespace fa {
namespace fwd {

constexpr int BM = 128;              // query rows per tile
constexpr int BN = 128;              // keys per tile

struct Params {
  int BH, N, nq, n_pairs, n_items, mask_kind;  // N, nq: query rows and tiles
  // Query tiles per work item: 2 (a pair, n_pairs = ceil(nq / 2)) or 1
  // (n_pairs = nq: one tile per item).
  int tiles_per_item;
  int Nk, nk, off;  // key rows and tiles; causal: query i sees keys j <= i + off
  int H;            // heads per batch element (a head's batch element is bh / H)
  // Optional per-batch-element lengths (device int [B], nullptr: N and Nk):
  // query rows and keys at or past them are padding.
  const int* seqlens_q;
  const int* seqlens_k;
  int group;  // heads per scheduling group
  const uint8_t* block_mask;
  float scale_log2;
  __nv_bfloat16* O;
  float* LSE;
  uint64_t timeout_ns;
  uint32_t* status;
  uint32_t slot;  // scheduler counter slot of this launch
};

// Heads per scheduling group.  The group's K and V tiles are the forward's
// working set in L2, kept to about 32 MiB; above that, more heads per group
// spread the longest-first order over more items, which evens out the CTAs'
// work under a causal mask (short sequences: all heads in one group).  At
// least 8 heads, or all of them.
__host__ __device__ inline int sched_group(int BH, int Nk, int d) {
  const long long per_head = 4LL * (Nk > 0 ? Nk : 1) * d;  // K and V, bf16
  const long long fit = (32LL << 20) / per_head;
  const long long g = fit > 8 ? fit : 8;
  return (int)(g < BH ? g : BH);
}

struct Item {
  int bh, q0, q1;
  bool has1;
  int Lq, Lk, off, nkb;  // this sequence's query rows and keys, causal offset, key tiles
};

// Work item idx -> (head, pair of query tiles, or one query tile).  Heads are taken in groups
// of p.group so that the K/V tiles in flight belong to a few heads and stay
// in L2; within a group later query tiles come first, so that under a causal
// mask the longest items start earliest (and, claimed dynamically, the short
// ones fill in at the end).
template <bool VARLEN>
__host__ __device__ __forceinline__ Item item_at(const Params& p, int idx) {
  Item it;
  const int per_group = p.group * p.n_pairs;
  const int g = idx / per_group, r = idx % per_group;
  const int gsize = min(p.group, p.BH - g * p.group);
  const int c = p.n_pairs - 1 - r / gsize;
  it.bh = g * p.group + r % gsize;
  it.q0 = p.tiles_per_item * c;
  it.q1 = it.q0 + 1;
  it.has1 = p.tiles_per_item == 2 && it.q1 < p.nq;
  if (VARLEN) {
    const int b = it.bh / p.H;
    const bool bok = FA_IN_BOUNDS(p.status, b, 1, p.BH / p.H);
    it.Lq = p.seqlens_q ? (bok ? min(max(ld_ro(p.seqlens_q + b), 0), p.N) : 0) : p.N;
    it.Lk = p.seqlens_k ? (bok ? min(max(ld_ro(p.seqlens_k + b), 0), p.Nk) : 0) : p.Nk;
    it.off = it.Lk - it.Lq;
    it.nkb = (it.Lk + BN - 1) / BN;
  } else {  // every sequence fills its slice: the launch's own sizes
    it.Lq = p.N;
    it.Lk = p.Nk;
    it.off = p.off;
    it.nkb = p.nk;
  }
  return it;
}

// Last key a query row of tile qt may see under the causal mask (the tile's
// last row of the sequence, shifted by the alignment; negative: none).
__host__ __device__ __forceinline__ int causal_last_key(const Item& it, int qt) {
  return min(qt * BM + BM - 1, it.Lq - 1) + it.off;
}

// Does query tile qt attend to key tile j?  (With per-sequence lengths,
// tiles past the sequence's query rows or keys attend to nothing; without,
// every tile an item or a key loop reaches is inside.)
template <bool VARLEN>
__host__ __device__ __forceinline__ bool member(const Params& p, const Item& it, int qt, int j) {
  if (VARLEN && (qt * BM >= it.Lq || j >= it.nkb)) return false;
  if (p.mask_kind == FA_MASK_CAUSAL) return j * BN <= causal_last_key(it, qt);
  if (p.mask_kind == FA_MASK_BLOCK)
    return FA_IN_BOUNDS(p.status, (size_t)qt * p.nk + j, 1, (size_t)p.nq * p.nk) &&
           ld_ro(p.block_mask + (size_t)qt * p.nk + j) != 0;
  return true;
}

// One past the last key tile either query tile of the item may need.
template <bool VARLEN>
__host__ __device__ __forceinline__ int kv_end(const Params& p, const Item& it) {
  if (VARLEN && it.q0 * BM >= it.Lq) return 0;
  if (p.mask_kind == FA_MASK_CAUSAL) {
    const int last = causal_last_key(it, (it.has1 && (!VARLEN || it.q1 * BM < it.Lq)) ? it.q1 : it.q0);
    return last < 0 ? 0 : min(it.nkb, last / BN + 1);
  }
  return it.nkb;
}

// Next key tile >= j needed by either query tile of the item (kv_end if none).
template <bool VARLEN>
__host__ __device__ __forceinline__ int next_union(const Params& p, const Item& it, int j) {
  const int e = kv_end<VARLEN>(p, it);
  if (p.mask_kind != FA_MASK_BLOCK) return j < e ? j : e;
  for (; j < e; ++j)
    if (member<VARLEN>(p, it, it.q0, j) || (it.has1 && member<VARLEN>(p, it, it.q1, j))) return j;
  return e;
}

}  // namespace fwd
}  // namespace fa
