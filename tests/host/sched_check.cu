// sched_check.cu -- the kernels' work schedules, walked on the host.
//
// The forward and backward kernels decide which tiles to compute with the
// functions in fwd_sched.cuh and bwd_sched.cuh (host-callable).  This program
// builds their launch parameters the way the launchers do, walks every work
// item exactly as the kernels' loops do, and compares what is visited with
// what the visibility rule requires, written row by row:
//   - every (head, query tile) of the forward belongs to exactly one item,
//     and every (head, key tile) of the backward is exactly one item;
//   - a query tile visits exactly the key tiles holding at least one
//     (row, key) pair that row may see, and the backward's key tile visits
//     exactly the query tiles with such a pair;
//   - for the deterministic backward, the place add_rank gives the addition of
//     key tile j to query tile i is the number of key tiles before j that
//     also visit i (the order the turn counters enforce).
// The visibility rule, per sequence of Lq query rows and Lk keys (padding
// beyond them sees and is seen by nothing): no mask, every key; causal, key c
// for row r iff c <= r + (Lk - Lq); block, the tile pair's mask entry.
//
// Usage: sched_check  -> runs a sweep of problem sizes, masks and lengths,
// prints "ok <cases>" and exits 0, or prints the first mismatch and exits 1.
#include <stdio.h>
#include <stdlib.h>

#include <vector>

#include "bwd_sched.cuh"
#include "fwd_sched.cuh"

namespace {

struct Problem {
  int B, H, Nq, Nk, kind;
  std::vector<uint8_t> mask;  // [nq, nk] for the block kind
  std::vector<int> lq, lk;    // per batch element; empty: full lengths
  bool varlen() const { return !lq.empty(); }
  int nq() const { return (Nq + 127) / 128; }
  int nk() const { return (Nk + 127) / 128; }
  int Lq(int b) const { return varlen() ? lq[b] : Nq; }
  int Lk(int b) const { return varlen() ? lk[b] : Nk; }
};

// Does tile pair (query tile i, key tile j) of batch element b hold a visible pair?
bool needed(const Problem& pr, int b, int i, int j) {
  const int Lq = pr.Lq(b), Lk = pr.Lk(b);
  const int r0 = i * 128, r1 = r0 + 128 < Lq ? r0 + 128 : Lq;  // real rows [r0, r1)
  const int c0 = j * 128, c1 = c0 + 128 < Lk ? c0 + 128 : Lk;  // real keys [c0, c1)
  if (r0 >= r1 || c0 >= c1) return false;
  if (pr.kind == FA_MASK_BLOCK) return pr.mask[(size_t)i * pr.nk() + j] != 0;
  if (pr.kind == FA_MASK_NONE) return true;
  for (int r = r0; r < r1; ++r)
    for (int c = c0; c < c1; ++c)
      if (c <= r + (Lk - Lq)) return true;
  return false;
}

uint32_t g_status = 0;
int g_fail = 0;

void fail(const char* what, const Problem& pr, int a, int b, int c) {
  if (g_fail++ == 0)
    printf("MISMATCH %s: B=%d H=%d Nq=%d Nk=%d kind=%d varlen=%d at (%d, %d, %d)\n", what, pr.B, pr.H, pr.Nq,
           pr.Nk, pr.kind, (int)pr.varlen(), a, b, c);
}

template <bool VARLEN>
void check_fwd(const Problem& pr, int tiles_per_item, int group) {
  using namespace fa::fwd;
  Params p = {};
  p.tiles_per_item = tiles_per_item;
  const int BH = pr.B * pr.H;
  p.BH = BH; p.N = pr.Nq; p.nq = pr.nq(); p.Nk = pr.Nk; p.nk = pr.nk(); p.off = pr.Nk - pr.Nq; p.H = pr.H;
  p.seqlens_q = VARLEN ? pr.lq.data() : nullptr;
  p.seqlens_k = VARLEN ? pr.lk.data() : nullptr;
  p.n_pairs = (p.nq + tiles_per_item - 1) / tiles_per_item;
  p.n_items = p.n_pairs * BH;
  p.group = group;
  p.mask_kind = pr.kind;
  p.block_mask = pr.kind == FA_MASK_BLOCK ? pr.mask.data() : nullptr;
  p.status = &g_status;
  std::vector<int> owner((size_t)BH * p.nq, 0);
  for (int idx = 0; idx < p.n_items; ++idx) {
    const Item it = item_at<VARLEN>(p, idx);
    if (it.bh < 0 || it.bh >= BH || it.q0 < 0 || it.q0 >= p.nq || (it.has1 && it.q1 >= p.nq)) {
      fail("fwd item out of range", pr, idx, it.bh, it.q0);
      return;
    }
    const int b = it.bh / pr.H;
    owner[(size_t)it.bh * p.nq + it.q0]++;
    if (it.has1) owner[(size_t)it.bh * p.nq + it.q1]++;
    // the key tiles each query tile computes: the union walk, filtered per tile
    const int e = kv_end<VARLEN>(p, it);
    if (e < 0 || e > p.nk) { fail("fwd kv_end out of range", pr, idx, e, 0); return; }
    std::vector<char> seen0(p.nk, 0), seen1(p.nk, 0);
    int last = -1;
    for (int j = next_union<VARLEN>(p, it, 0); j < e; j = next_union<VARLEN>(p, it, j + 1)) {
      if (j <= last) { fail("fwd key walk not increasing", pr, idx, j, last); return; }
      last = j;
      if (member<VARLEN>(p, it, it.q0, j)) seen0[j] = 1;
      if (it.has1 && member<VARLEN>(p, it, it.q1, j)) seen1[j] = 1;
    }
    for (int j = 0; j < p.nk; ++j) {
      if (seen0[j] != (char)needed(pr, b, it.q0, j)) fail("fwd key tiles of q0", pr, it.bh, it.q0, j);
      if (it.has1 && seen1[j] != (char)needed(pr, b, it.q1, j)) fail("fwd key tiles of q1", pr, it.bh, it.q1, j);
    }
  }
  for (size_t t = 0; t < owner.size(); ++t)
    if (owner[t] != 1) fail("fwd query tile not in exactly one item", pr, (int)(t / p.nq), (int)(t % p.nq), owner[t]);
}

template <bool VARLEN>
void check_bwd(const Problem& pr, int group) {
  using namespace fa::bwd;
  Params p = {};
  const int BH = pr.B * pr.H;
  p.BH = BH; p.N = pr.Nq; p.nq = pr.nq(); p.Npad = p.nq * 128; p.Nk = pr.Nk; p.nk = pr.nk();
  p.off = pr.Nk - pr.Nq; p.H = pr.H;
  p.seqlens_q = VARLEN ? pr.lq.data() : nullptr;
  p.seqlens_k = VARLEN ? pr.lk.data() : nullptr;
  p.n_items = BH * p.nk;
  p.mask_kind = pr.kind;
  p.block_mask = pr.kind == FA_MASK_BLOCK ? pr.mask.data() : nullptr;
  p.group = group;
  p.status = &g_status;
  std::vector<int> owner((size_t)BH * p.nk, 0);
  // visits[bh][i] = key tiles that visit query tile i, in ascending order
  std::vector<std::vector<int>> visits((size_t)BH * p.nq);
  for (int idx = 0; idx < p.n_items; ++idx) {
    const Item it = item_at<VARLEN>(p, idx);
    if (it.bh < 0 || it.bh >= BH || it.j < 0 || it.j >= p.nk) { fail("bwd item out of range", pr, idx, it.bh, it.j); return; }
    owner[(size_t)it.bh * p.nk + it.j]++;
    const int b = it.bh / pr.H;
    std::vector<char> seen(p.nq, 0);
    int last = -1;
    for (int i = next_q<VARLEN>(p, it, 0); i < p.nq; i = next_q<VARLEN>(p, it, i + 1)) {
      if (i <= last || i < 0) { fail("bwd query walk not increasing", pr, idx, i, last); return; }
      last = i;
      seen[i] = 1;
    }
    for (int i = 0; i < p.nq; ++i)
      if (seen[i] != (char)needed(pr, b, i, it.j)) fail("bwd query tiles of a key tile", pr, it.bh, i, it.j);
  }
  for (size_t t = 0; t < owner.size(); ++t)
    if (owner[t] != 1) fail("bwd key tile not in exactly one item", pr, (int)(t / p.nk), (int)(t % p.nk), owner[t]);
  // deterministic order: rank of (j, i) = key tiles before j that visit i
  for (int bh = 0; bh < BH; ++bh) {
    const int b = bh / pr.H;
    for (int i = 0; i < p.nq; ++i) {
      uint32_t before = 0;
      for (int j = 0; j < p.nk; ++j) {
        if (!needed(pr, b, i, j)) continue;
        if (add_rank(p, j, i) != before) fail("bwd add_rank", pr, bh, i, j);
        ++before;
      }
    }
  }
}

uint64_t g_rng = 88172645463325252ull;
uint32_t rnd() {  // xorshift64
  g_rng ^= g_rng << 13; g_rng ^= g_rng >> 7; g_rng ^= g_rng << 17;
  return (uint32_t)(g_rng >> 11);
}

}  // namespace

int main() {
  // The group sizes the launches choose for the benchmark shapes: 8 heads
  // where a head's tiles are large (long causal, block-sparse), every head
  // where they are small (BERT- and GPT-2-shaped).
  struct GroupCase { int BH, N, d, fwd, bwd; };
  const GroupCase gc[] = {{32, 8192, 128, 8, 8}, {8, 16384, 64, 8, 8}, {256, 512, 64, 256, 256},
                          {96, 1024, 64, 96, 96}, {3, 100, 64, 3, 3}, {1000, 65536, 128, 8, 8}};
  for (const GroupCase& c : gc) {
    const int f = fa::fwd::sched_group(c.BH, c.N, c.d), b = fa::bwd::sched_group(c.BH, c.N, c.d);
    if (f != c.fwd || b != c.bwd) {
      printf("MISMATCH group size for BH=%d N=%d d=%d: fwd %d (want %d), bwd %d (want %d)\n", c.BH, c.N, c.d, f,
             c.fwd, b, c.bwd);
      return 1;
    }
  }
  const int sizes[] = {1, 100, 127, 128, 129, 256, 300, 640, 1000};
  const int nsz = sizeof(sizes) / sizeof(sizes[0]);
  long cases = 0;
  for (int B : {1, 2, 3})
    for (int H : {1, 3})
      for (int a = 0; a < nsz; ++a)
        for (int c = 0; c < nsz; ++c)
          for (int kind = 0; kind < 3; ++kind)
            for (int var = 0; var < 2; ++var) {
              Problem pr;
              pr.B = B; pr.H = H; pr.Nq = sizes[a]; pr.Nk = sizes[c]; pr.kind = kind;
              if (kind == FA_MASK_BLOCK) {
                pr.mask.resize((size_t)pr.nq() * pr.nk());
                for (auto& m : pr.mask) m = (rnd() % 10) < 4;   // may leave rows or columns empty
              }
              if (var) {
                for (int b = 0; b < B; ++b) {
                  const uint32_t u = rnd() % 4;   // empty, full, or random lengths
                  pr.lq.push_back(u == 0 ? 0 : u == 1 ? pr.Nq : (int)(rnd() % (pr.Nq + 1)));
                  pr.lk.push_back(u == 0 ? pr.Nk : u == 1 ? pr.Nk : (int)(rnd() % (pr.Nk + 1)));
                }
              }
              // the launches' own group sizes for this shape lie in [1, BH];
              // the schedules are walked for those and for every other size
              // from one head to all of them
              const int BH = B * H;
              const int own[] = {fa::fwd::sched_group(BH, pr.Nk, 64), fa::fwd::sched_group(BH, pr.Nk, 128),
                                 fa::bwd::sched_group(BH, pr.Nq, 64), fa::bwd::sched_group(BH, pr.Nq, 128)};
              for (int g : own)
                if (g < 1 || g > BH) { fail("group size out of range", pr, g, BH, 0); return 1; }
              for (int g = 1; g <= BH; ++g) {
                if (var) {
                  check_fwd<true>(pr, 2, g);
                  check_fwd<true>(pr, 1, g);
                  check_bwd<true>(pr, g);
                } else {
                  check_fwd<false>(pr, 2, g);
                  check_fwd<false>(pr, 1, g);
                  check_bwd<false>(pr, g);
                }
              }
              ++cases;
              if (g_fail) return 1;
            }
  if (g_status != 0) {
    printf("an index check recorded a failure\n");
    return 1;
  }
  printf("ok %ld\n", cases);
  return 0;
}
