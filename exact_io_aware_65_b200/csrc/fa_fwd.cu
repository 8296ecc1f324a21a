// fa_fwd.cu -- forward pass of exact attention on sm_100a.
//
// The method ("FlashAttention: making attention fast by respecting the memory
// hierarchy", tiling paragraph; "FlashAttention: Fast and Memory-Efficient
// Exact Attention with IO-Awareness", sections "Softmax / tiling" and
// "Implementation"): load a block of queries, stream blocks of keys and
// values past it, and keep a running row maximum and row sum so that the
// softmax is completed incrementally; the N x N scores live only on chip.
//
// B200 mapping (one persistent CTA per SM, 384 threads), d = 128:
//   warp 0        TMA producer: two 128-row Q tiles per work item, then a ring
//                 of K and V tiles (128 keys x d, 128-byte swizzle).
//   warps 1(, 2)  MMA issuer(s), one thread each (Cfg::ISSUERS): S_t = Q_t K_j^T
//                 into tensor memory (fp32), and O_t += P_t V_j with P_t read
//                 from tensor memory.
//   warps 4..7    softmax for query tile 0; warps 8..11 for query tile 1.
//                 Thread r owns query row r: it reads its score row from
//                 tensor memory, keeps the row max m and row sum l in
//                 registers, writes P (bf16) into tensor memory, and does
//                 the final O / l and LSE epilogue.
// At d = 64 the CTA runs two independent pipelines (Cfg::DUAL): warps 0 and
// 3 produce, 1 and 2 issue, 4..7 and 8..11 do the softmax, each pipeline with
// its own Q tile, K/V ring and work items of one query tile.
// Tensor memory (512 columns):
//   d = 128: S/P of tile t at [128 t, 128 t + 128) (P, bf16, over the scores),
//            O of tile t at [256 + 128 t, 384 + 128 t).  A tile's next QK^T
//            waits for its PV, which reads P from the same columns; the two
//            query tiles ping-pong, so while one softmax group works on its
//            scores the tensor cores run the other tile's PV and next QK^T.
//   d = 64:  S of tile t at [128 t, 128 t + 128), P of tile t at
//            [256 + 64 t, 320 + 64 t), O of tile t at [384 + 64 t, 448 + 64 t).
//            P has columns of its own, so the next QK^T overwrites S as soon
//            as the softmax has read it (barrier s_free) and the scores of key
//            tile j + 1 are ready when the softmax finishes tile j: each
//            softmax group runs its key steps back to back.
//
// The O rescale is lazy: each row takes its reference maximum from its first
// key tile and keeps it while the exponentials stay below 2^16 (a row sum of
// one key tile below 2^16), so no later key tile needs a row maximum.  A key
// tile that breaks the bound is redone on its own row maximum and l and O
// move to the new reference; l and O always share the reference, so the
// final O / l is unchanged (exact in exact arithmetic).
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "fa_internal.h"
#include "sm100.cuh"
#include "fwd_sched.cuh"

namespace fa {
namespace fwd {

constexpr int NUM_THREADS = 384;
constexpr int RING = 4;              // depth of the item ring the producer fills

// Dynamic schedule.  CTA b starts on item b; after that each CTA claims
// items gridDim.x, gridDim.x + 1, ... from a counter.  Each launch takes one
// of SCHED_SLOTS counters (in turn, on the host), and the last CTA to stop
// claiming puts it back to zero.  Launches that run at the same time (other
// streams) use other slots, so at most SCHED_SLOTS forward launches may be
// in flight at once.
constexpr uint32_t SCHED_SLOTS = 4096;
__device__ uint32_t g_claim[SCHED_SLOTS];  // dynamic claims so far
__device__ uint32_t g_done[SCHED_SLOTS];   // CTAs that stopped claiming
constexpr float LN2 = 0.69314718055994530942f;

template <int D, int PIPES>
struct Cfg {
  static constexpr int TILE_BYTES = BN * D * 2;  // one Q, K or V tile
  static constexpr int CHUNKS = D / 64;          // 64-column (128-byte) chunks per row
  static constexpr int CHUNK_BYTES = BN * 128;   // one chunk of a tile
  // PIPES = 2 (d = 64): two independent pipelines per CTA.  Each has its own
  // producer warp (0, 3), MMA issuer (1, 2), softmax warpgroup (4..7,
  // 8..11), Q tile, K/V ring and stream of work items, one query tile each;
  // they share only the CTA's shared and tensor memory, so one pipeline's
  // softmax, item change or load wait overlaps the other's work, and neither
  // loads key tiles only the other needs.  PIPES = 1 (d = 128): one
  // pipeline, work items of two query tiles sharing one K/V stream.
  static_assert(PIPES == (D == 64 ? 2 : 1), "d = 64 runs two pipelines, d = 128 one");
  static constexpr bool DUAL = PIPES == 2;
  static constexpr int NPIPE = PIPES;
  static constexpr int NSLOT = 4;  // K/V ring slots per pipeline
  // Each softmax warp stages 64 columns of its 32 rows of O (bf16, 4 KB) at
  // a time here, in the 128-byte swizzle, and writes them out with one
  // tensor store.
  static constexpr int OSTAGE_BYTES = 8 * 32 * 128;
  static constexpr int SMEM_BYTES = 2 * TILE_BYTES + NPIPE * NSLOT * TILE_BYTES + OSTAGE_BYTES + 1024;
  // MMA issuer threads.  Issuing blocks while the tensor core's queue is
  // full, so with one issuer a tile's PV can wait behind the other tile's
  // products.  d = 64: one issuer per pipeline (short products, so the
  // decoupling wins).  d = 128: one issuer for both tiles, which keeps each
  // tile's PV and next QK^T back to back on the tensor core (interleaving
  // the two tiles' products delays both tiles' next scores).
  static constexpr int ISSUERS = D == 64 ? 2 : 1;
  // P in columns of its own (needs 2 x (128 + 64 + d) <= 512 columns).
  static constexpr bool SPLIT_P = D == 64;
  static constexpr uint32_t COL_P = 256;                   // + 64 t (SPLIT_P)
  static constexpr uint32_t COL_O = SPLIT_P ? 384 : 256;   // + d t
  // Consumers of a pipeline's item ring: its issuer(s) and softmax warps.
  static constexpr int CONSUMERS = DUAL ? 1 + 4 : ISSUERS + 8;
  static constexpr int PIPE_ISSUERS = DUAL ? 1 : ISSUERS;  // commits per Q / K/V release
  // Registers per thread after the split (launch: 168): producer and issuer
  // warpgroup, then each softmax warpgroup.  The d = 64 softmax holds a
  // whole score row and spills below 224.
  static constexpr int REG_CTL = D == 64 ? 56 : 72;
  static constexpr int REG_SMX = D == 64 ? 224 : 216;
  static_assert(REG_CTL + 2 * REG_SMX <= 3 * 168, "register split exceeds the launch");
};

// VARLEN: per-sequence lengths are read (else every sequence has N, Nk and
// the sizes stay compile-time-free of extra registers).
template <int D, bool VARLEN, int PIPES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
               const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapO,
               const Params p) {
  using C = Cfg<D, PIPES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                        // 2 tiles (DUAL: pipeline q's at q)
  uint8_t* sKV = smem + 2 * C::TILE_BYTES;   // NPIPE rings of NSLOT tiles
  uint8_t* sO = sKV + C::NPIPE * C::NSLOT * C::TILE_BYTES;  // OSTAGE_BYTES

  // Per pipeline: Q, K/V ring, item ring.
  __shared__ __align__(8) uint64_t q_full[2], q_empty[2], mma_drain[2];
  __shared__ __align__(8) uint64_t kv_full[2][C::NSLOT], kv_empty[2][C::NSLOT];
  __shared__ __align__(8) uint64_t s_full[2], p_full[2], o_full[2];
  __shared__ __align__(8) uint64_t s_free[2], pv_done[2];  // SPLIT_P only
  // A pipeline's producer claims work items and passes them to its other roles.
  __shared__ __align__(8) uint64_t item_full[2][RING], item_empty[2][RING];
  __shared__ int item_ring[2][RING];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&mma_drain[0], 1);
    mbar_init(&mma_drain[1], 1);
    for (int q = 0; q < C::NPIPE; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], C::PIPE_ISSUERS);  // one commit from each of its MMA issuers
      for (int i = 0; i < C::NSLOT; ++i) {
        mbar_init(&kv_full[q][i], 1);
        mbar_init(&kv_empty[q][i], C::PIPE_ISSUERS);
      }
      for (int r = 0; r < RING; ++r) {
        mbar_init(&item_full[q][r], 1);
        mbar_init(&item_empty[q][r], C::CONSUMERS);
      }
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], BM);
      mbar_init(&o_full[t], 1);
      mbar_init(&s_free[t], BM);
      mbar_init(&pv_done[t], 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if ((warp == 0 || (C::DUAL && warp == 3)) && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = tmem_base_sh;
  const WaitCtx w{p.timeout_ns, &abort_flag, p.status};

  auto take_item = [&](int q, uint32_t k, int& idx) -> bool {
    const uint32_t slot = k % RING;
    if (!mbar_wait(&item_full[q][slot], (k / RING) & 1, w)) return false;
    idx = *reinterpret_cast<volatile int*>(&item_ring[q][slot]);
    mbar_arrive(&item_empty[q][slot]);
    return true;
  };
  auto take_item_warp = [&](int q, uint32_t k, int& idx) -> bool {
    const uint32_t slot = k % RING;
    if (!mbar_wait_warp(&item_full[q][slot], (k / RING) & 1, w)) return false;
    idx = *reinterpret_cast<volatile int*>(&item_ring[q][slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[q][slot]);
    return true;
  };

  // Registers: 384 threads x 168 at launch; the producer/MMA warpgroup gives
  // much of its share to the two softmax warpgroups (Cfg::REG_CTL,
  // Cfg::REG_SMX; 128 x (56 + 224 + 224) = 128 x (88 + 208 + 208) = 64512,
  // the launch total).
  if (warp < 4) {
    regs_dec<C::REG_CTL>();  // may only lower the 168 registers of the launch
  if (warp == 0 || (C::DUAL && warp == 3)) {
    // ------------------------------------------------------------ producer
    // (of pipeline q)
    if (lane == 0) {
      const int q = warp == 0 ? 0 : 1;
      uint32_t kv_iter = 0, item_iter = 0;
      bool q_loading = false;  // this item's Q load was issued
      bool ok = true;
      for (;; ++item_iter) {
        const uint32_t slot = item_iter % RING;
        ok = mbar_wait(&item_empty[q][slot], ((item_iter / RING) & 1) ^ 1, w);
        if (!ok) break;
        // Pipeline q of CTA b starts on item NPIPE b + q, then claims items
        // NPIPE gridDim.x, NPIPE gridDim.x + 1, ...
        int idx = item_iter == 0 ? (int)(blockIdx.x * C::NPIPE) + q
                                 : (int)(gridDim.x * C::NPIPE) + (int)atomicAdd(&g_claim[p.slot], 1u);
        if (idx > p.n_items) idx = p.n_items;
        item_ring[q][slot] = idx;
        mbar_arrive(&item_full[q][slot]);
        if (idx >= p.n_items) break;
        const Item it = item_at<VARLEN>(p, idx);
        q_loading = false;
        ok = mbar_wait(&q_empty[q], (item_iter & 1) ^ 1, w);
        if (!ok) break;
        mbar_arrive_expect_tx(&q_full[q], C::TILE_BYTES * (it.has1 ? 2 : 1));
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_3d(sQ + q * C::TILE_BYTES + c * C::CHUNK_BYTES, &mapQ, &q_full[q], c * 64, it.q0 * BM, it.bh);
        if (it.has1) {
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(sQ + C::TILE_BYTES + c * C::CHUNK_BYTES, &mapQ, &q_full[q], c * 64, it.q1 * BM, it.bh);
        }
        q_loading = true;
        const int e = kv_end<VARLEN>(p, it);
        for (int j = next_union<VARLEN>(p, it, 0); ok && j < e; j = next_union<VARLEN>(p, it, j + 1)) {
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t slot = kv_iter % C::NSLOT;
            ok = mbar_wait(&kv_empty[q][slot], ((kv_iter / C::NSLOT) & 1) ^ 1, w);
            if (!ok) break;
            mbar_arrive_expect_tx(&kv_full[q][slot], C::TILE_BYTES);
            uint8_t* dst = sKV + (q * C::NSLOT + slot) * C::TILE_BYTES;
            const CUtensorMap* m = kv == 0 ? &mapK : &mapV;
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c)
              tma_load_3d(dst + c * C::CHUNK_BYTES, m, &kv_full[q][slot], c * 64, j * BN, it.bh);
            ++kv_iter;
          }
        }
        if (!ok) break;
      }
      // This pipeline claims no more (its last claim ran past the end, or it
      // aborted); the last pipeline of the launch to get here resets the
      // counter slot.
      if (atomicAdd(&g_done[p.slot], 1u) == gridDim.x * C::NPIPE - 1) {
        g_claim[p.slot] = 0u;
        g_done[p.slot] = 0u;
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory
        // is released (bounded).
        const uint64_t dl = globaltimer_ns() + 100000000ull;
        const uint32_t n = kv_iter < (uint32_t)C::NSLOT ? kv_iter : (uint32_t)C::NSLOT;
        for (uint32_t i = 0; i < n; ++i) {
          const uint32_t k = kv_iter - 1 - i;
          mbar_drain_wait(&kv_full[q][k % C::NSLOT], (k / C::NSLOT) & 1, dl);
        }
        // the last Q load issued: this item's, or the previous item's
        const uint32_t last_q = q_loading ? item_iter : item_iter - 1;
        if (q_loading || item_iter > 0) mbar_drain_wait(&q_full[q], last_q & 1, dl);
      }
    }
  } else if (warp == 1 || (C::ISSUERS == 2 && warp == 2)) {
    // ------------------------------------------------------------ MMA issuers
    // Cfg::ISSUERS threads; issuer u handles query tiles [t_lo, t_hi).  Each
    // walks every key step of every item and commits every K/V slot and the
    // Q tiles once (those barriers count one arrival per issuer).  Per key
    // step and tile: O_t += P_t V_j, then S_t = Q_t K_{j+1}^T into the same
    // columns (after the PV that reads P_t, in issue order).
    if (lane == 0) {
      const int t_lo = C::ISSUERS == 2 ? warp - 1 : 0;
      const int t_hi = C::ISSUERS == 2 ? warp : 2;
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t sQ_addr = smem_u32(sQ);
      const uint32_t sKV_addr = smem_u32(sKV);
      uint32_t kv_iter = 0, item_iter = 0, p_cnt[2] = {0, 0};
      bool ok = true, issued = false;

      // Descriptors of the Q tiles and of ring slot 0, built once; the
      // products below only move them (one 32-bit add per operand).
      const Desc dQ0 = desc_sw128(sQ_addr, 16, 1024);             // K-major, K = d
      const Desc dK0 = desc_sw128(sKV_addr, 16, 1024);            // K-major, K = d
      const Desc dV0 = desc_sw128(sKV_addr, C::CHUNK_BYTES, 1024);  // MN-major, N = d
      auto issue_s = [&](int t, uint32_t kslot) {
        const Desc qa = desc_at(dQ0, t * C::TILE_BYTES);
        const Desc ka = desc_at(dK0, kslot * C::TILE_BYTES);
        const uint32_t d_s = tmem + t * 128;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s >> 2) * C::CHUNK_BYTES + (s & 3) * 32;
          mma_ss(d_s, desc_at(qa, off), desc_at(ka, off), IDESC_S, s > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
        issued = true;
      };
      auto issue_pv = [&](int t, uint32_t vslot, uint32_t acc) {
        const Desc va = desc_at(dV0, vslot * C::TILE_BYTES);
        const uint32_t d_o = tmem + C::COL_O + t * D;
        const uint32_t a_p = tmem + (C::SPLIT_P ? C::COL_P + t * 64 : t * 128);
#pragma unroll
        for (int s = 0; s < BN / 16; ++s)
          mma_ts(d_o, a_p + s * 8, desc_at(va, s * 2048), IDESC_O, (s > 0 || acc) ? 1u : 0u);
      };

      if constexpr (C::SPLIT_P) {
        // The issuer of query tile t: with two pipelines the one tile of
        // pipeline t's items, else tile t of the pipeline's pairs.  Per key
        // step j (K of j at ring index kv_iter, its V at kv_iter + 1):
        // S = Q K_j^T once the softmax has read the previous scores, then
        // O += P V for the key tile before j once its P is written.  Every
        // S, P and PV is counted over the whole launch, so the n-th of each
        // pairs with the n-th arrival.
        const int t = warp - 1;
        const int q = C::DUAL ? t : 0;         // pipeline
        const uint32_t ring0 = q * C::NSLOT;  // its first ring slot
        uint32_t s_iss = 0, pv_iss = 0;
        for (;; ++item_iter) {
          int idx;
          ok = take_item(q, item_iter, idx);
          if (!ok || idx >= p.n_items) break;
          const Item it = item_at<VARLEN>(p, idx);
          const bool mine = C::DUAL || t == 0 || it.has1;
          const int qt = (C::DUAL || t == 0) ? it.q0 : it.q1;
          ok = mbar_wait(&q_full[q], item_iter & 1, w);
          if (!ok) break;
          tc_fence_after();
          const int e = kv_end<VARLEN>(p, it);
          int j = next_union<VARLEN>(p, it, 0), jp = -1;
          if (j >= e) tc_commit(&q_empty[q]);  // no key tile: Q was not read
          bool first_pv = true;
          while (ok && (j < e || jp >= 0)) {
            const int jn = j < e ? next_union<VARLEN>(p, it, j + 1) : e;
            if (j < e) {
              const uint32_t ks = kv_iter % C::NSLOT;
              ok = mbar_wait(&kv_full[q][ks], (kv_iter / C::NSLOT) & 1, w);
              if (!ok) break;
              tc_fence_after();
              if (mine && member<VARLEN>(p, it, qt, j)) {
                if (s_iss > 0) {
                  ok = mbar_wait(&s_free[t], (s_iss - 1) & 1, w);
                  if (!ok) break;
                  tc_fence_after();
                }
                issue_s(t, ring0 + ks);
                ++s_iss;
              }
              tc_commit(&kv_empty[q][ks]);
              if (jn >= e) tc_commit(&q_empty[q]);  // the item's last QK^T
            }
            if (jp >= 0) {
              const uint32_t vi = kv_iter - 1, vs = vi % C::NSLOT;  // V of key tile jp
              ok = mbar_wait(&kv_full[q][vs], (vi / C::NSLOT) & 1, w);
              if (!ok) break;
              tc_fence_after();
              if (mine && member<VARLEN>(p, it, qt, jp)) {
                ok = mbar_wait(&p_full[t], pv_iss & 1, w);
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, ring0 + vs, first_pv ? 0u : 1u);
                tc_commit(&pv_done[t]);
                first_pv = false;
                ++pv_iss;
              }
              tc_commit(&kv_empty[q][vs]);
            }
            if (j < e) kv_iter += 2;
            jp = j < e ? j : -1;
            j = jn;
          }
          if (!ok) break;
        }
      } else {
      for (;; ++item_iter) {
        int idx;
        ok = take_item(0, item_iter, idx);
        if (!ok || idx >= p.n_items) break;
        const Item it = item_at<VARLEN>(p, idx);
        const int tiles = it.has1 ? 2 : 1;  // tiles [0, tiles) exist
        ok = mbar_wait(&q_full[0], item_iter & 1, w);
        if (!ok) break;
        tc_fence_after();
        const int e = kv_end<VARLEN>(p, it);
        int j = next_union<VARLEN>(p, it, 0);
        int jn = j < e ? next_union<VARLEN>(p, it, j + 1) : e;  // the key tile after j
        bool first_pv[2] = {true, true};
        // Q is read only by the QK^T products: it goes back to the producer
        // once the item's last one has been issued, so the next item's Q
        // loads while this item's last softmax, PV and epilogue run.
        bool q_released = false;
        if (j < e) {
          const uint32_t ks = kv_iter % C::NSLOT;
          ok = mbar_wait(&kv_full[0][ks], (kv_iter / C::NSLOT) & 1, w);
          if (!ok) break;
          tc_fence_after();
          for (int t = t_lo; t < t_hi && t < tiles; ++t)
            if (member<VARLEN>(p, it, t == 0 ? it.q0 : it.q1, j)) issue_s(t, ks);
          tc_commit(&kv_empty[0][ks]);
          ++kv_iter;
          if (jn >= e) {
            tc_commit(&q_empty[0]);
            q_released = true;
          }
        }
        while (ok && j < e) {
          const int jnn = jn < e ? next_union<VARLEN>(p, it, jn + 1) : e;
          const uint32_t vs = kv_iter % C::NSLOT;
          const uint32_t ksn = (kv_iter + 1) % C::NSLOT;
          ok = mbar_wait(&kv_full[0][vs], (kv_iter / C::NSLOT) & 1, w);
          if (ok && jn < e) ok = mbar_wait(&kv_full[0][ksn], ((kv_iter + 1) / C::NSLOT) & 1, w);
          if (!ok) break;
          tc_fence_after();
          for (int t = t_lo; t < t_hi && t < tiles && ok; ++t) {
            const int qt = t == 0 ? it.q0 : it.q1;
            if (member<VARLEN>(p, it, qt, j)) {
              ok = mbar_wait(&p_full[t], p_cnt[t] & 1, w);
              if (!ok) break;
              ++p_cnt[t];
              tc_fence_after();
              issue_pv(t, vs, first_pv[t] ? 0u : 1u);
              first_pv[t] = false;
            }
            if (jn < e && member<VARLEN>(p, it, qt, jn)) issue_s(t, ksn);
          }
          if (!ok) break;
          tc_commit(&kv_empty[0][vs]);
          if (jn < e) {
            tc_commit(&kv_empty[0][ksn]);
            kv_iter += 2;
            if (!q_released && jnn >= e) {
              tc_commit(&q_empty[0]);
              q_released = true;
            }
          } else {
            kv_iter += 1;
          }
          j = jn;
          jn = jnn;
        }
        if (!ok) break;
        for (int t = t_lo; t < t_hi && t < tiles; ++t) tc_commit(&o_full[t]);
        if (!q_released) tc_commit(&q_empty[0]);
      }
      }
      if (issued) {
        // Every MMA issued by this thread must be finished before tensor
        // memory is released.
        const int u = C::ISSUERS == 2 ? warp - 1 : 0;
        tc_commit(&mma_drain[u]);
        mbar_drain_wait(&mma_drain[u], 0, globaltimer_ns() + 100000000ull);
      }
    }
  }
  } else {
    regs_inc<C::REG_SMX>();  // may only raise them
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;         // query tile of this warpgroup
    const int quarter = warp & 3;          // tensor-memory lane quarter
    const int r = quarter * 32 + lane;     // row within the tile
    const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_bits + t * 128;
    const uint32_t t_o = tmem + lane_bits + C::COL_O + t * D;
    const uint32_t t_p = tmem + lane_bits + C::COL_P + t * 64;  // SPLIT_P
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;
    uint32_t np = 0;  // P tiles written so far (SPLIT_P)
    bool ok = true;

    for (uint32_t k = 0;; ++k) {
      int idx;
      ok = take_item_warp(C::DUAL ? t : 0, k, idx);
      if (!ok || idx >= p.n_items) break;
      const Item it = item_at<VARLEN>(p, idx);
      if (!C::DUAL && t == 1 && !it.has1) continue;
      const int qt = (C::DUAL || t == 0) ? it.q0 : it.q1;  // DUAL: each pipeline's item is one tile
      const int row = qt * BM + r;
      float m = -INFINITY;  // reference maximum, scaled log2 units
      float l = 0.0f;
      bool first = true;  // no PV has written this tile's O yet
      const int e = kv_end<VARLEN>(p, it);
      // The key tiles this query tile visits, in order.  Under a block mask
      // the warp reads its row of the mask 32 key tiles at a time (one byte a
      // lane, then a ballot) instead of one dependent load per key tile.
      uint32_t mbits = 0;
      int mbase = -64;  // first key tile of the 32 in mbits
      auto next_key = [&](int j) -> int {
        if (p.mask_kind != FA_MASK_BLOCK) {
          while (j < e && !member<VARLEN>(p, it, qt, j)) ++j;
          return j < e ? j : e;
        }
        while (j < e) {
          if (j < mbase || j >= mbase + 32) {
            mbase = j & ~31;
            const int jj = mbase + lane;
            mbits = __ballot_sync(0xffffffffu, jj < e && member<VARLEN>(p, it, qt, jj));
          }
          const uint32_t rest = mbits >> (j - mbase);
          if (rest) return j + __ffs(rest) - 1;
          j = mbase + 32;
        }
        return e;
      };
      for (int j = next_key(0); j < e; j = next_key(j + 1)) {
        ok = mbar_wait_warp(&s_full[t], s_cnt & 1, w);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        uint32_t sraw[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32) FA_TMEM_LD_X32(t_s + c, (sraw + c));
        tc_wait_ld();
        if constexpr (C::SPLIT_P) {
          tc_fence_before();
          mbar_arrive(&s_free[t]);  // the next QK^T may overwrite the scores
        }
        float x[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) x[c] = __uint_as_float(sraw[c]);
        // valid columns [0, lim): keys that exist and, under the causal mask,
        // keys <= row + off
        const int key0 = j * BN;
        int lim = min(BN, it.Lk - key0);
        if (p.mask_kind == FA_MASK_CAUSAL) lim = max(0, min(lim, row + it.off + 1 - key0));
        if (lim < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) x[c] = -INFINITY;
        }
        // Reference maximum m.  A row takes it from its scores when it has
        // none yet (its first key tile, or every key so far masked); after
        // that the exponentials use the reference they have, and only a key
        // tile whose row sum reaches 2^16 (or is not finite) moves it: that
        // tile is then redone on its own row maximum, and l and O are brought
        // onto the new reference.  O / l does not depend on the reference.
        auto row_max = [&]() {
          float ma[8];  // eight independent chains, then a tree
#pragma unroll
          for (int k = 0; k < 8; ++k) ma[k] = x[k];
#pragma unroll
          for (int c = 8; c < BN; c += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) ma[k] = fmaxf(ma[k], x[c + k]);
          return sl2 * fmaxf(fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3])),
                             fmaxf(fmaxf(ma[4], ma[5]), fmaxf(ma[6], ma[7])));
        };
        // P = 2^(x sl2 - m) as bf16 into tensor memory (over the scores, or
        // into P's own columns); returns the row sum of this key tile.
        const uint32_t t_pw = C::SPLIT_P ? t_p : t_s;
        auto exp_pass = [&]() {
          const float m_use = (m == -INFINITY) ? 0.0f : m;  // a row with no key yet: P = 0
          // Two columns per instruction (packed fp32 pairs) for the scaling
          // and the row sum; each lane of a pair rounds as the scalar form.
          const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_use, -m_use);
          float2 rsa[4] = {};  // row sum, eight chains in four pairs
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float2 y = __ffma2_rn(make_float2(x[64 * h + 2 * i], x[64 * h + 2 * i + 1]), sl2x2, nm2);
              const float2 pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
              rsa[i & 3] = __fadd2_rn(rsa[i & 3], pp);
              pk[i] = pack_bf16x2(pp.x, pp.y);
            }
            FA_TMEM_ST_X32(t_pw + 32 * h, pk);
          }
          return ((rsa[0].x + rsa[0].y) + (rsa[1].x + rsa[1].y)) + ((rsa[2].x + rsa[2].y) + (rsa[3].x + rsa[3].y));
        };
        const bool need_m = m == -INFINITY;
        if (__any_sync(0xffffffffu, need_m)) {
          const float mx = row_max();
          if (need_m) m = mx;  // l and O are still zero for such a row
        }
        if constexpr (C::SPLIT_P) {
          if (np > 0) {
            // The previous PV has finished: it no longer reads P's columns,
            // and O holds every product so far (for a rescale below).
            ok = mbar_wait_warp(&pv_done[t], (np - 1) & 1, w);
            if (!ok) break;
            tc_fence_after();
          }
          ++np;
        }
        float rs = exp_pass();
        const bool redo = !(rs < 65536.0f);
        if (__any_sync(0xffffffffu, redo)) {
          float a = 1.0f;
          if (redo) {
            const float mx = row_max();  // >= m + 9 here, since rs >= 2^16
            a = ex2_approx(m - mx);
            m = mx;
            l *= a;
          }
          // Bring O onto the new reference (rows that kept theirs multiply by
          // 1).  Before the item's first PV there is nothing to rescale: that
          // PV overwrites O.
          if (!first) {
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t v[32];
              FA_TMEM_LD_X32(t_o + c, v);
              tc_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
              FA_TMEM_ST_X32(t_o + c, v);
            }
          }
          tc_wait_st();
          rs = exp_pass();
        }
        first = false;
        l += rs;
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // ---- epilogue: O / l and LSE
      if constexpr (C::SPLIT_P) {
        // the tile's last PV (none if no key tile reached the tile: then
        // l = 0 and O is written as zeros)
        if (!first) ok = mbar_wait_warp(&pv_done[t], (np - 1) & 1, w);
      } else {
        ok = mbar_wait_warp(&o_full[t], o_cnt & 1, w);
        ++o_cnt;
      }
      if (!ok) break;
      tc_fence_after();
      const bool live = l > 0.0f && row < it.Lq;  // false for a row that sees no key, or padding
      const float inv_l = live ? 1.0f / l : 0.0f;
      {
        // Per 64 columns: lane i puts row i of the warp's 32 (128 bytes:
        // eight 16-byte chunks, chunk k at slot k ^ (i & 7), which is the
        // 128-byte swizzle), then lane 0 stores the 32 x 64 box with one
        // tensor store (rows past N are not written).
        uint8_t* ws = sO + (warp - 4) * 4096;
        const int row0 = qt * BM + quarter * 32;
#pragma unroll
        for (int g = 0; g < D / 64; ++g) {
          if (lane == 0) bulk_wait_read_all();  // the warp's previous store has read the buffer
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 64; c += 32) {
            uint32_t v[32];
            FA_TMEM_LD_X32(t_o + 64 * g + c, v);
            tc_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])),
                                          make_float2(inv_l, inv_l));
              pk[i] = live ? pack_bf16x2(o.x, o.y) : 0u;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k = c / 8 + i;
              *reinterpret_cast<uint4*>(ws + lane * 128 + ((k ^ (lane & 7)) * 16)) =
                  make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
          fence_proxy_async_smem();  // the generic-proxy writes, before the tensor store reads them
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&mapO, ws, 64 * g, row0, it.bh);
            bulk_commit_group();
          }
        }
      }
      if (row < p.N && FA_IN_BOUNDS(p.status, (size_t)it.bh * p.N + row, 1, (size_t)p.BH * p.N))
        p.LSE[(size_t)it.bh * p.N + row] = live ? (m + log2f(l)) * LN2 : -INFINITY;
      tc_fence_before();
    }
    if (lane == 0) bulk_wait_all();  // this warp's O stores are done before the CTA leaves
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fwd

fa_status launch_fwd(const Problem& pr, const void* Q, const void* K, const void* V, void* O, float* LSE,
                     cudaStream_t s) {
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  CUtensorMap mQ, mK, mV, mO;
  if (!make_map_bf16(&mQ, Q, pr.BH, pr.N, pr.d, fwd::BM) || !make_map_bf16(&mK, K, pr.BH, pr.Nk, pr.d, fwd::BN) ||
      !make_map_bf16(&mV, V, pr.BH, pr.Nk, pr.d, fwd::BN) || !make_map_bf16_box(&mO, O, pr.BH, pr.N, pr.d, 64, 32))
    return FA_ERR_CUDA;
  fwd::Params p;
  p.BH = pr.BH;
  p.N = pr.N;
  p.nq = pr.nq;
  p.Nk = pr.Nk;
  p.nk = pr.nk;
  p.off = pr.off;
  p.H = pr.H;
  p.seqlens_q = pr.seqlens_q;
  p.seqlens_k = pr.seqlens_k;
  // d = 64: two pipelines of one-tile items; d = 128: pairs
  const bool dual = pr.d == 64;
  p.tiles_per_item = dual ? 1 : 2;
  p.n_pairs = (pr.nq + p.tiles_per_item - 1) / p.tiles_per_item;
  p.n_items = p.n_pairs * pr.BH;
  p.group = fwd::sched_group(pr.BH, pr.Nk, pr.d);
  p.mask_kind = pr.mask_kind;
  p.block_mask = pr.block_mask;
  p.scale_log2 = pr.scale_log2;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  p.timeout_ns = wait_timeout_ns();
  p.status = st;
  static std::atomic<uint32_t> next_slot{0};
  p.slot = next_slot.fetch_add(1u, std::memory_order_relaxed) % fwd::SCHED_SLOTS;
  const int npipe = dual ? 2 : 1;
  const int want = (p.n_items + npipe - 1) / npipe;  // CTAs that get a first item in every pipeline
  const int grid = want < num_sms() ? want : num_sms();
  auto run = [&](auto kern, int smem) -> bool {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return false;
    kern<<<grid, fwd::NUM_THREADS, smem, s>>>(mQ, mK, mV, mO, p);
    return true;
  };
  const bool varlen = pr.seqlens_q || pr.seqlens_k;
  bool ok;
  if (dual)
    ok = varlen ? run(fwd::fwd_kernel<64, true, 2>, fwd::Cfg<64, 2>::SMEM_BYTES)
                : run(fwd::fwd_kernel<64, false, 2>, fwd::Cfg<64, 2>::SMEM_BYTES);
  else
    ok = varlen ? run(fwd::fwd_kernel<128, true, 1>, fwd::Cfg<128, 1>::SMEM_BYTES)
                : run(fwd::fwd_kernel<128, false, 1>, fwd::Cfg<128, 1>::SMEM_BYTES);
  if (!ok) return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
