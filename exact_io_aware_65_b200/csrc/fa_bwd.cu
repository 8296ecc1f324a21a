// fa_bwd.cu -- backward pass of exact attention on sm_100a.
//
// The pages fix the strategy ("FlashAttention: Fast and Memory-Efficient
// Exact Attention with IO-Awareness", section "Backward / recomputation"):
// the forward keeps only the per-row softmax statistic (here LSE), and the
// backward rebuilds the attention probabilities on chip instead of reading an
// N x N matrix back.  The gradient formulas are the calculus of softmax
// attention:
//     P_ij  = exp(scale q_i.k_j - LSE_i)           (recomputed)
//     dV_j  = sum_i P_ij dO_i
//     dP_ij = dO_i . v_j,   D_i = dO_i . O_i = sum_j P_ij dP_ij
//     dS_ij = P_ij (dP_ij - D_i)
//     dK_j  = scale sum_i dS_ij q_i,   dQ_i = scale sum_j dS_ij k_j
//
// Three kernels, all on the caller's stream:
//   prep     -D_i, -LSE_i * log2(e) (negated, so that the softmax adds them;
//            padded to whole tiles) and a zeroed fp32 dQ accumulator, in the
//            workspace.
//   main     one persistent CTA per SM; a work item is one (head, 128-key
//            tile).  K_j and V_j stay in shared memory, dK_j and dV_j
//            accumulate in tensor memory across the query tiles that see
//            them, so they need no atomics.  Per query tile:
//              S^T  = K_j Q_i^T,  dP^T = V_j dO_i^T        (tensor cores)
//              P^T, dS^T                                   (softmax warps)
//              dV  += P^T dO_i,   dK += dS^T Q_i            (A from tensor memory)
//              dQ_i = dS K_j                                 (A = dS^T in smem)
//            Four drain warps read dQ_i out of tensor memory, stage it in a
//            dead shared-memory buffer and add it to the fp32 accumulator
//            with bulk reduce-adds (cp.reduce.async.bulk, add.f32).
//   convert  dQ = bf16(scale * dQ_acc).
//
// CTA roles (512 threads): warp 0 TMA producer; warp 1 MMA issuer; warps
// 4..11 softmax (thread = key row; warps 4..7 take query columns 0..63,
// warps 8..11 columns 64..127); warps 12..15 dQ drain (thread = query row).
// Tensor memory: S^T [0,128), then P^T (bf16) in [0,32) and [64,96); dP^T
// [128,256), then dS^T (bf16) in [128,160) and [192,224); dV [256, 256+d);
// dK [256+d, 256+2d).  The
// MMA order per query tile is dV, next S^T, dK, dQ, next dP^T, so the
// softmax of the next tile overlaps three products.  The dQ tile reuses the
// dP^T columns for d = 128 (the next dP^T waits for the drain) and has two
// buffers at [384,448) and [448,512) for d = 64.
#include <cuda_bf16.h>
#include <limits.h>
#include <math.h>

#include "fa_internal.h"
#include "sm100.cuh"
#include "bwd_sched.cuh"

namespace fa {
namespace bwd {

constexpr int NUM_THREADS = 512;
constexpr float LOG2E = 1.4426950408889634074f;

__host__ __device__ constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace carve-up (all offsets 256-byte aligned).  The fp32 dQ
// accumulator is tiled: within each (head, 128-query tile) block the element
// (query r, column c) sits at (c / 4) * 512 + r * 4 + c % 4, so that one warp
// adding four columns of 32 consecutive query rows touches 512 contiguous
// bytes.  `sched` is the work counter of the main kernel's dynamic scheduler;
// `turn` holds one counter per (head, query tile) for the deterministic
// order of the dQ additions (how many key tiles have added their part).
struct Workspace {
  size_t dq_off, d_off, l2_off, sched_off, turn_off, total;
};
__host__ __device__ inline Workspace workspace_layout(int BH, int Npad, int d) {
  Workspace w;
  w.dq_off = 0;
  w.d_off = align256((size_t)BH * Npad * d * sizeof(float));
  w.l2_off = w.d_off + align256((size_t)BH * Npad * sizeof(float));
  w.sched_off = w.l2_off + align256((size_t)BH * Npad * sizeof(float));
  w.turn_off = w.sched_off + 256;
  w.total = w.turn_off + align256((size_t)BH * (Npad / 128) * sizeof(uint32_t));
  return w;
}

// ------------------------------------------------------------------ prep ---
// One group of d/8 lanes per row; each lane covers 8 elements (16 bytes).
template <int D>
__global__ void __launch_bounds__(256) prep_kernel(const __nv_bfloat16* __restrict__ O,
                                                   const __nv_bfloat16* __restrict__ dO,
                                                   const float* __restrict__ LSE, float* __restrict__ Dw,
                                                   float* __restrict__ L2w, float* __restrict__ dq_acc,
                                                   uint32_t* __restrict__ sched, uint32_t* __restrict__ turn,
                                                   int BH, int N, int Npad, int H,
                                                   const int* __restrict__ seqlens_q, uint32_t* status) {
  constexpr int LPR = D / 8;
  if (blockIdx.x == 0 && threadIdx.x == 0) *sched = 0u;
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  const long long total = (long long)BH * Npad;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long r0 = ((long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * RPW; r0 < total;
       r0 += warps * RPW) {
    const long long r = r0 + sub;
    const int bh = (int)(r / Npad), n = (int)(r % Npad);
    // rows past the sequence's length (or the padded count) are padding: P = 0
    const int Lq = seqlens_q && r < total
                       ? (FA_IN_BOUNDS(status, bh / H, 1, BH / H) ? min(max(__ldg(seqlens_q + bh / H), 0), N) : 0)
                       : N;
    const bool real = r < total && n < Lq;
    float acc = 0.0f;
    if (real && FA_IN_BOUNDS(status, ((size_t)bh * N + n) * D + li * 8, 8, (size_t)BH * N * D)) {
      const size_t e = ((size_t)bh * N + n) * D + li * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(O + e);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + e);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[i]));
        const float2 fb2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[i]));
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < total && FA_IN_BOUNDS(status, r, 1, total) && FA_IN_BOUNDS(status, r * D + li * 8, 8, total * D)) {
      if (li == 0) {
        if ((n & 127) == 0 && FA_IN_BOUNDS(status, (size_t)bh * (Npad / 128) + n / 128, 1, total / 128))
          turn[(size_t)bh * (Npad / 128) + n / 128] = 0u;
        Dw[r] = -acc;
        float l2 = INFINITY;  // padding rows and rows that saw no key: P = 0
        if (real && FA_IN_BOUNDS(status, (size_t)bh * N + n, 1, (size_t)BH * N)) {
          const float lse = LSE[(size_t)bh * N + n];
          if (lse > -INFINITY) l2 = lse * LOG2E;
        }
        L2w[r] = -l2;
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + (size_t)r * D + li * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// --------------------------------------------------------------- convert ---
// Each thread takes 16 columns of one query row: four float4 column groups
// of the tiled accumulator.  Consecutive threads take consecutive rows, so
// every load instruction reads 512 contiguous bytes per warp, and each thread
// writes one whole 32-byte sector of the bf16 row.
template <int D>
__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ dq_acc,
                                                         __nv_bfloat16* __restrict__ dQ, int BH, int N, int Npad,
                                                         float scale, uint32_t* status) {
  constexpr int G = 4;                         // column groups per thread
  constexpr int PER_TILE = 128 * (D / (4 * G));
  const int nq = Npad / 128;
  const long long total = (long long)BH * nq * PER_TILE;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const long long tile = g / PER_TILE;  // bh * nq + qt
    const int rem = (int)(g % PER_TILE);
    const int eb = rem / 128, r = rem % 128;
    const int bh = (int)(tile / nq), qt = (int)(tile % nq);
    const int n = qt * 128 + r;
    // float4 f of a tile: column group f / 128, row f % 128
    const float4* t = reinterpret_cast<const float4*>(dq_acc + (size_t)tile * 128 * D);
    float4 v[G];
#pragma unroll
    for (int j = 0; j < G; ++j)
      v[j] = FA_IN_BOUNDS(status, tile * 128 * D + 4 * ((eb * G + j) * 128 + r), 4, total / PER_TILE * 128 * D)
                 ? t[(eb * G + j) * 128 + r]
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    if (n >= N || !FA_IN_BOUNDS(status, ((size_t)bh * N + n) * D + 4 * G * eb, 4 * G, (size_t)BH * N * D)) continue;
    uint4* dst = reinterpret_cast<uint4*>(dQ + ((size_t)bh * N + n) * D + 4 * G * eb);
#pragma unroll
    for (int h = 0; h < G / 2; ++h) {
      const float4 a = v[2 * h], b = v[2 * h + 1];
      dst[h] = make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                          pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
    }
  }
}

// ------------------------------------------------------------------ main ---
template <int D>
struct Cfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int CHUNK_BYTES = 128 * 128;  // 128 rows x 128 bytes
  static constexpr int NST = D == 64 ? 4 : 2;    // Q/dO stages
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_BYTES;
  static constexpr int OFF_DS = 2 * TILE_BYTES;           // dS^T, 128 x 128 bf16 (2 chunks)
  static constexpr int OFF_QD = 2 * TILE_BYTES + 32768;   // stages of (Q, dO)
  // Per stage: the 128 -LSE*log2(e) values then the 128 -D values of the
  // stage's query tile (fp32, 1 KB).
  static constexpr int OFF_LD = OFF_QD + NST * 2 * TILE_BYTES;
  // The dynamic region starts 1024-byte aligned (the extern declaration
  // asks for it), so no slack is added: at d = 128 this is 226 KB, which
  // with the static barriers fills the 227 KB a CTA may use.
  // d = 64: each softmax warp stages its 32 rows of dV, then of dK (its 32
  // of the 64 columns, bf16: 2 KB) so that they leave eight rows per store
  // instruction.  (At d = 128 shared memory is full; there an item spans
  // many query tiles and its epilogue matters little.)
  static constexpr int OFF_EPI = OFF_LD + NST * 1024;
  static constexpr int EPI_BYTES = D == 64 ? 8 * 32 * 64 : 0;
  static constexpr int SMEM_BYTES = OFF_EPI + EPI_BYTES;
  // Tensor memory columns.  S^T fp32 in [0,128); once read, P^T (bf16
  // pairs) goes to [0,32) and [64,96): each column half of the softmax packs
  // its 64 queries into the first 32 of its own 64 score columns, so neither
  // half writes where the other is still reading.  Likewise dP^T fp32 in
  // [128,256), then dS^T in [128,160) and [192,224).  The score columns are
  // free as soon as dV has been issued, so the next tile's S^T can follow it
  // directly.
  static constexpr int COL_S = 0, COL_P = 0, COL_DP = 128, COL_DS = 128;
  // Column of the s-th 16-query slice (K = 16 of a gradient product) of
  // packed P^T or dS^T starting at `base`.
  __host__ __device__ static constexpr uint32_t col_packed(int base, int s) { return base + (s >> 2) * 64 + (s & 3) * 8; }
  static constexpr int COL_DV = 256, COL_DK = 256 + D;
  // dQ: d = 128 reuses the dP^T columns once dK has read dS^T (one buffer,
  // so the next dP^T waits for the drain); d = 64 has two spare 64-column
  // buffers after dK.
  static constexpr int NDQ = D == 64 ? 2 : 1;
  __host__ __device__ static constexpr int col_dq(int b) { return D == 128 ? 128 : 384 + 64 * b; }
  // A dQ tile (fp32, 4 * 128 * D bytes) reaches the accumulator by bulk
  // reduce-adds from shared memory.  d = 64: the tile's whole Q/dO stage
  // (2 * TILE_BYTES, dead once dQ has been computed) holds it for one bulk
  // add, after which the drain returns both halves of the stage.  d = 128:
  // with two stages, holding the Q half that long would starve the producer,
  // so only the dO half holds it, in two halves added one after the other,
  // and the MMA warp returns the Q half right after the dQ product.
  static constexpr int DQ_PARTS = D == 128 ? 2 : 1;
  static constexpr int DQ_PART_BYTES = 4 * 128 * D / DQ_PARTS;
  static constexpr int DQ_SLOT_OFF = D == 128 ? TILE_BYTES : 0;  // within the stage
  static_assert(DQ_SLOT_OFF + DQ_PART_BYTES <= 2 * TILE_BYTES, "dQ part exceeds its stage");
  // Registers per thread of the producer/MMA, softmax and drain warpgroups
  // (setmaxnreg).  Launch: 512 threads x 128; 128 x (REG_CTL + 2 REG_SMX +
  // REG_DRN) must stay <= 65536.  ptxas spills nothing at either d; at
  // d = 128, 136 for the softmax rather than 128 took the main kernel from
  // 1.294 to 1.283 ms.
  static constexpr uint32_t REG_CTL = 88;
  static constexpr uint32_t REG_SMX = 136;
  static constexpr uint32_t REG_DRN = 152;
  static_assert(REG_CTL + 2 * REG_SMX + REG_DRN <= 512, "register split exceeds the launch");
  // setmaxnreg.dec may only lower and setmaxnreg.inc only raise the 128
  // registers a thread starts with (anything else is an illegal instruction).
  static_assert(REG_CTL <= 128 && REG_SMX >= 128 && REG_DRN >= 128, "setmaxnreg direction");
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_gpu(uint32_t* a, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Bounded wait until *a == want (another CTA's release); false on timeout or
// abort, with the CTA marked as aborting.
__device__ bool wait_turn(const uint32_t* a, uint32_t want, const WaitCtx& w) {
  uint64_t start = 0;
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_gpu(a) == want) return true;
    if ((it & 15u) == 15u) {
      if (*w.abort_flag) return false;
      const uint64_t now = globaltimer_ns();
      if (start == 0) {
        start = now;
      } else if (now - start > w.timeout_ns) {
        *w.abort_flag = 1;
        atomicCAS(w.status, FA_DEV_OK, FA_DEV_ERR_TIMEOUT);
        return false;
      }
    }
    __nanosleep(64);
  }
}

constexpr int RING = 4;     // depth of the item ring the producer fills
constexpr int CONSUMERS = 13;  // MMA warp + 8 softmax warps + 4 drain warps

// VARLEN: per-sequence lengths are read (else every sequence has N, Nk).
template <int D, bool VARLEN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    main_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapdO,
                const __grid_constant__ CUtensorMap mapdK, const __grid_constant__ CUtensorMap mapdV,
                const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];

  __shared__ __align__(8) uint64_t kv_full, kv_empty, s_full, dp_full, p_full, ds_full, dkdv_full, mma_drain;
  // The dQ drain stages a tile in shared memory, in one or two parts, before
  // each bulk reduce-add (dq_staged[h]: all 128 drain threads have written
  // part h; dq_half: the first part has been read out).  One barrier per
  // part, each completing one phase per tile.
  __shared__ __align__(8) uint64_t dq_staged[2], dq_half;
  // d = 128, unordered dQ: the second half of a dQ tile is staged in the dS
  // buffer (free once the tile's dQ product has read it), so both halves
  // are in flight at once.  dss_full: the softmax has written dS to shared
  // memory (the dQ product may read it); sds_free: the drain's bulk read of
  // the half staged there is done (the softmax may write the next dS).
  __shared__ __align__(8) uint64_t dss_full, sds_free;
  // Each stage holds a query tile's Q (with its LSE values) and dO (with its
  // D values), filled and released independently: the dQ drain releases
  // what held the tile's dQ for its bulk reduction, the MMA warp the Q half
  // when that was not needed (Cfg::DQ_PARTS).
  __shared__ __align__(8) uint64_t q_full[C::NST], q_empty[C::NST], do_full[C::NST], do_empty[C::NST];
  __shared__ __align__(8) uint64_t dq_full[C::NDQ], dq_free[C::NDQ];
  // Dynamic schedule: the producer claims work items from a global counter
  // and passes them to the other roles through this ring.
  __shared__ __align__(8) uint64_t item_full[RING], item_empty[RING];
  __shared__ int item_ring[RING];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&kv_full, 1);
    mbar_init(&kv_empty, 1);
    mbar_init(&s_full, 1);
    mbar_init(&dp_full, 1);
    mbar_init(&p_full, 256);
    mbar_init(&ds_full, 256);
    mbar_init(&dkdv_full, 1);
    mbar_init(&mma_drain, 1);
    mbar_init(&dq_staged[0], 128);
    mbar_init(&dq_staged[1], 128);
    mbar_init(&dq_half, 1);
    mbar_init(&dss_full, 256);
    mbar_init(&sds_free, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    for (int b = 0; b < C::NDQ; ++b) {
      mbar_init(&dq_full[b], 1);
      mbar_init(&dq_free[b], 128);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(&item_full[r], 1);
      mbar_init(&item_empty[r], CONSUMERS);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    tma_prefetch_desc(&mapdO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const WaitCtx w{p.timeout_ns, &abort_flag, p.status};

  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sDS = smem + C::OFF_DS;
  uint8_t* sQD = smem + C::OFF_QD;
  const float* sLD = reinterpret_cast<const float*>(smem + C::OFF_LD);

  // Consumer side of the item ring: the k-th item this CTA processes.
  auto take_item = [&](uint32_t k, int& idx) -> bool {
    const uint32_t slot = k % RING;
    if (!mbar_wait(&item_full[slot], (k / RING) & 1, w)) return false;
    idx = *reinterpret_cast<volatile int*>(&item_ring[slot]);
    mbar_arrive(&item_empty[slot]);
    return true;
  };
  auto take_item_warp = [&](uint32_t k, int& idx) -> bool {
    const uint32_t slot = k % RING;
    if (!mbar_wait_warp(&item_full[slot], (k / RING) & 1, w)) return false;
    idx = *reinterpret_cast<volatile int*>(&item_ring[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[slot]);
    return true;
  };

  if (warp < 4) {
    regs_dec<C::REG_CTL>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t item_iter = 0, qd_iter = 0;
      bool ok = true, q_only = false;  // q_only: the last tile's dO load was never issued
      for (;; ++item_iter) {
        const uint32_t slot = item_iter % RING;
        ok = mbar_wait(&item_empty[slot], ((item_iter / RING) & 1) ^ 1, w);
        if (!ok) break;
        // CTA b starts on item b, then claims items gridDim.x, gridDim.x + 1, ...
        int idx = item_iter == 0 ? (int)blockIdx.x : (int)gridDim.x + (int)atomicAdd(p.sched, 1u);
        if (idx > p.n_items) idx = p.n_items;
        item_ring[slot] = idx;
        mbar_arrive(&item_full[slot]);
        if (idx >= p.n_items) break;
        const Item it = item_at<VARLEN>(p, idx);
        ok = mbar_wait(&kv_empty, (item_iter & 1) ^ 1, w);
        if (!ok) break;
        mbar_arrive_expect_tx(&kv_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c) {
          tma_load_3d(sK + c * C::CHUNK_BYTES, &mapK, &kv_full, c * 64, it.j * BK, it.bh);
          tma_load_3d(sV + c * C::CHUNK_BYTES, &mapV, &kv_full, c * 64, it.j * BK, it.bh);
        }
        for (int i = next_q<VARLEN>(p, it, 0); i < p.nq; i = next_q<VARLEN>(p, it, i + 1)) {
          const uint32_t st = qd_iter % C::NST;
          const uint32_t par = ((qd_iter / C::NST) & 1) ^ 1;
          uint8_t* q = sQD + st * 2 * C::TILE_BYTES;
          const size_t row0 = (size_t)it.bh * p.Npad + (size_t)i * BQ;
          uint8_t* ld = smem + C::OFF_LD + st * 1024;
          ok = mbar_wait(&q_empty[st], par, w);
          if (!ok) break;
          mbar_arrive_expect_tx(&q_full[st], C::TILE_BYTES + 512);
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(q + c * C::CHUNK_BYTES, &mapQ, &q_full[st], c * 64, i * BQ, it.bh);
          // (a debug build that finds row0 out of range loads the first rows
          // instead, so the barrier still gets its bytes)
          bulk_load(ld, p.L2w + (FA_IN_BOUNDS(p.status, row0, 128, (size_t)p.BH * p.Npad) ? row0 : 0), 512,
                    &q_full[st]);
          ok = mbar_wait(&do_empty[st], par, w);
          if (!ok) {
            ++qd_iter;
            q_only = true;
            break;
          }
          mbar_arrive_expect_tx(&do_full[st], C::TILE_BYTES + 512);
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_3d(q + C::TILE_BYTES + c * C::CHUNK_BYTES, &mapdO, &do_full[st], c * 64, i * BQ, it.bh);
          bulk_load(ld + 512, p.Dw + (FA_IN_BOUNDS(p.status, row0, 128, (size_t)p.BH * p.Npad) ? row0 : 0), 512,
                    &do_full[st]);
          ++qd_iter;
        }
        if (!ok) break;
      }
      if (!ok) {
        const uint64_t dl = globaltimer_ns() + 100000000ull;
        const uint32_t n = qd_iter < (uint32_t)C::NST ? qd_iter : (uint32_t)C::NST;
        for (uint32_t k = 0; k < n; ++k) {
          const uint32_t q = qd_iter - 1 - k;
          mbar_drain_wait(&q_full[q % C::NST], (q / C::NST) & 1, dl);
          if (!(k == 0 && q_only)) mbar_drain_wait(&do_full[q % C::NST], (q / C::NST) & 1, dl);
        }
        if (item_iter > 0) mbar_drain_wait(&kv_full, (item_iter - 1) & 1, dl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_T = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T: K-major A and B
      constexpr uint32_t IDESC_G = idesc_bf16_f32(128, D, 0, 1);    // dV, dK: A in TMEM, B MN-major
      constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, D, 1, 1);    // dQ: both MN-major
      uint32_t item_iter = 0, qd_iter = 0, dq_iter = 0, p_cnt = 0, ds_cnt = 0, dss_cnt = 0;
      bool ok = true, issued = false;
      // Descriptors built once; the products below only move them (one
      // 32-bit add per operand).  K-major forms (K = d) for the score
      // products, MN-major forms for the gradient products.
      const Desc kK = desc_sw128(smem_u32(sK), 16, 1024), kV = desc_sw128(smem_u32(sV), 16, 1024);
      const Desc kQD = desc_sw128(smem_u32(sQD), 16, 1024);
      const Desc mQD = desc_sw128(smem_u32(sQD), C::CHUNK_BYTES, 1024);
      const Desc mDS = desc_sw128(smem_u32(sDS), C::CHUNK_BYTES, 1024);
      const Desc mK = desc_sw128(smem_u32(sK), C::CHUNK_BYTES, 1024);

      // S^T = K Q^T into the score columns (M = keys, N = queries, K = d).
      auto issue_s = [&](uint32_t st) {
        const Desc q = desc_at(kQD, st * 2 * C::TILE_BYTES);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s >> 2) * C::CHUNK_BYTES + (s & 3) * 32;
          mma_ss(tmem + C::COL_S, desc_at(kK, off), desc_at(q, off), IDESC_T, s > 0 ? 1u : 0u);
        }
        tc_commit(&s_full);
      };
      // dP^T = V dO^T.  With d = 128 the dP^T columns hold the previous dQ
      // tile until the drain warps have read it.
      auto issue_dp = [&](uint32_t tile) -> bool {
        const uint32_t st = tile % C::NST;
        if (!mbar_wait(&do_full[st], (tile / C::NST) & 1, w)) return false;
        if (D == 128 && dq_iter > 0) {
          if (!mbar_wait(&dq_free[0], (dq_iter - 1) & 1, w)) return false;
        }
        tc_fence_after();
        const Desc dO = desc_at(kQD, st * 2 * C::TILE_BYTES + C::TILE_BYTES);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s >> 2) * C::CHUNK_BYTES + (s & 3) * 32;
          mma_ss(tmem + C::COL_DP, desc_at(kV, off), desc_at(dO, off), IDESC_T, s > 0 ? 1u : 0u);
        }
        tc_commit(&dp_full);
        return true;
      };

      for (;; ++item_iter) {
        int idx;
        ok = take_item(item_iter, idx);
        if (!ok || idx >= p.n_items) break;
        const Item it = item_at<VARLEN>(p, idx);
        ok = mbar_wait(&kv_full, item_iter & 1, w);
        if (!ok) break;
        int i = next_q<VARLEN>(p, it, 0);
        if (i < p.nq) {
          ok = mbar_wait(&q_full[qd_iter % C::NST], (qd_iter / C::NST) & 1, w);
          if (!ok) break;
          tc_fence_after();
          issue_s(qd_iter % C::NST);
          issued = true;
          ok = issue_dp(qd_iter);
          if (!ok) break;
        }
        for (int n = 0; ok && i < p.nq; ++n) {
          const int inext = next_q<VARLEN>(p, it, i + 1);
          const uint32_t st = qd_iter % C::NST;         // stage of query tile i
          const uint32_t stn = (qd_iter + 1) % C::NST;  // stage of query tile inext
          const Desc gQ = desc_at(mQD, st * 2 * C::TILE_BYTES);  // MN-major Q of tile i
          const Desc gdO = desc_at(gQ, C::TILE_BYTES);          // MN-major dO of tile i
          // dV += P^T dO (A = P^T in TMEM, K = 128 queries)
          ok = mbar_wait(&p_full, p_cnt & 1, w);
          if (!ok) break;
          ++p_cnt;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < BQ / 16; ++s)
            mma_ts(tmem + C::COL_DV, tmem + C::col_packed(C::COL_P, s), desc_at(gdO, s * 2048), IDESC_G,
                   (n > 0 || s > 0) ? 1u : 0u);
          // S^T of the next query tile goes in now: its columns were last read
          // by the dV product just issued, and its softmax can then overlap
          // the dK, dQ and next dP products.
          if (inext < p.nq) {
            ok = mbar_wait(&q_full[stn], ((qd_iter + 1) / C::NST) & 1, w);
            if (!ok) break;
            tc_fence_after();
            issue_s(stn);
          }
          // dK += dS^T Q (A = dS^T in TMEM); dQ_i = dS K
          ok = mbar_wait(&ds_full, ds_cnt & 1, w);
          if (!ok) break;
          ++ds_cnt;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < BQ / 16; ++s)
            mma_ts(tmem + C::COL_DK, tmem + C::col_packed(C::COL_DS, s), desc_at(gQ, s * 2048), IDESC_G,
                   (n > 0 || s > 0) ? 1u : 0u);
          const uint32_t b = dq_iter % C::NDQ;
          if (D == 64 && dq_iter >= (uint32_t)C::NDQ) {
            ok = mbar_wait(&dq_free[b], ((dq_iter / C::NDQ) - 1) & 1, w);
            if (!ok) break;
            tc_fence_after();
          }
          ok = mbar_wait(&dss_full, dss_cnt & 1, w);  // dS in shared memory
          if (!ok) break;
          ++dss_cnt;
#pragma unroll
          for (int s = 0; s < BK / 16; ++s)
            mma_ss(tmem + C::col_dq(b), desc_at(mDS, s * 2048), desc_at(mK, s * 2048), IDESC_Q, s > 0 ? 1u : 0u);
          tc_commit(&dq_full[b]);
          if (C::DQ_PARTS == 2) tc_commit(&q_empty[st]);  // the rest goes back via the dQ drain
          ++qd_iter;
          ++dq_iter;
          // dP^T of the next query tile (after the dQ drain when they share columns)
          if (inext < p.nq) ok = issue_dp(qd_iter);
          i = inext;
        }
        if (!ok) break;
        tc_commit(&dkdv_full);
        tc_commit(&kv_empty);
      }
      if (issued) {
        tc_commit(&mma_drain);
        mbar_drain_wait(&mma_drain, 0, globaltimer_ns() + 100000000ull);
      }
    }
  }
  } else if (warp < 12) {
    regs_inc<C::REG_SMX>();
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int hf = (warp - 4) >> 2;        // query half: columns [64 hf, 64 hf + 64)
    const int kr = quarter * 32 + lane;    // key row within the tile
    const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, dk_cnt = 0;
    bool ok = true;
    for (uint32_t k = 0;; ++k) {
      int idx;
      ok = take_item_warp(k, idx);
      if (!ok || idx >= p.n_items) break;
      const Item it = item_at<VARLEN>(p, idx);
      const int key = it.j * BK + kr;
      bool any = false;
      for (int i = next_q<VARLEN>(p, it, 0); i < p.nq; i = next_q<VARLEN>(p, it, i + 1)) {
        ok = mbar_wait_warp(&s_full, s_cnt & 1, w);
        if (!ok) break;
        const uint32_t par = s_cnt & 1;
        ++s_cnt;
        tc_fence_after();
        // this query tile's LSE and D values, staged in shared memory by the
        // producer with Q and dO (same stage index as the MMA warp uses)
        const float* sL = sLD + ((s_cnt - 1) % C::NST) * 256 + hf * 64;
        const float* sD = sL + 128;
        // causal: query row q sees this key iff key <= q + off; some pair in
        // the tile is hidden iff its last key exceeds its first row's limit
        const bool cmask = p.mask_kind == FA_MASK_CAUSAL && it.j * BK + BK - 1 > i * BQ + it.off;
        // element masks only where the causal boundary or a ragged last key
        // tile crosses the tile: column c of this thread is hidden iff
        // c < kq, kq folding both tests (a missing key hides every column)
        const bool masked = cmask || (it.j + 1) * BK > it.Lk;
        const int kq = key >= it.Lk ? INT_MAX : (cmask ? key - (i * BQ + hf * 64 + it.off) : INT_MIN);
        // ---- P^T = exp2(S^T * scale * log2e - LSE_i * log2e), kept packed
        // as bf16 pairs (the form the dV product reads) for the dS step too.
        uint32_t pk[32];
        {
          uint32_t sr[64];
          FA_TMEM_LD_X32(tmem + lane_bits + C::COL_S + hf * 64, sr);
          FA_TMEM_LD_X32(tmem + lane_bits + C::COL_S + hf * 64 + 32, (sr + 32));
          tc_wait_ld();
          // (-LSE * log2e and -D are stored negated: two columns per packed
          // fp32 instruction, each lane rounding as the scalar form)
          const float4* l4 = reinterpret_cast<const float4*>(sL);
          const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float4 lv = l4[u];
            const float2 y0 = __ffma2_rn(make_float2(__uint_as_float(sr[4 * u + 0]), __uint_as_float(sr[4 * u + 1])),
                                         sl2x2, make_float2(lv.x, lv.y));
            const float2 y1 = __ffma2_rn(make_float2(__uint_as_float(sr[4 * u + 2]), __uint_as_float(sr[4 * u + 3])),
                                         sl2x2, make_float2(lv.z, lv.w));
            float pv[4] = {ex2_approx(y0.x), ex2_approx(y0.y), ex2_approx(y1.x), ex2_approx(y1.y)};
            if (masked) {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (kq > 4 * u + e) pv[e] = 0.0f;
            }
            pk[2 * u] = pack_bf16x2(pv[0], pv[1]);
            pk[2 * u + 1] = pack_bf16x2(pv[2], pv[3]);
          }
        }
        // over the first 32 of this half's own 64 score columns, all loaded
        FA_TMEM_ST_X32(tmem + lane_bits + C::COL_P + hf * 64, pk);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full);
        // ---- dS^T = P^T * (dP^T - D), with P as the bf16 values above
        ok = mbar_wait_warp(&dp_full, par, w);
        if (!ok) break;
        tc_fence_after();
        uint32_t dk[32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t dr[32];
          FA_TMEM_LD_X32(tmem + lane_bits + C::COL_DP + hf * 64 + cc * 32, dr);
          tc_wait_ld();
          const float4* d4 = reinterpret_cast<const float4*>(sD + cc * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 dv = d4[u];
            const uint32_t w0 = pk[cc * 16 + 2 * u], w1 = pk[cc * 16 + 2 * u + 1];
            const float2 t0 = __fadd2_rn(make_float2(__uint_as_float(dr[u * 4 + 0]), __uint_as_float(dr[u * 4 + 1])),
                                         make_float2(dv.x, dv.y));
            const float2 t1 = __fadd2_rn(make_float2(__uint_as_float(dr[u * 4 + 2]), __uint_as_float(dr[u * 4 + 3])),
                                         make_float2(dv.z, dv.w));
            const float2 g01 = __fmul2_rn(make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xffff0000u)), t0);
            const float2 g23 = __fmul2_rn(make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xffff0000u)), t1);
            dk[cc * 16 + u * 2 + 0] = pack_bf16x2(g01.x, g01.y);
            dk[cc * 16 + u * 2 + 1] = pack_bf16x2(g23.x, g23.y);
          }
        }
        // over the first 32 of this half's own 64 dP^T columns, all loaded
        FA_TMEM_ST_X32(tmem + lane_bits + C::COL_DS + hf * 64, dk);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&ds_full);  // dK may start
        // Shared-memory copy of dS^T (the A operand of dQ = dS K), 128-byte
        // swizzle: 16-byte unit u of row kr lives at unit (u ^ (kr & 7)).
        // With the split drain the buffer may still hold half of the
        // previous dQ tile on its way to the accumulator.  Otherwise its
        // only other reader, the previous dQ product, has completed: the MMA
        // warp issues this tile's dP^T after that product, and dp_full (the
        // commit of both) was waited for above.
        if (D == 128 && !p.deterministic && s_cnt > 1) {
          ok = mbar_wait_warp(&sds_free, (s_cnt - 2) & 1, w);
          if (!ok) break;
        }
        uint8_t* ds_row = sDS + hf * C::CHUNK_BYTES + kr * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int unit = u ^ (kr & 7);
          *reinterpret_cast<uint4*>(ds_row + unit * 16) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&dss_full);
        any = true;
      }
      if (!ok) break;
      // ---- epilogue: dV and dK rows of this key tile
      ok = mbar_wait_warp(&dkdv_full, dk_cnt & 1, w);
      if (!ok) break;
      ++dk_cnt;
      tc_fence_after();
      const bool store = key < p.Nk;
      const size_t gbase = ((size_t)it.bh * p.Nk + key) * D;
#pragma unroll
      for (int g = 0; g < 2; ++g) {  // 0: dV, 1: dK
        const float mul = g == 0 ? 1.0f : p.scale;
        __nv_bfloat16* dst = (g == 0 ? p.dV : p.dK) + gbase;
        const int colbase = (g == 0 ? C::COL_DV : C::COL_DK) + hf * (D / 2);
        if constexpr (C::EPI_BYTES > 0) {
          // Lane i puts its 64 bytes (four 16-byte chunks, chunk c at slot
          // c ^ ((i >> 1) & 3), which is the 64-byte swizzle) into the warp's
          // 2 KB; then lane 0 stores the 32 x 32 box with one tensor store
          // (keys past Nk are not written).
          uint8_t* ws = smem + C::OFF_EPI + (warp - 4) * 2048;
          uint32_t v[32];
          FA_TMEM_LD_X32(tmem + lane_bits + colbase, v);
          tc_wait_ld();
          if (lane == 0) bulk_wait_read_all();  // the warp's previous store has read the buffer
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t q[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(v[8 * c + 2 * e]), __uint_as_float(v[8 * c + 2 * e + 1])),
                                          make_float2(mul, mul));
              q[e] = any ? pack_bf16x2(o.x, o.y) : 0u;
            }
            *reinterpret_cast<uint4*>(ws + lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16)) = make_uint4(q[0], q[1], q[2], q[3]);
          }
          fence_proxy_async_smem();  // the generic-proxy writes, before the tensor store reads them
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(g == 0 ? &mapdV : &mapdK, ws, hf * 32, it.j * BK + quarter * 32, it.bh);
            bulk_commit_group();
          }
        } else {
#pragma unroll
          for (int c = 0; c < D / 2; c += 32) {
            uint32_t v[32];
            FA_TMEM_LD_X32(tmem + lane_bits + colbase + c, v);
            tc_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])),
                                          make_float2(mul, mul));
              pk[e] = any ? pack_bf16x2(o.x, o.y) : 0u;
            }
            if (store && FA_IN_BOUNDS(p.status, gbase + hf * (D / 2) + c, 32, (size_t)p.BH * p.Nk * D)) {
              uint4* o = reinterpret_cast<uint4*>(dst + hf * (D / 2) + c);
#pragma unroll
              for (int e = 0; e < 4; ++e) o[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
          }
        }
      }
      tc_fence_before();
    }
    if (C::EPI_BYTES > 0 && lane == 0) bulk_wait_all();  // this warp's dK/dV stores are done before the CTA leaves
  } else {
    regs_inc<C::REG_DRN>();
    // ------------------------------------------------------------ dQ drain
    // Read the whole dQ tile out of tensor memory, hand the columns back to
    // the MMA warp, then add the tile into the fp32 accumulator with bulk
    // reduce-adds (the TMA engine: vector reductions from the threads
    // saturated the load/store pipe that everything else here also uses).
    const int quarter = warp & 3;
    const int qr = quarter * 32 + lane;
    const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
    const bool leader = warp == 12 && lane == 0;
    uint32_t dq_iter = 0;
    bool ok = true, bulk_issued = false;
    for (uint32_t k = 0;; ++k) {
      int idx;
      ok = take_item_warp(k, idx);
      if (!ok || idx >= p.n_items) break;
      const Item it = item_at<VARLEN>(p, idx);
      for (int i = next_q<VARLEN>(p, it, 0); i < p.nq; i = next_q<VARLEN>(p, it, i + 1)) {
        const uint32_t b = dq_iter % C::NDQ;
        const uint32_t st = dq_iter % C::NST;
        ok = mbar_wait_warp(&dq_full[b], (dq_iter / C::NDQ) & 1, w);
        if (!ok) break;
        tc_fence_after();
        // With the split drain (d = 128, unordered) columns 64..127 are
        // staged first: they go to v[0, 64) and columns 0..63 to v[64, 128).
        const bool split = D == 128 && !p.deterministic;
        uint32_t v[D];
#pragma unroll
        for (int c = 0; c < D; c += 32)
          FA_TMEM_LD_X32(tmem + lane_bits + C::col_dq(b) + (split ? (c + D / 2) % D : c), (v + c));
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&dq_free[b]);
        // Stage the tile in its dead stage (the products that read it have
        // completed) in the accumulator's tiled layout, columns 4e..4e+3 of
        // row qr at byte e * 2048 + qr * 16 of a part, and add each part with
        // one bulk reduce-add (Cfg::DQ_PARTS).
        constexpr int GROUPS = D / 4 / C::DQ_PARTS;  // 4-column groups per part
        uint8_t* slot = sQD + st * 2 * C::TILE_BYTES + C::DQ_SLOT_OFF;
        float* dst = p.dq_acc + ((size_t)it.bh * p.Npad + (size_t)i * BQ) * D;
        if (D == 128 && !p.deterministic) {
          // Both halves in flight at once: columns 64..127 staged in the dS
          // buffer (its dQ product has completed) and added first, columns
          // 0..63 in the tile's dO half.  The dS buffer goes back to the
          // softmax once its half has been read, the dO half to the producer
          // once the second has.
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // h = 0: columns 64..127 (v[0, 64)) into the dS buffer;
            // h = 1: columns 0..63 (v[64, 128)) into the dO half
            uint8_t* buf = h == 0 ? sDS : slot;
            const int part = 1 - h;  // which half of the accumulator tile
#pragma unroll
            for (int e = 0; e < GROUPS; ++e) {
              const int g = h * GROUPS + e;
              *reinterpret_cast<uint4*>(buf + e * 2048 + qr * 16) =
                  make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
            }
            fence_proxy_async_smem();
            // a warp that has run ahead arrives only once the previous
            // tile's phase of this barrier is complete
            if (dq_iter > 0) {
              ok = mbar_wait_warp(&dq_staged[h], (dq_iter - 1) & 1, w);
              if (!ok) break;
            }
            mbar_arrive(&dq_staged[h]);
            if (leader) {
              ok = mbar_wait(&dq_staged[h], dq_iter & 1, w);
              if (ok && FA_IN_BOUNDS(p.status, ((size_t)it.bh * p.Npad + (size_t)i * BQ) * D + part * GROUPS * 512,
                                     C::DQ_PART_BYTES / 4, (size_t)p.BH * p.Npad * D))
                bulk_reduce_add_f32(dst + part * GROUPS * 512, buf, C::DQ_PART_BYTES);
              bulk_commit_group();
              bulk_issued = true;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
          }
          if (!ok) break;
          if (leader) {
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");  // the dS-buffer half
            mbar_arrive(&sds_free);
            bulk_wait_read_all();
            mbar_arrive(&do_empty[st]);
          }
          __syncwarp();
          ++dq_iter;
          continue;
        }
#pragma unroll
        for (int h = 0; h < C::DQ_PARTS; ++h) {
          if (h == 1) {
            ok = mbar_wait_warp(&dq_half, dq_iter & 1, w);  // first part read out
            if (!ok) break;
          }
#pragma unroll
          for (int e = 0; e < GROUPS; ++e) {
            const int g = h * GROUPS + e;
            *reinterpret_cast<uint4*>(slot + e * 2048 + qr * 16) =
                make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
          }
          fence_proxy_async_smem();
          // A warp that has run ahead arrives only once the previous tile's
          // phase of this barrier is complete (else its arrival would count
          // toward that phase).
          if (dq_iter > 0) {
            ok = mbar_wait_warp(&dq_staged[h], (dq_iter - 1) & 1, w);
            if (!ok) break;
          }
          mbar_arrive(&dq_staged[h]);
          if (leader) {
            ok = mbar_wait(&dq_staged[h], dq_iter & 1, w);
            uint32_t* turn = p.turn + (size_t)it.bh * p.nq + i;
            const bool turn_ok = !p.deterministic ||
                                 FA_IN_BOUNDS(p.status, (size_t)it.bh * p.nq + i, 1, (size_t)p.BH * p.nq);
            if (ok && p.deterministic && h == 0 && turn_ok) {
              ok = wait_turn(turn, add_rank(p, it.j, i), w);
              fence_proxy_async_global();
            }
            if (ok) {
              if (FA_IN_BOUNDS(p.status, ((size_t)it.bh * p.Npad + (size_t)i * BQ) * D + h * GROUPS * 512,
                               C::DQ_PART_BYTES / 4, (size_t)p.BH * p.Npad * D))
                bulk_reduce_add_f32(dst + h * GROUPS * 512, slot, C::DQ_PART_BYTES);
              bulk_commit_group();
              bulk_issued = true;
              bulk_wait_read_all();
              if (p.deterministic && h + 1 == C::DQ_PARTS && turn_ok) {
                // the additions are complete in global memory before the turn passes
                bulk_wait_all();
                fence_proxy_async_global();
                red_release_add_gpu(turn, 1u);
              }
              if (h + 1 < C::DQ_PARTS) {
                mbar_arrive(&dq_half);
              } else {
                if (C::DQ_PARTS == 1) mbar_arrive(&q_empty[st]);
                mbar_arrive(&do_empty[st]);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
        if (!ok) break;
        ++dq_iter;
      }
    }
    if (leader && bulk_issued) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bwd

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
  const int Npad = ((N + 127) / 128) * 128;
  return bwd::workspace_layout(B * H, Npad, d).total;
}

template <int D>
static fa_status launch_bwd_d(const Problem& pr, const CUtensorMap& mQ, const CUtensorMap& mK, const CUtensorMap& mV,
                              const CUtensorMap& mdO, const void* O, const void* dO, const float* LSE, void* dQ,
                              void* dK, void* dV, void* workspace, cudaStream_t s, uint32_t* st, int stage) {
  const int Npad = pr.nq * 128;
  const bwd::Workspace wl = bwd::workspace_layout(pr.BH, Npad, D);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws + wl.dq_off);
  float* Dw = reinterpret_cast<float*>(ws + wl.d_off);
  float* L2w = reinterpret_cast<float*>(ws + wl.l2_off);
  uint32_t* sched = reinterpret_cast<uint32_t*>(ws + wl.sched_off);
  uint32_t* turn = reinterpret_cast<uint32_t*>(ws + wl.turn_off);
  const int sms = num_sms();

  if (stage < 0 || stage == 0) {
    const long long rows = (long long)pr.BH * Npad;
    const long long warps_needed = (rows + (32 / (D / 8)) - 1) / (32 / (D / 8));
    long long blocks = (warps_needed + 7) / 8;
    if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
    bwd::prep_kernel<D><<<(int)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(O),
                                                     static_cast<const __nv_bfloat16*>(dO), LSE, Dw, L2w, dq_acc,
                                                     sched, turn, pr.BH, pr.N, Npad, pr.H, pr.seqlens_q, st);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stage < 0 || stage == 1) {
    bwd::Params p;
    p.BH = pr.BH;
    p.N = pr.N;
    p.Npad = Npad;
    p.nq = pr.nq;
    p.Nk = pr.Nk;
    p.nk = pr.nk;
    p.off = pr.off;
    p.H = pr.H;
    p.seqlens_q = pr.seqlens_q;
    p.seqlens_k = pr.seqlens_k;
    p.n_items = pr.BH * pr.nk;
    p.mask_kind = pr.mask_kind;
    p.block_mask = pr.block_mask;
    p.scale = pr.scale;
    p.scale_log2 = pr.scale_log2;
    p.Dw = Dw;
    p.L2w = L2w;
    p.dq_acc = dq_acc;
    p.sched = sched;
    p.turn = turn;
    p.deterministic = pr.deterministic;
    p.group = bwd::sched_group(pr.BH, pr.N, pr.d);
    p.dK = static_cast<__nv_bfloat16*>(dK);
    p.dV = static_cast<__nv_bfloat16*>(dV);
    p.timeout_ns = wait_timeout_ns();
    p.status = st;
    // dK and dV as 32 x 32 boxes for the d = 64 epilogue's tensor stores
    CUtensorMap mdK, mdV;
    if (!make_map_bf16_box(&mdK, dK, pr.BH, pr.Nk, pr.d, 32, 32) || !make_map_bf16_box(&mdV, dV, pr.BH, pr.Nk, pr.d, 32, 32))
      return FA_ERR_CUDA;
    constexpr int smem = bwd::Cfg<D>::SMEM_BYTES;
    const int grid = p.n_items < sms ? p.n_items : sms;
    auto run = [&](auto kern) -> bool {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return false;
      kern<<<grid, bwd::NUM_THREADS, smem, s>>>(mQ, mK, mV, mdO, mdK, mdV, p);
      return true;
    };
    const bool varlen = pr.seqlens_q || pr.seqlens_k;
    if (!(varlen ? run(bwd::main_kernel<D, true>) : run(bwd::main_kernel<D, false>))) return FA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stage < 0 || stage == 2) {
    // one thread per 16 columns of a padded row; the loop covers any excess
    const long long threads = (long long)pr.BH * Npad * (D / 16);
    const long long blocks = (threads + 255) / 256;
    const unsigned grid = (unsigned)(blocks < 0x7fffffffll ? blocks : 0x7fffffffll);
    bwd::dq_convert_kernel<D><<<grid, 256, 0, s>>>(dq_acc, static_cast<__nv_bfloat16*>(dQ), pr.BH, pr.N, Npad,
                                                   pr.scale, st);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status launch_bwd(const Problem& pr, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const float* LSE, void* dQ, void* dK, void* dV, void* workspace, cudaStream_t s, int stage) {
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  CUtensorMap mQ, mK, mV, mdO;
  if (!make_map_bf16(&mQ, Q, pr.BH, pr.N, pr.d, 128) || !make_map_bf16(&mK, K, pr.BH, pr.Nk, pr.d, 128) ||
      !make_map_bf16(&mV, V, pr.BH, pr.Nk, pr.d, 128) || !make_map_bf16(&mdO, dO, pr.BH, pr.N, pr.d, 128))
    return FA_ERR_CUDA;
  if (pr.d == 64) return launch_bwd_d<64>(pr, mQ, mK, mV, mdO, O, dO, LSE, dQ, dK, dV, workspace, s, st, stage);
  return launch_bwd_d<128>(pr, mQ, mK, mV, mdO, O, dO, LSE, dQ, dK, dV, workspace, s, st, stage);
}

}  // namespace fa
