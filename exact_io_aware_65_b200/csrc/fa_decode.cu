// fa_decode.cu -- a few new queries against a long key/value history
// (decoding against a KV cache), split over the keys.
//
// The method is the same exact attention ("FlashAttention: making attention
// fast by respecting the memory hierarchy", tiling paragraph: blocks of keys
// and values stream past the queries with a running maximum and sum); the
// pages pair it with the KV cache of autoregressive generation ("Flash
// Attention", "Product And Infrastructure Pressure" and "Related Topics").
// With Nq <= 16 query rows per head and Nk keys, every K and V element is
// read once from HBM and used Nq times: the work is bound by HBM, so it runs
// on the CUDA cores (the tensor cores' 128-row tiles would be almost empty).
//
// Kernel 1 (partial): persistent CTAs of 128 threads take work units (head,
// chunk of CH keys) round-robin.  The 64-key tiles of K and V are contiguous
// in [B,H,Nk,d], so each arrives by one bulk copy into a two-stage ring.  Per
// tile and query: scores s = (scale log2 e) q . k, the running maximum m and
// sum l of the online softmax, and O_u += 2^(s - m) V.  A unit leaves its
// unnormalised O_u with m_u and l_u in the workspace.
// Kernel 2 (merge), per (head, query): M = max_u m_u,
// L = sum_u l_u 2^(m_u - M), O = sum_u 2^(m_u - M) O_u / L,
// LSE = (M + log2 L) ln 2.  A query that sees no key gets O = 0, LSE = -inf.
#include <cuda_bf16.h>
#include <math.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace dec {

constexpr int THREADS = 128;
constexpr int TK = 64;      // keys per tile
constexpr int NS = 2;       // ring stages (small, so that three CTAs fit per SM at d = 128:
                            // the per-tile block barriers are hidden by the other CTAs)
constexpr int NQ_MAX = 16;  // query rows per head
constexpr float LN2 = 0.69314718055994530942f;

template <int D>
struct Cfg {
  static constexpr int TILE_BYTES = TK * D * 2;            // one K or V tile (bf16)
  static constexpr int OFF_Q = NS * 2 * TILE_BYTES;        // the head's queries, bf16 [NQ_MAX][D]
  static constexpr int OFF_S = OFF_Q + NQ_MAX * D * 2;     // scores, then p: fp32 [NQ_MAX][TK]
  static constexpr int SMEM_BYTES = OFF_S + NQ_MAX * TK * 4;
};
// Queries a thread accumulates O for, for problems of up to NQT queries (a
// thread owns one column; at d = 64 the two thread halves split the queries).
template <int D, int NQT>
constexpr int qpt() { return D == 128 ? NQT : (NQT + 1) / 2; }

struct Params {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int BH, Nq, Nk, off;  // off = Nk - Nq: causal query i sees keys j <= i + off
  int causal;
  float sl2;            // scale * log2(e)
  int CH, nchunks, n_units;
  float* part;          // [n_units, Nq, D] unnormalised O
  float2* ml;           // [n_units, Nq] (m, l), m in scaled log2 units
  uint64_t timeout_ns;
  uint32_t* status;
};

// bf16 pair -> two floats (exact: a bf16 is the high half of an fp32)
__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

struct Unit {
  int bh, k_begin, k_end, ntile;
};
__device__ __forceinline__ Unit unit_at(const Params& p, int u) {
  Unit r;
  r.bh = u / p.nchunks;
  r.k_begin = (u % p.nchunks) * p.CH;
  r.k_end = min(r.k_begin + p.CH, p.Nk);
  r.ntile = (r.k_end - r.k_begin + TK - 1) / TK;
  return r;
}

template <int D, int NQT>
__global__ void __launch_bounds__(THREADS, 3) partial_kernel(const Params p) {
  using C = Cfg<D>;
  constexpr int QPT = qpt<D, NQT>();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[NS];
  __shared__ float m_run[NQ_MAX], l_run[NQ_MAX], alpha[NQ_MAX];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_Q);
  float* sS = reinterpret_cast<float*>(smem + C::OFF_S);
  const WaitCtx w{p.timeout_ns, &abort_flag, p.status};

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // Producer state (thread 0): the next tile to load, in the consumers' order.
  int pu = blockIdx.x, ptile = 0;
  uint32_t issued = 0;
  auto issue_next = [&]() {
    if (pu >= p.n_units) return;
    const Unit un = unit_at(p, pu);
    const int k0 = un.k_begin + ptile * TK;
    const int rows = min(TK, un.k_end - k0);
    const uint32_t bytes = (uint32_t)rows * D * 2;
    const uint32_t s = issued % NS;
    uint8_t* kdst = smem + s * 2 * C::TILE_BYTES;
    size_t src = ((size_t)un.bh * p.Nk + k0) * D;
    // (a debug build that finds the tile out of range copies the cache's
    // first rows instead, so the barrier still gets its bytes)
    if (!FA_IN_BOUNDS(p.status, src, (size_t)rows * D, (size_t)p.BH * p.Nk * D)) src = 0;
    mbar_arrive_expect_tx(&full[s], 2 * bytes);
    bulk_load(kdst, p.K + src, bytes, &full[s]);
    bulk_load(kdst + C::TILE_BYTES, p.V + src, bytes, &full[s]);
    ++issued;
    if (++ptile == un.ntile) {
      ptile = 0;
      pu += gridDim.x;
    }
  };
  if (tid == 0)
    for (int s = 0; s < NS; ++s) issue_next();

  uint32_t t = 0;  // tiles consumed
  bool ok = true;
  for (int u = blockIdx.x; ok && u < p.n_units; u += gridDim.x) {
    const Unit un = unit_at(p, u);
    // this head's queries (bf16, exact copies) and fresh softmax state
    for (int i = tid; i < p.Nq * D / 8; i += THREADS)
      reinterpret_cast<uint4*>(sQ)[i] =
          FA_IN_BOUNDS(p.status, (size_t)un.bh * p.Nq * D + 8 * i, 8, (size_t)p.BH * p.Nq * D)
              ? reinterpret_cast<const uint4*>(p.Q + (size_t)un.bh * p.Nq * D)[i]
              : make_uint4(0u, 0u, 0u, 0u);
    if (tid < NQ_MAX) {
      m_run[tid] = -INFINITY;
      l_run[tid] = 0.0f;
    }
    float acc[QPT];
#pragma unroll
    for (int q = 0; q < QPT; ++q) acc[q] = 0.0f;
    __syncthreads();

    for (int tile = 0; tile < un.ntile; ++tile, ++t) {
      const uint32_t s = t % NS;
      ok = mbar_wait_warp(&full[s], (t / NS) & 1, w);
      // every warp must leave the loop together: agree on the outcome
      ok = __syncthreads_and(ok ? 1 : 0) != 0;
      if (!ok) break;
      const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(smem + s * 2 * C::TILE_BYTES);
      const __nv_bfloat16* sV = sK + TK * D;
      const int k0 = un.k_begin + tile * TK;
      const int rows = min(TK, un.k_end - k0);

      // ---- scores: thread -> key kk, queries g, g + 2, ...  Chunks of 8
      // elements are read in a rotated order so the rows of a warp's keys
      // fall in different banks.
      {
        const int kk = tid & (TK - 1), g = tid >> 6;
        const int kabs = k0 + kk;
        for (int q = g; q < p.Nq; q += 2) {
          float sc = -INFINITY;
          if (kk < rows && (!p.causal || kabs <= q + p.off)) {
            const uint4* kr = reinterpret_cast<const uint4*>(sK + kk * D);
            const uint4* qr = reinterpret_cast<const uint4*>(sQ + q * D);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
              const int ci = (i + kk) & (D / 8 - 1);
              const uint4 kv = kr[ci], qv = qr[ci];
              a0 = fmaf(lo_f(kv.x), lo_f(qv.x), a0);
              a1 = fmaf(hi_f(kv.x), hi_f(qv.x), a1);
              a0 = fmaf(lo_f(kv.y), lo_f(qv.y), a0);
              a1 = fmaf(hi_f(kv.y), hi_f(qv.y), a1);
              a0 = fmaf(lo_f(kv.z), lo_f(qv.z), a0);
              a1 = fmaf(hi_f(kv.z), hi_f(qv.z), a1);
              a0 = fmaf(lo_f(kv.w), lo_f(qv.w), a0);
              a1 = fmaf(hi_f(kv.w), hi_f(qv.w), a1);
            }
            sc = (a0 + a1) * p.sl2;
          }
          sS[q * TK + kk] = sc;
        }
      }
      __syncthreads();

      // ---- online softmax: warp -> queries warp, warp + 4, ...
      for (int q = warp; q < p.Nq; q += 4) {
        const float a = sS[q * TK + lane], b = sS[q * TK + lane + 32];
        float mx = fmaxf(a, b);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mo = m_run[q];
        const float mn = fmaxf(mo, mx);
        float al = 1.0f, pa = 0.0f, pb = 0.0f;
        if (mn != -INFINITY) {  // else nothing seen yet: p = 0, state unchanged
          al = ex2_approx(mo - mn);  // 0 when mo == -inf
          pa = ex2_approx(a - mn);
          pb = ex2_approx(b - mn);
        }
        sS[q * TK + lane] = pa;
        sS[q * TK + lane + 32] = pb;
        float sm = pa + pb;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        if (lane == 0) {
          m_run[q] = mn;
          l_run[q] = l_run[q] * al + sm;
          alpha[q] = al;
        }
      }
      __syncthreads();

      // ---- O_u = alpha O_u + p V over the tile's valid rows
      {
        const int c = D == 128 ? tid : (tid & 63);
        const int q0 = D == 128 ? 0 : (tid >> 6), qs = D == 128 ? 1 : 2;
        const __nv_bfloat16* vc = sV + c;
#pragma unroll
        for (int qi = 0; qi < QPT; ++qi) {
          const int q = q0 + qi * qs;
          if (q < p.Nq) acc[qi] *= alpha[q];
        }
        // unrolled so that the loads of several keys are in flight at once
#pragma unroll 8
        for (int kk = 0; kk < rows; ++kk) {
          const float v = __bfloat162float(vc[kk * D]);
#pragma unroll
          for (int qi = 0; qi < QPT; ++qi) {
            const int q = q0 + qi * qs;
            if (q < p.Nq) acc[qi] = fmaf(sS[q * TK + kk], v, acc[qi]);
          }
        }
      }
      __syncthreads();  // the stage and the scores are free again
      if (tid == 0) issue_next();
    }
    if (!ok) break;

    // ---- this unit's partial result
    {
      const int c = D == 128 ? tid : (tid & 63);
      const int q0 = D == 128 ? 0 : (tid >> 6), qs = D == 128 ? 1 : 2;
#pragma unroll
      for (int qi = 0; qi < QPT; ++qi) {
        const int q = q0 + qi * qs;
        if (q < p.Nq && FA_IN_BOUNDS(p.status, ((size_t)u * p.Nq + q) * D + c, 1, (size_t)p.n_units * p.Nq * D))
          p.part[((size_t)u * p.Nq + q) * D + c] = acc[qi];
      }
      if (tid < p.Nq && FA_IN_BOUNDS(p.status, (size_t)u * p.Nq + tid, 1, (size_t)p.n_units * p.Nq))
        p.ml[(size_t)u * p.Nq + tid] = make_float2(m_run[tid], l_run[tid]);
    }
    __syncthreads();  // sQ and the softmax state are reused by the next unit
  }
  if (!ok && tid == 0) {
    // let the copies already issued land before the CTA's memory is released
    const uint64_t dl = globaltimer_ns() + 100000000ull;
    for (uint32_t k = t; k < issued; ++k) mbar_drain_wait(&full[k % NS], (k / NS) & 1, dl);
  }
}

template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const Params p, __nv_bfloat16* O, float* LSE) {
  const int bh = blockIdx.x / p.Nq, q = blockIdx.x % p.Nq, c = threadIdx.x;
  const int u0 = bh * p.nchunks;
  if (!FA_IN_BOUNDS(p.status, ((size_t)bh * p.Nq + q) * D + c, 1, (size_t)p.BH * p.Nq * D) ||
      !FA_IN_BOUNDS(p.status, (size_t)(u0 + p.nchunks - 1) * p.Nq + q, 1, (size_t)p.n_units * p.Nq))
    return;
  float M = -INFINITY;
  for (int ch = 0; ch < p.nchunks; ++ch) M = fmaxf(M, p.ml[(size_t)(u0 + ch) * p.Nq + q].x);
  __nv_bfloat16* o = O + ((size_t)bh * p.Nq + q) * D;
  if (M == -INFINITY) {  // this query sees no key
    o[c] = __float2bfloat16(0.0f);
    if (c == 0) LSE[(size_t)bh * p.Nq + q] = -INFINITY;
    return;
  }
  float L = 0.0f, acc = 0.0f;
  for (int ch = 0; ch < p.nchunks; ++ch) {
    const int u = u0 + ch;
    const float2 ml = p.ml[(size_t)u * p.Nq + q];
    if (ml.x == -INFINITY) continue;  // a chunk of keys this query does not see
    const float f = ex2_approx(ml.x - M);
    L = fmaf(ml.y, f, L);
    acc = fmaf(p.part[((size_t)u * p.Nq + q) * D + c], f, acc);
  }
  o[c] = __float2bfloat16(acc / L);
  if (c == 0) LSE[(size_t)bh * p.Nq + q] = (M + log2f(L)) * LN2;
}

// Units and grid for a problem on the current device.
struct Plan {
  int grid, CH, nchunks, n_units;
};
template <int D>
static bool plan(int BH, int Nk, Plan* pl) {
  int per_sm = 0;
  // every instantiation uses the same shared memory; the largest sets the pace
  if (cudaFuncSetAttribute(partial_kernel<D, NQ_MAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg<D>::SMEM_BYTES) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, partial_kernel<D, NQ_MAX>, THREADS,
                                                    Cfg<D>::SMEM_BYTES) != cudaSuccess ||
      per_sm <= 0)
    return false;
  const long long slots = (long long)num_sms() * per_sm;
  // about four units per resident CTA, chunks of at least 256 keys
  const long long want = (4 * slots + BH - 1) / BH;
  long long ch = ((long long)Nk + want - 1) / want;
  ch = ((ch + TK - 1) / TK) * TK;
  if (ch < 256) ch = 256;
  pl->CH = (int)ch;
  pl->nchunks = (int)((Nk + ch - 1) / ch);
  pl->n_units = BH * pl->nchunks;
  pl->grid = (int)(pl->n_units < slots ? pl->n_units : slots);
  return true;
}

}  // namespace dec

static size_t decode_ws(const dec::Plan& pl, int Nq, int d) {
  const size_t part = (size_t)pl.n_units * Nq * d * sizeof(float);
  const size_t ml = (size_t)pl.n_units * Nq * sizeof(float2);
  return ((part + 255) & ~size_t(255)) + ml;
}

size_t decode_workspace_bytes(int BH, int Nq, int Nk, int d) {
  dec::Plan pl;
  if (!(d == 64 ? dec::plan<64>(BH, Nk, &pl) : dec::plan<128>(BH, Nk, &pl))) return 0;
  return decode_ws(pl, Nq, d);
}

template <int D>
static fa_status launch_decode_d(const Problem& pr, const void* Q, const void* K, const void* V, void* O, float* LSE,
                                 void* workspace, size_t workspace_bytes, cudaStream_t s) {
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  dec::Plan pl;
  if (!dec::plan<D>(pr.BH, pr.Nk, &pl)) return FA_ERR_CUDA;
  const size_t part_bytes = ((size_t)pl.n_units * pr.N * D * sizeof(float) + 255) & ~size_t(255);
  if (workspace_bytes < decode_ws(pl, pr.N, D)) return FA_ERR_WORKSPACE;
  dec::Params p;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.BH = pr.BH;
  p.Nq = pr.N;
  p.Nk = pr.Nk;
  p.off = pr.off;
  p.causal = pr.mask_kind == FA_MASK_CAUSAL;
  p.sl2 = pr.scale_log2;
  p.CH = pl.CH;
  p.nchunks = pl.nchunks;
  p.n_units = pl.n_units;
  p.part = static_cast<float*>(workspace);
  p.ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + part_bytes);
  p.timeout_ns = wait_timeout_ns();
  p.status = st;
  auto run = [&](auto kern) -> bool {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::Cfg<D>::SMEM_BYTES) !=
        cudaSuccess)
      return false;
    kern<<<pl.grid, dec::THREADS, dec::Cfg<D>::SMEM_BYTES, s>>>(p);
    return cudaGetLastError() == cudaSuccess;
  };
  const int nq = pr.N;
  const bool launched = nq <= 1   ? run(dec::partial_kernel<D, 1>)
                        : nq <= 2 ? run(dec::partial_kernel<D, 2>)
                        : nq <= 4 ? run(dec::partial_kernel<D, 4>)
                        : nq <= 8 ? run(dec::partial_kernel<D, 8>)
                                  : run(dec::partial_kernel<D, 16>);
  if (!launched) return FA_ERR_CUDA;
  dec::merge_kernel<D><<<pr.BH * pr.N, D, 0, s>>>(p, static_cast<__nv_bfloat16*>(O), LSE);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status launch_decode(const Problem& pr, const void* Q, const void* K, const void* V, void* O, float* LSE,
                        void* workspace, size_t workspace_bytes, cudaStream_t s) {
  if (pr.d == 64) return launch_decode_d<64>(pr, Q, K, V, O, LSE, workspace, workspace_bytes, s);
  return launch_decode_d<128>(pr, Q, K, V, O, LSE, workspace, workspace_bytes, s);
}

}  // namespace fa
