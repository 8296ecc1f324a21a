// fa_selftest.cu -- two small self-tests of the sm_100a machinery the
// attention kernels are built from:
//   * a bounded wait on an mbarrier that nothing completes (must time out,
//     record the status and return);
//   * one 128 x n x k tensor-core tile in the two operand forms attention
//     uses: S = A B^T with both operands K-major in shared memory, and
//     C = A B with A packed into tensor memory and B MN-major in shared memory.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

__global__ void selftest_wait_kernel(uint64_t timeout_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{timeout_ns, &abort_flag, status};
    // Phase 0 never completes: nobody arrives.  The wait must give up.
    (void)mbar_wait(&bar, 0, w);
  }
  __syncthreads();
}

fa_status launch_selftest_wait(uint64_t timeout_ns, cudaStream_t s) {
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, s>>>(timeout_ns, st);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// One CTA of 128 threads.  Shared memory: A tile (128 x k bf16, SW128, k/64
// chunks of 16 KB), B tile (n x k or k x n bf16, SW128).
__global__ void __launch_bounds__(128, 1)
    selftest_mma_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                        const __nv_bfloat16* __restrict__ A, float* __restrict__ C, int n, int k, int mode,
                        uint64_t timeout_ns, uint32_t* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                  // 32 KB max
  uint8_t* sB = smem + 32768;          // 32 KB max
  __shared__ __align__(8) uint64_t bar_load, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar_load, 1);
    mbar_init(&bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  WaitCtx w{timeout_ns, &abort_flag, status};

  // C occupies columns [0, n); A (mode 1) occupies columns [128, 128 + k/2).
  const uint32_t t_c = tbase;
  const uint32_t t_a = tbase + 128;

  if (mode == 1) {
    // Each thread packs its row of A into tensor memory: two bf16 per column.
    const int row = threadIdx.x;
    const uint32_t* arow = reinterpret_cast<const uint32_t*>(A + (size_t)row * k);
    for (int c0 = 0; c0 < k / 2; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = arow[c0 + i];
      const uint32_t addr = t_a + (uint32_t(warp * 32) << 16) + c0;
      FA_TMEM_ST_X16(addr, r);
    }
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  bool ok = true;
  if (threadIdx.x == 0) {
    const uint32_t bytesA = (mode == 0) ? 128u * k * 2 : 0u;
    const uint32_t bytesB = (uint32_t)n * k * 2;
    mbar_arrive_expect_tx(&bar_load, bytesA + bytesB);
    if (mode == 0) {
      for (int c = 0; c < k / 64; ++c) tma_load_3d(sA + c * 16384, &mapA, &bar_load, c * 64, 0, 0);
      for (int c = 0; c < k / 64; ++c) tma_load_3d(sB + c * (n * 128), &mapB, &bar_load, c * 64, 0, 0);
    } else {
      // B is [k x n] row-major: n/64 column chunks of k rows x 128 bytes.
      for (int c = 0; c < n / 64; ++c) tma_load_3d(sB + c * (k * 128), &mapB, &bar_load, c * 64, 0, 0);
    }
    ok = mbar_wait(&bar_load, 0, w);
    if (ok) {
      tc_fence_after();
      if (mode == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, n, 0, 0);
        for (int s = 0; s < k / 16; ++s) {
          const uint32_t off = (s & 3) * 32;
          const uint64_t da = smem_desc_sw128(smem_u32(sA) + (s >> 2) * 16384 + off, 16, 1024);
          const uint64_t db = smem_desc_sw128(smem_u32(sB) + (s >> 2) * (n * 128) + off, 16, 1024);
          mma_ss(t_c, da, db, idesc, s > 0 ? 1u : 0u);
        }
      } else {
        const uint32_t idesc = idesc_bf16_f32(128, n, 0, 1);
        for (int s = 0; s < k / 16; ++s) {
          const uint64_t db = smem_desc_sw128(smem_u32(sB) + s * 2048, (uint32_t)k * 128, 1024);
          mma_ts(t_c, t_a + s * 8, db, idesc, s > 0 ? 1u : 0u);
        }
      }
      tc_commit(&bar_mma);
    }
  }
  __syncwarp();
  // All threads wait for the MMA chain, then read their row of C.
  if (mbar_wait_warp(&bar_mma, 0, w)) {
    tc_fence_after();
    const int row = threadIdx.x;
    for (int c0 = 0; c0 < n; c0 += 32) {
      uint32_t r[32];
      const uint32_t addr = t_c + (uint32_t(warp * 32) << 16) + c0;
      FA_TMEM_LD_X32(addr, r);
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) C[(size_t)row * n + c0 + i] = __uint_as_float(r[i]);
    }
  }
  (void)ok;
  (void)lane;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

fa_status launch_selftest_mma(const void* A, const void* B, float* C, int n, int k, int mode, cudaStream_t s) {
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  CUtensorMap mA, mB;
  if (!make_map_bf16_2d(&mA, A, 128, k, 128)) return FA_ERR_CUDA;
  if (mode == 0) {
    if (!make_map_bf16_2d(&mB, B, n, k, n)) return FA_ERR_CUDA;
  } else {
    if (!make_map_bf16_2d(&mB, B, k, n, k)) return FA_ERR_CUDA;
  }
  const int smem = 65536 + 1024;
  if (cudaFuncSetAttribute(selftest_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_CUDA;
  selftest_mma_kernel<<<1, 128, smem, s>>>(mA, mB, static_cast<const __nv_bfloat16*>(A), C, n, k, mode,
                                           wait_timeout_ns(), st);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
