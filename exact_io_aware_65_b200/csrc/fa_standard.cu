// fa_standard.cu -- standard (materialising) attention: the baseline the
// pages set the method against ("FlashAttention: Fast and Memory-Efficient
// Exact Attention with IO-Awareness", sections "Attention hurts on long
// sequences" and "GPUs are often memory-bound"; "FlashAttention: making
// attention fast by respecting the memory hierarchy", cost paragraph).
//   S = scale Q K^T      written to HBM (fp32, [BH, N, N])
//   P = softmax(S)       read back, masked, normalised, written (bf16)
//   O = P V              read back once more
// The N x N grid makes two round trips through HBM and the memory grows as
// N^2.  The two products are plain batched GEMMs from cuBLAS, resolved at
// run time (so the library itself does not depend on it); the softmax is
// this file's kernel.  Forward only: it is there to measure against.
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <dlfcn.h>
#include <math.h>

#include <mutex>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace stdattn {

constexpr int THREADS = 256;
constexpr float LOG2E = 1.4426950408889634074f;
constexpr float LN2 = 0.69314718055994530942f;

// One row of S per CTA: the row is read once into shared memory, then the
// masked maximum, the sum of exponentials and the normalised bf16 P row.
__global__ void __launch_bounds__(THREADS) softmax_kernel(const float* __restrict__ S,
                                                          __nv_bfloat16* __restrict__ P, float* __restrict__ LSE,
                                                          int N, int mask_kind, const uint8_t* __restrict__ bm,
                                                          int nb, uint32_t* status) {
  extern __shared__ float row[];
  __shared__ float red[THREADS / 32];
  const size_t r = blockIdx.x;  // row index over B*H*N
  const int i = (int)(r % N);
  const float* s = S + r * N;
  // the grid is one CTA per row of S, so every index below is in range; the
  // debug build checks the row anyway
  if (!FA_IN_BOUNDS(status, r * N, N, (size_t)gridDim.x * N)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float mx = -INFINITY;
  for (int j = tid; j < N; j += THREADS) {
    bool keep = true;
    if (mask_kind == FA_MASK_CAUSAL) keep = j <= i;
    else if (mask_kind == FA_MASK_BLOCK)
      keep = FA_IN_BOUNDS(status, (size_t)(i / 128) * nb + j / 128, 1, (size_t)nb * nb) &&
             bm[(size_t)(i / 128) * nb + j / 128] != 0;
    const float v = keep ? s[j] * LOG2E : -INFINITY;  // log2 units
    row[j] = v;
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int k = 1; k < THREADS / 32; ++k) mx = fmaxf(mx, red[k]);
  __syncthreads();
  const float m = mx == -INFINITY ? 0.0f : mx;  // a row that sees nothing: all p = 0
  float sum = 0.0f;
  for (int j = tid; j < N; j += THREADS) {
    const float p = ex2_approx(row[j] - m);
    row[j] = p;
    sum += p;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = 0.0f;
  for (int k = 0; k < THREADS / 32; ++k) sum += red[k];
  const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
  __nv_bfloat16* prow = P + r * N;
  for (int j = tid; j < N; j += THREADS) prow[j] = __float2bfloat16(row[j] * inv);
  if (tid == 0) LSE[r] = sum > 0.0f ? (mx + log2f(sum)) * LN2 : -INFINITY;
}

// cuBLAS, opened on first use.  A soname already loaded in the process (for
// example by PyTorch) is reused.
struct Blas {
  bool tried = false, ok = false;
  decltype(&cublasCreate_v2) create = nullptr;
  decltype(&cublasSetStream_v2) set_stream = nullptr;
  // the exported C symbol (compute type as cublasComputeType_t)
  using gemm_t = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                    const void*, const void*, cudaDataType, int, long long, const void*,
                                    cudaDataType, int, long long, const void*, void*, cudaDataType, int, long long,
                                    int, cublasComputeType_t, cublasGemmAlgo_t);
  gemm_t gemm = nullptr;
  cublasHandle_t handle[64] = {};  // per device
  std::mutex mu;
};
static Blas g_blas;

static cublasHandle_t blas_handle() {
  std::lock_guard<std::mutex> lock(g_blas.mu);
  if (!g_blas.tried) {
    g_blas.tried = true;
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
    if (h) {
      g_blas.create = reinterpret_cast<decltype(g_blas.create)>(dlsym(h, "cublasCreate_v2"));
      g_blas.set_stream = reinterpret_cast<decltype(g_blas.set_stream)>(dlsym(h, "cublasSetStream_v2"));
      g_blas.gemm = reinterpret_cast<Blas::gemm_t>(dlsym(h, "cublasGemmStridedBatchedEx"));
      g_blas.ok = g_blas.create && g_blas.set_stream && g_blas.gemm;
    }
  }
  if (!g_blas.ok) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!g_blas.handle[dev] && g_blas.create(&g_blas.handle[dev]) != CUBLAS_STATUS_SUCCESS) return nullptr;
  return g_blas.handle[dev];
}

}  // namespace stdattn

size_t standard_workspace_bytes(int BH, int N) {
  const size_t nn = (size_t)BH * N * N;
  return ((nn * 4 + 255) & ~size_t(255)) + nn * 2;  // S fp32, then P bf16
}

fa_status launch_standard_fwd(const Problem& pr, const void* Q, const void* K, const void* V, void* O, float* LSE,
                              void* workspace, cudaStream_t s) {
  using namespace stdattn;
  cublasHandle_t h = blas_handle();
  if (!h) return FA_ERR_CUDA;
  uint32_t* st = status_word();
  if (!st) return FA_ERR_CUDA;
  const int N = pr.N, d = pr.d, BH = pr.BH;
  const size_t nn = (size_t)BH * N * N;
  float* S = static_cast<float*>(workspace);
  __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + ((nn * 4 + 255) & ~size_t(255)));
  if (g_blas.set_stream(h, s) != CUBLAS_STATUS_SUCCESS) return FA_ERR_CUDA;
  // Row-major X [r, c] is column-major X^T.  S (row-major N x N) is stored
  // as the column-major product K Q^T: A = K (stored d x N, transposed),
  // B = Q (stored d x N).
  const float alpha = pr.scale, beta = 0.0f, one = 1.0f;
  if (g_blas.gemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, N, d, &alpha, K, CUDA_R_16BF, d, (long long)N * d, Q, CUDA_R_16BF,
                  d, (long long)N * d, &beta, S, CUDA_R_32F, N, (long long)N * N, BH, CUBLAS_COMPUTE_32F,
                  CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  const int nb = (N + 127) / 128;
  if (cudaFuncSetAttribute(softmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, N * (int)sizeof(float)) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  softmax_kernel<<<(unsigned)((size_t)BH * N), THREADS, (size_t)N * sizeof(float), s>>>(
      S, P, LSE, N, pr.mask_kind, pr.block_mask, nb, st);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  // O (row-major N x d) is stored as the column-major product V^T P^T:
  // A = V (stored d x N), B = P (stored N x N).
  if (g_blas.gemm(h, CUBLAS_OP_N, CUBLAS_OP_N, d, N, N, &one, V, CUDA_R_16BF, d, (long long)N * d, P, CUDA_R_16BF,
                  N, (long long)N * N, &beta, O, CUDA_R_16BF, d, (long long)N * d, BH, CUBLAS_COMPUTE_32F,
                  CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  return FA_OK;
}

}  // namespace fa
