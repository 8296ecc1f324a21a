// fa_api.cu -- the extern "C" entry points of libfa.so: argument checks,
// TMA map encoding, the device status word, and dispatch to the kernels.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

__device__ uint32_t g_status = 0;

uint32_t* status_word() {
  static uint32_t* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

static std::atomic<uint64_t> g_wait_timeout_ns{4000000000ull};
uint64_t wait_timeout_ns() { return g_wait_timeout_ns.load(); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// cuTensorMapEncodeTiled is fetched through the runtime so the library does
// not link against libcuda directly.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_bf16(CUtensorMap* map, const void* base, int BH, int N, int d, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)N};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_bf16_box(CUtensorMap* map, const void* base, int BH, int N, int d, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn || (box_cols != 32 && box_cols != 64)) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)N};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  // the box's rows are 64 or 128 bytes: the swizzle of that width
  const CUtensorMapSwizzle sw = box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_bf16_2d(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  return make_map_bf16(map, base, 1, rows, cols, box_rows);
}

}  // namespace fa

using namespace fa;

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The kernels count work items (heads x 128-row tiles) and tile rows in
// 32-bit ints: B*H*N up to 2^37 keeps both below 2^31 (and is far beyond
// what fits in device memory at d = 64).
static bool sizes_supported(long long bh, int N) {
  return bh <= (1ll << 30) && N <= (1 << 30) && bh * (long long)N <= (1ll << 37);
}

static fa_status check_common(const void* Q, const void* K, const void* V, int B, int H, int N, int Nk, int d,
                              int mask_kind, const uint8_t* block_mask, float scale, Problem* p) {
  if (!Q || !K || !V) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || Nk <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (mask_kind != FA_MASK_NONE && mask_kind != FA_MASK_CAUSAL && mask_kind != FA_MASK_BLOCK)
    return FA_ERR_INVALID_ARG;
  if (mask_kind == FA_MASK_BLOCK && !block_mask) return FA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long bh = (long long)B * H;
  if (!sizes_supported(bh, N) || !sizes_supported(bh, Nk)) return FA_ERR_UNSUPPORTED;
  p->B = B; p->H = H; p->N = N; p->Nk = Nk; p->d = d;
  p->BH = (int)bh;
  p->nq = (N + 127) / 128;
  p->nk = (Nk + 127) / 128;
  p->off = Nk - N;
  p->mask_kind = mask_kind;
  p->block_mask = mask_kind == FA_MASK_BLOCK ? block_mask : nullptr;
  p->scale = scale;
  p->scale_log2 = (float)((double)scale * 1.4426950408889634074);
  return FA_OK;
}

extern "C" {

fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk, int d,
                    int mask_kind, const uint8_t* block_mask, float scale, void* O, float* LSE, void* stream) {
  Problem p;
  fa_status st = check_common(Q, K, V, B, H, Nq, Nk, d, mask_kind, block_mask, scale, &p);
  if (st != FA_OK) return st;
  if (!O || !LSE || !aligned(O, 16) || !aligned(LSE, 4)) return FA_ERR_INVALID_ARG;
  return launch_fwd(p, Q, K, V, O, LSE, (cudaStream_t)stream);
}

fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk, int d,
                        int mask_kind, const uint8_t* block_mask, float scale, const int* seqlens_q,
                        const int* seqlens_k, void* O, float* LSE, void* stream) {
  if (!aligned(seqlens_q, 4) || !aligned(seqlens_k, 4)) return FA_ERR_INVALID_ARG;
  Problem p;
  fa_status st = check_common(Q, K, V, B, H, Nq, Nk, d, mask_kind, block_mask, scale, &p);
  if (st != FA_OK) return st;
  if (!O || !LSE || !aligned(O, 16) || !aligned(LSE, 4)) return FA_ERR_INVALID_ARG;
  p.seqlens_q = seqlens_q;
  p.seqlens_k = seqlens_k;
  return launch_fwd(p, Q, K, V, O, LSE, (cudaStream_t)stream);
}

fa_status fa_fwd(const void* Q, const void* K, const void* V, int B, int H, int N, int d, int mask_kind,
                 const uint8_t* block_mask, float scale, void* O, float* LSE, void* stream) {
  return fa_fwd_qk(Q, K, V, B, H, N, N, d, mask_kind, block_mask, scale, O, LSE, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
  if (!sizes_supported((long long)B * H, N)) return 0;
  return bwd_workspace_bytes(B, H, N, d);
}

size_t fa_bwd_workspace_size_qk(int B, int H, int Nq, int Nk, int d) {
  if (Nk <= 0 || !sizes_supported((long long)B * H, Nk)) return 0;
  return fa_bwd_workspace_size(B, H, Nq, d);  // the workspace is per query row
}

static fa_status bwd_common(int stage, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                            const float* LSE, int B, int H, int N, int Nk, int d, int mask_kind,
                            const uint8_t* block_mask, float scale, void* dQ, void* dK, void* dV, void* workspace,
                            size_t workspace_bytes, void* stream, int deterministic = 0,
                            const int* seqlens_q = nullptr, const int* seqlens_k = nullptr) {
  Problem p;
  fa_status st = check_common(Q, K, V, B, H, N, Nk, d, mask_kind, block_mask, scale, &p);
  p.deterministic = deterministic;
  p.seqlens_q = seqlens_q;
  p.seqlens_k = seqlens_k;
  if (st != FA_OK) return st;
  if (!O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (!aligned(O, 16) || !aligned(dO, 16) || !aligned(LSE, 4) || !aligned(dQ, 16) || !aligned(dK, 16) ||
      !aligned(dV, 16))
    return FA_ERR_INVALID_ARG;
  const size_t need = bwd_workspace_bytes(B, H, N, d);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
  return launch_bwd(p, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, (cudaStream_t)stream, stage);
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                 int B, int H, int N, int d, int mask_kind, const uint8_t* block_mask, float scale, void* dQ,
                 void* dK, void* dV, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(-1, Q, K, V, O, dO, LSE, B, H, N, N, d, mask_kind, block_mask, scale, dQ, dK, dV, workspace,
                    workspace_bytes, stream);
}

fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                    int B, int H, int Nq, int Nk, int d, int mask_kind, const uint8_t* block_mask, float scale,
                    void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(-1, Q, K, V, O, dO, LSE, B, H, Nq, Nk, d, mask_kind, block_mask, scale, dQ, dK, dV, workspace,
                    workspace_bytes, stream);
}

fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                        const float* LSE, int B, int H, int Nq, int Nk, int d, int mask_kind,
                        const uint8_t* block_mask, float scale, const int* seqlens_q, const int* seqlens_k,
                        int deterministic, void* dQ, void* dK, void* dV, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!aligned(seqlens_q, 4) || !aligned(seqlens_k, 4)) return FA_ERR_INVALID_ARG;
  return bwd_common(-1, Q, K, V, O, dO, LSE, B, H, Nq, Nk, d, mask_kind, block_mask, scale, dQ, dK, dV, workspace,
                    workspace_bytes, stream, deterministic ? 1 : 0, seqlens_q, seqlens_k);
}

fa_status fa_bwd_qk_deterministic(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                  const float* LSE, int B, int H, int Nq, int Nk, int d, int mask_kind,
                                  const uint8_t* block_mask, float scale, void* dQ, void* dK, void* dV,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(-1, Q, K, V, O, dO, LSE, B, H, Nq, Nk, d, mask_kind, block_mask, scale, dQ, dK, dV, workspace,
                    workspace_bytes, stream, 1);
}

fa_status fa_bwd_stage(int stage, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                       const float* LSE, int B, int H, int N, int d, int mask_kind, const uint8_t* block_mask,
                       float scale, void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (stage < 0 || stage > 2) return FA_ERR_INVALID_ARG;
  return bwd_common(stage, Q, K, V, O, dO, LSE, B, H, N, N, d, mask_kind, block_mask, scale, dQ, dK, dV, workspace,
                    workspace_bytes, stream);
}

// fa_decode hands problems with at least this many queries per head (and at
// least one head per SM) to the tensor-core forward.
constexpr int DECODE_TC_MIN_NQ = 4;

size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nq > 16 || Nk <= 0 || (d != 64 && d != 128)) return 0;
  const long long bh = (long long)B * H;
  if (!sizes_supported(bh, Nk)) return 0;
  return decode_workspace_bytes((int)bh, Nq, Nk, d);
}

fa_status fa_decode(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk, int d, int mask_kind,
                    float scale, void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream) {
  if (mask_kind == FA_MASK_BLOCK) return FA_ERR_UNSUPPORTED;
  Problem p;
  fa_status st = check_common(Q, K, V, B, H, Nq, Nk, d, mask_kind, nullptr, scale, &p);
  if (st != FA_OK) return st;
  if (Nq > 16) return FA_ERR_UNSUPPORTED;
  if (!O || !LSE || !aligned(O, 16) || !aligned(LSE, 4)) return FA_ERR_INVALID_ARG;
  const size_t need = decode_workspace_bytes(p.BH, Nq, Nk, d);
  if (need == 0) return FA_ERR_CUDA;
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
  // With several queries per head and a head for every SM, the tensor-core
  // forward (one work item per head, the cache read once per head) fills the
  // GPU and outruns the split-key kernel, whose per-query work runs on the
  // CUDA cores.
  if (Nq >= DECODE_TC_MIN_NQ && p.BH >= num_sms()) return launch_fwd(p, Q, K, V, O, LSE, (cudaStream_t)stream);
  return launch_decode(p, Q, K, V, O, LSE, workspace, workspace_bytes, (cudaStream_t)stream);
}

size_t fa_standard_fwd_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || N > 16384 || (d != 64 && d != 128)) return 0;
  const long long bh = (long long)B * H;
  if (!sizes_supported(bh, N) || bh > (1 << 30) / 16) return 0;
  return standard_workspace_bytes((int)bh, N);
}

fa_status fa_standard_fwd(const void* Q, const void* K, const void* V, int B, int H, int N, int d, int mask_kind,
                          const uint8_t* block_mask, float scale, void* O, float* LSE, void* workspace,
                          size_t workspace_bytes, void* stream) {
  Problem p;
  fa_status st = check_common(Q, K, V, B, H, N, N, d, mask_kind, block_mask, scale, &p);
  if (st != FA_OK) return st;
  if (N > 16384) return FA_ERR_UNSUPPORTED;
  if (!O || !LSE || !aligned(O, 16) || !aligned(LSE, 4)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_standard_fwd_workspace_size(B, H, N, d);
  if (need == 0) return FA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
  return launch_standard_fwd(p, Q, K, V, O, LSE, workspace, (cudaStream_t)stream);
}

fa_status fa_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (v == 0) return FA_OK;
  if (v == FA_DEV_ERR_TIMEOUT) return FA_ERR_TIMEOUT;
  return v == FA_DEV_ERR_BOUNDS ? FA_ERR_BOUNDS : FA_ERR_CUDA;
}

void fa_set_wait_timeout_ns(uint64_t ns) { g_wait_timeout_ns.store(ns ? ns : 4000000000ull); }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported problem";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case FA_ERR_BOUNDS: return "a device-side index check failed (debug build)";
  }
  return "unknown status";
}

fa_status fa_selftest_bounded_wait(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return FA_ERR_INVALID_ARG;
  return launch_selftest_wait(timeout_ns, (cudaStream_t)stream);
}

fa_status fa_selftest_mma_tile(const void* A, const void* B, float* C, int n, int k, int mode, void* stream) {
  if (!A || !B || !C) return FA_ERR_INVALID_ARG;
  if ((n != 64 && n != 128) || (k != 64 && k != 128) || (mode != 0 && mode != 1)) return FA_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16)) return FA_ERR_INVALID_ARG;
  return launch_selftest_mma(A, B, C, n, k, mode, (cudaStream_t)stream);
}

}  // extern "C"
