// fa_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"

namespace fa {

// Problem description after validation.
struct Problem {
  int B, H, N, d;  // N: query rows
  int Nk;          // key rows (N for self-attention)
  int BH;          // B * H
  int nq, nk;      // ceil(N / 128) query tiles, ceil(Nk / 128) key tiles
  int off;         // Nk - N: causal alignment (query i sees keys j <= i + off)
  int mask_kind;
  const uint8_t* block_mask;  // device [nq, nk] or nullptr
  int deterministic = 0;      // backward: fixed order of the dQ additions
  // Optional per-batch-element lengths (device int [B]; nullptr: N, Nk).
  const int* seqlens_q = nullptr;
  const int* seqlens_k = nullptr;
  float scale;
  float scale_log2;  // scale * log2(e), computed in double and rounded once
};

// Encode a 3-D tiled TMA map over a contiguous bf16 [BH, N, d] tensor:
// dims (d, N, BH), box (64, box_rows, 1), 128-byte swizzle, zero fill out of
// bounds.  Returns false on failure.
bool make_map_bf16(CUtensorMap* map, const void* base, int BH, int N, int d, int box_rows);
// The same [BH, N, d] view with a box of box_cols (32 or 64) x box_rows and the
// swizzle of the box's row width (64 or 128 bytes): for tiled stores.
bool make_map_bf16_box(CUtensorMap* map, const void* base, int BH, int N, int d, int box_cols, int box_rows);

// Same for a 2-D row-major bf16 matrix [rows, cols] (used by the self-test).
bool make_map_bf16_2d(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);

uint64_t wait_timeout_ns();
// Device address of the calling device's status word (nullptr on failure).
uint32_t* status_word();
int num_sms();

// Kernel launchers (defined next to their kernels).
fa_status launch_fwd(const Problem& p, const void* Q, const void* K, const void* V, void* O, float* LSE,
                     cudaStream_t s);
// stage < 0: all three stages; otherwise only the given one (0, 1 or 2).
fa_status launch_bwd(const Problem& p, const void* Q, const void* K, const void* V, const void* O,
                     const void* dO, const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                     cudaStream_t s, int stage);
size_t bwd_workspace_bytes(int B, int H, int N, int d);
// Decode (few queries, long key history): workspace for the split-key
// partial results on the current device (0 on failure), and the launch.
size_t decode_workspace_bytes(int BH, int Nq, int Nk, int d);
fa_status launch_decode(const Problem& p, const void* Q, const void* K, const void* V, void* O, float* LSE,
                        void* workspace, size_t workspace_bytes, cudaStream_t s);
// Standard (materialising) attention, the baseline: workspace for S (fp32)
// and P (bf16), and the launch.
size_t standard_workspace_bytes(int BH, int N);
fa_status launch_standard_fwd(const Problem& p, const void* Q, const void* K, const void* V, void* O, float* LSE,
                              void* workspace, cudaStream_t s);
fa_status launch_selftest_wait(uint64_t timeout_ns, cudaStream_t s);
fa_status launch_selftest_mma(const void* A, const void* B, float* C, int n, int k, int mode, cudaStream_t s);

}  // namespace fa
