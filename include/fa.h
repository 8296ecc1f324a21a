/*
 * fa.h -- C ABI of libfa.so: exact, IO-aware scaled-dot-product attention
 * (forward and backward) for NVIDIA B200 (sm_100a).
 *
 * What is computed.  For every head (b, h) of [B, H, N, d] tensors:
 *     S = scale * Q K^T   (with a mask applied as -inf),
 *     P = softmax(S) row by row,   O = P V,   LSE_i = ln sum_j exp(S_ij).
 * The method is the one described on the pages "FlashAttention: making
 * attention fast by respecting the memory hierarchy" (tiling paragraph:
 * blocks of queries against blocks of keys and values, an online softmax,
 * the full score grid never written to slow memory) and "FlashAttention:
 * Fast and Memory-Efficient Exact Attention with IO-Awareness" (sections
 * "What FlashAttention targets": exact, same outputs as naive attention;
 * "Softmax / tiling"; "Backward / recomputation": the forward stores the
 * softmax normalisation statistics -- here the per-row log-sum-exp -- and the
 * backward recomputes the attention values on chip from them).
 *
 * Conventions shared by every call:
 *   - Q, K, V, O, dO, dQ, dK, dV: bf16, contiguous [B, H, N, d] (d fastest),
 *     DEVICE pointers, 16-byte aligned.  N_q = N_k = N (self-attention).
 *   - LSE: fp32 [B, H, N], natural log, DEVICE pointer, 4-byte aligned.
 *   - d must be 64 or 128.  N >= 1 is any length (a last partial tile of
 *     128 rows is handled by masking).
 *   - mask_kind: FA_MASK_NONE, FA_MASK_CAUSAL (key j visible to query i iff
 *     j <= i, top-left aligned) or FA_MASK_BLOCK.  For FA_MASK_BLOCK,
 *     `block_mask` is a DEVICE uint8 array [nb, nb], nb = ceil(N / 128),
 *     row-major, entry (I, J) != 0 keeping the 128 x 128 score tile of query
 *     rows [128 I, 128 I + 128) and key columns [128 J, 128 J + 128); one mask
 *     serves every batch and head (block-sparse FlashAttention, "Paper
 *     Abstract" of the summary page).  It is ignored for the other kinds.
 *     A query row with no visible key gets O = 0, LSE = -inf, and contributes
 *     nothing to the gradients.
 *   - scale: finite, > 0 (usually 1/sqrt(d)).
 *   - stream: a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call is asynchronous on it.
 *   - Ownership: the caller allocates and owns every buffer and the stream;
 *     the library keeps no allocation between calls.
 *   - Outputs must not alias inputs.
 *   - CUDA graphs: every call can be captured into a graph, after one
 *     eager call on the device has set up the per-device state.  Each
 *     forward launch takes one of 4096 per-device work-counter slots when it
 *     is issued, and a captured launch keeps its slot, so one graph must not
 *     be replayed on two streams at once.
 *   - Errors: argument problems are reported synchronously, before anything
 *     is launched.  A failed launch returns FA_ERR_CUDA.  Every wait inside
 *     the kernels is bounded in time; a wait that runs out records
 *     FA_ERR_TIMEOUT in a per-device status word that fa_device_status()
 *     reads (the outputs of that call are then undefined).
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad scale, bad mask kind */
  FA_ERR_UNSUPPORTED = 2, /* valid request outside this build: d not 64/128, B*H*N or B*H*Nk above 2^37 */
  FA_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
  FA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than fa_bwd_workspace_size() */
  FA_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (see fa_device_status) */
  FA_ERR_BOUNDS = 6       /* debug build only (libfa_debug.so): a kernel's index check
                             found an access outside its buffer and skipped it */
} fa_status;

typedef enum { FA_MASK_NONE = 0, FA_MASK_CAUSAL = 1, FA_MASK_BLOCK = 2 } fa_mask_kind;

/* Forward pass.
 * In:  Q, K, V [B,H,N,d] bf16; mask (kind + optional device block mask); scale.
 * Out: O [B,H,N,d] bf16 (round to nearest even); LSE [B,H,N] fp32, the
 *      natural-log normaliser of the scaled, masked scores of each row.
 * The N x N score grid never leaves the chip. */
fa_status fa_fwd(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                 int mask_kind, const uint8_t* block_mask, float scale, void* O, float* LSE,
                 void* stream);

/* Bytes of device workspace fa_bwd needs for this problem size: an fp32 dQ
 * accumulator [B,H,ceil(N/128)*128,d], the fp32 row terms D_i = dO_i . O_i
 * [B,H,ceil(N/128)*128], plus alignment padding.  Linear in N.  Returns 0 for
 * sizes fa_bwd would reject. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/* Backward pass, recomputing P on chip from Q, K and the forward's LSE.
 * In:  Q, K, V, O, dO [B,H,N,d] bf16; LSE [B,H,N] fp32 from fa_fwd with the
 *      same mask and scale; workspace (DEVICE, 256-byte aligned, at least
 *      fa_bwd_workspace_size() bytes, contents irrelevant on entry).
 * Out: dQ, dK, dV [B,H,N,d] bf16, gradients of sum(dO * O) with respect to
 *      Q, K and V.  dQ is summed over key tiles in fp32 in an unspecified
 *      order, so its last bits may differ from run to run
 *      (fa_bwd_qk_deterministic fixes the order). */
fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, int B, int H, int N, int d, int mask_kind,
                 const uint8_t* block_mask, float scale, void* dQ, void* dK, void* dV,
                 void* workspace, size_t workspace_bytes, void* stream);

/* The three launches fa_bwd makes, callable one at a time with fa_bwd's
 * arguments (each call checks them the same way).  stage 0: prep -- the row
 * terms D_i = dO_i . O_i and LSE scaled to log2 units (both stored negated)
 * and a zeroed fp32 dQ accumulator, all in the workspace; stage 1: main --
 * recompute P, produce dK and dV, add dQ partial sums into the accumulator;
 * stage 2: write dQ = bf16(scale * accumulator).  fa_bwd(...) is exactly
 * stages 0, 1, 2 in order on one stream; a stage reads what the previous
 * one left in the workspace, so they must run in that order on the same
 * workspace. */
fa_status fa_bwd_stage(int stage, const void* Q, const void* K, const void* V, const void* O,
                       const void* dO, const float* LSE, int B, int H, int N, int d, int mask_kind,
                       const uint8_t* block_mask, float scale, void* dQ, void* dK, void* dV,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Queries and keys of different counts (cross-attention, or a block of new
 * queries against a longer key/value history).  Same as fa_fwd, fa_bwd and
 * fa_bwd_workspace_size, which are these with Nq = Nk = N, except:
 *   - Q, O, dO, dQ are [B,H,Nq,d] and LSE [B,H,Nq]; K, V, dK, dV are
 *     [B,H,Nk,d].  Nq, Nk >= 1, any values (not multiples of 128).
 *   - FA_MASK_CAUSAL is aligned at the bottom right: query i sees key j iff
 *     j <= i + (Nk - Nq), so the last query sees every key (for Nq = Nk this
 *     is j <= i).  The pages do not treat Nq != Nk; this alignment keeps a
 *     suffix of the queries' outputs equal to those of the full square
 *     problem.  With Nq > Nk the first Nq - Nk queries see nothing: O = 0,
 *     LSE = -inf and no gradient, as for any row that sees no key.
 *   - FA_MASK_BLOCK takes a [ceil(Nq/128), ceil(Nk/128)] uint8 DEVICE grid
 *     (query tiles by key tiles, 1 = keep).
 *   - The workspace depends on Nq only.
 * Errors as for fa_fwd / fa_bwd (Nk <= 0 is FA_ERR_INVALID_ARG). */
fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk, int d,
                    int mask_kind, const uint8_t* block_mask, float scale, void* O, float* LSE,
                    void* stream);
size_t fa_bwd_workspace_size_qk(int B, int H, int Nq, int Nk, int d);

/* Variable-length batches in padded storage: batch element b holds
 * seqlens_q[b] query rows and seqlens_k[b] keys at the start of its
 * [Nq, d] / [Nk, d] slices; the rest of each slice is padding.  Each
 * sequence is its own attention problem (causal aligned at the bottom right
 * of that sequence: row i sees keys j <= i + seqlens_k[b] - seqlens_q[b]);
 * padding is never read as a key or a query, tiles wholly in padding do no
 * work, and padding rows of the outputs come out as O = 0, LSE = -inf and
 * zero gradients.  seqlens_q, seqlens_k: DEVICE int [B] (either may be NULL:
 * every sequence then has Nq, or Nk); values are clamped to [0, Nq] and
 * [0, Nk].  Otherwise as fa_fwd_qk / fa_bwd_qk (fa_bwd_qk_deterministic when
 * deterministic != 0), with the same workspace.  No page counterpart beyond
 * the batching of independent problems. */
fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk,
                        int d, int mask_kind, const uint8_t* block_mask, float scale,
                        const int* seqlens_q, const int* seqlens_k, void* O, float* LSE,
                        void* stream);
fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                        const float* LSE, int B, int H, int Nq, int Nk, int d, int mask_kind,
                        const uint8_t* block_mask, float scale, const int* seqlens_q,
                        const int* seqlens_k, int deterministic, void* dQ, void* dK, void* dV,
                        void* workspace, size_t workspace_bytes, void* stream);

/* fa_bwd_qk with run-to-run reproducible gradients: every element of dQ is
 * summed over key tiles in ascending key-tile order (each key tile waits
 * for its turn per query tile, through counters in the workspace), so the
 * result is the same bits on every run with the same inputs on the same
 * GPU.  dK and dV are always reproducible.  Same arguments, workspace size
 * and errors as fa_bwd_qk; slower, since the dQ additions of a query tile
 * are serialised.  It waits on other CTAs of the same launch: run it where
 * the launch can occupy the GPU (a launch whose CTAs cannot all become
 * resident within the wait limit ends with FA_ERR_TIMEOUT from
 * fa_device_status()).  No page counterpart: the pages do not address
 * reproducibility. */
fa_status fa_bwd_qk_deterministic(const void* Q, const void* K, const void* V, const void* O,
                                  const void* dO, const float* LSE, int B, int H, int Nq, int Nk,
                                  int d, int mask_kind, const uint8_t* block_mask, float scale,
                                  void* dQ, void* dK, void* dV, void* workspace,
                                  size_t workspace_bytes, void* stream);
fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, int B, int H, int Nq, int Nk, int d, int mask_kind,
                    const uint8_t* block_mask, float scale, void* dQ, void* dK, void* dV,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Decode: a few new queries per head against a long key/value history (a
 * KV cache), forward only.  The same exact attention as fa_fwd_qk, computed
 * by splitting the keys across the GPU and merging the partial softmax
 * results by their running maxima and sums (log-sum-exp); meant for the
 * shapes where fa_fwd_qk would leave most of the GPU idle.  With Nq >= 4
 * and at least as many heads (B H) as the GPU has SMs, the call runs the
 * tensor-core forward of fa_fwd_qk instead (one work item per head), which
 * then fills the GPU and reads the cache once per head at a higher rate;
 * the workspace is still required and goes unused.
 * In:  Q [B,H,Nq,d] bf16 with 1 <= Nq <= 16; K, V [B,H,Nk,d] bf16, Nk >= 1;
 *      mask_kind FA_MASK_NONE or FA_MASK_CAUSAL (bottom-right aligned as in
 *      fa_fwd_qk: query i sees keys j <= i + (Nk - Nq)); scale > 0;
 *      workspace (DEVICE, 256-byte aligned, at least
 *      fa_decode_workspace_size() bytes, contents irrelevant on entry).
 * Out: O [B,H,Nq,d] bf16, LSE [B,H,Nq] fp32, as fa_fwd_qk.  All DEVICE
 *      pointers, 16-byte aligned (LSE 4).
 * Errors: FA_ERR_INVALID_ARG (as fa_fwd_qk), FA_ERR_UNSUPPORTED (Nq > 16,
 * d not 64 or 128, a block mask), FA_ERR_WORKSPACE, FA_ERR_CUDA.  The pages
 * have no decode-specific algorithm; this is their tiling applied across
 * the keys, with the running statistics combined at the end. */
size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d);
fa_status fa_decode(const void* Q, const void* K, const void* V, int B, int H, int Nq, int Nk, int d,
                    int mask_kind, float scale, void* O, float* LSE, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Standard (materialising) attention, forward only: the baseline the pages
 * measure the method against, for speed and memory comparisons.  It writes
 * S = scale Q K^T to HBM in fp32, reads it back for a masked row softmax
 * that writes P in bf16, and reads P back for O = P V; the N x N grid makes
 * two round trips through HBM and the workspace grows as N^2.  The two
 * products are cuBLAS batched GEMMs (libcublas.so.12, opened at the first
 * call); the softmax is the library's own kernel.
 * In/out as fa_fwd (self-attention, N <= 16384, same masks and LSE
 * convention); workspace (DEVICE, 256-byte aligned) of at least
 * fa_standard_fwd_workspace_size() bytes: 6 * B * H * N^2 plus alignment.
 * Errors as fa_fwd, plus FA_ERR_UNSUPPORTED (N > 16384), FA_ERR_WORKSPACE,
 * and FA_ERR_CUDA when cuBLAS cannot be opened or fails. */
size_t fa_standard_fwd_workspace_size(int B, int H, int N, int d);
fa_status fa_standard_fwd(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                          int mask_kind, const uint8_t* block_mask, float scale, void* O, float* LSE,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Largest scratch, in bytes, that fa_bwd_static_workspace() can use: 64 MiB. */
#define FA_BWD_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)

/* fa_bwd without a caller-supplied workspace, for callers that cannot
 * allocate device memory: for example a runtime whose device memory is all
 * handed out up front by its own pool, so one more cudaMalloc would fail or
 * fragment it, or a latency-critical loop where cudaMalloc/cudaFree would
 * stall on an implicit device synchronisation.  This call allocates nothing.
 * Its scratch is a fixed 64 MiB array (FA_BWD_STATIC_WORKSPACE_BYTES) in the
 * library's own device memory; every GPU that loads the library holds it
 * until the process exits.  The paper has no counterpart to this call.
 *   - Arguments, outputs and results are those of fa_bwd, minus the
 *     workspace.  A problem whose fa_bwd_workspace_size() exceeds the array
 *     is refused with FA_ERR_WORKSPACE before anything runs (that allows
 *     B*H*ceil(N/128)*128 up to about 129,000 for d = 128 and about 254,000
 *     for d = 64).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current).  With the CUDA
 *     runtime's lazy module loading (the default since CUDA 12.2) that first
 *     call is also where the runtime reserves the 64 MiB on the device.  A
 *     caller whose pool takes the device's memory should therefore make its
 *     first call before the pool reserves that memory, and before any stream
 *     capture begins.  Later calls allocate nothing.
 *   - The looked-up address belongs to the device's context: after
 *     cudaDeviceReset() on a device, this library must not be called on that
 *     device again in the same process (this also holds for every other call
 *     here, whose device status word is looked up the same way).
 *   - All calls on a device share the one array, and it keeps whatever the
 *     last call left in it (each call clears what must start at zero).  Calls
 *     whose kernels overlap on the GPU -- on different streams, or from
 *     different host threads -- race on it and give wrong results: order
 *     them on one stream or synchronise between them. */
fa_status fa_bwd_static_workspace(const void* Q, const void* K, const void* V, const void* O,
                                  const void* dO, const float* LSE, int B, int H, int N, int d,
                                  int mask_kind, const uint8_t* block_mask, float scale, void* dQ,
                                  void* dK, void* dV, void* stream);

/* Synchronise `stream`, then read and clear the calling device's status
 * word.  Returns FA_OK, FA_ERR_TIMEOUT if a bounded wait ran out in a kernel
 * since the last call, FA_ERR_BOUNDS if (debug build only) an index check
 * failed, or FA_ERR_CUDA if the synchronisation itself failed. */
fa_status fa_device_status(void* stream);

/* Set the wall-clock limit, in nanoseconds, of every device-side wait in
 * later launches from this process (default 4e9 = 4 s).  0 restores the
 * default. */
void fa_set_wait_timeout_ns(uint64_t ns);

/* Human-readable name of a status code (static string). */
const char* fa_status_string(fa_status s);

/* Self-test of the bounded-wait machinery: launches one CTA whose thread
 * waits, for at most `timeout_ns`, on an mbarrier that nothing ever
 * completes, then returns.  After fa_device_status() the caller should see
 * FA_ERR_TIMEOUT.  No page counterpart: this exercises the library's own
 * failure detection. */
fa_status fa_selftest_bounded_wait(uint64_t timeout_ns, void* stream);

/* Self-test of the tensor-core path on one tile, used to validate the
 * shared-memory/TMEM descriptors in isolation.  A [128 x k] and Bt
 * [n x k] are bf16 row-major DEVICE arrays (k in {64, 128}; n in {64, 128});
 * C [128 x n] fp32 DEVICE receives A * Bt^T computed by TMA loads plus one
 * tcgen05.mma chain from shared memory (mode 0), or, in mode 1, by first
 * packing A into tensor memory and multiplying by Bt read as an MN-major
 * [k x n] operand -- the two forms that S = Q K^T and O += P V take. In
 * mode 1, B is passed as [k x n] row-major instead.  No page counterpart. */
fa_status fa_selftest_mma_tile(const void* A, const void* B, float* C, int n, int k, int mode,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
