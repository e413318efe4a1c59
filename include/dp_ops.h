/*
 * dp_ops.h -- single-kernel entry points of the dp library.
 *
 * Each call runs exactly one of the kernels that dp_queue_step launches, with
 * the same tile configuration, on caller-owned device memory.  They exist so
 * that each kernel can be checked element by element against an independent
 * reference at full workload sizes, and timed alone.
 *
 * All pointers are device pointers of the current device; all matrices are
 * row-major with the given leading dimension (in elements).  Calls enqueue on
 * `stream` (a cudaStream_t, NULL = legacy default) and return without waiting.
 * They allocate nothing.  Errors: DP_ERR_INVALID_ARG for a NULL pointer, a
 * non-positive or unsupported size, a misaligned pointer or leading dimension
 * (the bf16 tensor-core paths need 16-byte aligned rows); DP_ERR_CUDA if the
 * launch fails.  The message is in dp_last_error().  The extent behind a raw
 * pointer cannot be checked: the caller guarantees that every buffer holds the
 * rows and leading dimension its sizes imply.
 *
 * Method source: the DualParal write-up "双重并行：让AI视频生成突破时长限制…"
 * (techwalker.com) §三: self-attention of a chunk reads its neighbour's cached
 * K/V next to its own, without concatenating them; cross-attention and the
 * FFN are per chunk.  The block layout (adaLN LayerNorm, gated residuals,
 * GELU FFN) is the DiT family's, which the write-up names (Wan2.1) without
 * giving formulas.
 */
#ifndef DP_OPS_H
#define DP_OPS_H

#include "dp.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DP_DT_F32 = 0, DP_DT_BF16 = 1 } dp_dtype;

typedef enum {
  DP_EPI_STORE = 0,        /* out[r][c] = acc + bias[c]                         */
  DP_EPI_GELU = 1,         /* out[r][c] = gelu_erf(acc + bias[c])               */
  DP_EPI_RESID = 2,        /* resid[r][c] += acc + bias[c]                      */
  DP_EPI_RESID_GATED = 3   /* resid[r][c] += gate(r, c) * (acc + bias[c])       */
} dp_epilogue;

/* out/resid = epilogue(A[M][K] . W[N][K]^T + bias).
 * dtype: of A, W and (STORE/GELU) out.  bf16 runs on the tcgen05 tensor cores
 * with fp32 accumulation (needs K % 64 == 0, N % 32 == 0, lda and ldo
 * multiples of 8, 16-byte aligned pointers, and for a cache copy ldc % 8 == 0
 * and cache_col0 % 32 == 0); f32 runs FFMA.
 * gate(r, c) = gate[sel(r / rows_per_chunk) * gate_stride + c] with
 * sel(i) = chunk_sel[i] (device int array) or i when chunk_sel is NULL.
 * The optional cache copy also writes, for rows r in
 * [cache_row0, cache_row0 + cache_rows) and columns c >= cache_col0, the
 * stored value to cache[(r - cache_row0) * ldc + (c - cache_col0)] (STORE
 * only, same dtype as out). */
typedef struct {
  dp_dtype dtype;
  const void* A; long long lda;
  const void* W;
  const float* bias;              /* [N] or NULL */
  int M, N, K;
  dp_epilogue epi;
  void* out; long long ldo;
  float* resid; long long ldr;
  const float* gate; long long gate_stride; const int* chunk_sel; int rows_per_chunk;
  void* cache; long long cache_row0; int cache_rows; int cache_col0; long long ldc;
} dp_gemm_args;
DP_API dp_status dp_op_gemm(const dp_gemm_args* a, void* stream);

/* Chunked multi-head attention, softmax(q k^T / sqrt(head_dim)) v per head,
 * one joint softmax over the key buffers a chunk sees:
 *   - its own keys: rows [c * kv_chunk_rows, c * kv_chunk_rows + Lk) of k/v
 *     (kv_chunk_rows = 0: every chunk shares the same Lk keys, as in
 *     cross-attention to the prompt);
 *   - if pred_in_batch and c > 0: the own keys of chunk c - 1 (the
 *     neighbour's K/V already computed in this batch), read in place;
 *   - for c = 0: the Lk_pred keys k0_pred/v0_pred when not NULL (the
 *     neighbour's persisted K/V from the previous step);
 *   - if succ_in_batch and c < n_chunks - 1: the own keys of chunk c + 1.
 * Queries of chunk c are rows [c * Lq, (c + 1) * Lq) of q.  Head h uses
 * columns [h * head_dim, (h + 1) * head_dim) of q, k, v and out.
 * With per-chunk keys (kv_chunk_rows > 0), Lk <= kv_chunk_rows.
 * bf16 requires head_dim 64 or 128 (tcgen05 path), leading dimensions that
 * are multiples of 8 and 16-byte aligned pointers; f32 requires head_dim in
 * {16, 32, 64, 128}. */
typedef struct {
  dp_dtype dtype;
  int n_chunks, Lq, n_heads, head_dim;
  const void* q; long long ldq;
  const void* k; const void* v; long long ldkv; long long kv_chunk_rows; int Lk;
  int pred_in_batch;
  const void* k0_pred; const void* v0_pred; long long ld_pred; int Lk_pred;
  void* out; long long ldo;
  int succ_in_batch;
} dp_attn_args;
DP_API dp_status dp_op_attention(const dp_attn_args* a, void* stream);

/* out[r] = LN(x[r]) * (1 + scale(r)) + shift(r), LN over d columns without
 * affine (biased variance, eps 1e-6); shift(r)/scale(r) are the vectors
 * shift/scale + sel(r / rows_per_chunk) * mod_stride (sel as for the GEMM
 * gate); shift = scale = NULL gives plain LN.  x fp32, out fp32 or bf16. */
typedef struct {
  dp_dtype out_dtype;
  const float* x; long long ldx;
  int M, d;
  const float* shift; const float* scale; long long mod_stride;
  const int* chunk_sel; int rows_per_chunk;
  void* out; long long ldo;
} dp_ln_args;
DP_API dp_status dp_op_layernorm_mod(const dp_ln_args* a, void* stream);

/* The modulated projection of a DiT block, LN + adaLN (as dp_op_layernorm_mod)
 * followed by the GEMM that reads its output (as dp_op_gemm), for callers that
 * may not allocate device memory.  This is a library convenience: the
 * DualParal write-up has no counterpart to it.
 *
 * Who needs it: code that runs inside a host framework whose allocator owns
 * all device memory (memory taken with cudaMalloc behind its back can make it
 * run out, and cudaMalloc/cudaFree synchronise the device), and services that
 * plan their memory at start-up and must not allocate on the request path.
 * Such callers own their inputs and outputs but have nowhere to put the
 * normalised rows that pass from one kernel to the next.  This call keeps
 * them in one static device array of 32 MiB that the library holds on every
 * GPU that loads it, until the process exits.  It calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 * Arguments: `ln` and `gemm` as for the two calls above, with ln->out and
 * gemm->A NULL (the scratch takes their place, packed with leading dimension
 * ln->d); gemm->M == ln->M, gemm->K == ln->d and ln->out_dtype == gemm->dtype.
 * Limit: ln->M * ln->d * (2 for bf16, 4 for f32) <= 32 MiB, else
 * DP_ERR_INVALID_ARG with the sizes in dp_last_error().  Other errors as for
 * dp_op_layernorm_mod and dp_op_gemm.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call, on any stream, uses the same array, and each call
 * overwrites the rows it uses before reading them, so nothing needs clearing;
 * but calls whose work overlaps on the GPU (other streams, other host threads)
 * race on it: order them on one stream. */
DP_API dp_status dp_op_ln_gemm_noalloc(const dp_ln_args* ln, const dp_gemm_args* gemm, void* stream);

/* Exercises the bounded-wait failure path: launches one block that waits on
 * an mbarrier nothing arrives at, gives up after the kernels' wait limit
 * (2 s), sets the status word and returns; nothing faults.  A following
 * dp_op_check must then report DP_ERR_KERNEL (and clear the word). */
DP_API dp_status dp_op_selftest_timeout(void* stream);

/* Waits for `stream`, then reads and clears the status word that the
 * tensor-core kernels of the calls above set when one of their bounded waits
 * gives up (they then skip the rest of their work).  DP_ERR_KERNEL if set. */
DP_API dp_status dp_op_check(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DP_OPS_H */
