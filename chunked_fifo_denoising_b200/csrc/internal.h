// Internal declarations shared by the runtime (dp_api.cu) and the kernel files.
// Nothing here is part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dp.h"
#include "../../include/dp_ops.h"

namespace dp {

typedef __nv_bfloat16 bf16;

// Epilogue modes of the GEMM kernels (superset of dp_epilogue).
enum EpiMode : int {
  EPI_STORE = 0,        // out = acc + bias
  EPI_GELU = 1,         // out = gelu_erf(acc + bias)
  EPI_RESID = 2,        // resid += acc + bias
  EPI_RESID_GATED = 3,  // resid += gate * (acc + bias)
  EPI_SILU = 4,         // out = silu(acc + bias)             (init only)
  EPI_EULER = 5         // ring[...] += dsig(level) * (acc + bias)  (head)
};

struct EpiParams {
  int mode;
  int out_f32;                    // 1: out is float, 0: bf16
  const float* bias;              // [N] or null
  void* out; long long ldo;
  float* resid; long long ldr;
  // gate(r, c) = gate[sel(r / rows_per_chunk) * gate_stride + c]
  const float* gate; long long gate_stride; const int* chunk_sel; int rows_per_chunk;
  // optional copy of stored values: rows [cache_row0, +cache_rows), cols >= cache_col0
  void* cache; long long cache_row0; int cache_rows; int cache_col0; long long ldc;
  // Euler scatter into the latent ring (EPI_EULER): row r is token r % Lc of
  // batch chunk r / Lc; column = patch feature ((c*pt+dt)*ph+dy)*pw+dx.
  float* ring; long long chunk_numel;
  const int* chunk_slot;          // [batch chunk] -> ring slot
  const float* dsig;              // [batch chunk] -> sigma_{j-1} - sigma_j
  int lat_c, lat_f, lat_h, lat_w, pt, ph, pw;
  // QKV epilogue with per-head RMSNorm + rotary positions on the q and k
  // column blocks [0, 2 * rope_d) (bf16 tensor-core path; rows_per_chunk = Lc)
  int rope;
  int rope_d, rope_hd, rope_Fq, rope_Hq, rope_Wq, rope_nt, rope_nh;
  const float* q_w; const float* k_w;
  const float2* rope_t; const float2* rope_y; const float2* rope_x;
};

struct AttnParams {
  int f32;                        // 1: float operands, 0: bf16
  int n_chunks, Lq, n_heads, head_dim;
  const void* q; long long ldq;
  const void* k; const void* v; long long ldkv; long long kv_chunk_rows; int Lk;
  int pred_in_batch;
  const void* k0_pred; const void* v0_pred; long long ld_pred; int Lk_pred;
  void* out; long long ldo;
  int succ_in_batch;              // chunk c < n_chunks-1 also reads chunk c+1's own keys
  int qblocks_per_cta;            // tensor-core path: 256-query blocks per CTA (0 = choose)
  int dual_rem;                   // tensor-core path, set by the launcher: the last grid
                                  // column pairs two heads' one-tile remainder blocks
};

struct LnParams {
  int out_f32;
  const float* x; long long ldx;
  int M, d;
  const float* shift; const float* scale; long long mod_stride;
  const int* chunk_sel; int rows_per_chunk;
  void* out; long long ldo;
};

// ---- launchers (return cudaGetLastError() of the launch) -------------------
// SIMT FFMA GEMM: a_f32/w_f32 select float or bf16 operands.
cudaError_t gemm_simt(int a_f32, const void* A, long long lda, int w_f32, const void* W,
                      int M, int N, int K, const EpiParams& e, cudaStream_t s);
// tcgen05 tensor-core GEMM, bf16 operands, fp32 accumulation.
cudaError_t gemm_tc(const bf16* A, long long lda, const bf16* W, int M, int N, int K,
                    const EpiParams& e, int* status, cudaStream_t s);
bool gemm_tc_supported(long long lda, int M, int N, int K);

cudaError_t attention_simt(const AttnParams& p, cudaStream_t s);
cudaError_t attention_tc(const AttnParams& p, int* status, cudaStream_t s);
bool attention_tc_supported(const AttnParams& p);

cudaError_t layernorm_mod(const LnParams& p, cudaStream_t s);

// Per-head RMSNorm + 3-D rotary positions applied in place to the q and k
// column blocks of a [M][ld] qkv buffer (q at col 0, k at col d).  Tables hold
// (cos, sin) float pairs: rope_t [n_chunks * Fq][nt], rope_y [Hq][nh],
// rope_x [Wq][nw].  Rows of batch chunk 0 with cache != null also write the
// result of k to cache[row * ldc + col].
struct RopeParams {
  int f32;
  void* qkv; long long ld;
  int M, d, n_heads, Lc, Fq, Hq, Wq, nt, nh;
  const float* q_w; const float* k_w;
  const float2* rope_t; const float2* rope_y; const float2* rope_x;
  void* cache; long long ldc;
};
cudaError_t qk_norm_rope(const RopeParams& p, cudaStream_t s);

// ring [slots][C][F][H][W] fp32 -> patches [M][P] (float or bf16)
cudaError_t gather_patches(const float* ring, long long chunk_numel, const int* chunk_slot,
                           int n_chunks, int C, int F, int H, int W, int pt, int ph, int pw,
                           void* out, int out_f32, cudaStream_t s);

// sinusoid features of t_j = 1000 * j / T for j = 1..T -> out [T][D] fp32
cudaError_t timestep_features(int T, int D, float* out, cudaStream_t s);

// out[j][l][:] = m[j][:] + table[l][:]  (rows of width w)
cudaError_t add_layer_tables(const float* m, const float* table, int T, int L, int w,
                             float* out, cudaStream_t s);

// N(0,1) by the SplitMix64 + Box-Muller construction of the seeded generator
cudaError_t normal_fill(unsigned long long seed, unsigned long long a, unsigned long long b,
                        float* out, long long n, cudaStream_t s);

// Device status word of kernels launched from the single-kernel entry points.
int* op_status_word();
// A kernel whose only mbarrier wait times out (failure-path self test); it
// sets `status` (NULL: the status word of the single-kernel entry points).
cudaError_t selftest_timeout(int* status, cudaStream_t s);

// slot [C][F][HW] <- pool [2F][C][HW]: frame f of the chunk is pool frame src[f]
struct PoolGather { int src[64]; };
cudaError_t noise_from_pool(const float* pool, int C, int F, long long hw, PoolGather src,
                            float* slot, cudaStream_t s);

cudaError_t convert_f32_to_bf16(const float* in, bf16* out, long long n, cudaStream_t s);
cudaError_t convert_bf16_to_f32(const bf16* in, float* out, long long n, cudaStream_t s);
// strided 2-D copy/convert of a [rows][cols] block between float/bf16 buffers
cudaError_t copy_rows(const void* in, int in_f32, long long ldi, void* out, int out_f32,
                      long long ldo, long long rows, long long cols, cudaStream_t s);

}  // namespace dp
