// Single-kernel entry points (dp_ops.h): the kernels of dp_queue_step run alone
// on caller memory, same tile configurations, for parity checks and timing.
#include <cstring>

#include "runtime.h"

using namespace dp;

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

extern "C" {

dp_status dp_op_gemm(const dp_gemm_args* a, void* stream) {
  clear_error();
  if (!a || !a->A || !a->W) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (a->M <= 0 || a->N <= 0 || a->K <= 0 || a->lda < a->K)
    return fail(DP_ERR_INVALID_ARG, "bad GEMM sizes");
  if (a->epi < DP_EPI_STORE || a->epi > DP_EPI_RESID_GATED) return fail(DP_ERR_INVALID_ARG, "bad epilogue");
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.mode = (int)a->epi;
  e.out_f32 = a->dtype == DP_DT_F32;
  e.bias = a->bias;
  e.out = a->out;
  e.ldo = a->ldo;
  e.resid = a->resid;
  e.ldr = a->ldr;
  e.gate = a->gate;
  e.gate_stride = a->gate_stride;
  e.chunk_sel = a->chunk_sel;
  e.rows_per_chunk = a->rows_per_chunk > 0 ? a->rows_per_chunk : 1;
  e.cache = a->cache;
  e.cache_row0 = a->cache_row0;
  e.cache_rows = a->cache ? a->cache_rows : 0;
  e.cache_col0 = a->cache_col0;
  e.ldc = a->ldc;
  if ((a->epi == DP_EPI_STORE || a->epi == DP_EPI_GELU) && (!a->out || a->ldo < a->N))
    return fail(DP_ERR_INVALID_ARG, "STORE/GELU need out with ldo >= N");
  if ((a->epi == DP_EPI_RESID || a->epi == DP_EPI_RESID_GATED) && (!a->resid || a->ldr < a->N))
    return fail(DP_ERR_INVALID_ARG, "RESID needs resid with ldr >= N");
  if (a->epi == DP_EPI_RESID_GATED && !a->gate) return fail(DP_ERR_INVALID_ARG, "RESID_GATED needs gate");
  if (a->cache && (a->epi != DP_EPI_STORE || a->ldc < a->N - a->cache_col0))
    return fail(DP_ERR_INVALID_ARG, "cache copy needs STORE and ldc >= N - cache_col0");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (a->dtype == DP_DT_F32) {
    err = gemm_simt(1, a->A, a->lda, 1, a->W, a->M, a->N, a->K, e, s);
  } else if (a->dtype == DP_DT_BF16) {
    if (!gemm_tc_supported(a->lda, a->M, a->N, a->K) || !al16(a->A) || !al16(a->W))
      return fail(DP_ERR_INVALID_ARG, "bf16 GEMM needs K %% 64 == 0, N %% 32 == 0, lda %% 8 == 0, 16-byte aligned operands");
    if ((a->out && (a->ldo % 8 || !al16(a->out))) || (a->resid && (a->ldr % 4 || !al16(a->resid))) ||
        (a->bias && !al16(a->bias)) || (a->gate && (a->gate_stride % 4 || !al16(a->gate))) ||
        (a->cache && (a->ldc % 8 || a->cache_col0 % 32 || !al16(a->cache))))
      return fail(DP_ERR_INVALID_ARG, "bf16 GEMM epilogue pointers must be 16-byte aligned");
    err = gemm_tc(static_cast<const bf16*>(a->A), a->lda, static_cast<const bf16*>(a->W), a->M,
                  a->N, a->K, e, nullptr, s);
  } else {
    return fail(DP_ERR_INVALID_ARG, "bad dtype");
  }
  if (err != cudaSuccess) return fail(DP_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(err));
  return DP_OK;
}

dp_status dp_op_attention(const dp_attn_args* a, void* stream) {
  clear_error();
  if (!a || !a->q || !a->k || !a->v || !a->out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (a->n_chunks <= 0 || a->Lq <= 0 || a->Lk <= 0 || a->n_heads <= 0 || a->head_dim <= 0)
    return fail(DP_ERR_INVALID_ARG, "bad attention sizes");
  const long long w = (long long)a->n_heads * a->head_dim;
  if (a->ldq < w || a->ldkv < w || a->ldo < w) return fail(DP_ERR_INVALID_ARG, "leading dimension too small");
  if (a->k0_pred && (!a->v0_pred || a->Lk_pred <= 0 || a->ld_pred < w))
    return fail(DP_ERR_INVALID_ARG, "bad predecessor buffer");
  if ((a->pred_in_batch || a->succ_in_batch) && a->kv_chunk_rows <= 0)
    return fail(DP_ERR_INVALID_ARG, "pred_in_batch / succ_in_batch need per-chunk keys");
  if (a->kv_chunk_rows > 0 && a->Lk > a->kv_chunk_rows)
    return fail(DP_ERR_INVALID_ARG, "Lk %d exceeds kv_chunk_rows %lld: a chunk's keys would run into the next chunk's",
                a->Lk, a->kv_chunk_rows);
  AttnParams p;
  memset(&p, 0, sizeof(p));
  p.f32 = a->dtype == DP_DT_F32;
  p.n_chunks = a->n_chunks;
  p.Lq = a->Lq;
  p.n_heads = a->n_heads;
  p.head_dim = a->head_dim;
  p.q = a->q;
  p.ldq = a->ldq;
  p.k = a->k;
  p.v = a->v;
  p.ldkv = a->ldkv;
  p.kv_chunk_rows = a->kv_chunk_rows;
  p.Lk = a->Lk;
  p.pred_in_batch = a->pred_in_batch;
  p.k0_pred = a->k0_pred;
  p.v0_pred = a->v0_pred;
  p.ld_pred = a->ld_pred;
  p.Lk_pred = a->k0_pred ? a->Lk_pred : 0;
  p.out = a->out;
  p.ldo = a->ldo;
  p.succ_in_batch = a->succ_in_batch;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (a->dtype == DP_DT_F32) {
    if (a->head_dim != 16 && a->head_dim != 32 && a->head_dim != 64 && a->head_dim != 128)
      return fail(DP_ERR_INVALID_ARG, "f32 attention needs head_dim in {16,32,64,128}");
    err = attention_simt(p, s);
  } else if (a->dtype == DP_DT_BF16) {
    if (!attention_tc_supported(p)) return fail(DP_ERR_INVALID_ARG, "bf16 attention shape not supported");
    err = attention_tc(p, nullptr, s);
  } else {
    return fail(DP_ERR_INVALID_ARG, "bad dtype");
  }
  if (err != cudaSuccess) return fail(DP_ERR_CUDA, "attention launch: %s", cudaGetErrorString(err));
  return DP_OK;
}

dp_status dp_op_selftest_timeout(void* stream) {
  clear_error();
  cudaError_t err = selftest_timeout(nullptr, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(DP_ERR_CUDA, "self test launch: %s", cudaGetErrorString(err));
  return DP_OK;
}

dp_status dp_op_check(void* stream) {
  clear_error();
  DP_CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int* w = op_status_word();
  if (!w) return fail(DP_ERR_CUDA, "status word unavailable");
  int v = 0;
  DP_CK(cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost));
  if (v) {
    DP_CK(cudaMemset(w, 0, sizeof(int)));
    return fail(DP_ERR_KERNEL, "a kernel gave up a bounded wait (status 0x%x)", v);
  }
  return DP_OK;
}

dp_status dp_op_layernorm_mod(const dp_ln_args* a, void* stream) {
  clear_error();
  if (!a || !a->x || !a->out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (a->M <= 0 || a->d <= 0 || a->d % 4 || a->d > 6144 || a->ldx % 4 || a->ldo % 4)
    return fail(DP_ERR_INVALID_ARG, "bad layernorm sizes (d %% 4 == 0, d <= 6144)");
  if ((a->shift == nullptr) != (a->scale == nullptr)) return fail(DP_ERR_INVALID_ARG, "shift and scale go together");
  if (!al16(a->x) || !al16(a->out) || (a->shift && (!al16(a->shift) || !al16(a->scale) || a->mod_stride % 4)))
    return fail(DP_ERR_INVALID_ARG, "layernorm pointers must be 16-byte aligned");
  LnParams p;
  memset(&p, 0, sizeof(p));
  p.out_f32 = a->out_dtype == DP_DT_F32;
  p.x = a->x;
  p.ldx = a->ldx;
  p.M = a->M;
  p.d = a->d;
  p.shift = a->shift;
  p.scale = a->scale;
  p.mod_stride = a->mod_stride;
  p.chunk_sel = a->chunk_sel;
  p.rows_per_chunk = a->rows_per_chunk > 0 ? a->rows_per_chunk : 1;
  p.out = a->out;
  p.ldo = a->ldo;
  cudaError_t err = layernorm_mod(p, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(DP_ERR_CUDA, "layernorm launch: %s", cudaGetErrorString(err));
  return DP_OK;
}

}  // extern "C"
