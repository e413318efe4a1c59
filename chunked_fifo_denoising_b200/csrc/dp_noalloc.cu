// The modulated projection (LayerNorm + adaLN, then a GEMM) without any
// device allocation: the normalised rows live in one static device array of
// fixed size instead of a buffer the caller allocates.  See dp_op_ln_gemm_noalloc
// in include/dp_ops.h for who needs this and for its limits.
#include <mutex>

#include "runtime.h"

using namespace dp;

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device

// Held by every device that loads this library, until the process exits.
static __device__ __align__(256) unsigned char g_ln_gemm_scratch[kScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device.  Host code only
// holds a stand-in for the symbol; the real address differs per device and is
// looked up once per device, with that device current.
dp_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DP_ERR_INVALID_ARG, "device %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ln_gemm_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return fail(DP_ERR_CUDA, "address of the static scratch on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DP_OK;
}

}  // namespace

extern "C" {

dp_status dp_op_ln_gemm_noalloc(const dp_ln_args* ln, const dp_gemm_args* gemm, void* stream) {
  clear_error();
  if (!ln || !gemm) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (ln->out || gemm->A)
    return fail(DP_ERR_INVALID_ARG, "ln->out and gemm->A must be NULL: the static scratch takes their place");
  if (ln->M <= 0 || ln->d <= 0) return fail(DP_ERR_INVALID_ARG, "bad layernorm sizes");
  if (gemm->M != ln->M || gemm->K != ln->d)
    return fail(DP_ERR_INVALID_ARG, "the GEMM must read the normalised rows: M %d vs %d, K %d vs d %d",
                gemm->M, ln->M, gemm->K, ln->d);
  if (ln->out_dtype != gemm->dtype) return fail(DP_ERR_INVALID_ARG, "layernorm output and GEMM operand dtypes differ");
  const size_t elem = gemm->dtype == DP_DT_BF16 ? 2 : 4;
  const size_t bytes = (size_t)ln->M * (size_t)ln->d * elem;
  if (bytes > kScratchBytes)
    return fail(DP_ERR_INVALID_ARG,
                "normalised rows of %d x %d need %zu bytes, above the static scratch of %zu bytes",
                ln->M, ln->d, bytes, kScratchBytes);
  void* scratch = nullptr;
  DP_TRY(scratch_address(&scratch));
  // rows are packed (leading dimension d); every row is written before the GEMM reads it
  dp_ln_args l = *ln;
  l.out = scratch;
  l.ldo = ln->d;
  DP_TRY(dp_op_layernorm_mod(&l, stream));
  dp_gemm_args g = *gemm;
  g.A = scratch;
  g.lda = ln->d;
  return dp_op_gemm(&g, stream);
}

}  // extern "C"
