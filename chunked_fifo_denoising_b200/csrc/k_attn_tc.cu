// bf16 attention entry used by the production path.
#include "common.cuh"

namespace dp {

bool attention_tc_supported(const AttnParams& p) {
  return !p.f32 && (p.head_dim == 64 || p.head_dim == 128);
}

cudaError_t attention_tc(const AttnParams& p, int* status, cudaStream_t s) {
  (void)status;
  return attention_simt(p, s);
}

}  // namespace dp
