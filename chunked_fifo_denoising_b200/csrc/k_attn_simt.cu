// SIMT flash attention (fp32 arithmetic) over up to three key buffers per
// chunk: the predecessor's K/V (in-batch rows of chunk c-1, or the persisted
// K/V for the first chunk), the chunk's own K/V and, optionally, the
// successor's (in-batch rows of chunk c+1); one joint online softmax, no
// concatenation.  One thread per query row; key tiles staged in shared memory.
// Used by the fp32 validation mode.
#include "common.cuh"

namespace dp {

constexpr int SA_Q = 64;   // queries (threads) per block
constexpr int SA_KT = 32;  // keys per tile

template <typename T, int HD>
__global__ void __launch_bounds__(SA_Q) attn_simt_kernel(AttnParams p) {
  extern __shared__ float sm[];
  float* Ks = sm;                 // [SA_KT][HD]
  float* Vs = sm + SA_KT * HD;    // [SA_KT][HD]
  const int c = blockIdx.z, h = blockIdx.y;
  const int qi = blockIdx.x * SA_Q + threadIdx.x;
  const bool active = qi < p.Lq;
  const float scale = 1.0f / sqrtf((float)HD);
  float q[HD], acc[HD];
  const T* Q = (const T*)p.q + ((long long)c * p.Lq + (active ? qi : 0)) * p.ldq + h * HD;
#pragma unroll
  for (int i = 0; i < HD; ++i) {
    q[i] = to_f(Q[i]) * scale;
    acc[i] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;

  for (int src = 0; src < 3; ++src) {  // predecessor, own, successor
    const T* Kb;
    const T* Vb;
    long long ld;
    int n;
    if (src == 0) {  // predecessor
      if (c > 0 && p.pred_in_batch) {
        Kb = (const T*)p.k + (long long)(c - 1) * p.kv_chunk_rows * p.ldkv;
        Vb = (const T*)p.v + (long long)(c - 1) * p.kv_chunk_rows * p.ldkv;
        ld = p.ldkv;
        n = p.Lk;
      } else if (c == 0 && p.k0_pred) {
        Kb = (const T*)p.k0_pred;
        Vb = (const T*)p.v0_pred;
        ld = p.ld_pred;
        n = p.Lk_pred;
      } else {
        continue;
      }
    } else if (src == 1) {
      Kb = (const T*)p.k + (long long)c * p.kv_chunk_rows * p.ldkv;
      Vb = (const T*)p.v + (long long)c * p.kv_chunk_rows * p.ldkv;
      ld = p.ldkv;
      n = p.Lk;
    } else {  // successor
      if (!p.succ_in_batch || c + 1 >= p.n_chunks) continue;
      Kb = (const T*)p.k + (long long)(c + 1) * p.kv_chunk_rows * p.ldkv;
      Vb = (const T*)p.v + (long long)(c + 1) * p.kv_chunk_rows * p.ldkv;
      ld = p.ldkv;
      n = p.Lk;
    }
    for (int k0 = 0; k0 < n; k0 += SA_KT) {
      __syncthreads();
      for (int i = threadIdx.x; i < SA_KT * HD; i += SA_Q) {
        const int r = i / HD, col = i % HD;
        const bool ok = k0 + r < n;
        Ks[i] = ok ? to_f(Kb[(long long)(k0 + r) * ld + h * HD + col]) : 0.0f;
        Vs[i] = ok ? to_f(Vb[(long long)(k0 + r) * ld + h * HD + col]) : 0.0f;
      }
      __syncthreads();
      const int nt = min(SA_KT, n - k0);
      float s[SA_KT];
      float mt = m;
#pragma unroll
      for (int j = 0; j < SA_KT; ++j) {
        float d = 0.0f;
#pragma unroll
        for (int i = 0; i < HD; ++i) d = fmaf(q[i], Ks[j * HD + i], d);
        s[j] = j < nt ? d : -INFINITY;
        mt = fmaxf(mt, s[j]);
      }
      const float corr = (m == -INFINITY) ? 0.0f : expf(m - mt);
      l *= corr;
#pragma unroll
      for (int i = 0; i < HD; ++i) acc[i] *= corr;
#pragma unroll
      for (int j = 0; j < SA_KT; ++j) {
        const float pj = j < nt ? expf(s[j] - mt) : 0.0f;
        l += pj;
#pragma unroll
        for (int i = 0; i < HD; ++i) acc[i] = fmaf(pj, Vs[j * HD + i], acc[i]);
      }
      m = mt;
    }
  }
  if (active) {
    T* O = (T*)p.out + ((long long)c * p.Lq + qi) * p.ldo + h * HD;
    const float inv = 1.0f / l;
#pragma unroll
    for (int i = 0; i < HD; ++i) O[i] = from_f<T>(acc[i] * inv);
  }
}

template <typename T, int HD>
static cudaError_t launch_simt(const AttnParams& p, cudaStream_t s) {
  dim3 grid((p.Lq + SA_Q - 1) / SA_Q, p.n_heads, p.n_chunks);
  const size_t smem = 2 * SA_KT * HD * sizeof(float);
  attn_simt_kernel<T, HD><<<grid, SA_Q, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t dispatch_hd(const AttnParams& p, cudaStream_t s) {
  switch (p.head_dim) {
    case 16: return launch_simt<T, 16>(p, s);
    case 32: return launch_simt<T, 32>(p, s);
    case 64: return launch_simt<T, 64>(p, s);
    case 128: return launch_simt<T, 128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t attention_simt(const AttnParams& p, cudaStream_t s) {
  if (p.n_chunks <= 0 || p.Lq <= 0) return cudaSuccess;
  return p.f32 ? dispatch_hd<float>(p, s) : dispatch_hd<bf16>(p, s);
}

}  // namespace dp
