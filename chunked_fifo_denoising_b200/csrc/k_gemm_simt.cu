// SIMT FFMA GEMM with the fused epilogues: C = A[M][K] . W[N][K]^T (+ bias),
// fp32 accumulation in plain FFMA (no TF32).  Used by the fp32 validation mode
// for every contraction, and by both modes for the once-per-prompt/per-queue
// tables (timestep MLP, modulation projections, text projections).
#include "common.cuh"

namespace dp {

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16, SG_THREADS = 256;

template <typename TA, typename TW>
__global__ void __launch_bounds__(SG_THREADS)
gemm_simt_kernel(const TA* __restrict__ A, long long lda, const TW* __restrict__ W, int M, int N,
                 int K, EpiParams e) {
  __shared__ float As[SG_BK][SG_BM + 4];
  __shared__ float Ws[SG_BK][SG_BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 4x4 outputs each
  const int m0 = blockIdx.y * SG_BM, n0 = blockIdx.x * SG_BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SG_BK) {
    // each thread loads 4 elements of A and 4 of W (64 x 16 tiles)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + i * SG_THREADS;  // 0..1023
      const int r = idx / SG_BK, c = idx % SG_BK;
      const int gr = m0 + r, gc = k0 + c;
      As[c][r] = (gr < M && gc < K) ? to_f(A[(long long)gr * lda + gc]) : 0.0f;
      const int wr = n0 + r;
      Ws[c][r] = (wr < N && gc < K) ? to_f(W[(long long)wr * K + gc]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        w[i] = Ws[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c < N) apply_epi(e, r, c, acc[i][j]);
    }
  }
}

cudaError_t gemm_simt(int a_f32, const void* A, long long lda, int w_f32, const void* W,
                      int M, int N, int K, const EpiParams& e, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + SG_BN - 1) / SG_BN, (M + SG_BM - 1) / SG_BM);
  if (a_f32 && w_f32)
    gemm_simt_kernel<float, float><<<grid, SG_THREADS, 0, s>>>((const float*)A, lda,
                                                               (const float*)W, M, N, K, e);
  else if (a_f32)
    gemm_simt_kernel<float, bf16><<<grid, SG_THREADS, 0, s>>>((const float*)A, lda,
                                                              (const bf16*)W, M, N, K, e);
  else if (w_f32)
    gemm_simt_kernel<bf16, float><<<grid, SG_THREADS, 0, s>>>((const bf16*)A, lda,
                                                              (const float*)W, M, N, K, e);
  else
    gemm_simt_kernel<bf16, bf16><<<grid, SG_THREADS, 0, s>>>((const bf16*)A, lda,
                                                             (const bf16*)W, M, N, K, e);
  return cudaGetLastError();
}

}  // namespace dp
