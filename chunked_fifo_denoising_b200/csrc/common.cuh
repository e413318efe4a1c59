// Device helpers shared by the kernel files.
#pragma once

#include "internal.h"

namespace dp {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// GELU, exact form x * Phi(x) with Phi(x) = (1 + erf(x / sqrt 2)) / 2.
__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}
__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

// GELU x * Phi(x) with erf from Abramowitz and Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (|error of erf| <= 1.5e-7):
// erf(z) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2),
// t = 1 / (1 + p z), z >= 0; erf is odd.  Branch-free, used by the
// tensor-core GEMM epilogue; the reciprocal and 2^x run on the MUFU unit
// (approximate, relative error ~1e-7, well inside the formula's bound).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_approx_f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float gelu_as(float x) {
  const float z = fabsf(x) * 0.70710678118654752f;
  const float t = rcp_approx(fmaf(0.3275911f, z, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float e = ex2_approx_f(-z * z * 1.4426950408889634f);
  const float erf_abs = fmaf(-poly, e, 1.0f);
  const float erf_x = copysignf(erf_abs, x);
  return 0.5f * x * (1.0f + erf_x);
}

// Ring offset of (row, col) of the head output: row = token of batch chunk,
// col = patch feature.  Inverse of the patch gather.
__device__ __forceinline__ long long euler_index(const EpiParams& e, int row, int col, int Lc) {
  const int c = row / Lc, t = row - (row / Lc) * Lc;
  const int hq = e.lat_h / e.ph, wq = e.lat_w / e.pw;
  const int fq = t / (hq * wq), rem = t - fq * (hq * wq);
  const int yq = rem / wq, xq = rem - yq * wq;
  const int dx = col % e.pw, dy = (col / e.pw) % e.ph, dt = (col / (e.pw * e.ph)) % e.pt;
  const int cc = col / (e.pw * e.ph * e.pt);
  const long long lat = (((long long)cc * e.lat_f + fq * e.pt + dt) * e.lat_h + yq * e.ph + dy)
                            * e.lat_w + xq * e.pw + dx;
  return (long long)e.chunk_slot[c] * e.chunk_numel + lat;
}

// Applies the epilogue to one accumulator element (SIMT paths and tails).
__device__ __forceinline__ void apply_epi(const EpiParams& e, int row, int col, float acc) {
  float v = acc + (e.bias ? e.bias[col] : 0.0f);
  switch (e.mode) {
    case EPI_GELU: v = gelu_erf(v); break;
    case EPI_SILU: v = silu(v); break;
    default: break;
  }
  if (e.mode == EPI_RESID) {
    e.resid[(long long)row * e.ldr + col] += v;
    return;
  }
  if (e.mode == EPI_RESID_GATED) {
    const int c = row / e.rows_per_chunk;
    const int sel = e.chunk_sel ? e.chunk_sel[c] : c;
    e.resid[(long long)row * e.ldr + col] += e.gate[(long long)sel * e.gate_stride + col] * v;
    return;
  }
  if (e.mode == EPI_EULER) {
    const int c = row / e.rows_per_chunk;
    e.ring[euler_index(e, row, col, e.rows_per_chunk)] += e.dsig[c] * v;
    return;
  }
  if (e.out_f32) {
    ((float*)e.out)[(long long)row * e.ldo + col] = v;
  } else {
    ((bf16*)e.out)[(long long)row * e.ldo + col] = __float2bfloat16_rn(v);
  }
  if (e.cache && row >= e.cache_row0 && row < e.cache_row0 + e.cache_rows && col >= e.cache_col0) {
    const long long o = (long long)(row - e.cache_row0) * e.ldc + (col - e.cache_col0);
    if (e.out_f32) ((float*)e.cache)[o] = v;
    else ((bf16*)e.cache)[o] = __float2bfloat16_rn(v);
  }
}

template <int NW>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < NW; ++i) s += red[i];
  return s;
}

}  // namespace dp
