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

// Reciprocal on the MUFU unit (approximate, relative error ~1e-7).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU of two values, returned as a bf16 pair (low half = a), with erf from
// Abramowitz and Stegun, Handbook of Mathematical Functions, formula 7.1.28
// (|error of erf| <= 3e-7): erf(z) = 1 - 1 / (1 + a1 z + ... + a6 z^6)^16,
// z >= 0; erf is odd.  Both lanes go through the packed fp32x2 instructions
// of sm_100 (each lane rounded as the scalar instruction); the one
// reciprocal per value runs on the MUFU unit, and there is no exponential.
// For large z the 16th power overflows to +inf, whose reciprocal is 0:
// erf = 1, the limit.  Used by the tensor-core GEMM's GELU epilogue.
__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint32_t gelu2_bf16(float a, float b) {
  constexpr uint64_t kAbs = 0x7FFFFFFF7FFFFFFFull, kSign = 0x8000000080000000ull;
  const uint64_t x = f32x2_pack(a, b);
  const uint64_t z = f32x2_mul(x & kAbs, f32x2_pack(0.70710678118654752f, 0.70710678118654752f));
  uint64_t q = f32x2_fma(z, f32x2_pack(0.0000430638f, 0.0000430638f), f32x2_pack(0.0002765672f, 0.0002765672f));
  q = f32x2_fma(q, z, f32x2_pack(0.0001520143f, 0.0001520143f));
  q = f32x2_fma(q, z, f32x2_pack(0.0092705272f, 0.0092705272f));
  q = f32x2_fma(q, z, f32x2_pack(0.0422820123f, 0.0422820123f));
  q = f32x2_fma(q, z, f32x2_pack(0.0705230784f, 0.0705230784f));
  q = f32x2_fma(q, z, f32x2_pack(1.0f, 1.0f));
  q = f32x2_mul(q, q);  // ^2
  q = f32x2_mul(q, q);  // ^4
  q = f32x2_mul(q, q);  // ^8
  q = f32x2_mul(q, q);  // ^16
  float q0, q1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(q0), "=f"(q1) : "l"(q));
  // |erf| = 1 - 1/q; with the sign of x, Phi = (1 + erf) / 2 = 0.5 + 0.5 erf
  const uint64_t r = f32x2_pack(rcp_approx(q0), rcp_approx(q1));
  const uint64_t e = f32x2_fma(r, f32x2_pack(-1.0f, -1.0f), f32x2_pack(1.0f, 1.0f));
  const uint64_t es = (e & kAbs) | (x & kSign);
  const uint64_t phi = f32x2_fma(es, f32x2_pack(0.5f, 0.5f), f32x2_pack(0.5f, 0.5f));
  float g0, g1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(g0), "=f"(g1) : "l"(f32x2_mul(x, phi)));
  __nv_bfloat162 v = __floats2bfloat162_rn(g0, g1);
  return *reinterpret_cast<uint32_t*>(&v);
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
