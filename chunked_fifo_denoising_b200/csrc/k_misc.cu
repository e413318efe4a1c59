// Memory-bound kernels of the queue step: LayerNorm + adaLN modulation, the
// patch gather from the latent ring, per-level timestep features, table
// broadcast, the seeded noise generator and dtype conversions.
#include "common.cuh"

namespace dp {

static __device__ int g_op_status;

int* op_status_word() {
  // the symbol's device address differs per device: look it up per device
  static int* ptr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  if (!ptr[dev] && cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr[dev]), g_op_status) != cudaSuccess) {
    cudaGetLastError();
    ptr[dev] = nullptr;
  }
  return ptr[dev];
}

// ---------------------------------------------------------------------------
// LayerNorm (no affine, biased variance, eps 1e-6) + adaLN shift/scale.
// One 128-thread block per row, 128-bit loads of x; the row stays in
// registers between the mean, variance and output passes (d <= 6144).
// ---------------------------------------------------------------------------
constexpr int LN_THREADS = 128;
constexpr int LN_MAXV = 12;

template <bool OUT_F32>
__global__ void __launch_bounds__(LN_THREADS) ln_mod_kernel(LnParams p) {
  __shared__ float red[LN_THREADS / 32];
  const int row = blockIdx.x;
  const int nv = p.d >> 2;
  const float4* xr = reinterpret_cast<const float4*>(p.x + (long long)row * p.ldx);
  float4 v[LN_MAXV];
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int idx = threadIdx.x + i * LN_THREADS;
    if (idx < nv) {
      v[i] = xr[idx];
      s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
  }
  const float mean = block_sum<LN_THREADS / 32>(s, red) / (float)p.d;
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int idx = threadIdx.x + i * LN_THREADS;
    if (idx < nv) {
      const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
      ss += (a * a + b * b) + (c * c + d * d);
    }
  }
  const float var = block_sum<LN_THREADS / 32>(ss, red) / (float)p.d;
  const float rstd = 1.0f / sqrtf(var + 1e-6f);
  const float4* sh = nullptr;
  const float4* sc = nullptr;
  if (p.shift) {
    const int c = row / p.rows_per_chunk;
    const long long sel = p.chunk_sel ? p.chunk_sel[c] : c;
    sh = reinterpret_cast<const float4*>(p.shift + sel * p.mod_stride);
    sc = reinterpret_cast<const float4*>(p.scale + sel * p.mod_stride);
  }
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int idx = threadIdx.x + i * LN_THREADS;
    if (idx < nv) {
      float4 o;
      o.x = (v[i].x - mean) * rstd;
      o.y = (v[i].y - mean) * rstd;
      o.z = (v[i].z - mean) * rstd;
      o.w = (v[i].w - mean) * rstd;
      if (sh) {
        const float4 a = sh[idx], b = sc[idx];
        o.x = o.x * (1.0f + b.x) + a.x;
        o.y = o.y * (1.0f + b.y) + a.y;
        o.z = o.z * (1.0f + b.z) + a.z;
        o.w = o.w * (1.0f + b.w) + a.w;
      }
      if (OUT_F32) {
        reinterpret_cast<float4*>((float*)p.out + (long long)row * p.ldo)[idx] = o;
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>((bf16*)p.out + (long long)row * p.ldo)[idx] = pk;
      }
    }
  }
}

// One warp per row for narrow rows (d <= 512), where a 128-thread block per
// row would leave most threads idle: both reductions are warp shuffles, 8 rows
// per 256-thread block.
constexpr int LNW_MAXV = 16;

template <bool OUT_F32>
__global__ void __launch_bounds__(256) ln_mod_warp_kernel(LnParams p) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.M) return;
  const int nv = p.d >> 2;
  const float4* xr = reinterpret_cast<const float4*>(p.x + (long long)row * p.ldx);
  float4 v[LNW_MAXV];
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < LNW_MAXV; ++i) {
    const int idx = lane + i * 32;
    if (idx < nv) {
      v[i] = xr[idx];
      s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)p.d;
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < LNW_MAXV; ++i) {
    const int idx = lane + i * 32;
    if (idx < nv) {
      const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
      ss += (a * a + b * b) + (c * c + d * d);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = 1.0f / sqrtf(ss / (float)p.d + 1e-6f);
  const float4* sh = nullptr;
  const float4* sc = nullptr;
  if (p.shift) {
    const int c = row / p.rows_per_chunk;
    const long long sel = p.chunk_sel ? p.chunk_sel[c] : c;
    sh = reinterpret_cast<const float4*>(p.shift + sel * p.mod_stride);
    sc = reinterpret_cast<const float4*>(p.scale + sel * p.mod_stride);
  }
#pragma unroll
  for (int i = 0; i < LNW_MAXV; ++i) {
    const int idx = lane + i * 32;
    if (idx < nv) {
      float4 o;
      o.x = (v[i].x - mean) * rstd;
      o.y = (v[i].y - mean) * rstd;
      o.z = (v[i].z - mean) * rstd;
      o.w = (v[i].w - mean) * rstd;
      if (sh) {
        const float4 a = sh[idx], b = sc[idx];
        o.x = o.x * (1.0f + b.x) + a.x;
        o.y = o.y * (1.0f + b.y) + a.y;
        o.z = o.z * (1.0f + b.z) + a.z;
        o.w = o.w * (1.0f + b.w) + a.w;
      }
      if (OUT_F32) {
        reinterpret_cast<float4*>((float*)p.out + (long long)row * p.ldo)[idx] = o;
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>((bf16*)p.out + (long long)row * p.ldo)[idx] = pk;
      }
    }
  }
}

// Rows of d = 512 * NV: 8 consecutive rows per 128-thread block; the loads of
// row i+1 are issued before the reductions of row i, so every thread keeps
// 2 * NV 16-byte loads in flight.
constexpr int LN_ROWS = 8;

template <int NV, bool OUT_F32>
__global__ void __launch_bounds__(LN_THREADS) ln_rows_kernel(LnParams p) {
  __shared__ float red[2][LN_THREADS / 32];
  const int row0 = blockIdx.x * LN_ROWS;
  const int rend = min(row0 + LN_ROWS, p.M);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float4 v[NV], nx[NV];
  auto load = [&](float4 (&dst)[NV], int row) {
    const float4* xr = reinterpret_cast<const float4*>(p.x + (long long)row * p.ldx);
#pragma unroll
    for (int i = 0; i < NV; ++i) dst[i] = xr[threadIdx.x + i * LN_THREADS];
  };
  auto reduce = [&](float a, int b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) red[b][wid] = a;
    __syncthreads();
    float t = 0.0f;
#pragma unroll
    for (int i = 0; i < LN_THREADS / 32; ++i) t += red[b][i];
    return t;
  };
  if (row0 < rend) load(v, row0);
  for (int row = row0; row < rend; ++row) {
    if (row + 1 < rend) load(nx, row + 1);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < NV; ++i) s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    const float mean = reduce(s, 0) / (float)p.d;
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
      ss += (a * a + b * b) + (c * c + d * d);
    }
    const float var = reduce(ss, 1) / (float)p.d;
    const float rstd = 1.0f / sqrtf(var + 1e-6f);
    const float4* sh = nullptr;
    const float4* sc = nullptr;
    if (p.shift) {
      const int c = row / p.rows_per_chunk;
      const long long sel = p.chunk_sel ? p.chunk_sel[c] : c;
      sh = reinterpret_cast<const float4*>(p.shift + sel * p.mod_stride);
      sc = reinterpret_cast<const float4*>(p.scale + sel * p.mod_stride);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = threadIdx.x + i * LN_THREADS;
      float4 o;
      o.x = (v[i].x - mean) * rstd;
      o.y = (v[i].y - mean) * rstd;
      o.z = (v[i].z - mean) * rstd;
      o.w = (v[i].w - mean) * rstd;
      if (sh) {
        const float4 a = sh[idx], b = sc[idx];
        o.x = o.x * (1.0f + b.x) + a.x;
        o.y = o.y * (1.0f + b.y) + a.y;
        o.z = o.z * (1.0f + b.z) + a.z;
        o.w = o.w * (1.0f + b.w) + a.w;
      }
      if (OUT_F32) {
        reinterpret_cast<float4*>((float*)p.out + (long long)row * p.ldo)[idx] = o;
      } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>((bf16*)p.out + (long long)row * p.ldo)[idx] = pk;
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = nx[i];
  }
}

template <int NV>
static void launch_rows(const LnParams& p, cudaStream_t s) {
  const int blocks = (p.M + LN_ROWS - 1) / LN_ROWS;
  if (p.out_f32) ln_rows_kernel<NV, true><<<blocks, LN_THREADS, 0, s>>>(p);
  else ln_rows_kernel<NV, false><<<blocks, LN_THREADS, 0, s>>>(p);
}

cudaError_t layernorm_mod(const LnParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  if (p.d == 1536) {
    launch_rows<3>(p, s);
  } else if (p.d == 5120) {
    launch_rows<10>(p, s);
  } else if (p.d <= 512) {
    const int blocks = (p.M + 7) / 8;
    if (p.out_f32) ln_mod_warp_kernel<true><<<blocks, 256, 0, s>>>(p);
    else ln_mod_warp_kernel<false><<<blocks, 256, 0, s>>>(p);
  } else {
    if (p.out_f32) ln_mod_kernel<true><<<p.M, LN_THREADS, 0, s>>>(p);
    else ln_mod_kernel<false><<<p.M, LN_THREADS, 0, s>>>(p);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Per-head RMSNorm + 3-D rotary positions of q and k, in place.  One block
// per row: each thread owns pairs of channels; pass 1 stores every pair's
// sum of squares in shared memory, pass 2 reduces per head, pass 3 normalises,
// scales by the per-channel weight and rotates each pair by its angle.
// ---------------------------------------------------------------------------
constexpr int RP_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(RP_THREADS) qk_norm_rope_kernel(RopeParams p) {
  extern __shared__ float rp_sm[];  // [d/2] pair sums, then [n_heads] inverse rms
  float* ss = rp_sm;
  float* inv = rp_sm + p.d / 2;
  const int row = blockIdx.x;
  const int half = p.d / 2;               // pairs per part
  const int hp = (p.d / p.n_heads) / 2;   // pairs per head
  const int c = row / p.Lc, t = row - (row / p.Lc) * p.Lc;
  const int f = t / (p.Hq * p.Wq), y = (t / p.Wq) % p.Hq, x = t % p.Wq;
  T* base = (T*)p.qkv + (long long)row * p.ld;
  for (int part = 0; part < 2; ++part) {
    T* v = base + part * p.d;
    for (int i = threadIdx.x; i < half; i += RP_THREADS) {
      const float a = to_f(v[2 * i]), b = to_f(v[2 * i + 1]);
      ss[i] = a * a + b * b;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < p.n_heads; h += RP_THREADS) {
      float acc = 0.0f;
      for (int i = 0; i < hp; ++i) acc += ss[h * hp + i];
      inv[h] = 1.0f / sqrtf(acc / (float)(2 * hp) + 1e-6f);
    }
    __syncthreads();
    const float* w = part ? p.k_w : p.q_w;
    for (int i = threadIdx.x; i < half; i += RP_THREADS) {
      const int h = i / hp, l = i - (i / hp) * hp;
      const float r = inv[h];
      const float a = to_f(v[2 * i]) * r * w[2 * i];
      const float b = to_f(v[2 * i + 1]) * r * w[2 * i + 1];
      float2 cs;
      if (l < p.nt) cs = p.rope_t[(long long)(c * p.Fq + f) * p.nt + l];
      else if (l < p.nt + p.nh) cs = p.rope_y[(long long)y * p.nh + (l - p.nt)];
      else cs = p.rope_x[(long long)x * p.nh + (l - p.nt - p.nh)];
      const T ra = from_f<T>(a * cs.x - b * cs.y);
      const T rb = from_f<T>(a * cs.y + b * cs.x);
      v[2 * i] = ra;
      v[2 * i + 1] = rb;
      if (part == 1 && p.cache && row < p.Lc) {
        T* cr = (T*)p.cache + (long long)row * p.ldc;
        cr[2 * i] = ra;
        cr[2 * i + 1] = rb;
      }
    }
    __syncthreads();
  }
}

cudaError_t qk_norm_rope(const RopeParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  const size_t smem = (size_t)(p.d / 2 + p.n_heads) * sizeof(float);
  if (p.f32) qk_norm_rope_kernel<float><<<p.M, RP_THREADS, smem, s>>>(p);
  else qk_norm_rope_kernel<bf16><<<p.M, RP_THREADS, smem, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Patch gather: ring slot [C][F][H][W] -> token rows [Lc][C*pt*ph*pw].
// One thread per output element; consecutive threads walk the feature index.
// ---------------------------------------------------------------------------
template <typename TO>
__global__ void gather_kernel(const float* __restrict__ ring, long long chunk_numel,
                              const int* __restrict__ chunk_slot, long long total, int Lc,
                              int C, int F, int H, int W, int pt, int ph, int pw, TO* out) {
  const int P = C * pt * ph * pw;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / P;
    const int col = (int)(i - row * P);
    const int c = (int)(row / Lc), t = (int)(row - (long long)c * Lc);
    const int hq = H / ph, wq = W / pw;
    const int fq = t / (hq * wq), rem = t - fq * (hq * wq);
    const int yq = rem / wq, xq = rem - yq * wq;
    const int dx = col % pw, dy = (col / pw) % ph, dt = (col / (pw * ph)) % pt;
    const int cc = col / (pw * ph * pt);
    const long long lat = (((long long)cc * F + fq * pt + dt) * H + yq * ph + dy) * W + xq * pw + dx;
    out[i] = from_f<TO>(ring[(long long)chunk_slot[c] * chunk_numel + lat]);
  }
}

cudaError_t gather_patches(const float* ring, long long chunk_numel, const int* chunk_slot,
                           int n_chunks, int C, int F, int H, int W, int pt, int ph, int pw,
                           void* out, int out_f32, cudaStream_t s) {
  const int Lc = (F / pt) * (H / ph) * (W / pw);
  const long long total = (long long)n_chunks * Lc * C * pt * ph * pw;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  const int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
  if (out_f32)
    gather_kernel<float><<<grid, threads, 0, s>>>(ring, chunk_numel, chunk_slot, total, Lc, C, F,
                                                  H, W, pt, ph, pw, (float*)out);
  else
    gather_kernel<bf16><<<grid, threads, 0, s>>>(ring, chunk_numel, chunk_slot, total, Lc, C, F,
                                                 H, W, pt, ph, pw, (bf16*)out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Sinusoidal features of t_j = 1000 j / T, j = 1..T: [cos(t w_i), sin(t w_i)],
// w_i = 10000^(-i/(D/2)).  Evaluated in double, rounded once to float.
// ---------------------------------------------------------------------------
__global__ void timestep_kernel(int T, int D, float* out) {
  const int j = blockIdx.x + 1;
  const int half = D / 2;
  const double t = 1000.0 * ((double)j / (double)T);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double w = pow(10000.0, -(double)i / (double)half);
    out[(long long)(j - 1) * D + i] = (float)cos(t * w);
    out[(long long)(j - 1) * D + half + i] = (float)sin(t * w);
  }
}

cudaError_t timestep_features(int T, int D, float* out, cudaStream_t s) {
  timestep_kernel<<<T, 128, 0, s>>>(T, D, out);
  return cudaGetLastError();
}

__global__ void add_tables_kernel(const float* m, const float* table, int T, int L, int w,
                                  float* out) {
  const long long total = (long long)T * L * w;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(i % w);
    const long long jl = i / w;
    const int l = (int)(jl % L);
    const int j = (int)(jl / L);
    out[i] = m[(long long)j * w + c] + table[(long long)l * w + c];
  }
}

cudaError_t add_layer_tables(const float* m, const float* table, int T, int L, int w,
                             float* out, cudaStream_t s) {
  add_tables_kernel<<<1024, 256, 0, s>>>(m, table, T, L, w, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Seeded N(0,1): SplitMix64 (Steele, Lea, Flood 2014) stream keyed by
// (seed, a, b) and the Box-Muller transform (1958) in double, as in the
// host-side generator.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long mix64(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void normal_kernel(unsigned long long key, float* out, long long n) {
  const unsigned long long g = 0x9E3779B97F4A7C15ull;
  const long long npairs = (n + 1) / 2;
  for (long long p = blockIdx.x * (long long)blockDim.x + threadIdx.x; p < npairs;
       p += (long long)gridDim.x * blockDim.x) {
    const unsigned long long d0 = mix64(key + (unsigned long long)(2 * p + 1) * g) >> 11;
    const unsigned long long d1 = mix64(key + (unsigned long long)(2 * p + 2) * g) >> 11;
    const double u1 = ((double)d0 + 1.0) * 0x1.0p-53;
    const double u2 = (double)d1 * 0x1.0p-53;
    const double r = sqrt(-2.0 * log(u1));
    const double th = 6.283185307179586476925 * u2;
    out[2 * p] = (float)(r * cos(th));
    if (2 * p + 1 < n) out[2 * p + 1] = (float)(r * sin(th));
  }
}

static unsigned long long host_mix64(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

cudaError_t normal_fill(unsigned long long seed, unsigned long long a, unsigned long long b,
                        float* out, long long n, cudaStream_t s) {
  const unsigned long long g = 0x9E3779B97F4A7C15ull;
  unsigned long long k = host_mix64((seed + 1) * g);
  k = host_mix64(k + (a + 1) * g);
  k = host_mix64(k + (b + 1) * g);
  normal_kernel<<<148 * 4, 256, 0, s>>>(k, out, n);
  return cudaGetLastError();
}

// Coordinated noise: frames of the new chunk gathered from the noise pool.
__global__ void pool_gather_kernel(const float* __restrict__ pool, int C, int F, long long hw,
                                   PoolGather src, float* __restrict__ slot) {
  const long long total = (long long)C * F * hw;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i % hw;
    const int f = (int)((i / hw) % F);
    const int c = (int)(i / (hw * F));
    slot[i] = pool[((long long)src.src[f] * C + c) * hw + e];
  }
}

cudaError_t noise_from_pool(const float* pool, int C, int F, long long hw, PoolGather src,
                            float* slot, cudaStream_t s) {
  pool_gather_kernel<<<148 * 4, 256, 0, s>>>(pool, C, F, hw, src, slot);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Conversions
// ---------------------------------------------------------------------------
__global__ void f32_to_bf16_kernel(const float* in, bf16* out, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(in[i]);
}
__global__ void bf16_to_f32_kernel(const bf16* in, float* out, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = __bfloat162float(in[i]);
}

cudaError_t convert_f32_to_bf16(const float* in, bf16* out, long long n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  f32_to_bf16_kernel<<<148 * 8, 256, 0, s>>>(in, out, n);
  return cudaGetLastError();
}
cudaError_t convert_bf16_to_f32(const bf16* in, float* out, long long n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  bf16_to_f32_kernel<<<148 * 8, 256, 0, s>>>(in, out, n);
  return cudaGetLastError();
}

__global__ void copy_rows_kernel(const void* in, int in_f32, long long ldi, void* out,
                                 int out_f32, long long ldo, long long rows, long long cols) {
  const long long total = rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols, c = i - r * cols;
    const float v = in_f32 ? ((const float*)in)[r * ldi + c]
                           : __bfloat162float(((const bf16*)in)[r * ldi + c]);
    if (out_f32) ((float*)out)[r * ldo + c] = v;
    else ((bf16*)out)[r * ldo + c] = __float2bfloat16_rn(v);
  }
}

cudaError_t copy_rows(const void* in, int in_f32, long long ldi, void* out, int out_f32,
                      long long ldo, long long rows, long long cols, cudaStream_t s) {
  if (rows * cols <= 0) return cudaSuccess;
  copy_rows_kernel<<<148 * 8, 256, 0, s>>>(in, in_f32, ldi, out, out_f32, ldo, rows, cols);
  return cudaGetLastError();
}

}  // namespace dp
