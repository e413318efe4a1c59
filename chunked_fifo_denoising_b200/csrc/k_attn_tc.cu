// tcgen05 flash attention for sm_100a over up to two key buffers per chunk.
//
// DualParal write-up ("双重并行：让AI视频生成突破时长限制…", techwalker.com) §三:
// a chunk's self-attention also reads the K/V of its neighbour, reused from a
// cache rather than recomputed from a concatenated input.  Here the queries of
// chunk c stream the key tiles of the predecessor buffer (chunk c-1's rows of
// this batch, or the persisted K/V for the first chunk) and then of their own
// buffer through one online softmax; the buffers are never concatenated.  The
// same kernel with one shared buffer is the cross-attention to the prompt.
//
// CTA = one 128-query tile of one (chunk, head); 6 warps:
//   warp 0      TMA producer: Q once, then K and V tiles (128 keys) into a
//               2-stage ring, each tile from whichever buffer it belongs to
//   warp 1      TMEM owner + MMA issuer: S_j = Q K_j^T (M=128, N=128, K=hd)
//               into one of two TMEM S buffers, O += P_j V_j (N=hd, K=128)
//   warps 2..5  softmax, thread = query row: S row from TMEM, mask, online
//               max/sum in the log2 domain, P (bf16) into swizzled smem;
//               O is rescaled in TMEM only when a row maximum grows by more
//               than 2^8 (exact: the final division uses the same reference)
// Every mbarrier wait is bounded.
#include <mutex>

#include "tc_common.cuh"

namespace dp {

bool make_tmap_bf16(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
                    int box_rows, int box_cols);

using namespace tc;

namespace {

constexpr int BQ = 128, BKV = 128;

template <int HD>
struct Cfg {
  static constexpr int NSUB = HD / 64;              // 64-column (128-byte) sub-tiles
  static constexpr uint32_t SUB_BYTES = 128 * 128;  // 128 rows x 128 bytes
  static constexpr uint32_t Q_BYTES = NSUB * SUB_BYTES;
  static constexpr uint32_t K_BYTES = NSUB * SUB_BYTES;
  static constexpr uint32_t V_BYTES = NSUB * SUB_BYTES;
  static constexpr uint32_t P_BYTES = 2 * SUB_BYTES;  // 128 queries x 128 keys bf16
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = Q_BYTES;                 // 2 stages
  static constexpr uint32_t OFF_V = OFF_K + 2 * K_BYTES;     // 2 stages
  static constexpr uint32_t OFF_P = OFF_V + 2 * V_BYTES;     // 2 buffers
  static constexpr uint32_t SMEM = OFF_P + 2 * P_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;                 // S0, S1 (128 each), O (hd)
  static constexpr uint32_t O_COL = 256;
};

struct AttnMaps {
  CUtensorMap q, k, v, kp, vp;
};

__device__ __forceinline__ int tile_valid(int j, int tiles_p, int n_p, int n_o) {
  return j < tiles_p ? min(BKV, n_p - j * BKV) : min(BKV, n_o - (j - tiles_p) * BKV);
}

// Warp-uniform bounded wait: TMEM loads and stores that follow are
// warp-collective, so every lane takes the same branch.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  const bool w = mbar_wait(bar, parity, abort, status, ST_TIMEOUT_ATTN);
  return __all_sync(0xffffffffu, w);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) return;
  }
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
attn_tc_kernel(const __grid_constant__ AttnMaps maps, AttnParams p, int* status) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], s_empty[2], p_full[2],
      pv_done[2], done_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, c = blockIdx.z;
  // key sources of this chunk
  int n_p = 0;
  bool pred_cache = false;
  if (c > 0 && p.pred_in_batch) {
    n_p = p.Lk;
  } else if (c == 0 && p.k0_pred != nullptr) {
    n_p = p.Lk_pred;
    pred_cache = true;
  }
  const int n_o = p.Lk;
  const int tiles_p = (n_p + BKV - 1) / BKV;
  const int nt = tiles_p + (n_o + BKV - 1) / BKV;
  const int qrow0 = c * p.Lq + qt * BQ;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const int col0 = h * HD;
      mbar_arrive_expect_tx(&q_full, C::Q_BYTES);
#pragma unroll
      for (int s = 0; s < C::NSUB; ++s)
        tma_load_2d(smem + C::OFF_Q + s * C::SUB_BYTES, &maps.q, col0 + 64 * s, qrow0, &q_full);
      uint32_t issued = 0, issued_par = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j & 1;
        const uint32_t use = (uint32_t)(j >> 1);
        if (use > 0 && !mbar_wait(&kv_empty[st], (use - 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) break;
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        int row;
        if (j < tiles_p) {
          if (pred_cache) {
            mk = &maps.kp;
            mv = &maps.vp;
            row = j * BKV;
          } else {
            mk = &maps.k;
            mv = &maps.v;
            row = (int)((c - 1) * p.kv_chunk_rows) + j * BKV;
          }
        } else {
          mk = &maps.k;
          mv = &maps.v;
          row = (int)(c * p.kv_chunk_rows) + (j - tiles_p) * BKV;
        }
        mbar_arrive_expect_tx(&k_full[st], C::K_BYTES);
#pragma unroll
        for (int s = 0; s < C::NSUB; ++s)
          tma_load_2d(smem + C::OFF_K + st * C::K_BYTES + s * C::SUB_BYTES, mk, col0 + 64 * s, row, &k_full[st]);
        mbar_arrive_expect_tx(&v_full[st], C::V_BYTES);
#pragma unroll
        for (int s = 0; s < C::NSUB; ++s)
          tma_load_2d(smem + C::OFF_V + st * C::V_BYTES + s * C::SUB_BYTES, mv, col0 + 64 * s, row, &v_full[st]);
        issued |= 1u << st;
        issued_par = (issued_par & ~(1u << st)) | ((use & 1u) << st);
      }
      if (abort_flag) {
        drain_wait(&q_full, 0);
        for (int st = 0; st < 2; ++st)
          if (issued & (1u << st)) {
            drain_wait(&k_full[st], (issued_par >> st) & 1u);
            drain_wait(&v_full[st], (issued_par >> st) & 1u);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, HD, 0, 1);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      bool ok = mbar_wait(&q_full, 0, &abort_flag, status, ST_TIMEOUT_ATTN);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_full[st], (j >> 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) return false;
        if (j >= 2 && !mbar_wait(&s_empty[st], ((j >> 1) - 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN))
          return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + C::OFF_K + st * C::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::SUB_BYTES + (kk & 3) * 32;
          mma_bf16_ss(tmem + st * 128, desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024),
                      IDESC_S, kk > 0);
        }
        mma_commit(&s_full[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nt && ok; ++j) {
        if (j + 1 < nt && !issue_s(j + 1)) break;
        const int b = j & 1;
        if (!mbar_wait(&p_full[b], (j >> 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) break;
        if (!mbar_wait(&v_full[b], (j >> 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) break;
        tc_fence_after();
        const uint32_t sP = smem_u32(smem + C::OFF_P + b * C::P_BYTES);
        const uint32_t sV = smem_u32(smem + C::OFF_V + b * C::V_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t ad = desc_sw128(sP + (kk >> 2) * C::SUB_BYTES + (kk & 3) * 32, 16, 1024);
          // V is MN-major: 16 keys = 2 atoms of 8 rows (2048 B); hd groups of 64 are SUB_BYTES apart
          const uint64_t bd = desc_sw128(sV + kk * 2048, C::SUB_BYTES, 1024);
          mma_bf16_ss(tmem + C::O_COL, ad, bd, IDESC_O, (j | kk) != 0);
        }
        mma_commit(&pv_done[b]);
        mma_commit(&kv_empty[b]);
      }
      mma_commit(&done_bar);
      drain_wait(&done_bar, 0);
    }
    __syncwarp();
  } else {
    // ---------------- softmax + output (warps 2..5) ----------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row in the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!warp_wait(&s_full[b], (j >> 1) & 1, &abort_flag, status)) { ok = false; break; }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float t[32];
        tmem_ld32(tmem + lane_off + b * 128 + i * 32, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[i * 32 + e] = t[e];
      }
      tc_fence_before();
      mbar_arrive(&s_empty[b]);
      const int valid = tile_valid(j, tiles_p, n_p, n_o);
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        s[i] = i < valid ? s[i] * sl2 : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float m_new = fmaxf(m, mx);
      const bool want = (m == -INFINITY) || (m_new > m + 8.0f);
      const bool resc = __any_sync(0xffffffffu, want);  // TMEM access is warp-collective
      const float m_use = resc ? m_new : m;
      float sum = 0.0f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        s[i] = exp2f(s[i] - m_use);
        sum += s[i];
      }
      if (j >= 2 && !warp_wait(&pv_done[b], ((j - 2) >> 1) & 1, &abort_flag, status)) {
        ok = false;
        break;
      }
      if (resc && j > 0) {
        if (!warp_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, &abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float corr = exp2f(m - m_use);
        l *= corr;
#pragma unroll 1
        for (int i = 0; i < HD / 32; ++i) {
          float t[32];
          tmem_ld32(tmem + lane_off + C::O_COL + i * 32, t);
#pragma unroll
          for (int e = 0; e < 32; ++e) t[e] *= corr;
          tmem_st32(tmem + lane_off + C::O_COL + i * 32, t);
        }
      }
      l += sum;
      m = m_use;
      // P (bf16) row r into the K-major 128-byte-swizzled tile
      uint8_t* P = smem + C::OFF_P + b * C::P_BYTES;
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 pr = __floats2bfloat162_rn(s[jj * 8 + 2 * e], s[jj * 8 + 2 * e + 1]);
          w[e] = *reinterpret_cast<uint32_t*>(&pr);
        }
        const uint32_t off = (jj >> 3) * C::SUB_BYTES + r * 128 + ((((uint32_t)jj & 7u) ^ ((uint32_t)r & 7u)) << 4);
        *reinterpret_cast<uint4*>(P + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && nt > 0 &&
        warp_wait(&pv_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, &abort_flag, status)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      const bool row_ok = qt * BQ + r < p.Lq;
      bf16* O = (bf16*)p.out + (long long)(qrow0 + r) * p.ldo + h * HD;
#pragma unroll 1
      for (int i = 0; i < HD / 32; ++i) {
        float t[32];
        tmem_ld32(tmem + lane_off + C::O_COL + i * 32, t);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(O + i * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 pr = __floats2bfloat162_rn(t[q4 * 8 + 2 * e] * inv, t[q4 * 8 + 2 * e + 1] * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&pr);
            }
            d4[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<HD>::TMEM_COLS);
  }
}

template <int HD>
cudaError_t launch(const AttnParams& p, int* status, cudaStream_t s) {
  using C = Cfg<HD>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(attn_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int w = p.n_heads * HD;
  AttnMaps maps;
  const long long q_rows = (long long)p.n_chunks * p.Lq;
  const long long kv_rows = p.kv_chunk_rows > 0 ? (long long)p.n_chunks * p.kv_chunk_rows : p.Lk;
  if (!make_tmap_bf16(&maps.q, p.q, q_rows, w, p.ldq, 128, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&maps.k, p.k, kv_rows, w, p.ldkv, 128, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&maps.v, p.v, kv_rows, w, p.ldkv, 128, 64)) return cudaErrorInvalidValue;
  if (p.k0_pred) {
    if (!make_tmap_bf16(&maps.kp, p.k0_pred, p.Lk_pred, w, p.ld_pred, 128, 64)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&maps.vp, p.v0_pred, p.Lk_pred, w, p.ld_pred, 128, 64)) return cudaErrorInvalidValue;
  } else {
    maps.kp = maps.k;
    maps.vp = maps.v;
  }
  dim3 grid((p.Lq + BQ - 1) / BQ, p.n_heads, p.n_chunks);
  if (!status) status = op_status_word();
  attn_tc_kernel<HD><<<grid, 192, C::SMEM, s>>>(maps, p, status);
  return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(const AttnParams& p) {
  if (p.f32 || (p.head_dim != 64 && p.head_dim != 128)) return false;
  const long long w = (long long)p.n_heads * p.head_dim;
  if (p.ldq % 8 || p.ldkv % 8 || p.ldo % 8 || (p.k0_pred && p.ld_pred % 8)) return false;
  if (p.ldq < w || p.ldkv < w || p.ldo < w) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                      reinterpret_cast<uintptr_t>(p.v) | reinterpret_cast<uintptr_t>(p.out) |
                      reinterpret_cast<uintptr_t>(p.k0_pred) | reinterpret_cast<uintptr_t>(p.v0_pred);
  if (a & 15) return false;
  return p.n_chunks <= 65535 && p.n_heads <= 65535 && (long long)p.n_chunks * p.Lq < (1LL << 31);
}

cudaError_t attention_tc(const AttnParams& p, int* status, cudaStream_t s) {
  if (p.n_chunks <= 0 || p.Lq <= 0) return cudaSuccess;
  if (!attention_tc_supported(p)) return cudaErrorInvalidValue;
  return p.head_dim == 128 ? launch<128>(p, status, s) : launch<64>(p, status, s);
}

}  // namespace dp
