// tcgen05 flash attention for sm_100a over up to three key buffers per chunk.
//
// DualParal write-up ("双重并行：让AI视频生成突破时长限制…", techwalker.com) §三:
// a chunk's self-attention also reads the K/V of its neighbour, reused from a
// cache rather than recomputed from a concatenated input.  Here the queries of
// chunk c stream the key tiles of the predecessor buffer (chunk c-1's rows of
// this batch, or the persisted K/V for the first chunk), then of their own
// buffer and, with the bidirectional neighbourhood, of the successor (chunk
// c+1's rows of this batch) through one online softmax; the buffers are never
// concatenated.  The same kernel with one shared buffer is the cross-attention
// to the prompt.
//
// CTA = 256-query blocks (two 128-row tiles A and B each) of one (chunk, head),
// processed one after the other with TMEM and barriers kept (several blocks
// per CTA when the key set is short).  With a long key set, a chunk whose last
// block holds one tile of rows (3120 = 12 x 256 + 48) has the last blocks of
// heads h and h + 1 paired in one CTA as its tiles A and B, each with its own
// head's K/V.  10 warps:
//   warp 0      TMA producer: Q_A, Q_B per block; K and V tiles of 128 keys
//               into two 2-stage rings, each tile from whichever buffer it
//               belongs to
//   warp 1      TMEM owner + MMA issuer, tiles ping-ponged on the tensor core:
//               S_X = Q_X K_j^T (M=128, N=128, K=hd) into TMEM, then
//               O_X += P_X V_j with P_X read from TMEM (the TS form)
//   warps 2..5  softmax of tile A, warps 6..9 softmax of tile B; thread = query
//               row: S row from TMEM, online max/sum in the log2 domain, P as
//               bf16 written back over S in TMEM; O is rescaled in TMEM only when
//               a row maximum grows by more than 2^8 (exact: the final division
//               uses the same reference); O / l leaves through a swizzled 4 KB
//               box per warp and TMA stores that clip at the end of the chunk
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+hd) O_B [256+hd,256+2hd).
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
  static constexpr uint32_t T_BYTES = NSUB * SUB_BYTES;  // one 128-row tile of Q, K or V
  static constexpr uint32_t OFF_QA = 0;
  static constexpr uint32_t OFF_QB = T_BYTES;
  static constexpr uint32_t OFF_K = 2 * T_BYTES;             // 2 stages
  static constexpr uint32_t OFF_V = OFF_K + 2 * T_BYTES;     // 2 stages
  static constexpr uint32_t OFF_STG = OFF_V + 2 * T_BYTES;   // 8 x 4 KB output staging boxes
  static constexpr uint32_t SMEM = OFF_STG + 8 * 4096 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  __device__ static constexpr uint32_t s_col(int X) { return X ? 128u : 0u; }
  __device__ static constexpr uint32_t o_col(int X) { return 256u + (X ? (uint32_t)HD : 0u); }
};

struct AttnMaps {
  CUtensorMap q, k, v, kp, vp;
  CUtensorMap o;  // output as [chunk][row < Lq][column]: boxes clip at the end of each chunk
};

// One row of 64 bf16 (128 bytes, in 32 words) into a 32-row box with the
// 128-byte swizzle of the output tensor map.
__device__ __forceinline__ void stage_row(uint8_t* box, int r, const uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(box + r * 128 + ((j ^ (r & 7)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// 3-D tiled TMA store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int x, int y, int z, const void* smem_src) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(smem_u32(smem_src))
      : "memory");
}

// Key tiles of a chunk: predecessor [0, tp), own [tp, tp+to), successor after.
__device__ __forceinline__ int tile_valid(int j, int tp, int n_p, int to, int n_o, int n_s) {
  if (j < tp) return min(BKV, n_p - j * BKV);
  if (j < tp + to) return min(BKV, n_o - (j - tp) * BKV);
  return min(BKV, n_s - (j - tp - to) * BKV);
}

// Warp-uniform bounded wait: TMEM loads and stores that follow are
// warp-collective, so every lane takes the same branch.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  const bool w = mbar_wait(bar, parity, abort, status, ST_TIMEOUT_ATTN);
  return __all_sync(0xffffffffu, w);
}

// Packed fp32x2 arithmetic of sm_100 (two lanes per instruction, each lane
// rounded as the scalar instruction) and the three-input maximum.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// P = 2^(S * sl2 - m) of one thread's 128-key row of S (MUFU ex2), written
// back over S in TMEM as bf16 pairs; the fp32 values are summed into four
// packed partial sums.
__device__ __forceinline__ void exp_tile(const float (&s)[128], uint64_t sl2x2, uint64_t nmx2, uint32_t tS,
                                         uint64_t (&sp2)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float xa, xb;
      f2_unpack(f2_fma(f2_pack(s[32 * q + 2 * i], s[32 * q + 2 * i + 1]), sl2x2, nmx2), xa, xb);
      const float a = ex2_approx(xa);
      const float b = ex2_approx(xb);
      sp2[i & 3] = f2_add(sp2[i & 3], f2_pack(a, b));
      w[i] = pack_bf16(a, b);
    }
    tmem_st16_nowait(tS + q * 16, w);
  }
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) return;
  }
}

template <int HD>
__global__ void __launch_bounds__(320, 1)
attn_tc_kernel(const __grid_constant__ AttnMaps maps, AttnParams p, int* status) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t q_full, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2],
      p_full[2], pv_done[2], done_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, c = blockIdx.z;
  const int nqb = (p.Lq + 2 * BQ - 1) / (2 * BQ);
  // When the last 256-query block of a chunk holds at most 128 rows (one
  // tile), the last grid column pairs the last blocks of heads h and h + 1
  // (h even) as tiles A and B: each tile reads its own head's K/V, one ring
  // slot per head, and the column of odd h has nothing to do.  The other
  // columns cover blocks [qb0, qb1) of head h, one after the other.
  const bool dual = p.dual_rem && blockIdx.x == gridDim.x - 1;
  if (dual && (h & 1)) return;
  const int hB = dual ? h + 1 : h;  // head of tile B
  const int qb0 = dual ? nqb - 1 : blockIdx.x * p.qblocks_per_cta;
  const int qb1 = dual ? nqb : min(nqb - (p.dual_rem ? 1 : 0), qb0 + p.qblocks_per_cta);
  // key sources of this chunk (the same for every query block)
  int n_p = 0;
  bool pred_cache = false;
  if (c > 0 && p.pred_in_batch) {
    n_p = p.Lk;
  } else if (c == 0 && p.k0_pred != nullptr) {
    n_p = p.Lk_pred;
    pred_cache = true;
  }
  const int n_o = p.Lk;
  const int n_s = (p.succ_in_batch && c + 1 < p.n_chunks) ? p.Lk : 0;
  const int tiles_p = (n_p + BKV - 1) / BKV;
  const int tiles_o = (n_o + BKV - 1) / BKV;
  const int nt = tiles_p + tiles_o + (n_s + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
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
  if (warp == 0 && lane == 0) {  // tensor-map descriptors into the cache before the first copies
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.o);
    if (c == 0) {
      prefetch_tmap(&maps.kp);
      prefetch_tmap(&maps.vp);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const int col0 = h * HD, colB = hB * HD;
      uint32_t issued_k = 0, issued_v = 0, par = 0, q_issued = 0;
      // K/V tiles issued so far: a two-stage ring (stage gk & 1, use gk >> 1);
      // paired heads: one stage holding both heads' tiles (use gk)
      uint32_t gk = 0;
      bool ok = true;
      for (int qb = qb0; qb < qb1 && ok; ++qb) {
        const int bi = qb - qb0;
        const int q0 = qb * 2 * BQ;
        const bool has_b = dual || q0 + BQ < p.Lq;
        const int qrow0 = c * p.Lq + q0;
        const int qrowB = dual ? qrow0 : qrow0 + BQ;
        // Q of the previous block is read by its S MMAs only
        if (bi > 0 && !mbar_wait(&q_empty, (bi - 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) break;
        mbar_arrive_expect_tx(&q_full, (has_b ? 2 : 1) * C::T_BYTES);
#pragma unroll
        for (int s = 0; s < C::NSUB; ++s) {
          tma_load_2d(smem + C::OFF_QA + s * C::SUB_BYTES, &maps.q, col0 + 64 * s, qrow0, &q_full);
          if (has_b) tma_load_2d(smem + C::OFF_QB + s * C::SUB_BYTES, &maps.q, colB + 64 * s, qrowB, &q_full);
        }
        q_issued = bi + 1;
        for (int j = 0; j < nt; ++j, ++gk) {
          const int st = dual ? 0 : (int)(gk & 1);
          const uint32_t use = dual ? gk : gk >> 1;
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
          } else if (j < tiles_p + tiles_o) {
            mk = &maps.k;
            mv = &maps.v;
            row = (int)(c * p.kv_chunk_rows) + (j - tiles_p) * BKV;
          } else {  // successor: chunk c+1's own rows of this batch
            mk = &maps.k;
            mv = &maps.v;
            row = (int)((c + 1) * p.kv_chunk_rows) + (j - tiles_p - tiles_o) * BKV;
          }
          if (use > 0 && !mbar_wait(&k_empty[st], (use - 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[st], (dual ? 2 : 1) * C::T_BYTES);
#pragma unroll
          for (int s = 0; s < C::NSUB; ++s) {
            tma_load_2d(smem + C::OFF_K + st * C::T_BYTES + s * C::SUB_BYTES, mk, col0 + 64 * s, row, &k_full[st]);
            if (dual) tma_load_2d(smem + C::OFF_K + C::T_BYTES + s * C::SUB_BYTES, mk, colB + 64 * s, row, &k_full[st]);
          }
          issued_k |= 1u << st;
          par = (par & ~(1u << st)) | ((use & 1u) << st);
          if (use > 0 && !mbar_wait(&v_empty[st], (use - 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[st], (dual ? 2 : 1) * C::T_BYTES);
#pragma unroll
          for (int s = 0; s < C::NSUB; ++s) {
            tma_load_2d(smem + C::OFF_V + st * C::T_BYTES + s * C::SUB_BYTES, mv, col0 + 64 * s, row, &v_full[st]);
            if (dual) tma_load_2d(smem + C::OFF_V + C::T_BYTES + s * C::SUB_BYTES, mv, colB + 64 * s, row, &v_full[st]);
          }
          issued_v |= 1u << st;
        }
      }
      if (abort_flag) {  // let copies in flight land before the CTA exits
        if (q_issued > 0) drain_wait(&q_full, (q_issued - 1) & 1);
        for (int st = 0; st < 2; ++st) {
          if (issued_k & (1u << st)) drain_wait(&k_full[st], (par >> st) & 1u);
          if (issued_v & (1u << st)) drain_wait(&v_full[st], (par >> st) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, HD, 0, 1);
      // ring stage and phase of K/V tile g; with paired heads one stage holds
      // both heads' tiles (slot X) and its phase flips every tile
      auto kv_st = [&](uint32_t g) -> int { return dual ? 0 : (int)(g & 1); };
      auto kv_par = [&](uint32_t g) -> uint32_t { return dual ? (g & 1) : ((g >> 1) & 1); };
      auto kv_slot = [&](int X, uint32_t g) -> uint32_t { return dual ? (uint32_t)X : (g & 1); };
      // descriptors are built once per operand tile; a K step of 16 columns
      // adds 32 bytes (2 in the 16-byte address field), a 64-column sub-tile
      // SUB_BYTES, 16 rows of V 2048 bytes (the field stays below 2^14)
      auto issue_s = [&](int X, uint32_t g) {
        const uint64_t dq = desc_sw128(smem_u32(smem + (X ? C::OFF_QB : C::OFF_QA)), 16, 1024);
        const uint64_t dk = desc_sw128(smem_u32(smem + C::OFF_K + kv_slot(X, g) * C::T_BYTES), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * C::SUB_BYTES + (kk & 3) * 32) >> 4);
          mma_bf16_ss(tmem + C::s_col(X), dq + off, dk + off, IDESC_S, kk > 0);
        }
        mma_commit(&s_full[X]);
      };
      auto issue_pv = [&](int X, uint32_t g, int j) {
        const uint64_t dv = desc_sw128(smem_u32(smem + C::OFF_V + kv_slot(X, g) * C::T_BYTES), C::SUB_BYTES, 1024);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)  // 16 keys = 8 TMEM columns of packed P; 2 atoms of V
          mma_bf16_ts(tmem + C::o_col(X), tmem + C::s_col(X) + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), IDESC_O,
                      (j | kk) != 0);
        mma_commit(&pv_done[X]);
      };
      uint32_t gk = 0;          // K/V tiles consumed so far
      uint32_t gp[2] = {0, 0};  // P tiles of tile A / tile B consumed so far
      bool ok = true;
      // The first S of a block is issued at the end of the previous block,
      // right after that block's last PV of tile A, so the tensor core has work
      // while the softmax warps finish the last tile (several blocks per CTA).
      bool first_issued = false;
      for (int qb = qb0; qb < qb1 && ok; ++qb) {
        const int bi = qb - qb0;
        const bool has_b = dual || qb * 2 * BQ + BQ < p.Lq;
        if (!first_issued) {
          ok = mbar_wait(&q_full, bi & 1, &abort_flag, status, ST_TIMEOUT_ATTN) &&
               mbar_wait(&k_full[kv_st(gk)], kv_par(gk), &abort_flag, status, ST_TIMEOUT_ATTN);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, gk);
          if (has_b) issue_s(1, gk);
          mma_commit(&k_empty[kv_st(gk)]);
          if (nt == 1) mma_commit(&q_empty);  // last S of this block issued
        }
        first_issued = false;
        const bool more = qb + 1 < qb1;
        const bool next_has_b = (qb + 1) * 2 * BQ + BQ < p.Lq;
        for (int j = 0; j < nt; ++j) {
          const uint32_t g = gk + j;
          const bool next = j + 1 < nt;
          if (!mbar_wait(&v_full[kv_st(g)], kv_par(g), &abort_flag, status, ST_TIMEOUT_ATTN) ||
              !mbar_wait(&p_full[0], gp[0] & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(0, g, j);
          ++gp[0];
          if (next) {
            if (!mbar_wait(&k_full[kv_st(g + 1)], kv_par(g + 1), &abort_flag, status, ST_TIMEOUT_ATTN)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(0, g + 1);
          } else if (more) {
            // the next block's Q (loaded once this block's last S was issued)
            // and its first key tile
            if (!mbar_wait(&q_full, (bi + 1) & 1, &abort_flag, status, ST_TIMEOUT_ATTN) ||
                !mbar_wait(&k_full[kv_st(g + 1)], kv_par(g + 1), &abort_flag, status, ST_TIMEOUT_ATTN)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(0, g + 1);
          }
          if (has_b) {
            if (!mbar_wait(&p_full[1], gp[1] & 1, &abort_flag, status, ST_TIMEOUT_ATTN)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(1, g, j);
            ++gp[1];
          }
          mma_commit(&v_empty[kv_st(g)]);
          if (next) {
            if (has_b) issue_s(1, g + 1);
            mma_commit(&k_empty[kv_st(g + 1)]);
            if (j + 2 == nt) mma_commit(&q_empty);  // last S of this block issued
          } else if (more) {
            if (next_has_b) issue_s(1, g + 1);
            mma_commit(&k_empty[kv_st(g + 1)]);
            if (nt == 1) mma_commit(&q_empty);    // last S of the next block issued
            first_issued = true;
          }
        }
        gk += nt;
      }
      mma_commit(&done_bar);
      drain_wait(&done_bar, 0);
    }
    __syncwarp();
  } else {
    // ---------------- softmax + output (warps 2..9) ----------------
    const int X = warp >= 6 ? 1 : 0;
    const int quad = warp & 3;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::s_col(X);
    const uint32_t tO = tmem + lane_off + C::o_col(X);
    uint8_t* box = smem + C::OFF_STG + (warp - 2) * 4096;
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(hd)
    uint32_t gx = 0;  // tiles of this X processed so far (phases of s_full / p_full / pv_done)
    bool ok = true;
    for (int qb = qb0; qb < qb1 && ok; ++qb) {
      const int q0 = qb * 2 * BQ;
      if (X == 1 && !dual && !(q0 + BQ < p.Lq)) continue;  // this block has no tile B
      float m = -INFINITY, l = 0.0f;
      for (int j = 0; j < nt; ++j, ++gx) {
        if (!warp_wait(&s_full[X], gx & 1, &abort_flag, status)) { ok = false; break; }
        tc_fence_after();
        float s[128];
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld32_nowait(tS + i * 32, *reinterpret_cast<float(*)[32]>(s + i * 32));
        tmem_wait_ld();
        const int valid = tile_valid(j, tiles_p, n_p, tiles_o, n_o, n_s);
        if (valid < BKV) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= valid) s[i] = -INFINITY;
        }
        // row maximum with 8 independent partial maxima (short dependency chains)
        float mxp[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mxp[i] = s[i];
#pragma unroll
        for (int i = 8; i < 128; i += 2) mxp[(i >> 1) & 7] = max3f(mxp[(i >> 1) & 7], s[i], s[i + 1]);
        const float mx = fmaxf(max3f(mxp[0], mxp[1], mxp[2]),
                               fmaxf(max3f(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
        const float m_new = fmaxf(m, mx * sl2);
        const bool want = (m == -INFINITY) || (m_new > m + 8.0f);
        const bool resc = __any_sync(0xffffffffu, want);  // TMEM access is warp-collective
        const float m_use = resc ? m_new : m;
        const float nm = -m_use;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nmx2 = f2_pack(nm, nm);
        uint64_t sp2[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial row sums
        // P (bf16, two keys per 32-bit column) over the first 64 columns of S, 32
        // keys at a time; S is already in registers, and PV of the previous tile
        // (which read the old P) completed before S of this tile was written
        exp_tile(s, sl2x2, nmx2, tS, sp2);
        tmem_wait_st();
        if (resc && j > 0) {
          // O must hold PV of every earlier tile of this block before it is rescaled
          if (!warp_wait(&pv_done[X], (gx - 1) & 1, &abort_flag, status)) { ok = false; break; }
          tc_fence_after();
          const float corr = ex2_approx(m - m_use);
          l *= corr;
#pragma unroll 1
          for (int i = 0; i < HD / 32; ++i) {
            float t[32];
            tmem_ld32(tO + i * 32, t);
#pragma unroll
            for (int e = 0; e < 32; ++e) t[e] *= corr;
            tmem_st32(tO + i * 32, t);
          }
        }
        {
          float t0, t1;
          f2_unpack(f2_add(f2_add(sp2[0], sp2[1]), f2_add(sp2[2], sp2[3])), t0, t1);
          l += t0 + t1;
        }
        m = m_use;
        tc_fence_before();
        mbar_arrive(&p_full[X]);
      }
      if (!ok || nt == 0) break;
      if (!warp_wait(&pv_done[X], (gx - 1) & 1, &abort_flag, status)) { ok = false; break; }
      tc_fence_after();
      const float inv = 1.0f / l;
      // O / l as bf16, 64 columns at a time, through this warp's swizzled 32-row
      // box and a TMA store: whole 128-byte row segments instead of one row per
      // thread.  Rows at or past Lq fall outside the chunk in the output map and
      // are not written.  Tile B holds the next query rows, or (paired heads)
      // the same rows of head hB.
      const int y0 = q0 + (dual ? 0 : X * BQ) + quad * 32;
      const int x0 = (X ? hB : h) * HD;
#pragma unroll 1
      for (int i = 0; i < HD / 64; ++i) {
        float t[64];
        tmem_ld32_nowait(tO + i * 64, *reinterpret_cast<float(*)[32]>(t));
        tmem_ld32_nowait(tO + i * 64 + 32, *reinterpret_cast<float(*)[32]>(t + 32));
        tmem_wait_ld();
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = pack_bf16(t[2 * e] * inv, t[2 * e + 1] * inv);
        if (lane == 0) bulk_wait_read<0>();  // the previous store has read the box
        __syncwarp();
        stage_row(box, lane, w);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&maps.o, x0 + 64 * i, y0, c, box);
          bulk_commit();
        }
      }
      // the next block's PV overwrites O only after this thread's next P arrives
      tc_fence_before();
    }
    if (lane == 0) bulk_wait_all();  // output stores have landed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<HD>::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn3)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The bf16 output as a 3-D tensor [n_chunks][Lq][cols] (row stride ld
// elements), boxes of 32 rows x 64 columns of one chunk, 128-byte swizzle.
bool make_out_map(CUtensorMap* map, void* base, int n_chunks, int Lq, long long cols, long long ld) {
  static EncodeTiledFn3 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn3>(f);
  });
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)Lq, (cuuint64_t)n_chunks};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)Lq * (cuuint64_t)ld * 2};
  cuuint32_t box[3] = {64, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch(const AttnParams& p, int* status, cudaStream_t s) {
  using C = Cfg<HD>;
  // the shared-memory opt-in is a per-device attribute of the function
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    err = cudaFuncSetAttribute(attn_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (err != cudaSuccess) return err;
    done[dev] = true;
  }
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
  if (!make_out_map(&maps.o, p.out, p.n_chunks, p.Lq, w, p.ldo)) return cudaErrorInvalidValue;
  // query blocks of 256 per CTA: more when the key set is short (the setup of
  // a CTA, its Q loads and its O write-back are then amortised over more work)
  const long long keys = (long long)p.Lk * (1 + (p.pred_in_batch ? 1 : 0) + (p.succ_in_batch ? 1 : 0));
  AttnParams q = p;
  q.qblocks_per_cta = p.qblocks_per_cta > 0 ? p.qblocks_per_cta : (keys <= 1024 ? 5 : 1);
  const int nqb = (p.Lq + 2 * BQ - 1) / (2 * BQ);
  // A last block of one tile (Lq mod 256 in 1..128) costs a full block's
  // time for at most half its rows: pair the heads' last blocks in one column.
  // Only for long key sets (one block per CTA, self-attention): a paired block
  // has one K/V ring stage per head, which a short key set cannot hide
  // (cross-attention with 512 keys measured 6 % slower paired).
  const int last_rows = p.Lq - (nqb - 1) * 2 * BQ;
  q.dual_rem = (last_rows <= BQ && p.n_heads % 2 == 0 && q.qblocks_per_cta == 1) ? 1 : 0;
  const int main_blocks = nqb - q.dual_rem;
  dim3 grid((main_blocks + q.qblocks_per_cta - 1) / q.qblocks_per_cta + q.dual_rem, p.n_heads, p.n_chunks);
  if (!status) status = op_status_word();
  attn_tc_kernel<HD><<<grid, 320, C::SMEM, s>>>(maps, q, status);
  return cudaGetLastError();
}

}  // namespace

// One bounded wait on an mbarrier that nothing arrives at: exercises the
// give-up path of the tensor-core kernels (status word set, clean exit).
__global__ void selftest_timeout_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, ST_TIMEOUT_ATTN);
  __syncthreads();
}

cudaError_t selftest_timeout(int* status, cudaStream_t s) {
  if (!status) status = op_status_word();
  if (!status) return cudaErrorInvalidValue;
  selftest_timeout_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

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
