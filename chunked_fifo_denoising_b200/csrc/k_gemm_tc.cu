// Persistent tcgen05 GEMM for sm_100a: C = A[M][K] . W[N][K]^T with the fused
// epilogues of the DiT block (bias; bias+GELU; gated or plain residual add into
// the fp32 stream; bias + copy of the neighbour-cache columns; the head's
// Euler scatter into the latent ring).
//
// Layout: 128 x BN output tiles.  A ring stage holds KSUB sub-tiles of 64 K
// columns (one 128-byte swizzled row per operand row each).  One CTA per SM,
// 10 warps:
//   warp 0      TMA producer (one thread): A and W tiles into a STAGES-deep ring
//   warp 1      TMEM owner + MMA issuer (one thread): 4 x KSUB tcgen05.mma
//               (M=128, N=BN, K=16) per stage into one of two TMEM accumulators
//   warps 2..9  epilogue, two warps per TMEM lane quarter (each half of the
//               columns): tcgen05.ld of accumulator rows (thread = row), fused
//               epilogue into a 128-byte-swizzled smem box, TMA store or TMA
//               reduce-add; frees the accumulator so the next tile's MMAs
//               overlap this tile's epilogue.
// Tiles are walked row-block-major so the CTAs in flight share A row blocks
// through L2 while W stays L2-resident.  Every mbarrier wait is bounded.
//
// Pair mode (PAIR, N a multiple of 256): clusters of two CTAs on two SMs
// compute 256 x 256 tiles with tcgen05.mma.cta_group::2 (M = 256).  Each CTA
// loads its own 128 rows of A and 128 of the 256 rows of W, so an SM streams
// 64 instead of 96 bytes of operands per 8192 MMA FLOP.  The first CTA of the
// pair waits for both CTAs' loads on its own full barriers, issues the MMAs
// and commits them to the empty and accumulator barriers of both CTAs; each
// CTA runs the epilogue of its own 128 rows from its own tensor memory and
// releases the accumulator to the first CTA.  No load is multicast.  Pairs use
// stages of 128 K columns (KSUB = 2, three stages) when K allows: with half as
// many stage hand-offs per FLOP the K = 1536 GEMMs ran 5-7 % faster than with
// six 64-column stages.
#include <cstring>
#include <mutex>

#include "tc_common.cuh"

namespace dp {

using namespace tc;

namespace {

constexpr int BM = 128, BK = 64;

// Bias (and activation) for `n` consecutive columns starting at col0; columns
// at or beyond N read no bias.
template <int NV>
__device__ __forceinline__ void add_bias(const EpiParams& e, int col0, int N, float (&v)[NV]) {
  if (!e.bias) return;
#pragma unroll
  for (int i = 0; i < NV / 4; ++i) {
    if (col0 + 4 * i < N) {
      const float4 b = reinterpret_cast<const float4*>(e.bias + col0)[i];
      v[4 * i] += b.x;
      v[4 * i + 1] += b.y;
      v[4 * i + 2] += b.z;
      v[4 * i + 3] += b.w;
    }
  }
}

// One 128-byte row (8 chunks of 16 bytes) of a 128-byte-swizzled staging box:
// chunk j of row r lives at chunk position j ^ (r % 8), so the 8 rows a
// quarter-warp writes at once fall in distinct banks.
__device__ __forceinline__ void stage_row(uint8_t* box, int r, const uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(box + r * 128 + ((j ^ (r & 7)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) return;
  }
}

struct GemmMaps {
  CUtensorMap a, b;    // operands
  CUtensorMap out;     // STORE/GELU output (bf16 box 64x32 or fp32 box 32x32)
  CUtensorMap res;     // fp32 residual stream for the reduce-add epilogues
};

template <int BN, int STAGES, bool PAIR, int KSUB>
__global__ void __launch_bounds__(320, 1)
gemm_tc_kernel(const __grid_constant__ GemmMaps maps, int M, int N, int K, EpiParams e, int* status) {
  constexpr int BNL = PAIR ? BN / 2 : BN;  // rows of W this CTA loads per tile
  constexpr int TM = PAIR ? 2 * BM : BM;   // rows of an output tile
  constexpr uint32_t A_SUB = BM * BK * 2, B_SUB = BNL * BK * 2;  // one 64-column sub-tile
  constexpr uint32_t A_BYTES = A_SUB * KSUB;
  constexpr uint32_t B_BYTES = B_SUB * KSUB;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t STG_OFF = STAGES * STAGE_BYTES;  // 8 warps x one 4 KB staging box
  // columns per epilogue warp; with BN = 64 the second warp group has no columns
  // and only keeps in step with the accumulator barriers
  constexpr int HALF = BN >= 128 ? BN / 2 : BN;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16_f32(TM, BN, 0, 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES], tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pair mode: CTA `rank` of the pair owns rows rank*128.. of every tile; the
  // pairs walk the tiles together
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int tiles_n = (N + BN - 1) / BN;
  const int tiles_m = (M + TM - 1) / TM;
  const int num_tiles = tiles_n * tiles_m;
  const int kblocks = K / (BK * KSUB);  // ring stages per tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], PAIR ? 16 : 256);  // pair: one arrival per epilogue warp of each CTA
    }
    mbar_init(&done_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(&tmem_base_sh, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&tmem_base_sh, TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.b);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_par = 0;  // per-stage bit masks for the drain
      bool ok = true;
      for (int t = unit0; t < num_tiles && ok; t += units) {
        const int m0 = (t / tiles_n) * TM + (int)rank * BM, n0 = (t % tiles_n) * BN + (int)rank * BNL;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, status, ST_TIMEOUT_GEMM)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          if (PAIR) {
            // both CTAs' bytes land on the first CTA's full barrier
            if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * STAGE_BYTES);
            const uint32_t fb = cluster_addr(&full_bar[stage], 0);
            for (int q = 0; q < KSUB; ++q) {
              tma_load_2d_pair(sa + q * A_SUB, &maps.a, (kb * KSUB + q) * BK, m0, fb);
              tma_load_2d_pair(sa + A_BYTES + q * B_SUB, &maps.b, (kb * KSUB + q) * BK, n0, fb);
            }
          } else {
            mbar_arrive_expect_tx(&full_bar[stage], STAGE_BYTES);
            for (int q = 0; q < KSUB; ++q) {
              tma_load_2d(sa + q * A_SUB, &maps.a, (kb * KSUB + q) * BK, m0, &full_bar[stage]);
              tma_load_2d(sa + A_BYTES + q * B_SUB, &maps.b, (kb * KSUB + q) * BK, n0, &full_bar[stage]);
            }
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // the second CTA of a pair cannot see its copies complete (they count on
      // the first CTA's barriers): after a give-up it lets them settle for 1 ms
      if (abort_flag && !leader && issued) {
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 1000000ull) {
        }
      }
      if (abort_flag && leader) {  // let copies in flight land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) drain_wait(&full_bar[s], (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the first CTA of a pair) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = unit0; t < num_tiles && ok; t += units, ++it) {
        const int buf = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[buf], acc_phase ^ 1, &abort_flag, status, ST_TIMEOUT_GEMM)) break;
        tc_fence_after();
        const uint32_t dtm = tmem_base + buf * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status, ST_TIMEOUT_GEMM)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
#pragma unroll
          for (int q = 0; q < KSUB; ++q) {
            const uint64_t ad = desc_sw128(sa + q * A_SUB, 16, 1024);
            const uint64_t bd = desc_sw128(sa + A_BYTES + q * B_SUB, 16, 1024);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {  // +32 bytes along K per step = +2 in the address field
              if (PAIR) mma_bf16_ss_pair(dtm, ad + 2 * k, bd + 2 * k, IDESC, (kb | q | k) != 0);
              else mma_bf16_ss(dtm, ad + 2 * k, bd + 2 * k, IDESC, (kb | q | k) != 0);
            }
          }
          if (PAIR) {
            mma_commit_pair_both(&empty_bar[stage]);
          } else {
            mma_commit(&empty_bar[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) {
          if (PAIR) {
            mma_commit_pair_both(&tfull_bar[buf]);
          } else {
            mma_commit(&tfull_bar[buf]);
          }
        }
      }
      if (PAIR) mma_commit_pair(&done_bar);
      else mma_commit(&done_bar);
      drain_wait(&done_bar, 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    // warps w and w+4 share TMEM lanes 32*(w%4).. and split the tile's columns
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int half = (warp - 2) >> 2;
    uint8_t* box = smem + STG_OFF + (warp - 2) * 4096;
    const bool bf16_out = (e.mode == EPI_STORE && !e.out_f32) || e.mode == EPI_GELU;
    const bool reduce = e.mode == EPI_RESID || e.mode == EPI_RESID_GATED;
    // hands accumulator buffer `b` back to the MMA warp once this warp's TMEM
    // loads of it are complete
    auto release_acc = [&](int b) {
      tc_fence_before();
      if (PAIR) {
        __syncwarp();  // every lane's accumulator loads are complete
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&tempty_bar[b], 0));
      } else {
        mbar_arrive(&tempty_bar[b]);
      }
    };
    int it = 0;
    for (int t = unit0; t < num_tiles; t += units, ++it) {
      const int buf = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // warp-uniform: the TMEM loads below are warp-collective
      const bool waited = mbar_wait(&tfull_bar[buf], acc_phase, &abort_flag, status, ST_TIMEOUT_GEMM);
      if (!__all_sync(0xffffffffu, waited)) break;
      tc_fence_after();
      const int m0 = (t / tiles_n) * TM + (int)rank * BM, n0 = (t % tiles_n) * BN + half * HALF;
      const int row_base = m0 + quad * 32;
      const int row = row_base + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * BN + half * HALF;
      bool released = false;  // accumulator buffer handed back to the MMA warp
      if (half * HALF >= BN) {
        // no columns for this warp group
      } else if (e.rope && n0 < 2 * e.rope_d) {
        // q or k heads: per-head RMSNorm and rotary positions, head by head
        const int hd = e.rope_hd;
        const int grow = row < M ? row : M - 1;  // keep table lookups in range
        const int ci = grow / e.rows_per_chunk, tk = grow - ci * e.rows_per_chunk;
        const int fr = tk / (e.rope_Hq * e.rope_Wq);
        const int py = (tk / e.rope_Wq) % e.rope_Hq, px = tk % e.rope_Wq;
        const float2* tt = e.rope_t + (long long)(ci * e.rope_Fq + fr) * e.rope_nt;
        const float2* ty = e.rope_y + (long long)py * e.rope_nh;
        const float2* tx = e.rope_x + (long long)px * e.rope_nh;
#pragma unroll 1
        for (int hb = 0; hb < HALF / hd; ++hb) {
          const int colh = n0 + hb * hd;
          const int part = colh >= e.rope_d;
          const float* wn = (part ? e.k_w : e.q_w) + (colh - part * e.rope_d);
          // pass 1: sum of squares of the head's biased values
          float ss = 0.0f;
#pragma unroll 1
          for (int i = 0; i < hd / 32; ++i) {
            float v[32];
            tmem_ld32(tbase + hb * hd + i * 32, v);
            add_bias<32>(e, colh + i * 32, N, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) ss = fmaf(v[k], v[k], ss);
          }
          const float inv = 1.0f / sqrtf(ss / (float)hd + 1e-6f);
          // pass 2: normalise, scale, rotate each pair, store 64 columns at a time
#pragma unroll 1
          for (int g = 0; g < hd / 64; ++g) {
            const int col0 = colh + g * 64;
            float v[64];
            float* v0 = v;
            tmem_ld32(tbase + hb * hd + g * 64, *reinterpret_cast<float(*)[32]>(v0));
            tmem_ld32(tbase + hb * hd + g * 64 + 32, *reinterpret_cast<float(*)[32]>(v0 + 32));
            add_bias<64>(e, col0, N, v);
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int l = g * 32 + j;  // pair index within the head
              const float a = v[2 * j] * inv * wn[g * 64 + 2 * j];
              const float b = v[2 * j + 1] * inv * wn[g * 64 + 2 * j + 1];
              float2 cs;
              if (l < e.rope_nt) cs = tt[l];
              else if (l < e.rope_nt + e.rope_nh) cs = ty[l - e.rope_nt];
              else cs = tx[l - e.rope_nt - e.rope_nh];
              w[j] = pack_bf16(a * cs.x - b * cs.y, a * cs.y + b * cs.x);
            }
            if (e.cache && row < M && row >= e.cache_row0 && row < e.cache_row0 + e.cache_rows &&
                col0 >= e.cache_col0) {
              uint4* d = reinterpret_cast<uint4*>((bf16*)e.cache + (long long)(row - e.cache_row0) * e.ldc +
                                                  (col0 - e.cache_col0));
              for (int j = 0; j < 8; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            }
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            stage_row(box, lane, w);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&maps.out, col0, row_base, box);
              bulk_commit();
            }
          }
        }
      } else if (bf16_out) {
        // bias (+ GELU), bf16, optional cache copy, one TMA store of 64 columns
        auto convert_store = [&](int col0, float (&v)[64]) {
          add_bias<64>(e, col0, N, v);
          uint32_t w[32];
          if (e.mode == EPI_GELU) {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = gelu2_bf16(v[2 * i], v[2 * i + 1]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
          }
          if (e.cache && row < M && row >= e.cache_row0 && row < e.cache_row0 + e.cache_rows &&
              col0 >= e.cache_col0) {
            uint4* d = reinterpret_cast<uint4*>((bf16*)e.cache + (long long)(row - e.cache_row0) * e.ldc +
                                                (col0 - e.cache_col0));
            const int nchunk = min(8, (N - col0) / 8);
            for (int j = 0; j < nchunk; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
          if (lane == 0) bulk_wait_read<0>();  // the previous store has read the box
          __syncwarp();
          stage_row(box, lane, w);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&maps.out, col0, row_base, box);
            bulk_commit();
          }
        };
        // The accumulator goes back to the MMA warp as soon as this warp's
        // last column group is in registers; that group's conversion and
        // store run after the release (the GELU epilogue held the accumulator
        // for most of a tile's MMA time).
        float v[64];
        tmem_ld32(tbase, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(tbase + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        if (HALF / 64 == 2 && n0 + 64 < N) {
          convert_store(n0, v);
          tmem_ld32(tbase + 64, *reinterpret_cast<float(*)[32]>(v));
          tmem_ld32(tbase + 96, *reinterpret_cast<float(*)[32]>(v + 32));
          release_acc(buf);
          released = true;
          convert_store(n0 + 64, v);
        } else {
          release_acc(buf);
          released = true;
          convert_store(n0, v);
        }
      } else if (e.mode == EPI_EULER) {
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + c * 32, v);
          const int col0 = n0 + c * 32;
          if (row < M && col0 < N) {
            add_bias<32>(e, col0, N, v);
            const float ds = e.dsig[row / e.rows_per_chunk];
            for (int i = 0; i < 32; ++i) e.ring[euler_index(e, row, col0 + i, e.rows_per_chunk)] += ds * v[i];
          }
        }
      } else {
        // fp32 results: plain store (residual stream init) or reduce-add into it
        const int grow = row < M ? row : M - 1;  // rows past M are clipped by TMA; keep lookups in range
        const float* gate = nullptr;
        if (e.mode == EPI_RESID_GATED) {
          const int c = grow / e.rows_per_chunk;
          const long long sel = e.chunk_sel ? e.chunk_sel[c] : c;
          gate = e.gate + sel * e.gate_stride;
        }
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          const int col0 = n0 + c * 32;
          if (col0 >= N) break;  // uniform
          // gate loads first: their latency overlaps the TMEM load
          float4 gg[8];
          if (gate) {
#pragma unroll
            for (int i = 0; i < 8; ++i) gg[i] = reinterpret_cast<const float4*>(gate + col0)[i];
          }
          float v[32];
          tmem_ld32(tbase + c * 32, v);
          add_bias<32>(e, col0, N, v);
          if (gate) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[4 * i] *= gg[i].x;
              v[4 * i + 1] *= gg[i].y;
              v[4 * i + 2] *= gg[i].z;
              v[4 * i + 3] *= gg[i].w;
            }
          }
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i]);
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          stage_row(box, lane, w);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (reduce) tma_reduce_add_2d(&maps.res, col0, row_base, box);
            else tma_store_2d(&maps.out, col0, row_base, box);
            bulk_commit();
          }
        }
      }
      if (!released) release_acc(buf);
    }
    if (lane == 0) bulk_wait_all();  // stores and reductions have landed
  }
  tc_fence_before();
  __syncthreads();
  // pair: neither CTA frees tensor memory or leaves while the other may still
  // signal its barriers or the MMAs may still read its shared memory
  if (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (PAIR) cluster_sync();
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

// Row-major [rows][cols] (row stride `ld` elements) of bf16 or fp32, boxes of
// box_rows x box_cols with the 128-byte swizzle (box_cols * element = 128 B).
static bool make_tmap(CUtensorMap* map, bool f32, const void* base, long long rows, long long cols,
                      long long ld, int box_rows, int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * es};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 [rows][cols] row-major with row stride `ld` elements; box box_rows x 64.
bool make_tmap_bf16(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
                    int box_rows, int box_cols) {
  return make_tmap(map, false, base, rows, cols, ld, box_rows, box_cols);
}

bool gemm_tc_supported(long long lda, int M, int N, int K) {
  return M > 0 && N > 0 && K > 0 && K % BK == 0 && N % 32 == 0 && lda % 8 == 0 && lda >= K;
}

template <int BN, int STAGES, bool PAIR, int KSUB>
static cudaError_t launch_tc(const bf16* A, long long lda, const bf16* W, int M, int N, int K,
                             const EpiParams& e, int* status, cudaStream_t s) {
  constexpr int BNL = PAIR ? BN / 2 : BN;
  constexpr int TM = PAIR ? 2 * BM : BM;
  constexpr int SMEM = STAGES * KSUB * (BM * BK * 2 + BNL * BK * 2) + 8 * 4096 + 1024;
  // the shared-memory opt-in is a per-device attribute of the function
  static bool done[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    err = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES, PAIR, KSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM);
    if (err != cudaSuccess) return err;
    done[dev] = true;
  }
  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_tmap(&maps.a, false, A, M, K, lda, BM, BK)) return cudaErrorInvalidValue;
  if (!make_tmap(&maps.b, false, W, N, K, K, BNL, BK)) return cudaErrorInvalidValue;
  if (e.mode == EPI_GELU || (e.mode == EPI_STORE && !e.out_f32)) {
    if (!make_tmap(&maps.out, false, e.out, M, N, e.ldo, 32, 64)) return cudaErrorInvalidValue;
  } else if (e.mode == EPI_STORE) {
    if (!make_tmap(&maps.out, true, e.out, M, N, e.ldo, 32, 32)) return cudaErrorInvalidValue;
  } else if (e.mode == EPI_RESID || e.mode == EPI_RESID_GATED) {
    if (!make_tmap(&maps.res, true, e.resid, M, N, e.ldr, 32, 32)) return cudaErrorInvalidValue;
  } else if (e.mode != EPI_EULER) {
    return cudaErrorInvalidValue;
  }
  const int tiles = ((M + TM - 1) / TM) * ((N + BN - 1) / BN);
  if (!status) status = op_status_word();
  if (!PAIR) {
    const int grid = tiles < sm_count() ? tiles : sm_count();
    gemm_tc_kernel<BN, STAGES, PAIR, KSUB><<<grid, 320, SMEM, s>>>(maps, M, N, K, e, status);
    return cudaGetLastError();
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(320, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // pairs that fit on the device at once (one CTA per SM)
  static int max_pairs[64] = {};
  if (!max_pairs[dev]) {
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<BN, STAGES, PAIR, KSUB>, &cfg);
    if (err != cudaSuccess) return err;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    max_pairs[dev] = n;
  }
  const int pairs = tiles < max_pairs[dev] ? tiles : max_pairs[dev];
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, STAGES, PAIR, KSUB>, maps, M, N, K, e, status);
}

cudaError_t gemm_tc(const bf16* A, long long lda, const bf16* W, int M, int N, int K,
                    const EpiParams& e, int* status, cudaStream_t s) {
  if (!gemm_tc_supported(lda, M, N, K)) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(W)) & 15) return cudaErrorInvalidValue;
  if (N % 256 == 0 && K % 128 == 0) return launch_tc<256, 3, true, 2>(A, lda, W, M, N, K, e, status, s);
  if (N % 256 == 0) return launch_tc<256, 6, true, 1>(A, lda, W, M, N, K, e, status, s);
  if (N % 128 == 0) return launch_tc<128, 6, false, 1>(A, lda, W, M, N, K, e, status, s);
  return launch_tc<64, 8, false, 1>(A, lda, W, M, N, K, e, status, s);
}

}  // namespace dp
