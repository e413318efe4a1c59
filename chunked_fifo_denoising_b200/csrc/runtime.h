// Runtime objects behind the C ABI: device buffers, the model, the queue.
#pragma once

#include <deque>
#include <set>
#include <string>
#include <vector>

#include "internal.h"

namespace dp {

dp_status fail(dp_status s, const char* fmt, ...);
void clear_error();

#define DP_CK(call)                                                                       \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return ::dp::fail(DP_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                        __FILE__, __LINE__);                                              \
  } while (0)

#define DP_TRY(call)                  \
  do {                                \
    dp_status s_ = (call);            \
    if (s_ != DP_OK) return s_;       \
  } while (0)

struct DevBuf {
  void* p = nullptr;
  size_t bytes = 0;
  dp_free_fn fr = nullptr;
  void* ctx = nullptr;
  template <typename T> T* as() const { return static_cast<T*>(p); }
};
dp_status dev_alloc(DevBuf& b, size_t bytes, const char* what);
void dev_free(DevBuf& b);

// Per-kernel-class device timing with CUDA events on one stream.
struct Timer {
  bool on = false;
  cudaStream_t stream = nullptr;
  std::vector<cudaEvent_t> pool;
  struct Rec { int cls, e0, e1; double flops, bytes; };
  std::vector<Rec> pending;
  double ms[DP_KCLASS_COUNT] = {};
  long long n[DP_KCLASS_COUNT] = {};
  double fl[DP_KCLASS_COUNT] = {};
  double by[DP_KCLASS_COUNT] = {};
  int open = -1;
  dp_status begin(int cls);
  dp_status end(double flops, double bytes);
  dp_status collect();
  void reset();
  void release();
};

enum KClass { KC_GEMM = 0, KC_SELF_ATTN = 1, KC_CROSS_ATTN = 2, KC_LN = 3, KC_PATCH = 4,
              KC_HEAD = 5, KC_OTHER = 6 };

}  // namespace dp

struct dp_model {
  dp_model_config cfg;
  int device = 0;
  cudaStream_t stream = nullptr;
  bool f32 = false;  // validation mode
  int d = 0, H = 0, hd = 0, F = 0, P = 0, L = 0;
  struct Param {
    dp::DevBuf buf;
    bool act = false;         // stored in the compute dtype (else fp32)
    long long numel = 0;      // per layer (or total)
    int count = 0;            // layers (1 for global)
    std::vector<char> set;
  };
  Param params[DP_PARAM_COUNT];
  dp::DevBuf status;          // device status word(s) of bounded waits
  dp::DevBuf staging;         // fp32 staging for host -> device parameter copies
  std::set<dp_queue*> queues;

  const void* w(dp_param id, int layer = 0) const;
  const float* wf(dp_param id, int layer = 0) const;
  size_t act_size() const { return f32 ? 4 : 2; }
};

struct dp_queue {
  dp_model* m = nullptr;
  dp_queue_config qc;
  int Lc = 0;                 // tokens per chunk
  long long chunk_numel = 0;
  int n_slots = 0;
  long long Mmax = 0;
  dp::DevBuf ring, x, h, qkv, attn, u, textkv, cache[2], modtab, hmod;
  dp::DevBuf d_sel, d_slot, d_dsig;   // per batch chunk tables (device)
  dp::DevBuf rope_t, rope_y, rope_x;  // rotary (cos, sin) tables (qk_norm_rope)
  float* h_rope_t = nullptr;          // pinned staging of the per-step temporal table
  int rope_Fq = 0, rope_nt = 0, rope_nh = 0;
  dp::DevBuf noise_pool;              // [2F][C][H][W] (noise_mode 1)
  int* h_sel = nullptr;               // pinned staging
  int* h_slot = nullptr;
  float* h_dsig = nullptr;
  cudaEvent_t table_ev = nullptr;
  float* h_noise = nullptr;           // pinned copy of a pushed chunk given in host memory
  cudaEvent_t noise_ev = nullptr;     // its upload has left the staging
  // bookkeeping (host, exact)
  long long step = 0, next_id = 0, head_id = 0, ready_lo = 0;
  bool closed = false;
  std::deque<int> levels;             // levels of chunks [head_id, next_id)
  long long cache_id = -1;
  int cache_cur = 0;
  dp::Timer timer;
};
