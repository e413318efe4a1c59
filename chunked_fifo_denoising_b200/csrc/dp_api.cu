// C ABI: model creation, parameter upload, the FIFO queue and its step.
//
// Method: DualParal write-up "双重并行：让AI视频生成突破时长限制…" (techwalker.com).
// §二: a FIFO of chunks, levels T (tail) .. 1 (head); each step denoises every
// queued chunk once, moves each one place forward, pushes noise at the tail
// and releases the clean head.  §三: self-attention of a chunk reads its
// neighbour's K/V from a cache instead of a concatenated input; cross-
// attention and FFN are per chunk.  On one GPU every queued chunk goes through
// the DiT in one batched pass; the queue is a ring of latent slots whose shift
// is a change of indices, never a copy.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "runtime.h"

using namespace dp;

namespace dp {

static thread_local std::string g_err;
static std::mutex g_alloc_mu;
static dp_alloc_fn g_alloc = nullptr;
static dp_free_fn g_free = nullptr;
static void* g_ctx = nullptr;

dp_status fail(dp_status s, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}
void clear_error() { g_err.clear(); }

dp_status dev_alloc(DevBuf& b, size_t bytes, const char* what) {
  dev_free(b);
  if (bytes == 0) return DP_OK;
  bytes = (bytes + 255) & ~size_t(255);
  dp_alloc_fn a;
  dp_free_fn f;
  void* ctx;
  {
    std::lock_guard<std::mutex> lk(g_alloc_mu);
    a = g_alloc;
    f = g_free;
    ctx = g_ctx;
  }
  void* p = nullptr;
  if (a) {
    p = a(bytes, ctx);
    if (!p) return fail(DP_ERR_OOM, "allocator returned NULL for %s (%zu bytes)", what, bytes);
    b.fr = f;
    b.ctx = ctx;
  } else {
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(DP_ERR_OOM, "cudaMalloc of %s (%zu bytes) failed: %s", what, bytes,
                  cudaGetErrorString(e));
    }
    b.fr = nullptr;
  }
  b.p = p;
  b.bytes = bytes;
  return DP_OK;
}

void dev_free(DevBuf& b) {
  if (b.p) {
    if (b.fr) b.fr(b.p, b.ctx);
    else cudaFree(b.p);
  }
  b = DevBuf();
}

// ---------------------------------------------------------------------------
// Timer
// ---------------------------------------------------------------------------
dp_status Timer::begin(int cls) {
  if (!on) return DP_OK;
  while ((int)pool.size() < 2 * ((int)pending.size() + 1)) {
    cudaEvent_t e;
    DP_CK(cudaEventCreate(&e));
    pool.push_back(e);
  }
  Rec r{cls, 2 * (int)pending.size(), 2 * (int)pending.size() + 1, 0.0, 0.0};
  DP_CK(cudaEventRecord(pool[r.e0], stream));
  pending.push_back(r);
  open = (int)pending.size() - 1;
  return DP_OK;
}

dp_status Timer::end(double flops, double bytes) {
  if (!on || open < 0) return DP_OK;
  Rec& r = pending[open];
  r.flops = flops;
  r.bytes = bytes;
  DP_CK(cudaEventRecord(pool[r.e1], stream));
  open = -1;
  return DP_OK;
}

dp_status Timer::collect() {
  for (const Rec& r : pending) {
    DP_CK(cudaEventSynchronize(pool[r.e1]));
    float t = 0.f;
    DP_CK(cudaEventElapsedTime(&t, pool[r.e0], pool[r.e1]));
    ms[r.cls] += t;
    n[r.cls] += 1;
    fl[r.cls] += r.flops;
    by[r.cls] += r.bytes;
  }
  pending.clear();
  return DP_OK;
}

void Timer::reset() {
  pending.clear();
  for (int i = 0; i < DP_KCLASS_COUNT; ++i) ms[i] = fl[i] = by[i] = 0.0, n[i] = 0;
}

void Timer::release() {
  for (cudaEvent_t e : pool) cudaEventDestroy(e);
  pool.clear();
  pending.clear();
}

}  // namespace dp

// ---------------------------------------------------------------------------
// Parameters
// ---------------------------------------------------------------------------
static bool param_is_layer(dp_param id) { return id >= DP_L_MOD; }

static bool param_is_act(dp_param id) {
  switch (id) {
    case DP_PATCH_W: case DP_TEXT_W: case DP_OUT_W: case DP_L_QKV_W: case DP_L_O_W:
    case DP_L_CQ_W: case DP_L_CK_W: case DP_L_CV_W: case DP_L_CO_W: case DP_L_FFN1_W:
    case DP_L_FFN2_W:
      return true;
    default:
      return false;
  }
}

static long long param_numel(const dp_model_config& c, dp_param id) {
  const long long d = c.dim, F = c.ffn_dim, D = c.freq_dim;
  const long long P = (long long)c.latent_ch * c.patch_t * c.patch_h * c.patch_w;
  const bool text = c.text_in_dim != c.dim;
  switch (id) {
    case DP_PATCH_W: return d * P;
    case DP_PATCH_B: return d;
    case DP_TEXT_W: return text ? d * c.text_in_dim : 0;
    case DP_TEXT_B: return text ? d : 0;
    case DP_TIME1_W: return d * D;
    case DP_TIME1_B: return d;
    case DP_TIME2_W: return d * d;
    case DP_TIME2_B: return d;
    case DP_MOD_W: return 6 * d * d;
    case DP_MOD_B: return 6 * d;
    case DP_HEADMOD_W: return 2 * d * d;
    case DP_HEADMOD_B: return 2 * d;
    case DP_OUT_W: return P * d;
    case DP_OUT_B: return P;
    case DP_L_MOD: return 6 * d;
    case DP_L_QKV_W: return 3 * d * d;
    case DP_L_QKV_B: return 3 * d;
    case DP_L_O_W: case DP_L_CQ_W: case DP_L_CK_W: case DP_L_CV_W: case DP_L_CO_W: return d * d;
    case DP_L_O_B: case DP_L_CQ_B: case DP_L_CK_B: case DP_L_CV_B: case DP_L_CO_B: return d;
    case DP_L_FFN1_W: return F * d;
    case DP_L_FFN1_B: return F;
    case DP_L_FFN2_W: return d * F;
    case DP_L_FFN2_B: return d;
    case DP_L_QNORM_W: case DP_L_KNORM_W: return c.qk_norm_rope ? d : 0;
    default: return -1;
  }
}

const void* dp_model::w(dp_param id, int layer) const {
  const Param& p = params[id];
  return static_cast<const char*>(p.buf.p) + (size_t)layer * p.numel * (p.act ? act_size() : 4);
}
const float* dp_model::wf(dp_param id, int layer) const {
  return static_cast<const float*>(w(id, layer));
}

static dp_status check_config(const dp_model_config* c) {
  if (!c) return fail(DP_ERR_INVALID_ARG, "config is NULL");
  if (c->n_layers < 1 || c->dim < 16 || c->n_heads < 1 || c->dim % c->n_heads)
    return fail(DP_ERR_INVALID_ARG, "bad n_layers/dim/n_heads");
  const int hd = c->dim / c->n_heads;
  if (hd != 16 && hd != 32 && hd != 64 && hd != 128)
    return fail(DP_ERR_INVALID_ARG, "head_dim %d not in {16,32,64,128}", hd);
  if (c->dim % 8 || c->dim > 6144) return fail(DP_ERR_INVALID_ARG, "dim must be a multiple of 8 and <= 6144");
  if (c->ffn_dim < 1 || c->ffn_dim % 8) return fail(DP_ERR_INVALID_ARG, "ffn_dim must be a positive multiple of 8");
  if (c->freq_dim < 2 || c->freq_dim % 2) return fail(DP_ERR_INVALID_ARG, "freq_dim must be even");
  if (c->latent_ch < 1 || c->patch_t < 1 || c->patch_h < 1 || c->patch_w < 1)
    return fail(DP_ERR_INVALID_ARG, "bad latent/patch shape");
  if (c->text_len < 1 || c->text_in_dim < 1) return fail(DP_ERR_INVALID_ARG, "bad text shape");
  if (c->prec != DP_PREC_BF16 && c->prec != DP_PREC_FP32_VALIDATE)
    return fail(DP_ERR_INVALID_ARG, "bad precision");
  if (c->neighbours != DP_NEIGHBOURS_PRED && c->neighbours != DP_NEIGHBOURS_BOTH)
    return fail(DP_ERR_INVALID_ARG, "bad neighbours");
  if (c->qk_norm_rope != 0 && c->qk_norm_rope != 1) return fail(DP_ERR_INVALID_ARG, "bad qk_norm_rope");
  if (c->qk_norm_rope && hd < 6) return fail(DP_ERR_INVALID_ARG, "rotary positions need head_dim >= 6");
  if (c->prec == DP_PREC_BF16) {
    const int P = c->latent_ch * c->patch_t * c->patch_h * c->patch_w;
    if (hd != 64 && hd != 128) return fail(DP_ERR_INVALID_ARG, "bf16 path needs head_dim 64 or 128");
    if (c->dim % 64 || c->ffn_dim % 64 || P % 64)
      return fail(DP_ERR_INVALID_ARG, "bf16 path needs dim, ffn_dim and patch size multiples of 64");
  }
  return DP_OK;
}

extern "C" {

const char* dp_last_error(void) { return g_err.c_str(); }

dp_status dp_set_allocator(dp_alloc_fn alloc, dp_free_fn free_fn, void* ctx) {
  if (alloc && !free_fn) return fail(DP_ERR_INVALID_ARG, "allocator without free function");
  std::lock_guard<std::mutex> lk(g_alloc_mu);
  g_alloc = alloc;
  g_free = alloc ? free_fn : nullptr;
  g_ctx = alloc ? ctx : nullptr;
  return DP_OK;
}

dp_status dp_param_numel(const dp_model_config* cfg, dp_param id, long long* numel) {
  DP_TRY(check_config(cfg));
  if (!numel || id < 0 || id >= DP_PARAM_COUNT) return fail(DP_ERR_INVALID_ARG, "bad param id");
  *numel = param_numel(*cfg, id);
  return DP_OK;
}

dp_status dp_model_create(const dp_model_config* cfg, void* cuda_stream, dp_model** out) {
  clear_error();
  if (!out) return fail(DP_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  DP_TRY(check_config(cfg));
  dp_model* m = new dp_model();
  m->cfg = *cfg;
  DP_CK(cudaGetDevice(&m->device));
  m->stream = static_cast<cudaStream_t>(cuda_stream);
  m->f32 = cfg->prec == DP_PREC_FP32_VALIDATE;
  m->d = cfg->dim;
  m->H = cfg->n_heads;
  m->hd = cfg->dim / cfg->n_heads;
  m->F = cfg->ffn_dim;
  m->P = cfg->latent_ch * cfg->patch_t * cfg->patch_h * cfg->patch_w;
  m->L = cfg->n_layers;
  long long max_numel = 0;
  for (int i = 0; i < DP_PARAM_COUNT; ++i) {
    dp_param id = (dp_param)i;
    dp_model::Param& p = m->params[i];
    p.numel = param_numel(*cfg, id);
    p.count = param_is_layer(id) ? cfg->n_layers : 1;
    p.act = param_is_act(id);
    p.set.assign(p.count, p.numel == 0 ? 1 : 0);
    if (p.numel > max_numel) max_numel = p.numel;
    const size_t bytes = (size_t)p.numel * p.count * (p.act ? m->act_size() : 4);
    dp_status s = dev_alloc(p.buf, bytes, "parameter");
    if (s != DP_OK) { dp_destroy(m); return s; }
  }
  dp_status s = dev_alloc(m->status, 256, "status word");
  if (s == DP_OK) s = dev_alloc(m->staging, (size_t)max_numel * 4, "parameter staging");
  if (s != DP_OK) { dp_destroy(m); return s; }
  cudaError_t e = cudaMemsetAsync(m->status.p, 0, 256, m->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(m->stream);
  if (e != cudaSuccess) {
    dp_destroy(m);
    return fail(DP_ERR_CUDA, "status init: %s", cudaGetErrorString(e));
  }
  *out = m;
  return DP_OK;
}

dp_status dp_model_set_param(dp_model* m, dp_param id, int layer, const float* src,
                             long long numel, dp_loc loc) {
  clear_error();
  if (!m || !src) return fail(DP_ERR_INVALID_ARG, "NULL model or source");
  if (id < 0 || id >= DP_PARAM_COUNT) return fail(DP_ERR_INVALID_ARG, "bad param id %d", (int)id);
  dp_model::Param& p = m->params[id];
  if (!param_is_layer(id)) layer = 0;
  if (layer < 0 || layer >= p.count) return fail(DP_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (numel != p.numel)
    return fail(DP_ERR_INVALID_ARG, "param %d expects %lld elements, got %lld", (int)id, p.numel, numel);
  if (numel == 0) return DP_OK;
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  const float* dsrc = src;
  if (loc == DP_LOC_HOST) {
    DP_CK(cudaMemcpyAsync(m->staging.p, src, (size_t)numel * 4, cudaMemcpyHostToDevice, m->stream));
    dsrc = m->staging.as<float>();
  }
  void* dst = const_cast<void*>(m->w(id, layer));
  if (p.act && !m->f32) {
    DP_CK(convert_f32_to_bf16(dsrc, static_cast<bf16*>(dst), numel, m->stream));
  } else {
    DP_CK(cudaMemcpyAsync(dst, dsrc, (size_t)numel * 4, cudaMemcpyDeviceToDevice, m->stream));
  }
  DP_CK(cudaStreamSynchronize(m->stream));
  p.set[layer] = 1;
  return DP_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Queue
// ---------------------------------------------------------------------------
namespace {

const int kPredNone = 0, kPredCache = 2;
const unsigned long long kNoiseTensorId = 1001;    // tensor id of chunk noise in the generator
const unsigned long long kShuffleTensorId = 1002;  // draws of the coordinated-noise order
const unsigned long long kPoolTensorId = 1003;     // coordinated-noise pool frames

// SplitMix64 (Steele, Lea, Flood 2014): finaliser and keyed stream draws.
unsigned long long sm64_mix(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
unsigned long long sm64_key(unsigned long long seed, unsigned long long a, unsigned long long b) {
  const unsigned long long g = 0x9E3779B97F4A7C15ull;
  unsigned long long k = sm64_mix((seed + 1) * g);
  k = sm64_mix(k + (a + 1) * g);
  return sm64_mix(k + (b + 1) * g);
}

// Pool frames of chunk k (coordinated noise): the F frames chunk k-1 does not
// use, 0..F-1 for even k and F..2F-1 for odd k, shuffled by Fisher-Yates with
// the draws of stream (seed, 1002, k): for i = F-1 .. 1 swap i with draw mod (i+1).
PoolGather coordinated_frames(unsigned long long seed, long long k, int F) {
  PoolGather g;
  const int base = (k % 2 == 0) ? 0 : F;
  for (int f = 0; f < F; ++f) g.src[f] = base + f;
  const unsigned long long key = sm64_key(seed, kShuffleTensorId, (unsigned long long)k);
  unsigned long long t = 0;
  for (int i = F - 1; i >= 1; --i, ++t) {
    const unsigned long long draw = sm64_mix(key + (t + 1) * 0x9E3779B97F4A7C15ull);
    const int j = (int)(draw % (unsigned long long)(i + 1));
    const int tmp = g.src[i];
    g.src[i] = g.src[j];
    g.src[j] = tmp;
  }
  return g;
}

struct Plan {
  bool push = false;
  int n = 0;
  long long head = 0;
  std::vector<int> levels;
  int head_pred = kPredNone;
  bool writes_cache = false;
};

bool pushing(const dp_queue* q) {
  if (q->closed) return false;
  return q->qc.n_chunks < 0 || q->next_id < q->qc.n_chunks;
}

dp_status make_plan(const dp_queue* q, Plan& pl) {
  pl = Plan();
  pl.push = pushing(q);
  if (pl.push && q->next_id - q->ready_lo >= q->n_slots)
    return fail(DP_ERR_FULL, "no free ring slot for chunk %lld: pop ready chunks first", q->next_id);
  pl.levels.assign(q->levels.begin(), q->levels.end());
  if (pl.push) pl.levels.push_back(q->qc.T);
  pl.n = (int)pl.levels.size();
  if (pl.n == 0) return fail(DP_ERR_DRAINED, "queue drained");
  pl.head = q->head_id;
  pl.head_pred = pl.head == 0 ? kPredNone : kPredCache;
  pl.writes_cache = pl.levels[0] == 1;
  return DP_OK;
}

double gemm_flops(long long M, long long N, long long K) { return 2.0 * M * N * K; }

// Launch helpers bound to one queue.
struct Stepper {
  dp_queue* q;
  dp_model* m;
  cudaStream_t s;
  int* status;

  dp_status gemm(const void* A, long long lda, const void* W, int M, int N, int K,
                 const EpiParams& e, int cls = KC_GEMM) {
    DP_TRY(q->timer.begin(cls));
    cudaError_t err;
    if (m->f32) {
      err = gemm_simt(1, A, lda, 1, W, M, N, K, e, s);
    } else {
      if (!gemm_tc_supported(lda, M, N, K))
        return fail(DP_ERR_INVALID_ARG, "GEMM %dx%dx%d not supported by the tensor-core path", M, N, K);
      err = gemm_tc(static_cast<const bf16*>(A), lda, static_cast<const bf16*>(W), M, N, K, e,
                    status, s);
    }
    if (err != cudaSuccess) return fail(DP_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(err));
    return q->timer.end(gemm_flops(M, N, K), 0.0);
  }

  dp_status attention(const AttnParams& p, int cls, double flops) {
    DP_TRY(q->timer.begin(cls));
    cudaError_t err;
    if (m->f32) {
      err = attention_simt(p, s);
    } else {
      if (!attention_tc_supported(p)) return fail(DP_ERR_INVALID_ARG, "attention shape not supported");
      err = attention_tc(p, status, s);
    }
    if (err != cudaSuccess) return fail(DP_ERR_CUDA, "attention launch: %s", cudaGetErrorString(err));
    return q->timer.end(flops, 0.0);
  }

  dp_status ln(const LnParams& p) {
    DP_TRY(q->timer.begin(KC_LN));
    cudaError_t err = layernorm_mod(p, s);
    if (err != cudaSuccess) return fail(DP_ERR_CUDA, "layernorm launch: %s", cudaGetErrorString(err));
    const double bytes = (double)p.M * p.d * (4.0 + (p.out_f32 ? 4.0 : 2.0));
    return q->timer.end(0.0, bytes);
  }
};

EpiParams epi_base(int mode) {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.mode = mode;
  e.rows_per_chunk = 1;
  return e;
}

}  // namespace

// Runs the launch sequence of one step for the chunks of `pl` (device side).
static dp_status run_step(dp_queue* q, const Plan& pl) {
  dp_model* m = q->m;
  const int d = m->d, F = m->F, L = m->L, P = m->P, Lc = q->Lc, n = pl.n;
  const int M = n * Lc;
  const bool f32 = m->f32;
  const size_t as = m->act_size();
  Stepper st{q, m, m->stream, m->status.as<int>()};
  cudaStream_t s = m->stream;
  const dp_model_config& c = m->cfg;
  const dp_queue_config& qc = q->qc;
  const int* sel = q->d_sel.as<int>();
  const long long mstride = (long long)L * 6 * d;  // modtab stride per level
  float* modtab = q->modtab.as<float>();

  // patch embedding: gather 1 x ph x pw x C patches, then one GEMM (K = P)
  DP_TRY(q->timer.begin(KC_PATCH));
  DP_CK(gather_patches(q->ring.as<float>(), q->chunk_numel, q->d_slot.as<int>(), n, c.latent_ch,
                       qc.frames_per_chunk, qc.lat_h, qc.lat_w, c.patch_t, c.patch_h, c.patch_w,
                       q->h.p, f32 ? 1 : 0, s));
  DP_TRY(q->timer.end(0.0, (double)M * P * (4.0 + as)));
  {
    EpiParams e = epi_base(EPI_STORE);
    e.out_f32 = 1;
    e.bias = m->wf(DP_PATCH_B);
    e.out = q->x.p;
    e.ldo = d;
    DP_TRY(st.gemm(q->h.p, P, m->w(DP_PATCH_W), M, d, P, e, KC_PATCH));
  }
  void* cache_rd = q->cache[q->cache_cur].p;
  void* cache_wr = q->cache[1 - q->cache_cur].p;
  const long long cache_layer = (long long)Lc * 2 * d;  // elements per layer
  char* qkv = q->qkv.as<char>();
  const bool rope_fused = c.qk_norm_rope && !f32 && d % 256 == 0 && (m->hd == 64 || m->hd == 128);
  for (int l = 0; l < L; ++l) {
    float* mt = modtab + (long long)l * 6 * d;
    // --- self-attention block -------------------------------------------
    LnParams lp;
    memset(&lp, 0, sizeof(lp));
    lp.out_f32 = f32;
    lp.x = q->x.as<float>();
    lp.ldx = d;
    lp.M = M;
    lp.d = d;
    lp.shift = mt + 0 * d;
    lp.scale = mt + 1 * d;
    lp.mod_stride = mstride;
    lp.chunk_sel = sel;
    lp.rows_per_chunk = Lc;
    lp.out = q->h.p;
    lp.ldo = d;
    DP_TRY(st.ln(lp));
    {
      EpiParams e = epi_base(EPI_STORE);
      e.out_f32 = f32;
      e.bias = m->wf(DP_L_QKV_B, l);
      e.out = qkv;
      e.ldo = 3 * d;
      if (pl.writes_cache) {  // head chunk leaves after this step: keep its K/V
        e.cache = static_cast<char*>(cache_wr) + (size_t)l * cache_layer * as;
        e.cache_row0 = 0;
        e.cache_rows = Lc;
        e.cache_col0 = d;
        e.ldc = 2 * d;
      }
      // fused into the tensor-core epilogue when every 128-column half of a
      // 256-column tile holds whole heads of one part (q or k): d % 256 == 0
      if (rope_fused) {
        e.rope = 1;
        e.rows_per_chunk = Lc;
        e.rope_d = d;
        e.rope_hd = m->hd;
        e.rope_Fq = q->rope_Fq;
        e.rope_Hq = qc.lat_h / c.patch_h;
        e.rope_Wq = qc.lat_w / c.patch_w;
        e.rope_nt = q->rope_nt;
        e.rope_nh = q->rope_nh;
        e.q_w = m->wf(DP_L_QNORM_W, l);
        e.k_w = m->wf(DP_L_KNORM_W, l);
        e.rope_t = q->rope_t.as<float2>();
        e.rope_y = q->rope_y.as<float2>();
        e.rope_x = q->rope_x.as<float2>();
      }
      DP_TRY(st.gemm(q->h.p, d, m->w(DP_L_QKV_W, l), M, 3 * d, d, e));
    }
    if (c.qk_norm_rope && !rope_fused) {  // separate in-place kernel (fp32 mode, other widths)
      RopeParams rp;
      memset(&rp, 0, sizeof(rp));
      rp.f32 = f32;
      rp.qkv = qkv;
      rp.ld = 3 * d;
      rp.M = M;
      rp.d = d;
      rp.n_heads = m->H;
      rp.Lc = Lc;
      rp.Fq = q->rope_Fq;
      rp.Hq = qc.lat_h / c.patch_h;
      rp.Wq = qc.lat_w / c.patch_w;
      rp.nt = q->rope_nt;
      rp.nh = q->rope_nh;
      rp.q_w = m->wf(DP_L_QNORM_W, l);
      rp.k_w = m->wf(DP_L_KNORM_W, l);
      rp.rope_t = q->rope_t.as<float2>();
      rp.rope_y = q->rope_y.as<float2>();
      rp.rope_x = q->rope_x.as<float2>();
      if (pl.writes_cache) {  // the persisted K of the head chunk holds the rotated keys
        rp.cache = static_cast<char*>(cache_wr) + (size_t)l * cache_layer * as;
        rp.ldc = 2 * d;
      }
      DP_TRY(q->timer.begin(KC_OTHER));
      DP_CK(qk_norm_rope(rp, s));
      DP_TRY(q->timer.end(0.0, (double)M * 2 * d * 2 * as));
    }
    {
      AttnParams a;
      memset(&a, 0, sizeof(a));
      a.f32 = f32;
      a.n_chunks = n;
      a.Lq = Lc;
      a.n_heads = m->H;
      a.head_dim = m->hd;
      a.q = qkv;
      a.ldq = 3 * d;
      a.k = qkv + (size_t)d * as;
      a.v = qkv + (size_t)2 * d * as;
      a.ldkv = 3 * d;
      a.kv_chunk_rows = Lc;
      a.Lk = Lc;
      a.pred_in_batch = 1;
      a.succ_in_batch = c.neighbours == DP_NEIGHBOURS_BOTH;
      double keys = (double)n * Lc + (double)(n - 1) * Lc * (a.succ_in_batch ? 2 : 1);
      if (pl.head_pred == kPredCache) {
        a.k0_pred = static_cast<char*>(cache_rd) + (size_t)l * cache_layer * as;
        a.v0_pred = static_cast<char*>(cache_rd) + ((size_t)l * cache_layer + d) * as;
        a.ld_pred = 2 * d;
        a.Lk_pred = Lc;
        keys += Lc;
      }
      a.out = q->attn.p;
      a.ldo = d;
      DP_TRY(st.attention(a, KC_SELF_ATTN, 4.0 * Lc * keys * d));
    }
    {
      EpiParams e = epi_base(EPI_RESID_GATED);
      e.bias = m->wf(DP_L_O_B, l);
      e.resid = q->x.as<float>();
      e.ldr = d;
      e.gate = mt + 2 * d;
      e.gate_stride = mstride;
      e.chunk_sel = sel;
      e.rows_per_chunk = Lc;
      DP_TRY(st.gemm(q->attn.p, d, m->w(DP_L_O_W, l), M, d, d, e));
    }
    // --- cross-attention block (no modulation, no gate) -------------------
    lp.shift = lp.scale = nullptr;
    DP_TRY(st.ln(lp));
    {
      EpiParams e = epi_base(EPI_STORE);
      e.out_f32 = f32;
      e.bias = m->wf(DP_L_CQ_B, l);
      e.out = qkv;
      e.ldo = d;
      DP_TRY(st.gemm(q->h.p, d, m->w(DP_L_CQ_W, l), M, d, d, e));
    }
    {
      AttnParams a;
      memset(&a, 0, sizeof(a));
      a.f32 = f32;
      a.n_chunks = n;
      a.Lq = Lc;
      a.n_heads = m->H;
      a.head_dim = m->hd;
      a.q = qkv;
      a.ldq = d;
      char* tkv = q->textkv.as<char>() + (size_t)l * c.text_len * 2 * d * as;
      a.k = tkv;
      a.v = tkv + (size_t)d * as;
      a.ldkv = 2 * d;
      a.kv_chunk_rows = 0;
      a.Lk = c.text_len;
      a.out = q->attn.p;
      a.ldo = d;
      DP_TRY(st.attention(a, KC_CROSS_ATTN, 4.0 * M * (double)c.text_len * d));
    }
    {
      EpiParams e = epi_base(EPI_RESID);
      e.bias = m->wf(DP_L_CO_B, l);
      e.resid = q->x.as<float>();
      e.ldr = d;
      DP_TRY(st.gemm(q->attn.p, d, m->w(DP_L_CO_W, l), M, d, d, e));
    }
    // --- FFN block ----------------------------------------------------------
    lp.shift = mt + 3 * d;
    lp.scale = mt + 4 * d;
    DP_TRY(st.ln(lp));
    {
      EpiParams e = epi_base(EPI_GELU);
      e.out_f32 = f32;
      e.bias = m->wf(DP_L_FFN1_B, l);
      e.out = q->u.p;
      e.ldo = F;
      DP_TRY(st.gemm(q->h.p, d, m->w(DP_L_FFN1_W, l), M, F, d, e));
    }
    {
      EpiParams e = epi_base(EPI_RESID_GATED);
      e.bias = m->wf(DP_L_FFN2_B, l);
      e.resid = q->x.as<float>();
      e.ldr = d;
      e.gate = mt + 5 * d;
      e.gate_stride = mstride;
      e.chunk_sel = sel;
      e.rows_per_chunk = Lc;
      DP_TRY(st.gemm(q->u.p, F, m->w(DP_L_FFN2_W, l), M, d, F, e));
    }
  }
  // head: LN + head modulation, Linear to patch features, Euler update in the ring
  {
    LnParams lp;
    memset(&lp, 0, sizeof(lp));
    lp.out_f32 = f32;
    lp.x = q->x.as<float>();
    lp.ldx = d;
    lp.M = M;
    lp.d = d;
    lp.shift = q->hmod.as<float>();
    lp.scale = q->hmod.as<float>() + d;
    lp.mod_stride = 2 * d;
    lp.chunk_sel = sel;
    lp.rows_per_chunk = Lc;
    lp.out = q->h.p;
    lp.ldo = d;
    DP_TRY(st.ln(lp));
    EpiParams e = epi_base(EPI_EULER);
    e.bias = m->wf(DP_OUT_B);
    e.rows_per_chunk = Lc;
    e.ring = q->ring.as<float>();
    e.chunk_numel = q->chunk_numel;
    e.chunk_slot = q->d_slot.as<int>();
    e.dsig = q->d_dsig.as<float>();
    e.lat_c = c.latent_ch;
    e.lat_f = qc.frames_per_chunk;
    e.lat_h = qc.lat_h;
    e.lat_w = qc.lat_w;
    e.pt = c.patch_t;
    e.ph = c.patch_h;
    e.pw = c.patch_w;
    DP_TRY(st.gemm(q->h.p, d, m->w(DP_OUT_W), M, P, d, e, KC_HEAD));
  }
  return DP_OK;
}

static dp_status upload_tables(dp_queue* q, const Plan& pl) {
  DP_CK(cudaEventSynchronize(q->table_ev));  // previous upload has left the staging
  const int T = q->qc.T;
  for (int i = 0; i < pl.n; ++i) {
    const int j = pl.levels[i];
    q->h_sel[i] = j - 1;
    q->h_slot[i] = (int)((pl.head + i) % q->n_slots);
    q->h_dsig[i] = (float)((double)(j - 1) / T - (double)j / T);
  }
  cudaStream_t s = q->m->stream;
  if (q->m->cfg.qk_norm_rope) {
    // temporal rotary table of this step: absolute frame (chunk id * Fq + f)
    const int nt = q->rope_nt, Fq = q->rope_Fq;
    for (int c = 0; c < pl.n; ++c)
      for (int f = 0; f < Fq; ++f) {
        const double pos = (double)(pl.head + c) * Fq + f;
        for (int l = 0; l < nt; ++l) {
          const double a = std::fmod(pos * std::pow(10000.0, -(double)l / nt), 2.0 * M_PI);
          float* e = q->h_rope_t + 2 * (((size_t)c * Fq + f) * nt + l);
          e[0] = (float)std::cos(a);
          e[1] = (float)std::sin(a);
        }
      }
    DP_CK(cudaMemcpyAsync(q->rope_t.p, q->h_rope_t, (size_t)pl.n * Fq * nt * 2 * sizeof(float),
                          cudaMemcpyHostToDevice, s));
  }
  DP_CK(cudaMemcpyAsync(q->d_sel.p, q->h_sel, pl.n * sizeof(int), cudaMemcpyHostToDevice, s));
  DP_CK(cudaMemcpyAsync(q->d_slot.p, q->h_slot, pl.n * sizeof(int), cudaMemcpyHostToDevice, s));
  DP_CK(cudaMemcpyAsync(q->d_dsig.p, q->h_dsig, pl.n * sizeof(float), cudaMemcpyHostToDevice, s));
  DP_CK(cudaEventRecord(q->table_ev, s));
  return DP_OK;
}

// Reads and clears the model's device status word (the stream must have been
// synchronised): DP_ERR_KERNEL if a kernel gave up a bounded wait since the
// last check.
static dp_status check_status_word(dp_model* m) {
  int word = 0;
  DP_CK(cudaMemcpy(&word, m->status.p, sizeof(int), cudaMemcpyDeviceToHost));
  if (word != 0) {
    DP_CK(cudaMemset(m->status.p, 0, 256));
    return fail(DP_ERR_KERNEL, "a kernel gave up a bounded wait (status word 0x%x)", word);
  }
  return DP_OK;
}

static void free_queue(dp_queue* q) {
  DevBuf* bufs[] = {&q->ring, &q->x, &q->h, &q->qkv, &q->attn, &q->u, &q->textkv, &q->cache[0],
                    &q->cache[1], &q->modtab, &q->hmod, &q->d_sel, &q->d_slot, &q->d_dsig,
                    &q->rope_t, &q->rope_y, &q->rope_x, &q->noise_pool};
  for (DevBuf* b : bufs) dev_free(*b);
  if (q->h_rope_t) cudaFreeHost(q->h_rope_t);
  if (q->h_sel) cudaFreeHost(q->h_sel);
  if (q->h_slot) cudaFreeHost(q->h_slot);
  if (q->h_dsig) cudaFreeHost(q->h_dsig);
  if (q->table_ev) cudaEventDestroy(q->table_ev);
  if (q->h_noise) cudaFreeHost(q->h_noise);
  if (q->noise_ev) cudaEventDestroy(q->noise_ev);
  q->timer.release();
}

// Level tables and text K/V (once per queue).
static dp_status build_tables(dp_queue* q, const float* text, dp_loc loc) {
  dp_model* m = q->m;
  const dp_model_config& c = m->cfg;
  const int T = q->qc.T, d = m->d, D = c.freq_dim, L = m->L;
  cudaStream_t s = m->stream;
  DevBuf feats, h1, sv, mvec, textf, tp;
  dp_status st = DP_OK;
  auto cleanup = [&]() { dev_free(feats); dev_free(h1); dev_free(sv); dev_free(mvec); dev_free(textf); dev_free(tp); };
#define BT_TRY(x) do { st = (x); if (st != DP_OK) { cleanup(); return st; } } while (0)
#define BT_CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { cleanup(); return fail(DP_ERR_CUDA, "%s: %s", #x, cudaGetErrorString(e_)); } } while (0)
  BT_TRY(dev_alloc(feats, (size_t)T * D * 4, "timestep features"));
  BT_TRY(dev_alloc(h1, (size_t)T * d * 4, "time hidden"));
  BT_TRY(dev_alloc(sv, (size_t)T * d * 4, "time embedding"));
  BT_TRY(dev_alloc(mvec, (size_t)T * 6 * d * 4, "modulation"));
  BT_CK(timestep_features(T, D, feats.as<float>(), s));
  EpiParams e = epi_base(EPI_SILU);
  e.out_f32 = 1;
  e.bias = m->wf(DP_TIME1_B);
  e.out = h1.p;
  e.ldo = d;
  BT_CK(gemm_simt(1, feats.p, D, 1, m->w(DP_TIME1_W), T, d, D, e, s));
  e.bias = m->wf(DP_TIME2_B);
  e.out = sv.p;  // SiLU(e_j), the input of both modulation projections
  BT_CK(gemm_simt(1, h1.p, d, 1, m->w(DP_TIME2_W), T, d, d, e, s));
  e = epi_base(EPI_STORE);
  e.out_f32 = 1;
  e.bias = m->wf(DP_MOD_B);
  e.out = mvec.p;
  e.ldo = 6 * d;
  BT_CK(gemm_simt(1, sv.p, d, 1, m->w(DP_MOD_W), T, 6 * d, d, e, s));
  BT_CK(add_layer_tables(mvec.as<float>(), m->wf(DP_L_MOD), T, L, 6 * d, q->modtab.as<float>(), s));
  e.bias = m->wf(DP_HEADMOD_B);
  e.out = q->hmod.p;
  e.ldo = 2 * d;
  BT_CK(gemm_simt(1, sv.p, d, 1, m->w(DP_HEADMOD_W), T, 2 * d, d, e, s));
  // prompt: optional projection to the model width, then K/V of every layer
  const int Lt = c.text_len, Din = c.text_in_dim;
  BT_TRY(dev_alloc(textf, (size_t)Lt * Din * 4, "text"));
  BT_CK(cudaMemcpyAsync(textf.p, text, (size_t)Lt * Din * 4,
                        loc == DP_LOC_HOST ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, s));
  const float* t = textf.as<float>();
  if (Din != d) {
    BT_TRY(dev_alloc(tp, (size_t)Lt * d * 4, "projected text"));
    e = epi_base(EPI_STORE);
    e.out_f32 = 1;
    e.bias = m->wf(DP_TEXT_B);
    e.out = tp.p;
    e.ldo = d;
    BT_CK(gemm_simt(1, textf.p, Din, m->f32 ? 1 : 0, m->w(DP_TEXT_W), Lt, d, Din, e, s));
    t = tp.as<float>();
  }
  const size_t as = m->act_size();
  for (int l = 0; l < L; ++l) {
    char* dst = q->textkv.as<char>() + (size_t)l * Lt * 2 * d * as;
    e = epi_base(EPI_STORE);
    e.out_f32 = m->f32;
    e.ldo = 2 * d;
    e.bias = m->wf(DP_L_CK_B, l);
    e.out = dst;
    BT_CK(gemm_simt(1, t, d, m->f32 ? 1 : 0, m->w(DP_L_CK_W, l), Lt, d, d, e, s));
    e.bias = m->wf(DP_L_CV_B, l);
    e.out = dst + (size_t)d * as;
    BT_CK(gemm_simt(1, t, d, m->f32 ? 1 : 0, m->w(DP_L_CV_W, l), Lt, d, d, e, s));
  }
  BT_CK(cudaStreamSynchronize(s));
  cleanup();
#undef BT_TRY
#undef BT_CK
  return DP_OK;
}

extern "C" {

dp_status dp_queue_init(dp_model* m, const dp_queue_config* qc, const float* text,
                        dp_loc text_loc, dp_queue** out) {
  clear_error();
  if (!m || !qc || !text || !out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  const dp_model_config& c = m->cfg;
  if (qc->T < 1 || qc->ready_capacity < 1) return fail(DP_ERR_INVALID_ARG, "T and ready_capacity must be >= 1");
  if (qc->frames_per_chunk < 1 || qc->frames_per_chunk % c.patch_t || qc->lat_h < 1 ||
      qc->lat_h % c.patch_h || qc->lat_w < 1 || qc->lat_w % c.patch_w)
    return fail(DP_ERR_INVALID_ARG, "chunk shape not divisible by the patch size");
  if (qc->n_chunks == 0 || qc->n_chunks < -1) return fail(DP_ERR_INVALID_ARG, "n_chunks must be > 0 or -1");
  if (qc->noise_mode != 0 && qc->noise_mode != 1) return fail(DP_ERR_INVALID_ARG, "bad noise_mode");
  if (qc->noise_mode == 1 && qc->frames_per_chunk > 64)
    return fail(DP_ERR_INVALID_ARG, "coordinated noise supports at most 64 frames per chunk");
  if (text_loc != DP_LOC_DEVICE && text_loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  for (int i = 0; i < DP_PARAM_COUNT; ++i)
    for (char sset : m->params[i].set)
      if (!sset) return fail(DP_ERR_STATE, "parameter %d not set", i);
  {
    // kernels index rows with 32-bit integers and elements with 64-bit offsets
    const long long lc = (long long)(qc->frames_per_chunk / c.patch_t) * (qc->lat_h / c.patch_h) *
                         (qc->lat_w / c.patch_w);
    if ((long long)qc->T * lc >= (1LL << 31)) return fail(DP_ERR_INVALID_ARG, "too many rows for one queue step");
  }
  dp_queue* q = new dp_queue();
  q->m = m;
  q->qc = *qc;
  q->Lc = (qc->frames_per_chunk / c.patch_t) * (qc->lat_h / c.patch_h) * (qc->lat_w / c.patch_w);
  q->chunk_numel = (long long)c.latent_ch * qc->frames_per_chunk * qc->lat_h * qc->lat_w;
  q->n_slots = qc->T + qc->ready_capacity;
  q->Mmax = (long long)qc->T * q->Lc;
  q->timer.stream = m->stream;
  const int d = m->d, L = m->L;
  const size_t as = m->act_size();
  const long long Mm = q->Mmax;
  dp_status s = DP_OK;
#define QA(buf, bytes, what) if (s == DP_OK) s = dev_alloc(buf, bytes, what)
  QA(q->ring, (size_t)q->n_slots * q->chunk_numel * 4, "latent ring");
  QA(q->x, (size_t)Mm * d * 4, "residual stream");
  QA(q->h, (size_t)Mm * std::max(d, m->P) * as, "normalised activations");
  QA(q->qkv, (size_t)Mm * 3 * d * as, "qkv");
  QA(q->attn, (size_t)Mm * d * as, "attention output");
  QA(q->u, (size_t)Mm * m->F * as, "ffn hidden");
  QA(q->textkv, (size_t)L * c.text_len * 2 * d * as, "text K/V");
  QA(q->cache[0], (size_t)L * q->Lc * 2 * d * as, "predecessor K/V A");
  QA(q->cache[1], (size_t)L * q->Lc * 2 * d * as, "predecessor K/V B");
  QA(q->modtab, (size_t)qc->T * L * 6 * d * 4, "modulation table");
  QA(q->hmod, (size_t)qc->T * 2 * d * 4, "head modulation table");
  QA(q->d_sel, (size_t)qc->T * 4, "chunk levels");
  QA(q->d_slot, (size_t)qc->T * 4, "chunk slots");
  QA(q->d_dsig, (size_t)qc->T * 4, "chunk sigma steps");
  if (qc->noise_mode == 1) QA(q->noise_pool, (size_t)2 * q->chunk_numel * 4, "noise pool");
  if (c.qk_norm_rope) {
    q->rope_Fq = qc->frames_per_chunk / c.patch_t;
    q->rope_nh = (m->hd / 2) / 3;
    q->rope_nt = m->hd / 2 - 2 * q->rope_nh;
    QA(q->rope_t, (size_t)qc->T * q->rope_Fq * q->rope_nt * 2 * 4, "temporal rotary table");
    QA(q->rope_y, (size_t)(qc->lat_h / c.patch_h) * q->rope_nh * 2 * 4, "row rotary table");
    QA(q->rope_x, (size_t)(qc->lat_w / c.patch_w) * q->rope_nh * 2 * 4, "column rotary table");
  }
#undef QA
  if (s == DP_OK) {
    cudaError_t e = cudaMallocHost(&q->h_sel, qc->T * sizeof(int));
    if (e == cudaSuccess) e = cudaMallocHost(&q->h_slot, qc->T * sizeof(int));
    if (e == cudaSuccess) e = cudaMallocHost(&q->h_dsig, qc->T * sizeof(float));
    if (e == cudaSuccess && c.qk_norm_rope)
      e = cudaMallocHost(&q->h_rope_t, (size_t)qc->T * q->rope_Fq * q->rope_nt * 2 * sizeof(float));
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q->table_ev, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(q->table_ev, m->stream);
    if (e == cudaSuccess) e = cudaMallocHost(&q->h_noise, (size_t)q->chunk_numel * sizeof(float));
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q->noise_ev, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(q->noise_ev, m->stream);
    if (e != cudaSuccess) s = fail(DP_ERR_OOM, "pinned staging: %s", cudaGetErrorString(e));
  }
  if (s == DP_OK) s = build_tables(q, text, text_loc);
  if (s == DP_OK && qc->noise_mode == 1) {
    // default pool: 2F frames of N(0,1), frame b from stream (seed, 1003, b)
    const long long fe = (long long)c.latent_ch * qc->lat_h * qc->lat_w;
    for (int b = 0; b < 2 * qc->frames_per_chunk && s == DP_OK; ++b) {
      cudaError_t e = normal_fill(qc->seed, kPoolTensorId, (unsigned long long)b,
                                  q->noise_pool.as<float>() + (size_t)b * fe, fe, m->stream);
      if (e == cudaSuccess) e = cudaStreamSynchronize(m->stream);
      if (e != cudaSuccess) s = fail(DP_ERR_CUDA, "noise pool: %s", cudaGetErrorString(e));
    }
  }
  if (s == DP_OK && c.qk_norm_rope) {
    // row and column rotary tables, fixed for the queue: angle = pos * 10000^(-l/nh)
    const int nh = q->rope_nh;
    for (int axis = 0; axis < 2 && s == DP_OK; ++axis) {
      const int npos = axis == 0 ? qc->lat_h / c.patch_h : qc->lat_w / c.patch_w;
      std::vector<float> tab((size_t)npos * nh * 2);
      for (int pos = 0; pos < npos; ++pos)
        for (int l = 0; l < nh; ++l) {
          const double a = pos * std::pow(10000.0, -(double)l / nh);
          tab[2 * ((size_t)pos * nh + l)] = (float)std::cos(a);
          tab[2 * ((size_t)pos * nh + l) + 1] = (float)std::sin(a);
        }
      cudaError_t e = cudaMemcpy(axis == 0 ? q->rope_y.p : q->rope_x.p, tab.data(),
                                 tab.size() * sizeof(float), cudaMemcpyHostToDevice);
      if (e != cudaSuccess) s = fail(DP_ERR_CUDA, "rotary tables: %s", cudaGetErrorString(e));
    }
  }
  if (s != DP_OK) {
    std::string msg = dp_last_error();
    free_queue(q);
    delete q;
    return fail(s, "%s", msg.c_str());
  }
  m->queues.insert(q);
  *out = q;
  return DP_OK;
}

dp_status dp_queue_step(dp_queue* q, const float* noise, dp_loc loc) {
  clear_error();
  if (!q) return fail(DP_ERR_INVALID_ARG, "NULL queue");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  Plan pl;
  DP_TRY(make_plan(q, pl));
  if (pl.head_pred == kPredCache && q->cache_id != pl.head - 1)
    return fail(DP_ERR_STATE, "persisted K/V belong to chunk %lld, head needs chunk %lld",
                q->cache_id, pl.head - 1);
  // timing records are read back lazily (on query, or when many are pending)
  if (q->timer.on && q->timer.pending.size() > 16384) DP_TRY(q->timer.collect());
  dp_model* m = q->m;
  cudaStream_t s = m->stream;
  if (pl.push) {
    float* slot = q->ring.as<float>() + (size_t)(q->next_id % q->n_slots) * q->chunk_numel;
    if (noise && loc == DP_LOC_HOST) {
      // the caller may reuse its host buffer once the call returns: stage it
      // in pinned memory (the previous push has left the staging by now)
      DP_CK(cudaEventSynchronize(q->noise_ev));
      std::memcpy(q->h_noise, noise, (size_t)q->chunk_numel * 4);
      DP_CK(cudaMemcpyAsync(slot, q->h_noise, (size_t)q->chunk_numel * 4, cudaMemcpyHostToDevice, s));
      DP_CK(cudaEventRecord(q->noise_ev, s));
    } else if (noise) {
      DP_CK(cudaMemcpyAsync(slot, noise, (size_t)q->chunk_numel * 4, cudaMemcpyDeviceToDevice, s));
    } else if (q->qc.noise_mode == 1) {
      const int F = q->qc.frames_per_chunk;
      DP_CK(noise_from_pool(q->noise_pool.as<float>(), m->cfg.latent_ch, F,
                            (long long)q->qc.lat_h * q->qc.lat_w,
                            coordinated_frames(q->qc.seed, q->next_id, F), slot, s));
    } else {
      DP_CK(normal_fill(q->qc.seed, kNoiseTensorId, (unsigned long long)q->next_id, slot,
                        q->chunk_numel, s));
    }
  }
  DP_TRY(upload_tables(q, pl));
  DP_TRY(run_step(q, pl));
  // bookkeeping after the pass
  if (pl.push) {
    q->levels.push_back(q->qc.T);
    q->next_id += 1;
  }
  for (int& j : q->levels) j -= 1;
  if (pl.writes_cache) {
    q->cache_id = pl.head;
    q->cache_cur = 1 - q->cache_cur;
  }
  while (!q->levels.empty() && q->levels.front() == 0) {
    q->levels.pop_front();
    q->head_id += 1;
  }
  q->step += 1;
  return DP_OK;
}

dp_status dp_queue_pop(dp_queue* q, float* out, dp_loc loc, long long* chunk_id) {
  clear_error();
  if (!q || !out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  if (q->ready_lo >= q->head_id) return fail(DP_ERR_EMPTY, "no clean chunk is ready");
  cudaStream_t s = q->m->stream;
  const float* slot = q->ring.as<float>() + (size_t)(q->ready_lo % q->n_slots) * q->chunk_numel;
  DP_CK(cudaMemcpyAsync(out, slot, (size_t)q->chunk_numel * 4,
                        loc == DP_LOC_HOST ? cudaMemcpyDeviceToHost : cudaMemcpyDeviceToDevice, s));
  if (chunk_id) *chunk_id = q->ready_lo;
  q->ready_lo += 1;
  if (loc == DP_LOC_HOST) {
    // the copy has been waited for anyway: report a kernel that gave up a
    // bounded wait (and skipped its work) instead of returning its result as good
    DP_CK(cudaStreamSynchronize(s));
    DP_TRY(check_status_word(q->m));
  }
  return DP_OK;
}

dp_status dp_queue_set_noise_pool(dp_queue* q, const float* pool, dp_loc loc) {
  clear_error();
  if (!q || !pool) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (q->qc.noise_mode != 1) return fail(DP_ERR_STATE, "the queue does not use coordinated noise");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  DP_CK(cudaMemcpyAsync(q->noise_pool.p, pool, (size_t)2 * q->chunk_numel * 4,
                        loc == DP_LOC_HOST ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice,
                        q->m->stream));
  DP_CK(cudaStreamSynchronize(q->m->stream));
  return DP_OK;
}

dp_status dp_queue_close(dp_queue* q) {
  clear_error();
  if (!q) return fail(DP_ERR_INVALID_ARG, "NULL queue");
  q->closed = true;
  return DP_OK;
}

dp_status dp_queue_sync(dp_queue* q) {
  clear_error();
  if (!q) return fail(DP_ERR_INVALID_ARG, "NULL queue");
  dp_model* m = q->m;
  DP_CK(cudaStreamSynchronize(m->stream));
  return check_status_word(m);
}

dp_status dp_queue_selftest_timeout(dp_queue* q) {
  clear_error();
  if (!q) return fail(DP_ERR_INVALID_ARG, "NULL queue");
  cudaError_t err = selftest_timeout(q->m->status.as<int>(), q->m->stream);
  if (err != cudaSuccess) return fail(DP_ERR_CUDA, "self test launch: %s", cudaGetErrorString(err));
  return DP_OK;
}

dp_status dp_queue_inspect(const dp_queue* q, dp_queue_info* info, long long* ids, int* levels,
                           int* slots, int* positions, int cap) {
  clear_error();
  if (!q || !info) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  memset(info, 0, sizeof(*info));
  info->step = q->step;
  info->n_ready = (int)(q->head_id - q->ready_lo);
  info->next_pop_id = info->n_ready > 0 ? q->ready_lo : -1;
  const bool push = pushing(q);
  info->next_push_id = push ? q->next_id : -1;
  std::vector<int> lv(q->levels.begin(), q->levels.end());
  if (push) lv.push_back(q->qc.T);
  info->n = (int)lv.size();
  info->drained = info->n == 0;
  if (info->n > 0) {
    info->head_pred = q->head_id == 0 ? kPredNone : kPredCache;
    info->writes_cache = lv[0] == 1;
  }
  for (int i = 0; i < info->n && i < cap; ++i) {
    if (ids) ids[i] = q->head_id + i;
    if (levels) levels[i] = lv[i];
    if (slots) slots[i] = (int)((q->head_id + i) % q->n_slots);
    if (positions) positions[i] = lv[i] - 1;
  }
  return DP_OK;
}

dp_status dp_queue_read_latents(dp_queue* q, float* out, int n, dp_loc loc) {
  clear_error();
  if (!q || !out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  if (n != (int)q->levels.size())
    return fail(DP_ERR_INVALID_ARG, "queue holds %d chunks, asked for %d", (int)q->levels.size(), n);
  cudaStream_t s = q->m->stream;
  for (int i = 0; i < n; ++i) {
    const float* slot = q->ring.as<float>() + (size_t)((q->head_id + i) % q->n_slots) * q->chunk_numel;
    DP_CK(cudaMemcpyAsync(out + (size_t)i * q->chunk_numel, slot, (size_t)q->chunk_numel * 4,
                          loc == DP_LOC_HOST ? cudaMemcpyDeviceToHost : cudaMemcpyDeviceToDevice, s));
  }
  DP_CK(cudaStreamSynchronize(s));
  return DP_OK;
}

dp_status dp_queue_load_state(dp_queue* q, long long step, long long n_pushed, int n,
                              const float* latents, const float* pred_kv, dp_loc loc) {
  clear_error();
  if (!q || (n > 0 && !latents)) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  const int T = q->qc.T;
  if (n < 0 || n > T || n_pushed < n || step < n_pushed || (q->qc.n_chunks >= 0 && n_pushed > q->qc.n_chunks))
    return fail(DP_ERR_INVALID_ARG, "inconsistent state (step %lld, pushed %lld, n %d)", step, n_pushed, n);
  // Every check comes before the first copy, so a rejected state leaves the
  // queue as it was.  A FIFO stream pushes chunk k at step k and chunk k
  // leaves after step k + T - 1; before step `step` the queued chunks are
  // therefore exactly [max(0, step - T + 1), n_pushed).
  const long long head = n_pushed - n;
  std::deque<int> lv;
  for (long long k = head; k < n_pushed; ++k) {
    const long long j = T - (step - k);
    if (j < 1 || j > T) return fail(DP_ERR_INVALID_ARG, "chunk %lld would be at level %lld", k, j);
    lv.push_back((int)j);
  }
  if (head != std::max(0LL, step - T + 1) && !(n == 0 && head <= step - T + 1))
    return fail(DP_ERR_INVALID_ARG,
                "chunks [%lld, %lld) at step %lld: chunk %lld has not left the queue yet", head, n_pushed,
                step, head - 1);
  // Pushes stop when n_chunks are in, or when the stream was closed; a state
  // past its last push (step > n_pushed) with pushes still allowed by n_chunks
  // is a closed stream, and is restored closed.
  const bool closed = step > n_pushed;
  dp_model* m = q->m;
  const size_t blk = (size_t)q->Lc * m->d;
  if (pred_kv && loc == DP_LOC_HOST && blk * 4 > m->staging.bytes)
    return fail(DP_ERR_INVALID_ARG, "predecessor block of %zu floats larger than the staging buffer", blk);
  cudaStream_t s = m->stream;
  const cudaMemcpyKind kind = loc == DP_LOC_HOST ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice;
  for (int i = 0; i < n; ++i) {
    float* slot = q->ring.as<float>() + (size_t)((head + i) % q->n_slots) * q->chunk_numel;
    DP_CK(cudaMemcpyAsync(slot, latents + (size_t)i * q->chunk_numel, (size_t)q->chunk_numel * 4, kind, s));
  }
  if (pred_kv) {
    // fp32 source layout [L][2][Lc][d] -> cache layout [L][Lc][2d]; host
    // blocks pass through the model's staging buffer one at a time
    for (int l = 0; l < m->L; ++l) {
      for (int kv = 0; kv < 2; ++kv) {
        const float* part = pred_kv + ((size_t)l * 2 + kv) * blk;
        const float* dsrc = part;
        if (loc == DP_LOC_HOST) {
          DP_CK(cudaMemcpyAsync(m->staging.p, part, blk * 4, cudaMemcpyHostToDevice, s));
          dsrc = m->staging.as<float>();
        }
        char* dst = q->cache[q->cache_cur].as<char>() +
                    ((size_t)l * q->Lc * 2 * m->d + (size_t)kv * m->d) * m->act_size();
        DP_CK(copy_rows(dsrc, 1, m->d, dst, m->f32 ? 1 : 0, 2 * m->d, q->Lc, m->d, s));
        if (loc == DP_LOC_HOST) DP_CK(cudaStreamSynchronize(s));
      }
    }
    q->cache_id = head - 1;
  } else {
    q->cache_id = -1;
  }
  DP_CK(cudaStreamSynchronize(s));
  q->step = step;
  q->next_id = n_pushed;
  q->head_id = head;
  q->ready_lo = head;
  q->levels = lv;
  q->closed = closed;
  return DP_OK;
}

dp_status dp_queue_read_pred_kv(dp_queue* q, float* out, dp_loc loc, long long* chunk_id) {
  clear_error();
  if (!q || !out) return fail(DP_ERR_INVALID_ARG, "NULL argument");
  if (loc != DP_LOC_DEVICE && loc != DP_LOC_HOST) return fail(DP_ERR_INVALID_ARG, "bad location");
  dp_model* m = q->m;
  cudaStream_t s = m->stream;
  const size_t blk = (size_t)q->Lc * m->d;
  for (int l = 0; l < m->L; ++l) {
    for (int kv = 0; kv < 2; ++kv) {
      const char* src = q->cache[q->cache_cur].as<char>() +
                        ((size_t)l * q->Lc * 2 * m->d + (size_t)kv * m->d) * m->act_size();
      float* dst = out + ((size_t)l * 2 + kv) * blk;
      float* ddst = loc == DP_LOC_HOST ? m->staging.as<float>() : dst;
      if (loc == DP_LOC_HOST && blk * 4 > m->staging.bytes)
        return fail(DP_ERR_INVALID_ARG, "predecessor block larger than staging");
      DP_CK(copy_rows(src, m->f32 ? 1 : 0, 2 * m->d, ddst, 1, m->d, q->Lc, m->d, s));
      if (loc == DP_LOC_HOST) {
        DP_CK(cudaMemcpyAsync(dst, ddst, blk * 4, cudaMemcpyDeviceToHost, s));
        DP_CK(cudaStreamSynchronize(s));
      }
    }
  }
  DP_CK(cudaStreamSynchronize(s));
  if (chunk_id) *chunk_id = q->cache_id;
  return DP_OK;
}

dp_status dp_queue_set_timing(dp_queue* q, int enable) {
  clear_error();
  if (!q) return fail(DP_ERR_INVALID_ARG, "NULL queue");
  if (q->timer.on) DP_TRY(q->timer.collect());
  q->timer.on = enable != 0;
  q->timer.reset();
  return DP_OK;
}

dp_status dp_queue_timing(dp_queue* q, int kclass, double* total_ms, long long* launches,
                          double* flops, double* bytes) {
  clear_error();
  if (!q || kclass < 0 || kclass >= DP_KCLASS_COUNT) return fail(DP_ERR_INVALID_ARG, "bad argument");
  DP_TRY(q->timer.collect());
  if (total_ms) *total_ms = q->timer.ms[kclass];
  if (launches) *launches = q->timer.n[kclass];
  if (flops) *flops = q->timer.fl[kclass];
  if (bytes) *bytes = q->timer.by[kclass];
  return DP_OK;
}

void dp_queue_destroy(dp_queue* q) {
  if (!q) return;
  if (q->m) {
    cudaStreamSynchronize(q->m->stream);
    q->m->queues.erase(q);
  }
  free_queue(q);
  delete q;
}

void dp_destroy(dp_model* m) {
  if (!m) return;
  cudaStreamSynchronize(m->stream);
  std::set<dp_queue*> qs = m->queues;
  for (dp_queue* q : qs) dp_queue_destroy(q);
  for (int i = 0; i < DP_PARAM_COUNT; ++i) dev_free(m->params[i].buf);
  dev_free(m->status);
  dev_free(m->staging);
  delete m;
}

}  // extern "C"
