/*
 * dp.h -- C ABI of a single-GPU (B200, sm_100a) block-wise FIFO video-denoising
 * queue in the style of DualParal.
 *
 * Method source: the DualParal write-up "双重并行：让AI视频生成突破时长限制，
 * 新加坡国立大学团队实现分钟级长视频创作" (techwalker.com), which describes
 * "Minute-Long Videos with Dual Parallelisms":
 *   §一  the video is cut into non-overlapping temporal chunks, each at its own
 *        noise level (later chunks noisier), and one inference step denoises
 *        all chunks together;
 *   §二  the chunks form a FIFO queue whose noise levels fall from T at the tail
 *        to 1 at the head; after each step every chunk moves one place forward,
 *        a new noisy chunk enters at the tail and the clean one leaves at the
 *        head; since a chunk holds a fixed number of frames, memory does not
 *        grow with video length;
 *   §三  in self-attention a chunk reuses its neighbour's cached K/V instead of
 *        concatenating the neighbour's input; cross-attention and the FFN are
 *        strictly per chunk.
 * On one GPU all T queued chunks run through the DiT as one batched pass.
 *
 * Conventions (all entry points):
 *   - Every call returns a dp_status and never aborts the process.  On error,
 *     dp_last_error() returns a message for the calling thread.
 *   - The library owns every device buffer it allocates; all allocation
 *     happens in dp_model_create, dp_model_set_param (none), dp_queue_init.
 *     dp_queue_step and dp_queue_pop allocate nothing, so device memory is
 *     flat in the length of the video.
 *   - Device work is enqueued on the stream given to dp_model_create and is
 *     asynchronous unless stated otherwise; host buffers passed with
 *     DP_LOC_HOST are read/written with stream-ordered copies and the call
 *     returns once the copy has completed (host memory may be reused).
 *   - Pointers marked "device" must be device memory of the model's device;
 *     pointers marked by a dp_loc follow that location.
 *   - Nothing here is sharded across GPUs and no collective runs.  Several
 *     GPUs serve independent queues (replicas).
 */
#ifndef DP_H
#define DP_H

#include <stddef.h>

/* Exported symbols of the shared library (built with hidden default visibility). */
#if defined(__GNUC__)
#define DP_API __attribute__((visibility("default")))
#else
#define DP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DP_OK = 0,
  DP_ERR_INVALID_ARG = 1,  /* a NULL pointer, a size out of range or a bad enum */
  DP_ERR_OOM = 2,          /* a device or pinned-host allocation failed        */
  DP_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                */
  DP_ERR_EMPTY = 4,        /* dp_queue_pop: no clean chunk is waiting          */
  DP_ERR_FULL = 5,         /* dp_queue_step: a push is due but ready_capacity
                              clean chunks are waiting to be popped            */
  DP_ERR_DRAINED = 6,      /* dp_queue_step: every chunk has left the queue     */
  DP_ERR_STATE = 7,        /* call out of order (e.g. parameters missing)      */
  DP_ERR_KERNEL = 8        /* a kernel reported a bounded wait that timed out
                              (device status word set); the context stays usable */
} dp_status;

typedef enum {
  DP_PREC_BF16 = 0,           /* production: bf16 operands, fp32 accumulate,
                                 fp32 residual stream and latents           */
  DP_PREC_FP32_VALIDATE = 1   /* fp32 operands, fp32 FFMA accumulation
                                 everywhere (no TF32)                       */
} dp_precision;

typedef enum {
  DP_LOC_DEVICE = 0,
  DP_LOC_HOST = 1
} dp_loc;

/* Which neighbours a chunk's self-attention reads besides its own tokens.
 * PRED: the preceding chunk k-1 (its K/V from this pass, or persisted from the
 * previous step once it has left the queue).  BOTH: also the following chunk
 * k+1 when it is queued in the same pass (the chunk pushed last has none). */
typedef enum {
  DP_NEIGHBOURS_PRED = 0,
  DP_NEIGHBOURS_BOTH = 1
} dp_neighbours;

/* Model shape.  dim % n_heads == 0; head_dim = dim / n_heads must be 16, 32,
 * 64 or 128 (the production path needs 64 or 128); freq_dim even;
 * patch = patch_t x patch_h x patch_w over latent_ch channels. */
typedef struct {
  int n_layers;
  int dim;
  int n_heads;
  int ffn_dim;
  int freq_dim;     /* width of the sinusoidal timestep features */
  int latent_ch;
  int patch_t, patch_h, patch_w;
  int text_len;     /* prompt tokens                                  */
  int text_in_dim;  /* prompt feature width; != dim adds a projection */
  dp_precision prec;
  dp_neighbours neighbours;
  int qk_norm_rope;  /* 1: self-attention q and k get a per-head RMSNorm (eps 1e-6,
                        weights L_QNORM_W / L_KNORM_W) and 3-D rotary positions
                        (temporal = chunk id * frames + frame, row, column; the
                        head_dim/2 pairs split into temporal / height / width
                        bands, height = width = floor(head_dim/6) pairs) */
} dp_model_config;

/* Queue shape.  One chunk = latent_ch x frames_per_chunk x lat_h x lat_w fp32,
 * laid out [C][F][H][W] row-major. */
typedef struct {
  int T;                  /* number of noise levels = queue length (>= 1)    */
  int frames_per_chunk;   /* multiple of patch_t                            */
  int lat_h, lat_w;       /* multiples of patch_h, patch_w                  */
  long long n_chunks;     /* chunks in the stream; -1 = until dp_queue_close */
  int ready_capacity;     /* clean chunks that may wait for dp_queue_pop (>=1) */
  unsigned long long seed;/* seed of the internal noise generator           */
  int noise_mode;         /* initial latent of a chunk pushed without caller
                             noise: 0 = fresh N(0,1) per chunk; 1 = coordinated:
                             from a pool of 2F noise frames, the F frames the
                             previous chunk did not use (frames 0..F-1 for even
                             chunk ids, F..2F-1 for odd), in a Fisher-Yates order
                             driven by SplitMix64 stream (seed, 1002, chunk id) */
} dp_queue_config;

/* Parameters.  Linear weights are [out][in] row-major fp32; biases [out].
 * Per-layer entries (DP_L_*) are set once per layer index.  Shapes, with
 * d = dim, F = ffn_dim, D = freq_dim, P = latent_ch*patch_t*patch_h*patch_w:
 *   PATCH_W [d][P]  PATCH_B [d]      TEXT_W [d][text_in_dim]  TEXT_B [d]
 *   TIME1_W [d][D]  TIME1_B [d]      TIME2_W [d][d]  TIME2_B [d]
 *   MOD_W [6d][d]   MOD_B [6d]       HEADMOD_W [2d][d] HEADMOD_B [2d]
 *   OUT_W [P][d]    OUT_B [P]
 *   L_MOD [6d]  L_QKV_W [3d][d] L_QKV_B [3d]  L_O_W [d][d] L_O_B [d]
 *   L_CQ_W, L_CK_W, L_CV_W, L_CO_W [d][d] with biases [d]
 *   L_FFN1_W [F][d] L_FFN1_B [F]  L_FFN2_W [d][F] L_FFN2_B [d]
 *   L_QNORM_W [d] L_KNORM_W [d] (only with qk_norm_rope)
 * TEXT_* exist only when text_in_dim != dim. */
typedef enum {
  DP_PATCH_W = 0, DP_PATCH_B, DP_TEXT_W, DP_TEXT_B,
  DP_TIME1_W, DP_TIME1_B, DP_TIME2_W, DP_TIME2_B,
  DP_MOD_W, DP_MOD_B, DP_HEADMOD_W, DP_HEADMOD_B, DP_OUT_W, DP_OUT_B,
  DP_L_MOD, DP_L_QKV_W, DP_L_QKV_B, DP_L_O_W, DP_L_O_B,
  DP_L_CQ_W, DP_L_CQ_B, DP_L_CK_W, DP_L_CK_B, DP_L_CV_W, DP_L_CV_B,
  DP_L_CO_W, DP_L_CO_B, DP_L_FFN1_W, DP_L_FFN1_B, DP_L_FFN2_W, DP_L_FFN2_B,
  DP_L_QNORM_W, DP_L_KNORM_W,
  DP_PARAM_COUNT
} dp_param;

typedef struct dp_model dp_model;
typedef struct dp_queue dp_queue;

/* Optional device allocator (e.g. a framework's caching allocator).  NULL
 * alloc restores cudaMalloc/cudaFree.  Applies to models and queues created
 * afterwards; the library frees each buffer with the allocator that made it. */
typedef void* (*dp_alloc_fn)(size_t bytes, void* ctx);
typedef void (*dp_free_fn)(void* ptr, void* ctx);
DP_API dp_status dp_set_allocator(dp_alloc_fn alloc, dp_free_fn free_fn, void* ctx);

/* Number of elements of parameter `id` for this config (0 if absent). */
DP_API dp_status dp_param_numel(const dp_model_config* cfg, dp_param id, long long* numel);

/* Creates a model on the current CUDA device and allocates its weights.
 * The model is the per-chunk-timestep DiT of the write-up's section 一 (every
 * chunk of the queue carries its own noise level into the block's adaLN).
 * `cuda_stream` is a cudaStream_t (NULL = legacy default stream) on which all
 * later work of this model and its queues runs. */
DP_API dp_status dp_model_create(const dp_model_config* cfg, void* cuda_stream, dp_model** out);

/* Copies one parameter (fp32, `numel` elements, from host or device memory)
 * into the model, converting to the compute precision.  `layer` is ignored for
 * non-layer parameters.  Every parameter must be set before dp_queue_init. */
DP_API dp_status dp_model_set_param(dp_model* m, dp_param id, int layer, const float* src,
                             long long numel, dp_loc loc);

/* Starts a queue (section 二: a FIFO of chunks, levels T at the tail down to 1
 * at the head; section 三: the prompt's cross-attention K/V serve every chunk
 * and every step, so they are projected once, here).
 * Allocates the latent ring (T + ready_capacity chunk slots),
 * the activations for T chunks and the double-buffered predecessor K/V cache;
 * projects the prompt `text` ([text_len][text_in_dim] fp32) to the per-layer
 * cross-attention K/V once; builds the per-level modulation tables.  The queue
 * starts empty.  Synchronous. */
DP_API dp_status dp_queue_init(dp_model* m, const dp_queue_config* qc, const float* text,
                        dp_loc text_loc, dp_queue** out);

/* One queue step (section 二: every queued chunk is denoised once and moves one
 * place toward the head, a noisy chunk enters at the tail, the clean one
 * leaves at the head; section 三: a chunk's self-attention reads its
 * neighbour's K/V next to its own, never a concatenated input).
 * If a chunk is due (fewer than n_chunks pushed and the queue
 * not closed), it is pushed at the tail at level T first, its latent taken
 * from `new_chunk_noise` ([C][F][H][W] fp32 at `loc`), or drawn N(0,1) by the
 * internal generator when `new_chunk_noise` is NULL.  Then every queued chunk
 * runs through the DiT once, is advanced by one Euler step
 * x <- x + (sigma_{j-1} - sigma_j) v with sigma_j = j/T, and drops one level;
 * the chunk that reaches level 0 becomes ready for dp_queue_pop.
 * Errors: DP_ERR_FULL (push due, no free slot: pop first), DP_ERR_DRAINED
 * (nothing left to denoise), DP_ERR_STATE (the persisted K/V the head needs
 * are missing); after these nothing was enqueued and the queue is unchanged.
 * DP_ERR_CUDA / DP_ERR_INVALID_ARG from a failed launch inside the step leave
 * part of the step enqueued: the queue must then be destroyed (or reloaded
 * with dp_queue_load_state).  A queue is not safe to use from several host
 * threads at once.
 * Ownership: a host `new_chunk_noise` (pageable or page-locked) is copied into
 * the queue's pinned staging before the call returns and may be reused at
 * once; a device one is read in stream order, so it must not be overwritten
 * before the step has run (dp_queue_sync, or a later event on the stream). */
DP_API dp_status dp_queue_step(dp_queue* q, const float* new_chunk_noise, dp_loc loc);

/* Pop at the head of the FIFO (section 二: the clean chunk leaves for the
 * decoder).  Copies the oldest ready chunk ([C][F][H][W] fp32) to `out` at
 * `loc` and frees its slot; `chunk_id` (may be NULL) receives its id.  Chunk
 * ids pop in strictly increasing order.  DP_ERR_EMPTY if none is ready.  A
 * host `out` is complete when the call returns: the call waits for the stream
 * and then checks the device status word, returning DP_ERR_KERNEL (the chunk
 * is still consumed and `chunk_id` set) if a kernel gave up a bounded wait
 * since the last check, because the chunk may then hold skipped work; reload
 * the queue (dp_queue_load_state) or destroy it.  A device `out` is written in
 * stream order and not checked: call dp_queue_sync for that. */
DP_API dp_status dp_queue_pop(dp_queue* q, float* out, dp_loc loc, long long* chunk_id);

/* Coordinated noise initialisation (section 三: a new chunk's noise comes from
 * a pool, avoiding the frames its neighbour used, shuffled).
 * Replaces the coordinated-noise pool (noise_mode 1) with `pool`
 * ([2F][C][H][W] fp32 at `loc`).  By default the pool is drawn N(0,1) on the
 * device at dp_queue_init (frame b from stream (seed, 1003, b)).  Synchronous. */
DP_API dp_status dp_queue_set_noise_pool(dp_queue* q, const float* pool, dp_loc loc);

/* Ends an unbounded stream: no further chunk is pushed; steps drain the queue. */
DP_API dp_status dp_queue_close(dp_queue* q);

/* Waits for the queue's stream and checks the device status word.  Returns
 * DP_ERR_KERNEL if a kernel gave up a bounded wait since the last check. */
DP_API dp_status dp_queue_sync(dp_queue* q);

/* Exercises the failure path of the queue's bounded waits: enqueues on the
 * queue's stream one block that waits on an mbarrier nothing arrives at, gives
 * up after the kernels' wait limit (2 s), sets the queue's status word and
 * returns; nothing faults and the queue's data is untouched.  The next
 * dp_queue_sync or host dp_queue_pop then reports DP_ERR_KERNEL once. */
DP_API dp_status dp_queue_selftest_timeout(dp_queue* q);

/* Bookkeeping of the FIFO (section 二) for the NEXT step, as dp_queue_step
 * would run it now (including
 * the chunk it would push).  Arrays hold up to `cap` entries, head first:
 * chunk ids, levels (1..T), ring slots and queue positions (level - 1).
 * head_pred: 0 = none (head is chunk 0), 2 = persisted K/V of the chunk that
 * left last step.  writes_cache: the head is at level 1, so its K/V are kept
 * for the next step.  Exact integers. */
typedef struct {
  long long step;          /* index of the next step (0-based)         */
  long long next_push_id;  /* id of the chunk pushed next, -1 if none  */
  int n;                   /* queued chunks in the next step           */
  int head_pred;
  int writes_cache;
  int n_ready;             /* clean chunks waiting for dp_queue_pop     */
  long long next_pop_id;   /* -1 if none ready                          */
  int drained;             /* 1 if no step remains                      */
} dp_queue_info;
DP_API dp_status dp_queue_inspect(const dp_queue* q, dp_queue_info* info, long long* ids,
                           int* levels, int* slots, int* positions, int cap);

/* Latents of the chunks queued now (head first) to `out` [n][C][F][H][W]
 * fp32 at `loc`; `n` must equal the current number of queued chunks.  These
 * are the chunks after the last step (levels already lowered), before the
 * next push.  Synchronous.  For tests and checkpoints. */
DP_API dp_status dp_queue_read_latents(dp_queue* q, float* out, int n, dp_loc loc);

/* Sets the queue to the state it would have before step `step` of a stream
 * that has pushed `n_pushed` chunks: the queued chunks are ids
 * [n_pushed - n, n_pushed) with latents `latents` ([n][C][F][H][W] fp32 at
 * `loc`) and levels taken from the FIFO schedule; `pred_kv` ([n_layers][2]
 * [tokens_per_chunk][dim] fp32, K then V per layer, or NULL) are the persisted
 * self-attention K/V of chunk n_pushed - n - 1.  No chunk is ready after it.
 * Synchronous.  For per-step parity tests and resuming a checkpoint.
 * Only states a FIFO stream reaches are accepted (DP_ERR_INVALID_ARG
 * otherwise, with the queue unchanged): chunk k is pushed at step k and leaves
 * after step k + T - 1, so before `step` the queued chunks must be exactly
 * [max(0, step - T + 1), n_pushed), with step >= n_pushed.  A state with
 * step > n_pushed has stopped pushing: it is restored closed (as after
 * dp_queue_close); with step == n_pushed the queue is open and pushes while
 * n_chunks allows (call dp_queue_close after loading to end it there).  Leaving
 * `pred_kv` NULL while the head chunk has a predecessor makes the next step
 * fail with DP_ERR_STATE. */
DP_API dp_status dp_queue_load_state(dp_queue* q, long long step, long long n_pushed, int n,
                              const float* latents, const float* pred_kv, dp_loc loc);

/* Persisted predecessor K/V to `out` ([n_layers][2][tokens][dim] fp32 at
 * `loc`); `chunk_id` receives the id they belong to (-1 if none). Synchronous. */
DP_API dp_status dp_queue_read_pred_kv(dp_queue* q, float* out, dp_loc loc, long long* chunk_id);

/* Per-kernel-class device timing with CUDA events on the queue's stream.
 * Classes: 0 GEMM (tensor cores in bf16), 1 self-attention, 2 cross-attention,
 * 3 layer norm + modulation, 4 patch embed, 5 head + Euler, 6 other.
 * Enabling resets the counters.  `flops` is the algorithmic FLOP count of the
 * launches timed (0 for memory-bound classes); `bytes` their algorithmic
 * HBM bytes (0 for contractions). */
#define DP_KCLASS_COUNT 7
DP_API dp_status dp_queue_set_timing(dp_queue* q, int enable);
DP_API dp_status dp_queue_timing(dp_queue* q, int kclass, double* total_ms, long long* launches,
                          double* flops, double* bytes);

/* Releases one queue (its device memory). */
DP_API void dp_queue_destroy(dp_queue* q);
/* Releases a model and every queue still attached to it. */
DP_API void dp_destroy(dp_model* m);

/* Message of the last error on the calling thread ("" if none). */
DP_API const char* dp_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DP_H */
