/*
 * rc.h -- C ABI of the bounded ("rolling") KV cache for block-autoregressive
 * video diffusion on NVIDIA B200 (sm_100a).
 *
 * One call, rc_step, runs the per-chunk attention step the pages describe:
 * rotate the new chunk's queries and keys with a 3D (t, h, w) RoPE at their
 * assigned time index, append the chunk's K/V to a cache that pins sink
 * frames and evicts the oldest window frames, and run the chunk's queries
 * through softmax attention over sink + window + the chunk itself.
 *
 * Passages that define the operations (page title, section):
 *   - Causal-Forcing inference walkthrough (lqnn.cn), section 3 "KV Cache":
 *     per-layer k/v buffers [B, kv_cache_size, 12, 128] plus the two cursors
 *     global_end_index / local_end_index; only the current block's queries
 *     are computed; new frames' roped keys and values are appended;
 *     causal_rope_apply(start_frame) gives new frames their absolute time.
 *   - LingBot-World 2.0 rolling-cache explainer (icman.com.cn), sections
 *     "local_attn_size 滑动窗口", "sink_size 注意力汇聚" and the two
 *     easily-missed details: fixed-size cache of local_attn_size frames,
 *     num_evicted = new + local_end - capacity, the first sink_size frames
 *     never move, rolling fires only when the forward adds new content,
 *     attention reads the window up to local_end.
 *   - rCM length-extrapolation guide (dpshk.com), strategies 1-3: sliding
 *     window with sink blocks, Rolling Sink, Infinity-RoPE (block-relative
 *     time, clamp at 0, KV flush, RoPE cut); the cache bound is computed up
 *     front and preallocated. Strategy 4, Deep Forcing (deep sink + top-C
 *     tokens by attention score + recent tail, time encodings rewritten so no
 *     holes remain) and strategy 5, Relax Forcing (sink + history frames
 *     chosen by w * alignment + (1 - w) * complementarity + tail).
 *   - Rolling Sink digest (paper.rainbus.top/paper/2602.07775), method-step
 *     details: sink time indices slide to [i-K, i-(K-S)); sink content is a
 *     length-S segment of Roll(x_[0,K)), forward on even cycles, reversed on
 *     odd cycles; K=6, S=5.
 *
 * Conventions
 *   - Ownership: every device pointer (q, k_new, v_new, out, lse, scores,
 *     topc and the cache memory block) belongs to the caller. The library
 *     never frees them and keeps no pointer to q/k/v/out after a call
 *     returns; it keeps the cache block until rc_cache_destroy.
 *   - Asynchrony: device work is enqueued on the caller's stream
 *     (a cudaStream_t passed as void*, NULL = legacy default stream). Host
 *     state advances at enqueue time. Calls on one handle are not
 *     thread-safe; distinct handles are independent.
 *   - Layouts: q, k_new, v_new and out are [n_frames * frame_seqlen, heads,
 *     head_dim] bf16, contiguous, 16-byte aligned (token-major, as a DiT
 *     layer produces them). lse is [heads, n_frames * frame_seqlen] fp32.
 *   - Errors: every function returns an rc_status. Nothing throws across
 *     the ABI. rc_last_error() gives a message for the calling thread's
 *     last failure. On RC_EINVAL / RC_ESTATE / RC_ERANGE the cache state is
 *     unchanged and nothing was enqueued.
 */
#ifndef RC_H_
#define RC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rc_status {
  RC_OK = 0,
  RC_EINVAL = 1,    /* bad argument or config */
  RC_ESTATE = 2,    /* frame_start neither repeats the last chunk nor continues the stream */
  RC_ECUDA = 3,     /* a CUDA runtime/driver call failed */
  RC_ERANGE = 4,    /* a time index, size or count exceeds the configured maximum */
  RC_ETIMEOUT = 5,  /* a device-side bounded wait gave up (see rc_device_status) */
  RC_ENOMEM = 6     /* the caller's memory block is smaller than rc_cache_bytes() */
} rc_status;

typedef enum rc_policy {
  RC_NONE = 0,           /* unbounded baseline: keep every frame (capacity must cover the video) */
  RC_SLIDING = 1,        /* sliding window + attention sink (rCM strategy 1, LingBot) */
  RC_ROLLING_SINK = 2,   /* Rolling Sink: bank roll + sliding sink time indices */
  RC_INFINITY_ROPE = 3,  /* Infinity-RoPE: block-relative time, clamp at 0, flush + cut */
  RC_DEEP_FORCING = 4,   /* Deep Forcing: deep sink + top-C scored tokens + recent tail
                            (rCM length-extrapolation guide, strategy 4); see below */
  RC_RELAX_FORCING = 5,  /* Relax Forcing: sink + K history frames chosen by cosine
                            similarity + recent tail (strategy 5); see below */
  RC_MEMROPE = 6         /* MemRoPE: sink + long/short EMA memory frames of the evicted
                            frames + window (strategy 5's MemRoPE tip); see below */
} rc_policy;

/* rc_reindex flags */
#define RC_REINDEX_FLUSH 1u  /* Infinity-RoPE KV flush: keep sink + last block, drop the middle */
#define RC_REINDEX_CUT   2u  /* Infinity-RoPE RoPE cut: add t_delta to the time of all later frames */
#define RC_REINDEX_SINK  4u  /* sliding / none: add t_delta to the sink frames' time index */

#define RC_MAX_SLOTS 256        /* sink_frames + window_frames */
#define RC_MAX_CHUNK_FRAMES 16  /* chunk_frames */

typedef struct rc_config {
  int layers;             /* independent caches sharing one schedule */
  int heads;              /* attention heads per layer */
  int head_dim;           /* 64 or 128 */
  int frame_seqlen;       /* tokens per latent frame, = grid_h * grid_w */
  int grid_h, grid_w;     /* latent token grid of a frame; token n sits at (n / grid_w, n % grid_w) */
  int sink_frames;        /* pinned frames at the head of the cache (inside the footprint) */
  int window_frames;      /* rolling frames, including the current chunk */
  int chunk_frames;       /* frames per rc_step (the block size of block policies) */
  int mask_block_frames;  /* mask inside the current chunk: query frame r sees chunk frames
                             r' with r'/m <= r/m; 1 = frame-causal (default), chunk_frames = none */
  int rope_t_pairs, rope_h_pairs, rope_w_pairs;  /* 0,0,0 = default split of head_dim/2 pairs:
                             h = w = floor(c/3), t = c - 2 floor(c/3) */
  double theta;           /* RoPE base, default 10000 */
  int t_max;              /* largest RoPE time index + 1 the cache may use (table size) */
  rc_policy policy;
  int rs_bank_blocks;     /* Rolling Sink K: bank = first K blocks */
  int rs_sink_blocks;     /* Rolling Sink S: sink_frames must equal S * chunk_frames and
                             window_frames (K - S + 1) * chunk_frames */
  int rs_static_semantics;/* 1 = stage 2 only (sink shows blocks 0..S-1 at sliding times) */
  int ir_f_limit;         /* Infinity-RoPE: the newest block ends at time index f_limit */
  int ir_sink_blocks;     /* Infinity-RoPE: global sink blocks (sink_frames = this * chunk_frames) */
  int ir_cache_blocks;    /* Infinity-RoPE: blocks kept before the current one, sink included
                             (window_frames = (cache - sink + 1) * chunk_frames) */
  int df_budget_tokens;   /* Deep Forcing: tokens of the compressed region (a multiple of
                             frame_seqlen); sink_frames = deep sink, window_frames = recent
                             tail including the current chunk (>= 2 chunks) */
  int rf_history_frames;  /* Relax Forcing: K, history frames kept between sink and tail */
  double rf_weight;       /* Relax Forcing: w in score = w * alignment + (1 - w) * complement */
  double mr_alpha_long;   /* MemRoPE: EMA factor of the long-term memory frame */
  double mr_alpha_short;  /* MemRoPE: EMA factor of the short-term memory frame */
} rc_config;

/* MemRoPE (rCM length-extrapolation guide, the MemRoPE tip under strategy 5):
 * the cache is the sliding window (sink_frames + window_frames) plus two
 * memory frames. Every frame that leaves the window, oldest first, is folded
 * token by token into both memories, per head, for raw keys and values:
 * M = a M + (1 - a) X with a = mr_alpha_long / mr_alpha_short (the first
 * evicted frame initialises them), in fp32 on the device. Keys are kept raw and
 * positioned for attention at every step: the long-term memory at time
 * sink_frames (right after the sink), the short-term one at g_w - 1 (right
 * before the first window frame g_w), each token at its own (h, w).
 * rc_get_state lists them as history entries with content -1 (long) and -2
 * (short). Chunks are whole blocks. */

/* Relax Forcing (rCM length-extrapolation guide, strategy 5): the cache keeps
 * the sink (the first sink_frames frames), at most rf_history_frames history
 * frames and the recent tail (the newest window_frames frames up to the
 * current chunk's end). When a new chunk pushes the tail's oldest frames out
 * they join the history frames in a pool; if the pool holds more than K frames
 * the K with the highest score = w * alignment + (1 - w) * complement stay
 * (ties to the older frame), in time order. A frame's descriptor is the mean
 * over its tokens of its raw key, heads concatenated; alignment = cosine with
 * the mean descriptor of the tail (the new chunk included); complement = 1 -
 * the mean cosine with the other pool frames. Every frame keeps its own
 * absolute time index (nothing is re-rotated). Chunks are whole blocks. */

/* Deep Forcing (rCM length-extrapolation guide, strategy 4): the cache keeps
 * the deep sink (the first sink_frames frames), a compressed region of at most
 * df_budget_tokens tokens chosen by attention score, and the recent tail (the
 * newest window_frames frames up to the current chunk's end). Every rc_step
 * scores the cached tokens (the softmax mass each key receives, summed over
 * heads and queries, as rc_step's scores output). When a new chunk pushes the
 * tail's oldest frames out, they join the compressed region's tokens in a pool
 * and the df_budget_tokens highest-scoring pool tokens (scores of the last
 * step before the chunk, ties to the lower index) form the new region, in
 * time order. Time indices leave no holes: tail and chunk frames keep tau = g;
 * with g_t the first tail frame and V = region tokens / frame_seqlen, region
 * token i has tau = g_t - V + i / frame_seqlen and sink frame j has
 * tau = g_t - V - sink_frames + j, so sink, region and tail sit on
 * consecutive time positions; the region's and the sink's keys are rotated to
 * their new times on the device (the page's in-place rope_time_delta_).
 * Chunks are whole blocks of chunk_frames frames. */

/* Fill *cfg with defaults for the pages' short signature
 * (layers, heads, head_dim, frame_seqlen, sink_frames, window_frames):
 * sliding policy, chunk 3 frames, frame-causal chunk mask, theta 1e4,
 * t_max 4096, grid 1 x frame_seqlen (set grid_h/grid_w for a 2D grid). */
rc_status rc_config_init(rc_config* cfg, int layers, int heads, int head_dim,
                         int frame_seqlen, int sink_frames, int window_frames);

/* Bytes of device memory a cache with this config needs (K/V ring buffers
 * of every layer, pristine sources of the block policies, RoPE tables and
 * the step's scratch). The caller allocates them, 256-byte aligned. */
rc_status rc_cache_bytes(const rc_config* cfg, size_t* bytes);

/* Create a cache handle over the caller's memory block. dev_mem == NULL
 * creates a host-only handle: it tracks the cache state exactly as a device
 * handle would, enqueues nothing, and rc_step must then get NULL tensors.
 * A device handle zeroes its block and uploads the RoPE tables on the
 * current device's legacy default stream, then synchronizes. */
rc_status rc_cache_create(const rc_config* cfg, void* dev_mem, size_t bytes, void** out_handle);

/* Run one chunk through one layer.
 *   frame_start: stream frame index of the chunk's first frame. Equal to the
 *     layer's previous frame_start = another denoise pass of the same chunk
 *     (overwrites it, evicts nothing); equal to the layer's committed end =
 *     a new chunk; anything else = RC_ESTATE.
 *   n_frames: frames in this chunk (1..chunk_frames; block policies need
 *     exactly chunk_frames).
 *   policy: must equal cfg->policy (stated at each call site).
 *   q, k_new, v_new: [n_frames*F, heads, head_dim] bf16 device, read only.
 *   out: [n_frames*F, heads, head_dim] bf16 device, written.
 *   lse: NULL or [heads, n_frames*F] fp32 device (natural-log logsumexp of
 *     the scaled scores), written.
 *   scores / topc / C: NULL/NULL/0, or the Deep-Forcing token scores: scores
 *     [n_candidates] fp32 device receives, for every cached token that is
 *     neither sink nor current (logical order: oldest frame first, token in
 *     frame), the softmax mass it received summed over heads and queries;
 *     topc [C] int32 device receives the logical indices (over the whole
 *     kept list) of the C highest-scoring candidates, ties to the lower
 *     index, sorted ascending (fewer than C candidates: the tail is -1).
 *     rc_get_state reports n_candidates.
 *   stream: cudaStream_t as void*.
 */
rc_status rc_step(void* handle, int layer, const void* q, const void* k_new, const void* v_new,
                  int frame_start, int n_frames, rc_policy policy, void* out, float* lse,
                  float* scores, int32_t* topc, int C, void* stream);

/* Top-C over a score vector the caller supplies, in the candidate order of
 * `layer`'s last rc_step. For a stream whose heads are split across GPUs
 * (each rank's cache holds a head range, and its rc_step scores only those
 * heads): the ranks sum their score vectors with one all-reduce and select
 * from the sum. The selection is rc_step's (rCM length-extrapolation guide,
 * strategy 4, Deep Forcing: keep the candidate tokens with the highest
 * attention scores): ties to the lower index, output ascending, -1 tail when
 * there are fewer than C candidates.
 *   scores: [n_candidates] fp32 device, read only, in rc_step's scores order
 *     (rc_get_state reports n_candidates).
 *   topc: [C] int32 device, written: logical indices over the kept list.
 * Errors: RC_EINVAL (host-only handle, null pointer, C <= 0, bad layer),
 * RC_ESTATE (no rc_step has run on the layer). Enqueued on `stream`. */
rc_status rc_select_topc(void* handle, int layer, const float* scores, int C, int32_t* topc, void* stream);

/* rc_step for callers that cannot allocate device memory. The pages have no
 * counterpart; this is a deployment convenience.
 *
 * rc_step keeps each call's scratch (the rotated queries of the chunk, the
 * log-sum-exps the token scores need, and the score work buffers) inside the
 * caller's memory block. Some callers cannot provide device memory at all:
 * code that runs where no allocator may be called (a plugin handed a fixed
 * budget by its host, a real-time loop that forbids allocation after start-up,
 * a runtime whose memory accounting the library must not touch). For them this
 * entry point places that scratch in one array inside the library's own device
 * image instead (a file-scope __device__ array of 16 MiB, 256-byte aligned),
 * which every GPU that loads the library holds until the process exits. It
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments, layouts and results are those of rc_step. Differences:
 *   - Only device handles: a host-only handle (dev_mem == NULL) is rejected
 *     with RC_EINVAL (rc_step accepts it and only advances the state).
 *   - The scratch a call needs is heads * chunk_frames * frame_seqlen *
 *     (head_dim * 2 + 4) bytes (rotated queries and log-sum-exps) plus 8
 *     bytes per cache row for the two token-score buffers, each part rounded
 *     up to 256 bytes. The cache rows per head are rc_cache_layout's
 *     `capacity`: (sink_frames + window_frames) * frame_seqlen, plus
 *     2 * df_budget_tokens (Deep Forcing) or 2 * rf_history_frames *
 *     frame_seqlen (Relax Forcing), plus 2 * frame_seqlen (MemRoPE). A config
 *     needing more than 16 MiB is rejected with RC_ERANGE before anything is
 *     planned or enqueued (e.g. 12 heads x 128 with 4680-token chunks fits;
 *     40 heads does not).
 *   - The attention runs with one CTA per (head, 256-query block) and never
 *     splits a block between CTAs, so it needs no partial-result rows; with
 *     more blocks than SMs it runs in several waves.
 *   - Only the rotated queries, log-sum-exps and token-score buffers move to
 *     the static array. The device status word and, under Relax Forcing, the
 *     chunk's frame descriptors stay in the caller's block, as in rc_step.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current) and remembers it; make
 *     that first call before any stream capture.
 *   - Every call, from every handle on the device, shares the one array, which
 *     keeps the last call's contents (whatever must start at zero is cleared
 *     by the call itself). Calls whose work overlaps on the GPU -- different
 *     streams without ordering between them -- race on it: order them.
 *   - Errors: those of rc_step, plus RC_EINVAL for a host-only handle and
 *     RC_ERANGE for a config beyond the static maximum.
 */
rc_status rc_step_noalloc(void* handle, int layer, const void* q, const void* k_new,
                          const void* v_new, int frame_start, int n_frames, rc_policy policy,
                          void* out, float* lse, float* scores, int32_t* topc, int C, void* stream);

/* Sink / time-index rewrites between chunks, applied to every layer at its
 * next new chunk: RC_REINDEX_FLUSH and/or RC_REINDEX_CUT (Infinity-RoPE),
 * RC_REINDEX_SINK (sliding / none, t_delta added to the sink's time index).
 * The re-rotation of cached keys runs inside that next rc_step, on its
 * stream; `stream` is accepted for symmetry and may be NULL. */
rc_status rc_reindex(void* handle, rc_policy policy, int t_delta, unsigned flags, void* stream);

typedef struct rc_frame_state {
  int32_t content;      /* stream frame whose raw k/v the entry holds */
  int32_t tau;          /* RoPE time index the policy assigns */
  int32_t region;       /* 0 sink, 1 history, 2 current chunk */
  int32_t rank;         /* chunk-relative frame of a current entry, -1 otherwise */
  int32_t slot;         /* physical frame slot of the ring buffer */
  int32_t stored_time;  /* time index its keys are rotated to in memory (= tau + shift) */
} rc_frame_state;

typedef struct rc_state {
  int32_t n_kept;            /* entries below, logical order: sink, history (oldest first), current */
  int32_t frames_committed;  /* stream frames appended so far */
  int32_t chunk_start;       /* frame_start of the last rc_step */
  int32_t chunk_frames;      /* n_frames of the last rc_step */
  int32_t valid_tokens;      /* n_kept * frame_seqlen */
  int32_t shift;             /* stored_time - tau for unclamped frames (Infinity-RoPE), else 0 */
  int32_t n_candidates;      /* tokens scored by rc_step (history region) */
  int32_t n_jobs;            /* re-rotation jobs the last rc_step ran */
  int32_t evicted[RC_MAX_SLOTS];  /* contents that left the cache at the last new chunk */
  int32_t n_evicted;
  rc_frame_state kept[RC_MAX_SLOTS];
  int32_t comp_tokens;       /* Deep / Relax Forcing: tokens in the selected region (logically
                                between the sink and the tail frames; 0 for other policies) */
  int32_t comp_tau0;         /* Deep Forcing: region token i has tau = comp_tau0 + i / frame_seqlen;
                                Relax Forcing: -1 (each region frame keeps its own index) */
  int32_t comp_row0;         /* Deep / Relax Forcing: physical row (per head) of region token 0 in the K/V
                                buffers (rows past the ring: (sink + window) * F + b * budget) */
} rc_state;

/* Copy a layer's cache state (after its last rc_step) to host memory. */
rc_status rc_get_state(const void* handle, int layer, rc_state* out);

/* Deep Forcing / Relax Forcing: the source of each token of a layer's
 * selected region (Deep Forcing's compressed tokens, Relax Forcing's history
 * frames), in region order: frame[i] = stream frame, tok[i] = token index in
 * that frame (row-major h, w). frame and tok are host arrays of at least
 * rc_state.comp_tokens entries. Synchronizes `stream` (the selection lives on
 * the device). RC_EINVAL for other policies or a host-only handle. */
rc_status rc_comp_tokens(void* handle, int layer, int32_t* frame, int32_t* tok, void* stream);

/* Relax Forcing: the pool scores of a layer's last selection (pool order:
 * history frames, then the frames that left the tail), to host memory.
 * *n receives the pool size (0 if the last new chunk needed no selection);
 * scores must hold RC_MAX_SLOTS floats. Synchronizes `stream`. */
rc_status rc_pool_scores(void* handle, int layer, float* scores, int32_t* n, void* stream);

/* Synchronize `stream` and report the device-side status word: RC_OK, or
 * RC_ETIMEOUT if a kernel's bounded wait gave up since the last check
 * (the word is cleared). */
rc_status rc_device_status(void* handle, void* stream);

/* Host copy of the fp32 (cos, sin) RoPE tables the handle uploaded:
 * axis 0 = time [t_max][t_pairs], 1 = row [grid_h][h_pairs], 2 = column
 * [grid_w][w_pairs], interleaved cos, sin. Writes *count floats if dst is
 * NULL, else copies up to *count floats. */
rc_status rc_rope_table(const void* handle, int axis, float* dst, size_t* count);

typedef struct rc_layout {
  size_t kv_layer_stride;  /* bytes between one layer's K and the next layer's K */
  size_t k_offset;         /* layer 0's K ring buffer [heads][head_dim/64][capacity][64] bf16:
                              each head in 64-dim planes (dims 64p .. 64p+63 of token t at
                              plane p, row t) */
  size_t v_offset;         /* layer 0's V ring buffer, same layout */
  size_t raw_layer_stride; /* bytes between layers of the pristine source */
  size_t raw_k_offset;     /* pristine raw K [heads][raw_frames*F][head_dim] (0 if none) */
  size_t raw_v_offset;     /* pristine raw V (Rolling Sink bank, 0 if none) */
  size_t q_offset;         /* rotated-query scratch [heads][chunk_frames*F][head_dim] bf16 */
  int32_t capacity;        /* tokens per head of a ring buffer = (sink + window) * F */
  int32_t raw_frames;      /* frames of the pristine source */
  size_t total;            /* = rc_cache_bytes() */
} rc_layout;

/* Byte offsets of the regions inside the caller's memory block (to inspect
 * or checkpoint the raw cache next to rc_get_state's integer state). */
rc_status rc_cache_layout(const void* handle, rc_layout* out);

/* Failure-detection self-test: launches one CTA whose bounded wait on a
 * barrier that nothing completes gives up after `limit_us` microseconds and
 * records RC_ETIMEOUT in the status word, as a real kernel's wait would; the
 * next rc_device_status then returns RC_ETIMEOUT and the context stays
 * usable. Faults nothing. */
rc_status rc_watchdog_selftest(void* handle, unsigned limit_us, void* stream);

/* Per-kernel timing with CUDA events recorded on the launching stream
 * around every kernel a step enqueues (re-rotation, append, attention,
 * scores, top-C, compaction, and the merge of attention units split between
 * CTAs). rc_profile_begin arms it for up to max_launches launches (events
 * are created here, not in rc_step); rc_profile_end synchronizes the
 * recorded events and reports, per kernel kind, the launch count and the
 * summed device milliseconds, then disarms. Launches beyond the limit are
 * counted but not timed. */
enum { RC_KERNEL_REROTATE = 0, RC_KERNEL_APPEND = 1, RC_KERNEL_ATTENTION = 2,
       RC_KERNEL_SCORES = 3, RC_KERNEL_TOPC = 4, RC_KERNEL_COMBINE = 5, RC_KERNEL_COMPACT = 6,
       RC_KERNEL_KINDS = 7 };
typedef struct rc_profile {
  int64_t launches[RC_KERNEL_KINDS];
  int64_t timed[RC_KERNEL_KINDS];
  double ms[RC_KERNEL_KINDS];
  double flops[RC_KERNEL_KINDS];  /* algorithmic FLOPs (attention: 4*d*H*visible pairs) */
  double bytes[RC_KERNEL_KINDS];  /* algorithmic HBM bytes (append, re-rotate) */
} rc_profile;
rc_status rc_profile_begin(void* handle, int max_launches);
rc_status rc_profile_end(void* handle, rc_profile* out);

rc_status rc_cache_destroy(void* handle);

/* Message for the calling thread's last failed call ("" if none). */
const char* rc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RC_H_ */
