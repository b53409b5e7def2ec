/*
 * fd.h -- C ABI of the B200 (sm_100a) streaming chunk-attention library.
 *
 * One hot path: block-causal chunk attention over a bounded per-rollout KV
 * cache (sink frames + rolling window ring buffer) with 3D (t,h,w) RoPE on
 * Q and K, plus the ring-buffer commit that evicts the oldest window frame.
 *
 * Sources for the behaviour (the pages describe it in prose; no formula is
 * printed):
 *   [FD-BM]  "NVIDIA FlashDreams Is the Open-Source Inference Engine Robotics
 *            World Models Needed", section Bounded Memory for Infinite
 *            Rollouts: per-rollout cache of bounded size with eviction.
 *   [FD-HP]  same page, section Hot-Path Generation, Background State
 *            Updates: generate() (denoising) vs finalize() (cache update).
 *   [C3-MA]  "Cosmos3-H-Dreams" model card, Model Architecture: block-causal
 *            few-step student with a KV cache; conditioning frame prefilled
 *            once; each latent frame consumes 4 action vectors.
 *   [C3-SI]  "Cosmos3-H-Dreams" model card, Software Integration: static-shape
 *            KV cache, CUDA Graphs.
 *   [AD-VII] AlpaDreams GTC 2026 write-up, section VII: causal DiT attends to
 *            historical clean frames and the current noisy frame via a KV cache.
 *   [DZ-SR]  "Single-GPU inference for DreamZero", Sequential requests: KV and
 *            frame positions carry over between requests; explicit reset.
 *   [FD-CP]  "NVIDIA FlashDreams ...", section Multi-GPU Context Parallelism:
 *            one rollout's inference sharded across several GPUs.
 *
 * Readings where the pages are silent (the same ones the test oracle states):
 *   - scores q.k/sqrt(d), softmax over the whole key set, no bias or mask
 *     inside it; key set = valid cache tokens + every token of the block;
 *   - the first S frames of a rollout are sinks (never evicted); later frames
 *     go to slot S + ((m - S) mod W) of a W-slot ring; valid slots are always
 *     a prefix of the slot array;
 *   - 3D RoPE: pairs (2i, 2i+1) of the head dimension; the d/2 pairs split
 *     into contiguous t | h | w sections of d/2 - 2*floor(d/6), floor(d/6),
 *     floor(d/6) pairs; pair j of a section of n pairs turns by
 *     coord * theta^(-j/n); video token i of a frame is at
 *     (h, w) = (i / grid_w, i % grid_w), action tokens at (0, 0); t is the
 *     absolute frame index since the last reset;
 *   - the cache stores K/V as committed (pre-RoPE) plus an int32 frame
 *     position per slot; a cached key's rotation depends only on that
 *     position, so the commit also stores it rotated (krot).  Each attention
 *     call on the tensor cores first rotates the block's keys and queries
 *     once, into work areas (kblk, qblk) that the attention kernel copies
 *     tiles from (the CUDA-core kernel rotates both as it stages them).
 *
 * Conventions for every call:
 *   - all pointers to tensors are DEVICE pointers on the device that owns the
 *     cache storage; host arrays are marked (host);
 *   - a call on a cache needs that cache's device to be current (otherwise
 *     FD_ERR_INVALID_ARG, nothing launched); one process may drive caches on
 *     several devices (ordinals below 64), switching the current device
 *     between calls;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default);
 *     every call only enqueues work on it: no host synchronisation, no
 *     allocation, so a block of calls can be captured in a CUDA graph;
 *   - argument and shape errors return a status before anything is launched;
 *   - layouts are dense row-major, token-major then head then dim ("BSHD");
 *   - bf16 tensors are raw bfloat16 (uint16 bit patterns); f32 are IEEE float.
 */
#ifndef FD_H_
#define FD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FD_OK = 0,
  FD_ERR_INVALID_ARG = 1,     /* null pointer, index out of range           */
  FD_ERR_SHAPE = 2,           /* descriptor or call shape not allowed       */
  FD_ERR_DTYPE = 3,           /* dtype not known                            */
  FD_ERR_CAPACITY = 4,        /* storage too small / too many frames        */
  FD_ERR_CUDA = 5,            /* a CUDA runtime or driver call failed       */
  FD_ERR_DEVICE_TIMEOUT = 6,  /* a device-side wait gave up (see below)     */
  FD_ERR_UNSUPPORTED = 7,     /* valid request this build does not handle   */
  FD_ERR_ALIGNMENT = 8        /* a tensor base is not 16-byte aligned       */
} fd_status;

typedef enum { FD_BF16 = 0, FD_F32 = 1 } fd_dtype;

/* Geometry of one cache.  T = views*grid_h*grid_w video tokens per latent
 * frame (views of one frame side by side, view-major; a single view when
 * num_views is 0 or 1);
 * Tf = T + action_tokens key/value tokens per frame ([C3-MA]: 4 action
 * vectors per latent frame).  Requires 1 <= block_frames <= window_frames,
 * sink_frames >= 0, head_dim even and a multiple of 8.
 * Grouped-query attention (no counterpart on the pages; a variant of the
 * cache semantics): keys and values carry Hkv = num_kv_heads heads, queries
 * and outputs H = num_heads; Hkv divides H and query head h reads key/value
 * head h / (H / Hkv).  num_kv_heads = 0 means Hkv = H (multi-head). */
typedef struct {
  int32_t num_layers;     /* L: one independent cache per layer            */
  int32_t max_rollouts;   /* R: concurrent rollouts, each with its own cache */
  int32_t num_heads;      /* H query heads                                 */
  int32_t head_dim;       /* d                                             */
  int32_t grid_h;         /* latent grid height                            */
  int32_t grid_w;         /* latent grid width                             */
  int32_t action_tokens;  /* A extra K/V tokens per frame (no queries)     */
  int32_t block_frames;   /* F latent frames denoised together             */
  int32_t sink_frames;    /* S frames kept for the whole rollout           */
  int32_t window_frames;  /* W rolling window frames                       */
  float rope_theta;       /* RoPE base (1e4 in every shipped workload)     */
  int32_t dtype;          /* fd_dtype of q, k, v, out and the cache        */
  int32_t num_kv_heads;   /* Hkv key/value heads (0: = num_heads)          */
  int32_t num_views;      /* V camera views per frame (0: = 1); video
                           * token i sits at (h, w) of i mod (grid_h*grid_w)
                           * and all views share t (no counterpart on the
                           * pages beyond their four-view models)           */
  int32_t num_shards;     /* N context-parallel shards of the key set (0: 1)
                           * ([FD-CP]); this cache stores the ring slots s
                           * with s % N == shard_index at local index s / N,
                           * every shard counts all committed frames, and the
                           * block's own keys belong to shard 0              */
  int32_t shard_index;    /* this cache's shard, 0 <= shard_index < N      */
  int32_t num_work_sets;  /* Wk per-call work areas (0: 1), 1 <= Wk <= L: an
                           * attention call on layer l uses work set l mod
                           * Wk, and two attention calls on this cache may
                           * run at the same time on the GPU only when their
                           * layers differ modulo Wk.  One set (the default)
                           * keeps the storage to what one call at a time
                           * needs; Wk = L lets calls on any two layers
                           * overlap (no counterpart on the pages)          */
} fd_cache_desc;

/* Byte offsets of the regions inside the caller's storage buffer.
 *   k, v : [L][R][S+W][Tf][Hkv][d] elements of `dtype`, exactly as committed
 *   krot : [L][R][S+W][Tf][Hkv][d] the same keys rotated by 3D RoPE to their
 *          frame's position, written by the commit (a committed frame and its
 *          position never change, so its rotation is computed once instead
 *          of at every attention call); derived data, not part of the
 *          cache's observable state
 *   kblk : [Wk][R][F*Tf][Hkv][d] work area of fd_block_attention: the
 *          current block's keys rotated once per call, read by every query
 *          tile (one set per work set, see num_work_sets)
 *   qblk : [Wk][R][F*T][H][d] work area of the same calls: the block's
 *          queries rotated once per call (bf16 caches; empty for fp32)
 *   part : [Wk][148][2][256*128 + 512] float work area of the bf16 attention
 *          kernel: a CTA whose share of the work ends or begins inside a
 *          query tile pair leaves its partial result there (unnormalised
 *          output rows, running max, row sum), which a fold kernel launched
 *          right after combines; empty (size 0) for fp32
 *   pos  : [L][R][S+W] int32, frame index held by a slot, -1 = empty
 *   count: [L][R] int32, frames committed since the last reset (n)
 *   ttab : [L][R][S+W+F][p_t] float2 (cos, sin) of the t-section angles for
 *          every slot's frame and for the next block's frames n..n+F-1
 *   htab : [grid_h][p_h] float2, wtab : [grid_w][p_w] float2 (static)
 *   err  : int32 device error word (0 = none)                            */
typedef struct {
  size_t k, v, krot, kblk, qblk, part, pos, count, ttab, htab, wtab, err;
  size_t total;           /* == fd_cache_bytes(desc)                       */
  size_t layer_kv_bytes;  /* bytes of one layer's K (or V) region          */
  int32_t rope_pairs_t, rope_pairs_h, rope_pairs_w;
} fd_cache_layout;

typedef struct fd_cache fd_cache;

/* Bytes of device storage a cache with this geometry needs; 0 if the
 * descriptor is invalid.  Pure host function.  The storage is bounded by the
 * geometry alone, whatever the length of the rollouts ([FD-BM], [C3-SI]:
 * bounded, static-shape cache); its regions are those of fd_cache_layout
 * (the cache's reading: K/V as committed plus positions, see the readings
 * at the top of this file). */
size_t fd_cache_bytes(const fd_cache_desc* desc);

/* Region offsets of the storage layout above ([FD-BM], [C3-SI]; the regions
 * follow the readings at the top of this file).  Pure host function. */
fd_status fd_cache_get_layout(const fd_cache_desc* desc, fd_cache_layout* out);

/* Bind a cache object to caller-owned device storage of at least
 * fd_cache_bytes(desc) bytes (base 1024-byte aligned).  Clears the storage,
 * marks every slot empty, sets every counter to 0 and builds the RoPE tables,
 * then synchronises the device once.  The library allocates no device
 * memory, here or later: memory stays constant over unbounded rollouts
 * ([FD-BM], [C3-SI]).  The host object is freed by fd_cache_destroy.
 *
 * Snapshot and restore: every piece of a cache's state (K, V, rotated K,
 * slot positions, frame counters, RoPE tables) lives in the storage, so a
 * snapshot is a copy of the fd_cache_bytes bytes taken between calls (after
 * the stream's work is done), and a restore is fd_cache_create with the same
 * descriptor followed by a copy of the snapshot over the new storage.  The
 * calls then continue the snapshot's rollouts.  fd_cache_frames reads a host
 * mirror of the counters that only this object's commits and resets
 * update, so after a restore it counts from the restore. */
fd_status fd_cache_create(const fd_cache_desc* desc, void* dev_storage,
                          size_t bytes, fd_cache** out);

/* Frees the host object only; the storage stays the caller's. */
fd_status fd_cache_destroy(fd_cache* cache);

/* Copy of the descriptor / layout a cache was created with. */
fd_status fd_cache_get_desc(const fd_cache* cache, fd_cache_desc* out);
fd_status fd_cache_layout_of(const fd_cache* cache, fd_cache_layout* out);

/* Start a new sequence for the listed rollouts in every layer ([DZ-SR]):
 * counter n = 0, every slot empty (pos = -1), K/V of those rollouts zeroed,
 * t tables rebuilt for frames 0..F-1.  rollout_ids (host) [n_ids], each in
 * [0, max_rollouts). */
fd_status fd_cache_reset(fd_cache* cache, const int32_t* rollout_ids,
                         int32_t n_ids, void* stream);

/* 3D RoPE in place on a block tensor x of rollouts 0..n_rollouts-1.  The
 * pages name no positional encoding; this is the 3D (t,h,w) RoPE reading at
 * the top of this file (pair layout, t | h | w sections, frequencies), with
 * t the block's frames since the last reset ([DZ-SR]: frame positions carry
 * over between requests):
 *   x: [n_rollouts][F][tokens_per_frame][heads][d] of the cache dtype;
 *   tokens_per_frame = T (queries) or Tf (keys, action tokens at (t,0,0));
 *   heads = num_heads (queries) or Hkv (keys); anything else FD_ERR_SHAPE;
 * frame f of rollout r is at t = n_r + f with n_r that rollout's counter at
 * `layer`, i.e. the positions fd_block_attention gives the block.  This is the
 * same rotation fd_block_attention applies internally; it is exported for
 * callers that need rotated tensors and for tests.  n_rollouts x F x
 * tokens_per_frame of 2^31 or more returns FD_ERR_UNSUPPORTED (the kernel
 * counts token rows in 32 bits; fd_block_attention has the same limit for its
 * block keys). */
fd_status fd_rope3d(const fd_cache* cache, int32_t layer, int32_t n_rollouts,
                    void* x, int32_t tokens_per_frame, int32_t heads,
                    void* stream);

/* One denoising-step attention call for `layer` ([C3-MA], [AD-VII]):
 *   q   : [n_rollouts][F*T][H][d]   queries of the block, pre-RoPE
 *   k, v: [n_rollouts][F*Tf][Hkv][d] keys/values of the block, pre-RoPE
 *   out : [n_rollouts][F*T][H][d]   softmax(q'k'^T/sqrt(d)) v
 *   lse : [n_rollouts][H][F*T] fp32 natural-log sum of exp of the scaled
 *         scores, or NULL
 * For rollout r the key set is its valid cache slots (sinks + window, frame
 * positions from the slot table) plus all F*Tf block tokens at t = n_r + f.
 * The cache is read only: call it once per denoising step, then commit.
 * bf16 with head_dim 128 or 64 runs on tcgen05 tensor cores (fp32
 * accumulation, P rounded to bf16); f32, and bf16 with head_dim 32 or 96, on
 * CUDA cores in fp32 arithmetic (no TF32; bf16 output rounded once).  Other head sizes
 * return FD_ERR_UNSUPPORTED before any launch.  Tensor bases must be 16-byte
 * aligned.
 * On the tensor cores a pass first rotates the block's queries and keys into
 * the call's work set (qblk, kblk); the attention kernel is persistent (one
 * CTA per multiprocessor, at most 148) and splits the call's KV iterations
 * evenly over its CTAs; it returns FD_ERR_UNSUPPORTED when n_rollouts x H x
 * ceil(F*T/256) x (ceil((S+W)*Tf/128) + ceil(F*Tf/128)) x CTAs reaches 2^31.
 * A query-tile pair split between CTAs leaves its pieces in the work set's
 * `part` region; a fold kernel launched right after the attention kernel
 * combines them (a fixed order: results do not depend on timing).  The
 * attention and fold kernels are launched as programmatic dependents of the
 * kernel before them on the stream: each starts its prologue early and waits
 * on the device for its predecessor before reading that kernel's output, and
 * every block of the fold waits for the attention kernel, so work enqueued
 * after the call sees all of its results as with plain stream order.
 * Device-side waits are bounded: a wait that gives up sets the error word
 * (fd_get_device_error) instead of hanging. */
fd_status fd_block_attention(fd_cache* cache, int32_t layer,
                             int32_t n_rollouts, const void* q, const void* k,
                             const void* v, void* out, float* lse,
                             void* stream);

/* Allocation-free variant of fd_block_attention.  The pages have no
 * counterpart: it is an interface for callers that cannot set device memory
 * aside for the per-layer work area inside the cache storage -- storage
 * carved from a pool or arena someone else sizes, or a process that may not
 * call cudaMalloc at all (it can synchronise the device, which a real-time
 * serving loop cannot afford).  Same arguments, semantics and results as
 * fd_block_attention; the work area for the block's rotated keys and queries
 * (used by the tensor-core kernels; CUDA-core calls need none) is instead a
 * static device array of FD_STATIC_WORK_BYTES inside this library, which
 * every GPU that loads the library holds until the process exits.
 *   - FD_ERR_CAPACITY (before any launch) when a tensor-core call's
 *     n_rollouts*F*(Tf*Hkv + T*H)*d*2 bytes (the block's rotated keys with
 *     Hkv key/value heads and its rotated queries with H heads) exceed
 *     FD_STATIC_WORK_BYTES;
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress), so make that first call before any stream
 *     capture on that device;
 *   - every call shares the one array: calls that overlap on the GPU race
 *     and must be ordered (one stream, or events);
 *   - allocates nothing, neither on the device nor through any library. */
#define FD_STATIC_WORK_BYTES (32u << 20)
fd_status fd_block_attention_static(fd_cache* cache, int32_t layer,
                                    int32_t n_rollouts, const void* q,
                                    const void* k, const void* v, void* out,
                                    float* lse, void* stream);

/* Ring-buffer commit for layers [layer_begin, layer_end) -- the finalize()
 * half of [FD-HP]:  for every rollout r < n_rollouts and f < frames_r,
 * slot = slot_of(n_r + f) receives frame f of k[l]/v[l] bit for bit (and its
 * keys rotated to t = n_r + f in the krot region), pos[slot] = n_r + f; then
 * n_r += frames_r and the rollout's t table is rebuilt.  Once the window is
 * full this evicts the oldest window frames.
 *   frames (host) [n_rollouts], each in [0, F]; NULL = F for every rollout
 *   (a ragged prefill commits fewer frames for some rollouts);
 *   k, v (host arrays of device pointers) [layer_end - layer_begin], each
 *   [n_rollouts][F*Tf][Hkv][d] pre-RoPE (in practice the last step's k/v). */
fd_status fd_cache_commit(fd_cache* cache, int32_t layer_begin,
                          int32_t layer_end, int32_t n_rollouts,
                          const int32_t* frames, const void* const* k,
                          const void* const* v, void* stream);

/* Window-boundary policy of [DZ-SR], a second way to bound the cache next to
 * the rolling ring: the S + W slots hold one local-attention window of
 * consecutive frames; when the next block of `frames` frames does not fit
 * (n + frames > S + W, n the rollout's counter at `layer`), the window
 * restarts: the caller releases the old frames with fd_cache_reset, commits
 * the re-encoded conditioning frames (they take positions 0, 1, ...) with
 * fd_cache_commit, and then runs the block.  Used this way the ring never
 * wraps.  Sets *reached to 1 in that case and to 0 otherwise.  Host only:
 * reads the host mirror of the counter (fd_cache_frames); nothing is
 * launched.  frames in [1, F]. */
fd_status fd_cache_window_full(const fd_cache* cache, int32_t layer,
                               int32_t rollout, int32_t frames, int32_t* reached);

/* Host mirror of a rollout's counter (updated by commit/reset calls). */
fd_status fd_cache_frames(const fd_cache* cache, int32_t layer,
                          int32_t rollout, int64_t* n);

/* Reads (synchronously) and clears the device error word.  *code = 0 when no
 * device-side check fired; otherwise bits 0-7 give the kind (1 = a bounded
 * wait gave up) and bits 8-15 the site.  Returns FD_ERR_DEVICE_TIMEOUT when
 * *code != 0. */
fd_status fd_get_device_error(fd_cache* cache, int32_t* code);

/* Verification hook for the base-2 exponential of the bf16 softmax, which
 * computes part of its weights on the FMA pipe (Cody-Waite reduction and a
 * cubic, see the attention kernel) and the rest on the hardware unit.  For
 * each x[i] (device, n floats, each in [-126, 8]) writes (device, 3n floats)
 * y[3i] = the FMA-pipe value, y[3i+1] = the hardware approximation,
 * y[3i+2] = CUDA's exp2f(x[i]).  Asynchronous on `stream`. */
fd_status fd_exp2_selfcheck(const float* x, float* y, int64_t n, void* stream);

/* Failure-detection self-test (no counterpart on the pages).  Runs one
 * device-side wait on an mbarrier that nothing ever completes, through the
 * same bounded wait the attention kernel uses, limited to limit_ms (1..2000)
 * instead of the kernel's 2 s.  The wait gives up, records kind 1 (timeout)
 * and site 5 in the cache's error word and the kernel returns: nothing
 * faults or hangs and the context stays usable.  Read the result with
 * fd_get_device_error (FD_ERR_DEVICE_TIMEOUT, code 0x501). */
fd_status fd_selftest_bounded_wait(fd_cache* cache, int32_t limit_ms,
                                   void* stream);

/* Context parallelism ([FD-CP]): rows of attention over a key set split into
 * parts from each part's rows and log-sum-exp, e.g. the outputs of
 * fd_block_attention on the N shards of one cache (gathered onto one device,
 * by NCCL or a peer copy, before this call):
 *   outs[i]: [n_rollouts][rows][heads][head_dim] of `dtype`, normalised over
 *            part i's keys (device, host array of n_parts pointers)
 *   lses[i]: [n_rollouts][heads][rows] fp32 natural-log sum of exponentials
 *            of part i's scaled scores; -inf for a part with no key
 *   out    : the whole-set rows, same layout as outs[i]; lse: its
 *            log-sum-exp (or NULL)
 * O = sum_i exp(lse_i - M) O_i / sum_i exp(lse_i - M), M = max_i lse_i,
 * computed in fp32 and rounded once to `dtype`; rows no part has a key for
 * become 0 with lse -inf.  1 <= n_parts <= 16.  No counterpart formula on the
 * pages, which only name context parallelism. */
fd_status fd_attention_combine(int32_t n_parts, const void* const* outs,
                               const float* const* lses, int32_t n_rollouts,
                               int32_t rows, int32_t heads, int32_t head_dim,
                               int32_t dtype, void* out, float* lse, void* stream);

/* Number of kernels this library has launched in this process. */
uint64_t fd_launch_count(void);

const char* fd_status_string(fd_status status);

#ifdef __cplusplus
}
#endif

#endif /* FD_H_ */
