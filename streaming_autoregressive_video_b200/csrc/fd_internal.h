// Internal definitions shared by the host entry points and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "fd.h"

namespace fd {

// NVTX range over one entry point of the library, so that a profiler's
// timeline shows each call (header-only NVTX v3: without an attached tool a
// push or pop is one indirect call that returns at once).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Devices one process may drive (ordinals 0 .. kMaxDevices-1).
constexpr int kMaxDevices = 64;

// One-time setup per device.  Kernel attributes (cudaFuncSetAttribute) act
// on the current device only, so a process that drives several GPUs sets
// them once on each.  setup() runs until it succeeds once on a device; two
// threads may both run it on first use (it must be idempotent).
struct PerDeviceOnce {
  std::atomic<bool> done[kMaxDevices];
};

template <typename Setup>
cudaError_t once_per_device(PerDeviceOnce& once, Setup&& setup) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (once.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess) once.done[dev].store(true, std::memory_order_release);
  return e;
}

// Device error word: bits 0-7 kind, bits 8-15 site.
enum DevErrKind : int32_t { kDevErrTimeout = 1, kDevErrArgument = 2 };

// Exact division by a runtime constant for the index ranges used here
// (n * d < 2^40): q = (n * m) >> 40 with m = ceil(2^40 / d).
struct FastDiv {
  uint64_t m;
  uint32_t d;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.m = ((1ull << 40) + d - 1) / d;
  return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, FastDiv f) {
  return (uint32_t)(((uint64_t)n * f.m) >> 40);
}

// The RoPE pass walks token rows (rollout, frame, token) with a 32-bit
// counter that steps by the grid's warp count: rows stay below 2^31 so the
// counter cannot wrap.
inline bool rope_rows_ok(int n_rollouts, int F, int tokens) {
  return (uint64_t)n_rollouts * (uint64_t)F * (uint64_t)tokens < (1ull << 31);
}

// Valid cache frames of a rollout that committed n frames into a ring of S
// sinks and W window slots: the slot prefix [0, nv).  Of these, shard `shard`
// of N stores slots shard, shard + N, ... (local indices 0, 1, ...), which are
// again a prefix of its local storage.
__host__ __device__ __forceinline__ int valid_slots_global(int n, int S, int W) {
  const int win = n - S > 0 ? n - S : 0;
  return (n < S ? n : S) + (win < W ? win : W);
}
__host__ __device__ __forceinline__ int valid_slots_local(int nv, int N, int shard) {
  return nv > shard ? (nv - shard + N - 1) / N : 0;
}

// Device pointers into one cache's storage plus its geometry.
struct CacheView {
  uint8_t* k;
  uint8_t* v;
  uint8_t* krot;  // committed keys rotated to their frame's position
  uint8_t* kblk;  // work areas: the block's keys rotated per call
  uint8_t* qblk;  // work areas: the block's queries rotated per call (bf16)
  int32_t* pos;
  int32_t* count;
  float2* ttab;
  float2* htab;
  float2* wtab;
  float* part;    // [work_sets][kAttnMaxCtas][2][kPartSlotFloats] (bf16 caches)
  int32_t* err;
  int L, R, H, d, gh, gw, T, Tf, F, S, W, slots, pt, ph, pw, esz, nb;
  int Hkv;               // key/value heads (divides H)
  int Tv;                // video tokens per view (gh * gw); T = views * Tv
  // Context-parallel shard: this cache stores ring slots s with s % N == shard
  // at local index s / N; `slots` above counts local slots, S and W stay the
  // ring's global sink and window counts, count[] the global frame counter.
  int N, shard;
  int work_sets;  // per-call work areas; layer l uses set l % work_sets
  double theta;
  uint64_t frame_bytes;  // Tf * Hkv * d * esz (one frame of K or V)
};

// Persistent tensor-core attention: at most this many CTAs, each with two
// partial-result slots of kPartSlotFloats floats (O [256][128], m [256],
// l [256]) per work set.
constexpr int kAttnMaxCtas = 148;
constexpr size_t kPartSlotFloats = 256 * 128 + 2 * 256;

// Limits of one commit launch (host splits larger requests).
constexpr int kCommitMaxLayers = 32;
constexpr int kCommitMaxRollouts = 64;

struct CommitParams {
  const uint8_t* k[kCommitMaxLayers];
  const uint8_t* v[kCommitMaxLayers];
  int32_t frames[kCommitMaxRollouts];
  int layer0;    // first layer of this launch
  int nl;        // layers in this launch
  int rollout0;  // first rollout of this launch
  int nr;        // rollouts in this launch
  int src_rollouts;  // rollout extent of the k/v buffers (their stride)
};

struct ResetParams {
  int32_t ids[kCommitMaxRollouts];
  int n;
};

// Parameters of the attention kernels (the tensor maps travel separately).
struct AttnParams {
  const void* q;         // block queries and keys: rotated (work area) for the
  const void* k;         // tensor-core kernel, as given for the CUDA-core kernel
  const void* v;
  const int32_t* pos;    // [R][slots] of the layer
  const int32_t* count;  // [R] of the layer
  const float2* ttab;    // [R][slots+F][pt] of the layer
  const float2* htab;
  const float2* wtab;
  void* out;
  float* lse;
  int32_t* err;
  const uint8_t* kc;     // rotated cache K of the layer, rollout 0 (CUDA cores)
  const uint8_t* vc;
  float* part;           // per-CTA partial results of split units (tensor path)
  int H, d, T, Tf, gh, gw, F, S, W, slots, Mq, pt, ph, pw, n_rollouts;
  int nb;                // query-tile pairs per (rollout, head)
  int Hkv;               // key/value heads
  int kv_group;          // H / Hkv: query head h reads key/value head h / kv_group
  int Tv;                // video tokens per view
  FastDiv div_Tv;
  int N, shard;          // context-parallel shard of the key set (1, 0: whole)
  int G;                 // CTAs of the persistent launch
  int map_row0;          // layer * R: row offset of this layer in the cache maps
  int kb_row0;           // batch offset of rollout 0 in the rotated-block-key map
  FastDiv div_T, div_Tf, div_gw;
  float scale_log2;      // log2(e) / sqrt(d)
  float scale;           // 1 / sqrt(d)
};

// Launch helpers implemented in the .cu files.
cudaError_t launch_cache_init(const CacheView& c, cudaStream_t s);
cudaError_t launch_commit(const CacheView& c, const CommitParams& p,
                          cudaStream_t s);
cudaError_t launch_reset(const CacheView& c, const ResetParams& p,
                         cudaStream_t s);
cudaError_t launch_rope3d(const CacheView& c, int layer, int n_rollouts,
                          void* x, int tokens_per_frame, int heads,
                          cudaStream_t s);
// the block's queries q [n_rollouts][F*T][H][d] into q_out and (k not null)
// keys k [n_rollouts][F*Tf][Hkv][d] into k_out, rotated (positions from
// `layer`'s counters), same layouts, one launch (bf16)
cudaError_t launch_rope_block(const CacheView& c, int layer, int n_rollouts,
                              const void* q, void* q_out, const void* k, void* k_out,
                              cudaStream_t s);
// attention on CUDA cores in fp32 arithmetic: fp32 caches of any head size
// d in {32, 64, 96, 128}; bf16 caches (esz = 2) whose d is 32 or 96
cudaError_t launch_attn_cuda_core(const AttnParams& p, int esz, cudaStream_t s);
// bf16 output rows and log-sum-exp of rollouts with no key on this shard
cudaError_t launch_attn_zero_keyless(const AttnParams& p, cudaStream_t s);
// out = log-sum-exp weighted sum of n_parts partial results (context
// parallelism); rows = n_rollouts * Mq, heads H, head dim d
constexpr int kCombineMaxParts = 16;
struct CombineParams {
  const void* out[kCombineMaxParts];
  const float* lse[kCombineMaxParts];
  int n_parts, n_rollouts, Mq, H, d, esz;
  void* dst;
  float* dst_lse;
};
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);
// Dynamic shared memory the tensor-core kernel needs for this call (its
// operand stages, barriers and epilogue staging), 0 if that exceeds the limit.
size_t attn_bf16_smem_bytes(const AttnParams& p);
// Launches the persistent tensor-core attention kernel and, when it splits
// query-tile pairs between CTAs, the fold of those pairs.
cudaError_t launch_attn_bf16_sm100(const CUtensorMap& tm_q,
                                   const CUtensorMap& tm_kc,
                                   const CUtensorMap& tm_vc,
                                   const CUtensorMap& tm_kb,
                                   const CUtensorMap& tm_vb,
                                   const AttnParams& p, cudaStream_t s);
// Folds the split_units query-tile pairs past the whole-unit waves of the
// attention kernel just launched on `s` (fold.cu).
cudaError_t launch_fold_split_units(const AttnParams& p, uint64_t split_units,
                                    cudaStream_t s);

void count_launch(int n);
cudaError_t launch_bounded_wait_selftest(int32_t* err, uint64_t limit_ns,
                                         cudaStream_t s);

// Shared body of the attention entry points.  `work` is a device area for the
// block's rotated keys ([n_rollouts][F*Tf][Hkv][d]) followed by its rotated
// queries ([n_rollouts][F*T][H][d]; block_work_bytes bytes in all,
// 16-byte aligned) or nullptr for the call's work set in the cache storage.
fd_status block_attention_impl(fd_cache* cache, int32_t layer,
                               int32_t n_rollouts, const void* q,
                               const void* k, const void* v, void* out,
                               float* lse, void* stream, void* work);
size_t block_work_bytes(const fd_cache* cache, int32_t n_rollouts);
// whether attention calls on this cache run on the tensor-core kernels
bool tensor_core_call(const fd_cache* cache);

}  // namespace fd

namespace fd {
cudaError_t launch_exp2_selfcheck(const float* x, float* y, int64_t n,
                                  cudaStream_t s);
}  // namespace fd
