// Host side of the C ABI declared in include/fd.h: argument validation, the
// storage layout, TMA descriptor encoding and kernel launches.  No entry
// point allocates device memory: the caller owns every device buffer.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "fd.h"
#include "fd_internal.h"

struct fd_cache {
  fd_cache_desc desc;
  fd_cache_layout layout;
  fd::CacheView view;
  int device;
  int sms;                      // multiprocessors of the device
  std::vector<int64_t> host_n;  // [L][R] mirror of the device counters
  CUtensorMap tm_kc, tm_vc;     // bf16 caches: (d, Hkv, slots*Tf, L*R)
  CUtensorMap tm_kb;            // rotated block keys: (d, Hkv, F*Tf, work_sets*R)
  bool have_maps;
};

namespace fd {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n); }

namespace {

constexpr size_t kAlign = 1024;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool mul_ok(size_t a, size_t b, size_t* out) {
  if (a != 0 && b > SIZE_MAX / a) return false;
  *out = a * b;
  return true;
}

// Returns FD_OK and fills `lay` when the descriptor is valid.
fd_status compute_layout(const fd_cache_desc* d, fd_cache_layout* lay) {
  if (d == nullptr || lay == nullptr) return FD_ERR_INVALID_ARG;
  if (d->dtype != FD_BF16 && d->dtype != FD_F32) return FD_ERR_DTYPE;
  if (d->num_layers < 1 || d->max_rollouts < 1 || d->num_heads < 1 ||
      d->grid_h < 1 || d->grid_w < 1 || d->action_tokens < 0 ||
      d->block_frames < 1 || d->sink_frames < 0 || d->window_frames < 1)
    return FD_ERR_SHAPE;
  if (d->block_frames > d->window_frames) return FD_ERR_SHAPE;
  if (d->num_layers > 256 || d->max_rollouts > 65535 || d->num_heads > 65535 ||
      d->block_frames > 64)
    return FD_ERR_SHAPE;
  const int32_t hkv = d->num_kv_heads == 0 ? d->num_heads : d->num_kv_heads;
  if (hkv < 1 || hkv > d->num_heads || d->num_heads % hkv != 0) return FD_ERR_SHAPE;
  if (d->head_dim < 8 || d->head_dim % 8 != 0 || d->head_dim > 256)
    return FD_ERR_SHAPE;
  if (!(d->rope_theta > 1.0f) || !isfinite(d->rope_theta)) return FD_ERR_SHAPE;
  const int32_t views = d->num_views == 0 ? 1 : d->num_views;
  if (views < 1 || views > 64) return FD_ERR_SHAPE;
  const size_t T = (size_t)views * d->grid_h * d->grid_w;
  const size_t Tf = T + (size_t)d->action_tokens;
  if (Tf > (1u << 24) || T * d->block_frames > (1u << 30)) return FD_ERR_SHAPE;
  const size_t gslots = (size_t)d->sink_frames + d->window_frames;
  if (gslots * Tf > (1u << 30)) return FD_ERR_SHAPE;
  // context-parallel shard: ring slots s with s % N == shard_index, local s / N
  const int32_t shards = d->num_shards == 0 ? 1 : d->num_shards;
  if (shards < 1 || shards > 64 || (size_t)shards > gslots || d->shard_index < 0 ||
      d->shard_index >= shards)
    return FD_ERR_SHAPE;
  const size_t slots = (gslots + shards - 1) / shards;  // local slots
  // per-call work areas (rotated block keys and queries, split-pair partials)
  const int32_t sets = d->num_work_sets == 0 ? 1 : d->num_work_sets;
  if (sets < 1 || sets > d->num_layers) return FD_ERR_SHAPE;
  const size_t ws_r = (size_t)sets * d->max_rollouts;
  const size_t esz = d->dtype == FD_BF16 ? 2 : 4;
  const int d2 = d->head_dim / 2;
  const int p_hw = d->head_dim / 6;
  lay->rope_pairs_t = d2 - 2 * p_hw;
  lay->rope_pairs_h = p_hw;
  lay->rope_pairs_w = p_hw;
  if (p_hw < 1) return FD_ERR_SHAPE;

  size_t frame, layer_kv, kv, lr, x;
  if (!mul_ok(Tf * hkv, (size_t)d->head_dim * esz, &frame) ||
      !mul_ok(frame, slots * d->max_rollouts, &layer_kv) ||
      !mul_ok(layer_kv, (size_t)d->num_layers, &kv))
    return FD_ERR_CAPACITY;
  lr = (size_t)d->num_layers * d->max_rollouts;
  size_t off = 0;
  // Every region is kept below 2^56 bytes (far beyond any device memory), so
  // the dozen regions summed below cannot wrap a 64-bit size.
  constexpr size_t kRegionMax = (size_t)1 << 56;
  if (kv > kRegionMax) return FD_ERR_CAPACITY;
  lay->k = off;
  off = align_up(off + kv);
  lay->v = off;
  off = align_up(off + kv);
  lay->krot = off;
  off = align_up(off + kv);
  lay->kblk = off;
  size_t blk;
  if (!mul_ok(frame * d->block_frames, ws_r, &blk) || blk > kRegionMax) return FD_ERR_CAPACITY;
  off = align_up(off + blk);
  // the block's rotated queries and the partial results of the persistent
  // bf16 kernel
  const bool tensor_path = d->dtype == FD_BF16;
  lay->qblk = off;
  if (tensor_path) {
    if (!mul_ok(T * d->block_frames * d->num_heads, (size_t)d->head_dim * esz * ws_r, &x) ||
        x > kRegionMax)
      return FD_ERR_CAPACITY;
    off = align_up(off + x);
  }
  lay->part = off;
  if (tensor_path)
    off = align_up(off + (size_t)sets * kAttnMaxCtas * 2 * kPartSlotFloats * sizeof(float));
  lay->pos = off;
  off = align_up(off + lr * slots * sizeof(int32_t));
  lay->count = off;
  off = align_up(off + lr * sizeof(int32_t));
  lay->ttab = off;
  if (!mul_ok(lr * (slots + d->block_frames), (size_t)lay->rope_pairs_t * 8, &x) ||
      x > kRegionMax)
    return FD_ERR_CAPACITY;
  off = align_up(off + x);
  lay->htab = off;
  off = align_up(off + (size_t)d->grid_h * p_hw * 8);
  lay->wtab = off;
  off = align_up(off + (size_t)d->grid_w * p_hw * 8);
  lay->err = off;
  off = align_up(off + 16);
  lay->total = off;
  lay->layer_kv_bytes = layer_kv;
  return FD_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D bf16 map (d, H, rows, batch), box (64, 1, 128, 1), 128-byte swizzle.
bool encode_bf16_map(CUtensorMap* m, const void* base, int d, int H,
                     uint64_t rows, uint64_t batch) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, rows, batch};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2,
                           rows * H * d * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult res = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                     const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

fd_status check_device(const fd_cache* c) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FD_ERR_CUDA;
  return dev == c->device ? FD_OK : FD_ERR_INVALID_ARG;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

fd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FD_OK : FD_ERR_CUDA; }

}  // namespace
}  // namespace fd

extern "C" {

const char* fd_status_string(fd_status s) {
  switch (s) {
    case FD_OK: return "ok";
    case FD_ERR_INVALID_ARG: return "invalid argument";
    case FD_ERR_SHAPE: return "shape not allowed";
    case FD_ERR_DTYPE: return "unknown dtype";
    case FD_ERR_CAPACITY: return "capacity exceeded";
    case FD_ERR_CUDA: return "CUDA error";
    case FD_ERR_DEVICE_TIMEOUT: return "device-side wait gave up";
    case FD_ERR_UNSUPPORTED: return "unsupported configuration";
    case FD_ERR_ALIGNMENT: return "tensor not 16-byte aligned";
  }
  return "unknown status";
}

uint64_t fd_launch_count(void) { return fd::g_launches.load(); }

size_t fd_cache_bytes(const fd_cache_desc* desc) {
  fd_cache_layout lay;
  return fd::compute_layout(desc, &lay) == FD_OK ? lay.total : 0;
}

fd_status fd_cache_get_layout(const fd_cache_desc* desc, fd_cache_layout* out) {
  return fd::compute_layout(desc, out);
}

fd_status fd_cache_create(const fd_cache_desc* desc, void* dev_storage,
                          size_t bytes, fd_cache** out) {
  fd::NvtxRange nvtx_range("fd_cache_create");
  if (out == nullptr) return FD_ERR_INVALID_ARG;
  *out = nullptr;
  fd_cache_layout lay;
  fd_status st = fd::compute_layout(desc, &lay);
  if (st != FD_OK) return st;
  if (dev_storage == nullptr) return FD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dev_storage) & 1023) != 0) return FD_ERR_ALIGNMENT;
  if (bytes < lay.total) return FD_ERR_CAPACITY;

  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_storage) != cudaSuccess ||
      attr.type != cudaMemoryTypeDevice)
    return FD_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return FD_ERR_CUDA;
  if (cur != attr.device) return FD_ERR_INVALID_ARG;

  fd_cache* c = new (std::nothrow) fd_cache();
  if (c == nullptr) return FD_ERR_CAPACITY;
  c->desc = *desc;
  c->layout = lay;
  c->device = attr.device;
  if (cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device) !=
          cudaSuccess ||
      c->sms < 1) {
    delete c;
    return FD_ERR_CUDA;
  }
  uint8_t* base = static_cast<uint8_t*>(dev_storage);
  fd::CacheView& v = c->view;
  v.k = base + lay.k;
  v.v = base + lay.v;
  v.krot = base + lay.krot;
  v.kblk = base + lay.kblk;
  v.qblk = base + lay.qblk;
  v.part = reinterpret_cast<float*>(base + lay.part);
  v.pos = reinterpret_cast<int32_t*>(base + lay.pos);
  v.count = reinterpret_cast<int32_t*>(base + lay.count);
  v.ttab = reinterpret_cast<float2*>(base + lay.ttab);
  v.htab = reinterpret_cast<float2*>(base + lay.htab);
  v.wtab = reinterpret_cast<float2*>(base + lay.wtab);
  v.err = reinterpret_cast<int32_t*>(base + lay.err);
  v.L = desc->num_layers;
  v.R = desc->max_rollouts;
  v.H = desc->num_heads;
  v.Hkv = desc->num_kv_heads == 0 ? desc->num_heads : desc->num_kv_heads;
  v.d = desc->head_dim;
  v.gh = desc->grid_h;
  v.gw = desc->grid_w;
  v.Tv = desc->grid_h * desc->grid_w;
  v.T = (desc->num_views == 0 ? 1 : desc->num_views) * v.Tv;
  v.Tf = v.T + desc->action_tokens;
  v.F = desc->block_frames;
  v.S = desc->sink_frames;
  v.W = desc->window_frames;
  v.N = desc->num_shards == 0 ? 1 : desc->num_shards;
  v.shard = desc->shard_index;
  v.slots = (v.S + v.W + v.N - 1) / v.N;  // local slots of this shard
  v.work_sets = desc->num_work_sets == 0 ? 1 : desc->num_work_sets;
  v.nb = (v.F * v.T + 255) / 256;
  v.pt = lay.rope_pairs_t;
  v.ph = lay.rope_pairs_h;
  v.pw = lay.rope_pairs_w;
  v.esz = desc->dtype == FD_BF16 ? 2 : 4;
  v.theta = (double)desc->rope_theta;
  v.frame_bytes = (uint64_t)v.Tf * v.Hkv * v.d * v.esz;
  c->host_n.assign((size_t)v.L * v.R, 0);
  c->have_maps = false;
  if (desc->dtype == FD_BF16) {
    const uint64_t rows = (uint64_t)v.slots * v.Tf;
    const uint64_t batch = (uint64_t)v.L * v.R;
    if (!fd::encode_bf16_map(&c->tm_kc, v.krot, v.d, v.Hkv, rows, batch) ||
        !fd::encode_bf16_map(&c->tm_vc, v.v, v.d, v.Hkv, rows, batch) ||
        !fd::encode_bf16_map(&c->tm_kb, v.kblk, v.d, v.Hkv, (uint64_t)v.F * v.Tf,
                             (uint64_t)v.work_sets * v.R)) {
      // only the tensor-core path needs the maps; keep going without them
      c->have_maps = false;
    } else {
      c->have_maps = true;
    }
  }
  cudaError_t e = cudaMemsetAsync(dev_storage, 0, lay.total, 0);
  if (e == cudaSuccess) e = fd::launch_cache_init(v, 0);
  if (e == cudaSuccess) e = cudaStreamSynchronize(0);
  if (e != cudaSuccess) {
    delete c;
    return FD_ERR_CUDA;
  }
  *out = c;
  return FD_OK;
}

fd_status fd_cache_destroy(fd_cache* cache) {
  if (cache == nullptr) return FD_ERR_INVALID_ARG;
  delete cache;
  return FD_OK;
}

fd_status fd_cache_get_desc(const fd_cache* cache, fd_cache_desc* out) {
  if (cache == nullptr || out == nullptr) return FD_ERR_INVALID_ARG;
  *out = cache->desc;
  return FD_OK;
}

fd_status fd_cache_layout_of(const fd_cache* cache, fd_cache_layout* out) {
  if (cache == nullptr || out == nullptr) return FD_ERR_INVALID_ARG;
  *out = cache->layout;
  return FD_OK;
}

fd_status fd_cache_frames(const fd_cache* cache, int32_t layer,
                          int32_t rollout, int64_t* n) {
  if (cache == nullptr || n == nullptr) return FD_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cache->view.L || rollout < 0 ||
      rollout >= cache->view.R)
    return FD_ERR_INVALID_ARG;
  *n = cache->host_n[(size_t)layer * cache->view.R + rollout];
  return FD_OK;
}

fd_status fd_cache_window_full(const fd_cache* cache, int32_t layer,
                               int32_t rollout, int32_t frames, int32_t* reached) {
  if (cache == nullptr || reached == nullptr) return FD_ERR_INVALID_ARG;
  const fd::CacheView& v = cache->view;
  if (layer < 0 || layer >= v.L || rollout < 0 || rollout >= v.R) return FD_ERR_INVALID_ARG;
  if (frames < 1 || frames > v.F) return FD_ERR_INVALID_ARG;
  const int64_t n = cache->host_n[(size_t)layer * v.R + rollout];
  *reached = n + frames > (int64_t)v.S + v.W ? 1 : 0;
  return FD_OK;
}

fd_status fd_cache_reset(fd_cache* cache, const int32_t* rollout_ids,
                         int32_t n_ids, void* stream) {
  fd::NvtxRange nvtx_range("fd_cache_reset");
  if (cache == nullptr || (n_ids > 0 && rollout_ids == nullptr) || n_ids < 0)
    return FD_ERR_INVALID_ARG;
  const fd::CacheView& v = cache->view;
  for (int i = 0; i < n_ids; ++i)
    if (rollout_ids[i] < 0 || rollout_ids[i] >= v.R) return FD_ERR_INVALID_ARG;
  if (n_ids == 0) return FD_OK;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int i0 = 0; i0 < n_ids; i0 += fd::kCommitMaxRollouts) {
    fd::ResetParams p;
    p.n = n_ids - i0 < fd::kCommitMaxRollouts ? n_ids - i0 : fd::kCommitMaxRollouts;
    for (int i = 0; i < p.n; ++i) p.ids[i] = rollout_ids[i0 + i];
    st = fd::cuda_status(fd::launch_reset(v, p, s));
    if (st != FD_OK) return st;
  }
  for (int i = 0; i < n_ids; ++i)
    for (int l = 0; l < v.L; ++l)
      cache->host_n[(size_t)l * v.R + rollout_ids[i]] = 0;
  return FD_OK;
}

fd_status fd_rope3d(const fd_cache* cache, int32_t layer, int32_t n_rollouts,
                    void* x, int32_t tokens_per_frame, int32_t heads,
                    void* stream) {
  fd::NvtxRange nvtx_range("fd_rope3d");
  if (cache == nullptr || x == nullptr) return FD_ERR_INVALID_ARG;
  const fd::CacheView& v = cache->view;
  if (layer < 0 || layer >= v.L || n_rollouts < 1 || n_rollouts > v.R)
    return FD_ERR_INVALID_ARG;
  if (tokens_per_frame != v.T && tokens_per_frame != v.Tf) return FD_ERR_SHAPE;
  if (heads != v.H && heads != v.Hkv) return FD_ERR_SHAPE;
  if (!fd::aligned16(x)) return FD_ERR_ALIGNMENT;
  if (!fd::rope_rows_ok(n_rollouts, v.F, tokens_per_frame)) return FD_ERR_UNSUPPORTED;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;
  return fd::cuda_status(fd::launch_rope3d(v, layer, n_rollouts, x,
                                           tokens_per_frame, heads,
                                           static_cast<cudaStream_t>(stream)));
}

fd_status fd_block_attention(fd_cache* cache, int32_t layer,
                             int32_t n_rollouts, const void* q, const void* k,
                             const void* v_, void* out, float* lse,
                             void* stream) {
  fd::NvtxRange nvtx_range("fd_block_attention");
  return fd::block_attention_impl(cache, layer, n_rollouts, q, k, v_, out, lse,
                                  stream, nullptr);
}

}  // extern "C"

// Work-area bytes of a call: the block's rotated keys, then its rotated
// queries (tensor-core calls; the CUDA-core kernel rotates as it stages).
bool fd::tensor_core_call(const fd_cache* cache) {
  return cache->desc.dtype == FD_BF16 && (cache->view.d == 128 || cache->view.d == 64);
}

static size_t block_key_bytes(const fd::CacheView& c, int32_t n_rollouts) {
  return (size_t)n_rollouts * c.F * c.frame_bytes;
}

size_t fd::block_work_bytes(const fd_cache* cache, int32_t n_rollouts) {
  const fd::CacheView& c = cache->view;
  if (!tensor_core_call(cache)) return 0;
  return block_key_bytes(c, n_rollouts) +
         (size_t)n_rollouts * c.F * c.T * c.H * c.d * c.esz;
}

fd_status fd::block_attention_impl(fd_cache* cache, int32_t layer,
                                   int32_t n_rollouts, const void* q,
                                   const void* k, const void* v_, void* out,
                                   float* lse, void* stream, void* work) {
  if (cache == nullptr || q == nullptr || k == nullptr || v_ == nullptr ||
      out == nullptr)
    return FD_ERR_INVALID_ARG;
  const fd::CacheView& c = cache->view;
  if (layer < 0 || layer >= c.L || n_rollouts < 1 || n_rollouts > c.R)
    return FD_ERR_INVALID_ARG;
  if (!fd::aligned16(q) || !fd::aligned16(k) || !fd::aligned16(v_) ||
      !fd::aligned16(out) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return FD_ERR_ALIGNMENT;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;

  fd::AttnParams p;
  memset(&p, 0, sizeof(p));
  // bf16 with d = 128 or 64 runs on the tensor cores; fp32, and bf16 of the
  // other head sizes, on CUDA cores
  const bool tensor_cores = fd::tensor_core_call(cache);
  // the call's work set: the block's keys and queries, rotated once for all
  // query tiles (see fd.h, kblk and qblk), and the split-pair partials; the
  // rotated keys and queries go to the caller's `work` instead when one is
  // given
  const int ws = layer % c.work_sets;
  uint8_t* kblk = work != nullptr ? static_cast<uint8_t*>(work)
                                  : c.kblk + (size_t)ws * c.R * c.F * c.frame_bytes;
  uint8_t* qblk = work != nullptr
      ? static_cast<uint8_t*>(work) + block_key_bytes(c, n_rollouts)
      : c.qblk + (size_t)ws * c.R * c.F * c.T * c.H * c.d * c.esz;
  // the CUDA-core kernel reads the block as given and rotates as it stages
  p.q = tensor_cores ? static_cast<const void*>(qblk) : q;
  p.k = tensor_cores ? static_cast<const void*>(kblk) : k;
  p.v = v_;
  p.pos = c.pos + (size_t)layer * c.R * c.slots;
  p.count = c.count + (size_t)layer * c.R;
  p.ttab = c.ttab + (size_t)layer * c.R * (c.slots + c.F) * c.pt;
  p.htab = c.htab;
  p.wtab = c.wtab;
  p.out = out;
  p.lse = lse;
  p.N = c.N;
  p.shard = c.shard;
  p.err = c.err;
  p.kc = c.krot + (size_t)layer * cache->layout.layer_kv_bytes;
  p.vc = c.v + (size_t)layer * cache->layout.layer_kv_bytes;
  p.part = c.part + (size_t)ws * fd::kAttnMaxCtas * 2 * fd::kPartSlotFloats;
  p.nb = c.nb;
  p.H = c.H;
  p.Hkv = c.Hkv;
  p.kv_group = c.H / c.Hkv;
  p.d = c.d;
  p.T = c.T;
  p.Tf = c.Tf;
  p.gh = c.gh;
  p.gw = c.gw;
  p.F = c.F;
  p.S = c.S;
  p.W = c.W;
  p.slots = c.slots;
  p.Mq = c.F * c.T;
  p.pt = c.pt;
  p.ph = c.ph;
  p.pw = c.pw;
  p.n_rollouts = n_rollouts;
  p.map_row0 = layer * c.R;
  p.kb_row0 = work != nullptr ? 0 : ws * c.R;
  p.div_T = fd::make_fastdiv((uint32_t)c.T);
  p.div_Tf = fd::make_fastdiv((uint32_t)c.Tf);
  p.div_gw = fd::make_fastdiv((uint32_t)c.gw);
  p.div_Tv = fd::make_fastdiv((uint32_t)c.Tv);
  p.Tv = c.Tv;
  p.scale = (float)(1.0 / sqrt((double)c.d));
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c.d));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  if (tensor_cores ? !cache->have_maps : (c.d % 32 != 0 || c.d > 128))
    return FD_ERR_UNSUPPORTED;
  if (tensor_cores && fd::attn_bf16_smem_bytes(p) == 0) return FD_ERR_UNSUPPORTED;
  // a shard's result is only usable with its log-sum-exp (to be combined)
  if (c.N > 1 && lse == nullptr) return FD_ERR_INVALID_ARG;
  // the RoPE pass walks the block's query and key rows with a 32-bit row
  // counter
  if (!fd::rope_rows_ok(n_rollouts, c.F, c.T + c.Tf)) return FD_ERR_UNSUPPORTED;
  // Everything the tensor-core launch needs is prepared before the first
  // launch of the call, so a refusal leaves nothing half done.
  CUtensorMap tm_q, tm_vb, tm_kb_work;
  if (tensor_cores) {
    const uint64_t kb_rows = (uint64_t)c.F * c.Tf;
    if (!fd::encode_bf16_map(&tm_q, qblk, c.d, c.H, (uint64_t)p.Mq, n_rollouts) ||
        !fd::encode_bf16_map(&tm_vb, v_, c.d, c.Hkv, kb_rows, n_rollouts))
      return FD_ERR_CUDA;
    if (work != nullptr &&
        !fd::encode_bf16_map(&tm_kb_work, work, c.d, c.Hkv, kb_rows, n_rollouts))
      return FD_ERR_CUDA;
    // persistent grid: one CTA per multiprocessor, no more CTAs than KV
    // iterations the call can have (every rollout's cache full)
    const int64_t nt_max = ((int64_t)c.slots * c.Tf + 127) / 128 +
                           ((int64_t)c.F * c.Tf + 127) / 128;
    const int64_t it_max = (int64_t)n_rollouts * c.H * c.nb * nt_max;
    int64_t g = cache->sms < fd::kAttnMaxCtas ? cache->sms : fd::kAttnMaxCtas;
    if (it_max < g) g = it_max;
    // the kernel's schedule arithmetic is 32-bit
    if (it_max * g >= ((int64_t)1 << 31)) return FD_ERR_UNSUPPORTED;
    p.G = (int)g;
  }
  if (!tensor_cores) return fd::cuda_status(fd::launch_attn_cuda_core(p, c.esz, s));
  // one pass rotates the block's queries and (the block's keys belong to
  // shard 0; other shards never read them) its keys
  st = fd::cuda_status(fd::launch_rope_block(c, layer, n_rollouts, q, qblk,
                                             c.shard == 0 ? k : nullptr, kblk, s));
  if (st != FD_OK) return st;
  if (c.shard != 0) {
    // rollouts with no key on this shard get zero rows and lse = -inf here;
    // the tensor-core kernel skips them
    st = fd::cuda_status(fd::launch_attn_zero_keyless(p, s));
    if (st != FD_OK) return st;
  }
  return fd::cuda_status(fd::launch_attn_bf16_sm100(
      tm_q, cache->tm_kc, cache->tm_vc, work != nullptr ? tm_kb_work : cache->tm_kb,
      tm_vb, p, s));
}

extern "C" {

fd_status fd_cache_commit(fd_cache* cache, int32_t layer_begin,
                          int32_t layer_end, int32_t n_rollouts,
                          const int32_t* frames, const void* const* k,
                          const void* const* v, void* stream) {
  fd::NvtxRange nvtx_range("fd_cache_commit");
  if (cache == nullptr || k == nullptr || v == nullptr) return FD_ERR_INVALID_ARG;
  const fd::CacheView& c = cache->view;
  if (layer_begin < 0 || layer_end > c.L || layer_begin >= layer_end ||
      n_rollouts < 1 || n_rollouts > c.R)
    return FD_ERR_INVALID_ARG;
  const int nl = layer_end - layer_begin;
  for (int i = 0; i < nl; ++i) {
    if (k[i] == nullptr || v[i] == nullptr) return FD_ERR_INVALID_ARG;
    if (!fd::aligned16(k[i]) || !fd::aligned16(v[i])) return FD_ERR_ALIGNMENT;
  }
  if (frames != nullptr)
    for (int r = 0; r < n_rollouts; ++r)
      if (frames[r] < 0 || frames[r] > c.F) return FD_ERR_CAPACITY;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // one launch covers at most kCommitMaxLayers layers and kCommitMaxRollouts
  // rollouts, and its grid.y (layers x rollouts x 2 x F) stays below 65536
  const int r_chunk = fd::kCommitMaxRollouts;
  int l_chunk = 65535 / (r_chunk * 2 * c.F);
  if (l_chunk > fd::kCommitMaxLayers) l_chunk = fd::kCommitMaxLayers;
  if (l_chunk < 1) l_chunk = 1;
  if ((int64_t)r_chunk * 2 * c.F > 65535) return FD_ERR_UNSUPPORTED;
  for (int l0 = 0; l0 < nl; l0 += l_chunk) {
    for (int r0 = 0; r0 < n_rollouts; r0 += r_chunk) {
      fd::CommitParams p;
      memset(&p, 0, sizeof(p));
      p.layer0 = layer_begin + l0;
      p.nl = nl - l0 < l_chunk ? nl - l0 : l_chunk;
      p.rollout0 = r0;
      p.nr = n_rollouts - r0 < r_chunk ? n_rollouts - r0 : r_chunk;
      p.src_rollouts = n_rollouts;
      for (int i = 0; i < p.nl; ++i) {
        p.k[i] = static_cast<const uint8_t*>(k[l0 + i]);
        p.v[i] = static_cast<const uint8_t*>(v[l0 + i]);
      }
      for (int i = 0; i < p.nr; ++i) p.frames[i] = frames ? frames[r0 + i] : c.F;
      st = fd::cuda_status(fd::launch_commit(c, p, s));
      if (st != FD_OK) return st;
    }
  }
  for (int i = 0; i < nl; ++i)
    for (int r = 0; r < n_rollouts; ++r)
      cache->host_n[(size_t)(layer_begin + i) * c.R + r] += frames ? frames[r] : c.F;
  return FD_OK;
}

fd_status fd_get_device_error(fd_cache* cache, int32_t* code) {
  if (cache == nullptr || code == nullptr) return FD_ERR_INVALID_ARG;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;
  int32_t v = 0;
  if (cudaMemcpy(&v, cache->view.err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FD_ERR_CUDA;
  *code = v;
  if (v != 0) {
    if (cudaMemset(cache->view.err, 0, sizeof(int32_t)) != cudaSuccess) return FD_ERR_CUDA;
    return FD_ERR_DEVICE_TIMEOUT;
  }
  return FD_OK;
}

fd_status fd_attention_combine(int32_t n_parts, const void* const* outs,
                               const float* const* lses, int32_t n_rollouts,
                               int32_t rows, int32_t heads, int32_t head_dim,
                               int32_t dtype, void* out, float* lse, void* stream) {
  fd::NvtxRange nvtx_range("fd_attention_combine");
  if (outs == nullptr || lses == nullptr || out == nullptr) return FD_ERR_INVALID_ARG;
  if (n_parts < 1 || n_parts > fd::kCombineMaxParts) return FD_ERR_SHAPE;
  if (dtype != FD_BF16 && dtype != FD_F32) return FD_ERR_DTYPE;
  if (n_rollouts < 1 || rows < 1 || heads < 1 || head_dim < 1 || head_dim > 256)
    return FD_ERR_SHAPE;
  const size_t esz = dtype == FD_BF16 ? 2 : 4;
  auto misaligned = [&](const void* ptr, size_t a) {
    return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0;
  };
  fd::CombineParams p;
  memset(&p, 0, sizeof(p));
  for (int i = 0; i < n_parts; ++i) {
    if (outs[i] == nullptr || lses[i] == nullptr) return FD_ERR_INVALID_ARG;
    if (misaligned(outs[i], esz) || misaligned(lses[i], 4)) return FD_ERR_ALIGNMENT;
    p.out[i] = outs[i];
    p.lse[i] = lses[i];
  }
  if (misaligned(out, esz) || (lse != nullptr && misaligned(lse, 4))) return FD_ERR_ALIGNMENT;
  p.n_parts = n_parts;
  p.n_rollouts = n_rollouts;
  p.Mq = rows;
  p.H = heads;
  p.d = head_dim;
  p.esz = (int)esz;
  p.dst = out;
  p.dst_lse = lse;
  return fd::cuda_status(fd::launch_combine(p, static_cast<cudaStream_t>(stream)));
}

fd_status fd_selftest_bounded_wait(fd_cache* cache, int32_t limit_ms,
                                   void* stream) {
  if (cache == nullptr || limit_ms < 1 || limit_ms > 2000) return FD_ERR_INVALID_ARG;
  fd_status st = fd::check_device(cache);
  if (st != FD_OK) return st;
  return fd::cuda_status(fd::launch_bounded_wait_selftest(
      cache->view.err, (uint64_t)limit_ms * 1000000ull,
      static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

extern "C" fd_status fd_exp2_selfcheck(const float* x, float* y, int64_t n,
                                       void* stream) {
  if (x == nullptr || y == nullptr || n < 0) return FD_ERR_INVALID_ARG;
  if (n == 0) return FD_OK;
  return fd::cuda_status(
      fd::launch_exp2_selfcheck(x, y, n, static_cast<cudaStream_t>(stream)));
}
