// Context parallelism: attention over a key set split into parts, each part
// computed where its keys live ("NVIDIA FlashDreams Is the Open-Source
// Inference Engine Robotics World Models Needed", Multi-GPU Context
// Parallelism; AlpaDreams GTC 2026 write-up, section VIII: inference spread
// over up to 16 GPUs).  Each part returns its softmax-normalised rows O_i and
// natural-log sum of exponentials lse_i; the rows of the whole key set are
//   O = sum_i exp(lse_i - M) O_i / sum_i exp(lse_i - M),  M = max_i lse_i,
//   lse = M + log sum_i exp(lse_i - M),
// and a part with no key (lse_i = -inf) weighs 0.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fd_internal.h"

namespace fd {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float load_elem(const void* base, size_t i, int esz) {
  if (esz == 2) {
    const uint16_t b = static_cast<const uint16_t*>(base)[i];
    return __uint_as_float((uint32_t)b << 16);
  }
  return static_cast<const float*>(base)[i];
}

__device__ __forceinline__ void store_elem(void* base, size_t i, int esz, float v) {
  if (esz == 2) {
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    static_cast<__nv_bfloat16*>(base)[i] = b;
  } else {
    static_cast<float*>(base)[i] = v;
  }
}

// One warp per output row (rollout r, query q, head h): rows [r][q][h][d],
// log-sum-exps [r][h][q].
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    combine_kernel(CombineParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t rows = (size_t)p.n_rollouts * p.Mq * p.H;
  const size_t row = (size_t)blockIdx.x * kWarpsPerBlock + warp;
  if (row >= rows) return;
  const int h = (int)(row % p.H);
  const size_t rq = row / p.H;
  const int q = (int)(rq % p.Mq);
  const int r = (int)(rq / p.Mq);
  const size_t li = ((size_t)r * p.H + h) * p.Mq + q;
  float M = -INFINITY;
  for (int i = 0; i < p.n_parts; ++i) M = fmaxf(M, p.lse[i][li]);
  float w[kCombineMaxParts];
  float L = 0.f;
  for (int i = 0; i < p.n_parts; ++i) {
    const float l = p.lse[i][li];
    w[i] = (M == -INFINITY || l == -INFINITY) ? 0.f : expf(l - M);
    L += w[i];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const size_t base = row * p.d;
  for (int e = lane; e < p.d; e += 32) {
    float acc = 0.f;
    for (int i = 0; i < p.n_parts; ++i)
      if (w[i] != 0.f) acc = fmaf(w[i], load_elem(p.out[i], base + e, p.esz), acc);
    store_elem(p.dst, base + e, p.esz, acc * inv);
  }
  if (lane == 0 && p.dst_lse != nullptr) p.dst_lse[li] = L > 0.f ? M + logf(L) : -INFINITY;
}

// Rows of rollouts that have no key on this shard (no valid local cache slot;
// the block's keys belong to shard 0): zero output, lse = -inf.  One warp per
// (query, head) row; rollouts with keys return at once.
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    zero_keyless_kernel(AttnParams p) {
  const int r = blockIdx.y;
  const int nv = valid_slots_local(valid_slots_global(p.count[r], p.S, p.W), p.N, p.shard);
  if (nv > 0 || p.shard == 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * kWarpsPerBlock + warp;  // q * H + h
  if (row >= (size_t)p.Mq * p.H) return;
  uint16_t* out = static_cast<uint16_t*>(p.out) + ((size_t)r * p.Mq * p.H + row) * p.d;
  for (int e = lane; e < p.d; e += 32) out[e] = 0;
  if (lane == 0 && p.lse != nullptr) {
    const int q = (int)(row / p.H), h = (int)(row % p.H);
    p.lse[((size_t)r * p.H + h) * p.Mq + q] = -INFINITY;
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  const size_t rows = (size_t)p.n_rollouts * p.Mq * p.H;
  const size_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffull) return cudaErrorInvalidValue;
  combine_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(p);
  count_launch(1);
  return cudaGetLastError();
}

cudaError_t launch_attn_zero_keyless(const AttnParams& p, cudaStream_t s) {
  const size_t rows = (size_t)p.Mq * p.H;
  const size_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7fffffffull || p.n_rollouts > 65535) return cudaErrorInvalidValue;
  dim3 grid((unsigned)blocks, (unsigned)p.n_rollouts);
  zero_keyless_kernel<<<grid, kWarpsPerBlock * 32, 0, s>>>(p);
  count_launch(1);
  return cudaGetLastError();
}

}  // namespace fd
