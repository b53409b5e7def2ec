// Fold of the query-tile pairs that the persistent tensor-core attention
// kernel splits between CTAs (the split-KV combine of one unit's pieces).
// Reading and arithmetic: the pieces are partial online-softmax results over
// disjoint key ranges of the same rows, combined exactly as the streaming
// attention definition's softmax over the union of their keys (the rescaling
// of running sums by the exponential of the max difference).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_sched.cuh"
#include "fd_internal.h"
#include "sm100.cuh"

namespace fd {
namespace {

using namespace sm100;
using namespace attn;

// Folds the pieces of the query-tile pairs that the persistent kernel split
// between CTAs: row = sum_i O_i 2^(m_i - M) / sum_i l_i 2^(m_i - M) over the
// unit's pieces i in CTA order (a fixed order, so the rounding does not depend
// on which CTA finished first), M the largest max, written in bf16 with the
// log-sum-exp.  It runs after the attention kernel on the same stream, so
// every piece's slot is complete; no CTA of the attention kernel waits or
// folds.  An item is 32 of a split unit's 256 rows: lane = row, warp w = the
// w-th eighth of the columns (D/32 four-column chunks), so every load of a
// warp reads 512 contiguous bytes of a slot; the bf16 rows are staged in
// shared memory and written row by row.  The grid is at most three blocks per
// multiprocessor, each taking items blockIdx.x, + gridDim.x, ...; a block
// computes the schedule and the rollouts' iteration offsets once, before it
// waits for the attention kernel (they depend only on the parameters and the
// cache counters, which that kernel does not write).
constexpr int kFoldRows = 32;          // rows per item
constexpr int kFoldBlocksPerSm = 3;   // resident blocks per multiprocessor (registers)
constexpr int kFoldGridPerSm = 3;     // grid cap: blocks per multiprocessor
constexpr int kFoldCachedRollouts = 64;  // rollouts whose offsets a block keeps in smem

template <int D>
__global__ void __launch_bounds__(256, kFoldBlocksPerSm)
    fold_split_units(const __grid_constant__ AttnParams p) {
  constexpr int kChunks = D / 32;  // four-column chunks per thread
  constexpr size_t kOffM = 2 * kBM * D, kOffL = kOffM + 2 * kBM;
  constexpr int kItemsPerUnit = 2 * kBM / kFoldRows;
  __shared__ Sched s_sd;
  __shared__ int s_nt[kFoldCachedRollouts];       // KV iterations of a unit of rollout r
  __shared__ int s_pre[kFoldCachedRollouts + 1];  // iterations of the rollouts before r
  __shared__ int s_unit[6];  // r, h, b, U0, c_lo, c_hi (c_lo == c_hi: nothing to fold)
  __shared__ __align__(16) uint16_t s_out[kFoldRows][D];
  const int per_r = p.H * p.nb;
  const int cached = min(p.n_rollouts, kFoldCachedRollouts);
  for (int r = threadIdx.x; r < cached; r += blockDim.x) s_nt[r] = tile_counts(p, r).nt;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_sd = make_sched(p);
    s_pre[0] = 0;
    for (int r = 0; r < cached; ++r) s_pre[r + 1] = s_pre[r] + per_r * s_nt[r];
  }
  __syncthreads();
  // every block waits for the attention kernel (also those with nothing to
  // fold), so this grid completes after it and work later on the stream sees
  // both kernels' rows
  griddep_wait();
  const Sched sd = s_sd;
  const int n_items = (p.n_rollouts * per_r - sd.W * p.G) * kItemsPerUnit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ch0 = warp * kChunks;  // first chunk of this thread
  auto piece = [&](int c) { return cta_begin(c, sd, p.G) < cta_begin(c + 1, sd, p.G); };
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    if (threadIdx.x == 0) {
      const int unit = sd.W * p.G + item / kItemsPerUnit;
      const int r = unit / per_r;
      int U0, nt;  // the unit's first iteration and its iterations
      if (r < cached) {
        nt = s_nt[r];
        U0 = s_pre[r];
      } else {
        nt = tile_counts(p, r).nt;
        U0 = s_pre[cached];
        for (int rr = cached; rr < r; ++rr) U0 += per_r * tile_counts(p, rr).nt;
      }
      const int u = unit - r * per_r;
      U0 += u * nt;
      s_unit[0] = r;
      s_unit[1] = u / p.nb;
      s_unit[2] = u - (u / p.nb) * p.nb;
      s_unit[3] = U0;
      s_unit[4] = nt > 0 ? cta_of(U0, sd, p.G) : 0;
      s_unit[5] = nt > 0 ? cta_of(U0 + nt - 1, sd, p.G) : 0;
    }
    __syncthreads();
    const int c_lo = s_unit[4], c_hi = s_unit[5];
    const int r = s_unit[0], h = s_unit[1], b = s_unit[2], U0 = s_unit[3];
    if (c_lo != c_hi) {  // else whole: the attention kernel wrote its rows
      const int row_b = (item % kItemsPerUnit) * kFoldRows;  // item's first row
      const int row = row_b + lane;
      // pieces in groups of two, every load of a group in flight together;
      // M is the running max over the groups so far
      constexpr int kGroup = 2;
      float M = -INFINITY, L = 0.f;
      float4 acc[kChunks];
#pragma unroll
      for (int e = 0; e < kChunks; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c0 = c_lo; c0 <= c_hi; c0 += kGroup) {
        bool has[kGroup];
        float mv[kGroup], lv[kGroup];
        float4 ov[kGroup][kChunks];
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
          has[i] = c0 + i <= c_hi && piece(c0 + i);
          mv[i] = -INFINITY;
          lv[i] = 0.f;
          if (has[i]) {
            const float* sl = part_slot(p, c0 + i, U0, sd);
            mv[i] = __ldcg(sl + kOffM + row);
            lv[i] = __ldcg(sl + kOffL + row);
#pragma unroll
            for (int e = 0; e < kChunks; ++e)
              ov[i][e] =
                  __ldcg(reinterpret_cast<const float4*>(sl) + (size_t)(ch0 + e) * 2 * kBM + row);
          }
        }
        float Mg = M;
#pragma unroll
        for (int i = 0; i < kGroup; ++i) Mg = fmaxf(Mg, mv[i]);
        if (Mg > M) {  // rescale what earlier groups left (nothing in the first group)
          const float sc = ex2_approx(M - Mg);
          L *= sc;
#pragma unroll
          for (int e = 0; e < kChunks; ++e) {
            acc[e].x *= sc;
            acc[e].y *= sc;
            acc[e].z *= sc;
            acc[e].w *= sc;
          }
          M = Mg;
        }
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
          if (!has[i]) continue;
          const float w = mv[i] == M ? 1.f : ex2_approx(mv[i] - M);
          L += lv[i] * w;
#pragma unroll
          for (int e = 0; e < kChunks; ++e) {
            acc[e].x += w * ov[i][e].x;
            acc[e].y += w * ov[i][e].y;
            acc[e].z += w * ov[i][e].z;
            acc[e].w += w * ov[i][e].w;
          }
        }
      }
      const float inv_l = 1.f / L;
#pragma unroll
      for (int e = 0; e < kChunks; ++e)
        *reinterpret_cast<uint2*>(&s_out[lane][(ch0 + e) * 4]) =
            make_uint2(pack_bf16(acc[e].x * inv_l, acc[e].y * inv_l),
                       pack_bf16(acc[e].z * inv_l, acc[e].w * inv_l));
      const int qrow = b * 2 * kBM + row;
      if (warp == 0 && p.lse != nullptr && qrow < p.Mq)
        p.lse[((size_t)r * p.H + h) * p.Mq + qrow] = (M + log2f(L)) * 0.69314718055994530942f;
      __syncthreads();
      // rows of D bf16 = D / 8 sixteen-byte vectors; the block's 256 threads
      // write 256 vectors per round
      constexpr int kVecRow = D / 8;
      for (int t = threadIdx.x; t < kFoldRows * kVecRow; t += 256) {
        const int i = t / kVecRow, v = t % kVecRow;
        const int q = b * 2 * kBM + row_b + i;
        if (q >= p.Mq) continue;
        uint16_t* out = static_cast<uint16_t*>(p.out) + (((size_t)r * p.Mq + q) * p.H + h) * D;
        reinterpret_cast<uint4*>(out)[v] = *reinterpret_cast<const uint4*>(&s_out[i][v * 8]);
      }
    }
    __syncthreads();  // s_unit and s_out are rewritten by the next item
  }
}

}  // namespace

cudaError_t launch_fold_split_units(const AttnParams& p, uint64_t split_units, cudaStream_t s) {
  if (split_units == 0) return cudaSuccess;
  const uint64_t items = split_units * (2 * kBM / kFoldRows);
  const uint64_t cap = (uint64_t)p.G * kFoldGridPerSm;
  // launched as a programmatic dependent of the attention kernel: the blocks
  // start on multiprocessors it leaves and wait on the device for it
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(items < cap ? items : cap));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, p.d == 128 ? fold_split_units<128> : fold_split_units<64>, p);
}

}  // namespace fd
