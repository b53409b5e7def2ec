// Block-causal chunk attention on CUDA cores, arithmetic in fp32 (no TF32).
//
// Same definition as the tensor-core kernel: for every query of the block,
// softmax(q' k'^T / sqrt(d)) v over the rollout's valid cache tokens (sinks +
// window, positions from the slot table) and all tokens of the block, with 3D
// RoPE applied to q and k as they are staged ("Cosmos3-H-Dreams" model card,
// Model Architecture: block-causal student with a KV cache; AlpaDreams GTC
// 2026 write-up, section VII: next frame from historical clean frames and the
// current noisy frame).  It serves fp32 caches, where the tolerance leaves no
// room for TF32 rounding, and bf16 caches whose head size the tensor-core
// kernel does not take (d = 32, 96): bf16 values are widened to fp32 as
// they are staged and the output is rounded to bf16 once, at the end.
//
// One CTA = (query tile of 8 x kRowsPerWarp rows, head, rollout); 8 warps,
// each kRowsPerWarp rows (4 for calls with many rows; 1 when 4 would leave
// most multiprocessors idle, as in launch-sized calls, where the warps' serial
// row loops are the latency).  Keys are staged 64 at a time in smem (the
// cache's keys arrive rotated, the block's keys are rotated in fp32 as they
// are staged); within a warp lane j scores key j (four independent partial
// sums over the head dimension), then the warp forms the online softmax and
// each lane accumulates d/32 output dimensions.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fd_internal.h"

namespace fd {
namespace {

constexpr int kWarps = 8;
constexpr int kKeys = 64;                     // keys per staged tile

struct KeyCoord {
  int tidx;  // row of the rollout's t table
  int h, w;
};

__device__ __forceinline__ float2 rope_cs(const AttnParams& p,
                                          const float2* tt, int pair,
                                          const KeyCoord& kc) {
  if (pair < p.pt) return tt[kc.tidx * p.pt + pair];
  if (pair < p.pt + p.ph) return p.htab[kc.h * p.ph + (pair - p.pt)];
  return p.wtab[kc.w * p.pw + (pair - p.pt - p.ph)];
}

// Elements (2i, 2i+1) of a stored row as fp32: fp32 storage, or bf16 bit
// patterns (the lower address in the low half of the 32-bit word).
__device__ __forceinline__ float2 load_pair(const float* x) {
  return *reinterpret_cast<const float2*>(x);
}
__device__ __forceinline__ float2 load_pair(const uint16_t* x) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(x);
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ void store_elem(float* x, float v) { *x = v; }
__device__ __forceinline__ void store_elem(uint16_t* x, float v) {
  *x = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Elem: float (fp32 cache) or uint16_t (bf16 bit patterns)
template <typename Elem, int D, int kRowsPerWarp>
__global__ void __launch_bounds__(kWarps * 32)
    attn_cuda_core_kernel(AttnParams p) {
  constexpr int kRows = kWarps * kRowsPerWarp;  // query rows per CTA
  constexpr int kPerLane = D / 32;
  extern __shared__ float sm[];
  float* Qs = sm;                          // [kRows][D]
  float* Ks = Qs + kRows * D;              // [kKeys][D + 1]
  float* Vs = Ks + kKeys * (D + 1);        // [kKeys][D]

  const int r = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = valid_slots_local(valid_slots_global(p.count[r], p.S, p.W), p.N, p.shard);
  const int n1 = nv * p.Tf, n2 = p.shard == 0 ? p.F * p.Tf : 0;
  const float2* tt = p.ttab + (size_t)r * (p.slots + p.F) * p.pt;
  const Elem* qg = static_cast<const Elem*>(p.q);
  const Elem* kg = static_cast<const Elem*>(p.k);
  const Elem* vg = static_cast<const Elem*>(p.v);
  const Elem* kcg = reinterpret_cast<const Elem*>(p.kc);
  const Elem* vcg = reinterpret_cast<const Elem*>(p.vc);

  // rotated queries
  for (int e = threadIdx.x; e < kRows * (D / 2); e += blockDim.x) {
    const int row = e / (D / 2), pair = e % (D / 2);
    const int q = q0 + row;
    float a = 0.f, b = 0.f;
    if (q < p.Mq) {
      const int f = q / p.T, tok = (q - f * p.T) % p.Tv;  // inside its view
      const KeyCoord kc{p.slots + f, tok / p.gw, tok % p.gw};
      const float2 x = load_pair(qg + (((size_t)r * p.Mq + q) * p.H + h) * D + 2 * pair);
      const float2 cs = rope_cs(p, tt, pair, kc);
      a = x.x * cs.x - x.y * cs.y;
      b = x.x * cs.y + x.y * cs.x;
    }
    Qs[row * D + 2 * pair] = a;
    Qs[row * D + 2 * pair + 1] = b;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][kPerLane];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) o[i][e] = 0.f;
  }

  const int nt1 = (n1 + kKeys - 1) / kKeys, nt2 = (n2 + kKeys - 1) / kKeys;
  for (int j = 0; j < nt1 + nt2; ++j) {
    const bool seg1 = j < nt1;
    const int key0 = seg1 ? j * kKeys : (j - nt1) * kKeys;
    const int nseg = seg1 ? n1 : n2;
    __syncthreads();
    for (int e = threadIdx.x; e < kKeys * (D / 2); e += blockDim.x) {
      const int kr = e / (D / 2), pair = e % (D / 2);
      const int key = key0 + kr;
      float a = 0.f, b = 0.f, va = 0.f, vb = 0.f;
      if (key < nseg) {
        // key/value head of this query head (grouped-query attention)
        const int hk = h / p.kv_group;
        const size_t off = seg1
            ? (((size_t)r * p.slots * p.Tf + key) * p.Hkv + hk) * D + 2 * pair
            : (((size_t)r * p.F * p.Tf + key) * p.Hkv + hk) * D + 2 * pair;
        // cached frames' keys arrive rotated (at commit); the block's keys
        // are rotated here, frame f of the block at t-row slots + f
        const float2 kx = load_pair((seg1 ? kcg : kg) + off);
        const float2 vx = load_pair((seg1 ? vcg : vg) + off);
        a = kx.x;
        b = kx.y;
        if (!seg1) {
          const int f = key / p.Tf, tok = key - f * p.Tf;
          const int tv = tok % p.Tv;  // inside its view; action tokens at (0, 0)
          const KeyCoord kc{p.slots + f, tok < p.T ? tv / p.gw : 0,
                            tok < p.T ? tv % p.gw : 0};
          const float2 cs = rope_cs(p, tt, pair, kc);
          a = kx.x * cs.x - kx.y * cs.y;
          b = kx.x * cs.y + kx.y * cs.x;
        }
        va = vx.x;
        vb = vx.y;
      }
      Ks[kr * (D + 1) + 2 * pair] = a;
      Ks[kr * (D + 1) + 2 * pair + 1] = b;
      Vs[kr * D + 2 * pair] = va;
      Vs[kr * D + 2 * pair + 1] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const float* qrow = Qs + (warp * kRowsPerWarp + i) * D;
#pragma unroll
      for (int sub = 0; sub < kKeys / 32; ++sub) {
        const int kr = sub * 32 + lane;
        const bool valid = key0 + kr < nseg;
        // four independent partial sums shorten the dependent FMA chain
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int e = 0; e < D; e += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            s4[u] = fmaf(qrow[e + u], Ks[kr * (D + 1) + e + u], s4[u]);
        }
        float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        s = valid ? s * p.scale : -INFINITY;
        float mt = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        if (mt == -INFINITY) continue;  // whole sub-tile past the segment end
        const float m_new = fmaxf(m[i], mt);
        const float alpha = expf(m[i] - m_new);
        const float pj = valid ? expf(s - m_new) : 0.f;
        float ps = pj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l[i] = l[i] * alpha + ps;
        m[i] = m_new;
#pragma unroll
        for (int e = 0; e < kPerLane; ++e) o[i][e] *= alpha;
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
          const float pb = __shfl_sync(0xffffffffu, pj, jj);
          const float* vrow = Vs + (sub * 32 + jj) * D;
#pragma unroll
          for (int e = 0; e < kPerLane; ++e)
            o[i][e] = fmaf(pb, vrow[lane + 32 * e], o[i][e]);
        }
      }
    }
  }

  Elem* outg = static_cast<Elem*>(p.out);
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int q = q0 + warp * kRowsPerWarp + i;
    if (q >= p.Mq) continue;
    // a shard may hold no key of this rollout: zero row, log-sum-exp -inf
    const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
    Elem* dst = outg + (((size_t)r * p.Mq + q) * p.H + h) * D;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) store_elem(dst + lane + 32 * e, o[i][e] * inv);
    if (p.lse != nullptr && lane == 0)
      p.lse[((size_t)r * p.H + h) * p.Mq + q] = l[i] > 0.f ? m[i] + logf(l[i]) : -INFINITY;
  }
}

template <typename Elem, int D, int kRowsPerWarp>
cudaError_t launch_rows(const AttnParams& p, cudaStream_t s) {
  constexpr int kRows = kWarps * kRowsPerWarp;
  const size_t smem = sizeof(float) * (kRows * D + kKeys * (D + 1) + kKeys * D);
  static PerDeviceOnce attr;
  cudaError_t e = once_per_device(attr, [smem] {
    return cudaFuncSetAttribute(attn_cuda_core_kernel<Elem, D, kRowsPerWarp>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid((p.Mq + kRows - 1) / kRows, p.H, p.n_rollouts);
  attn_cuda_core_kernel<Elem, D, kRowsPerWarp><<<grid, kWarps * 32, smem, s>>>(p);
  count_launch(1);
  return cudaGetLastError();
}

// Four rows per warp unless that leaves fewer CTAs than multiprocessors
// (148 on B200): then one row per warp, four times the CTAs.
template <typename Elem, int D>
cudaError_t launch_d(const AttnParams& p, cudaStream_t s) {
  const int64_t ctas4 = (int64_t)((p.Mq + 4 * kWarps - 1) / (4 * kWarps)) * p.H * p.n_rollouts;
  if (ctas4 < kAttnMaxCtas) return launch_rows<Elem, D, 1>(p, s);
  return launch_rows<Elem, D, 4>(p, s);
}

}  // namespace

template <typename Elem>
cudaError_t launch_elem(const AttnParams& p, cudaStream_t s) {
  switch (p.d) {
    case 32: return launch_d<Elem, 32>(p, s);
    case 64: return launch_d<Elem, 64>(p, s);
    case 96: return launch_d<Elem, 96>(p, s);
    case 128: return launch_d<Elem, 128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_cuda_core(const AttnParams& p, int esz, cudaStream_t s) {
  if (esz == 2) return launch_elem<uint16_t>(p, s);
  return launch_elem<float>(p, s);
}

}  // namespace fd
