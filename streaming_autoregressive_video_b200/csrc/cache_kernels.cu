// Cache maintenance kernels: storage initialisation, ring-buffer commit,
// rollout reset and the standalone 3D RoPE.
//
// The commit is the finalize() half of the generate()/finalize() split in
// "NVIDIA FlashDreams Is the Open-Source Inference Engine Robotics World
// Models Needed" (Hot-Path Generation, Background State Updates), and the
// ring keeps memory bounded as that page's Bounded Memory for Infinite
// Rollouts section requires.  The slot rule (sinks first, then a W-slot ring)
// and the RoPE layout are the readings documented in include/fd.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fd_internal.h"

namespace fd {
namespace {

__device__ __forceinline__ int slot_of(int m, int S, int W) {
  return m < S ? m : S + (m - S) % W;
}

// t-section (cos, sin) of one rollout/layer: rows 0..slots-1 for the frame
// held by each slot (identity for empty slots), rows slots..slots+F-1 for the
// next block's frames n..n+F-1.  Angles in fp64, rounded once to fp32.
__device__ void fill_ttab(const CacheView& c, int l, int r, int n,
                          const int32_t* pos_lr) {
  float2* tab = c.ttab + ((size_t)l * c.R + r) * (c.slots + c.F) * c.pt;
  const int rows = c.slots + c.F;
  for (int e = threadIdx.x; e < rows * c.pt; e += blockDim.x) {
    const int row = e / c.pt, j = e % c.pt;
    const long long t = row < c.slots ? (long long)pos_lr[row]
                                      : (long long)n + (row - c.slots);
    float2 cs = make_float2(1.f, 0.f);
    if (t >= 0) {
      const double inv_freq = pow(c.theta, -(double)j / (double)c.pt);
      double s, co;
      sincos((double)t * inv_freq, &s, &co);
      cs = make_float2((float)co, (float)s);
    }
    tab[e] = cs;
  }
}

// grid: L*R blocks for slot metadata + 1 block for the static h/w tables.
__global__ void cache_init_kernel(CacheView c) {
  const int b = blockIdx.x;
  if (b < c.L * c.R) {
    const int l = b / c.R, r = b % c.R;
    int32_t* pos = c.pos + (size_t)b * c.slots;
    for (int s = threadIdx.x; s < c.slots; s += blockDim.x) pos[s] = -1;
    if (threadIdx.x == 0) c.count[b] = 0;
    __syncthreads();
    fill_ttab(c, l, r, 0, pos);
    return;
  }
  for (int e = threadIdx.x; e < c.gh * c.ph; e += blockDim.x) {
    const int h = e / c.ph, j = e % c.ph;
    double s, co;
    sincos((double)h * pow(c.theta, -(double)j / (double)c.ph), &s, &co);
    c.htab[e] = make_float2((float)co, (float)s);
  }
  for (int e = threadIdx.x; e < c.gw * c.pw; e += blockDim.x) {
    const int w = e / c.pw, j = e % c.pw;
    double s, co;
    sincos((double)w * pow(c.theta, -(double)j / (double)c.pw), &s, &co);
    c.wtab[e] = make_float2((float)co, (float)s);
  }
  if (threadIdx.x == 0) c.err[0] = 0;
}

// cos/sin of the kPairs rotation pairs from `pair0` on, for a token whose
// t-section row is `tt_row` and whose grid coordinates are (hh, ww).
template <int kPairs>
__device__ __forceinline__ void rope_cs(float2 (&cs)[kPairs], int pair0, const CacheView& c,
                                        const float2* tt_row, int hh, int ww) {
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const int pair = pair0 + i;
    if (pair < c.pt) cs[i] = __ldg(tt_row + pair);
    else if (pair < c.pt + c.ph) cs[i] = __ldg(c.htab + hh * c.ph + (pair - c.pt));
    else cs[i] = __ldg(c.wtab + ww * c.pw + (pair - c.pt - c.ph));
  }
}

// 3D RoPE of the pairs held by one 16-byte vector (4 bf16 pairs or 2 fp32
// pairs), given their cos/sin.
template <typename Elem>
__device__ __forceinline__ uint4 rotate16_cs(uint4 u, const float2 (&cs)[8 / sizeof(Elem)]) {
  constexpr int kPairs = 8 / sizeof(Elem);
  float vals[2 * kPairs];
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
  if constexpr (sizeof(Elem) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      vals[2 * i] = __uint_as_float(w4[i] << 16);
      vals[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) vals[i] = __uint_as_float(w4[i]);
  }
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const float a = vals[2 * i], b = vals[2 * i + 1];
    vals[2 * i] = a * cs[i].x - b * cs[i].y;
    vals[2 * i + 1] = a * cs[i].y + b * cs[i].x;
  }
  uint32_t o4[4];
  if constexpr (sizeof(Elem) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(vals[2 * i], vals[2 * i + 1]);
      o4[i] = *reinterpret_cast<const uint32_t*>(&b2);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) o4[i] = __float_as_uint(vals[i]);
  }
  return make_uint4(o4[0], o4[1], o4[2], o4[3]);
}

// The same for a vector whose first pair is `pair0`, looking its cos/sin up.
template <typename Elem>
__device__ __forceinline__ uint4 rotate16(uint4 u, int pair0, const CacheView& c,
                                          const float2* tt_row, int hh, int ww) {
  float2 cs[8 / sizeof(Elem)];
  rope_cs(cs, pair0, c, tt_row, hh, ww);
  return rotate16_cs<Elem>(u, cs);
}

// Commit copy: every CTA takes a run of token rows of one frame of one
// (layer, rollout); one warp per token row.  For its row a warp loads the
// block's K and V chunks (16-byte vectors, up to 2 x 8 per lane in flight),
// then stores K and V into the frame's ring slot and K, rotated to the frame's
// position t = n + f, into the rotated-key region.  K and V of a row travel
// together, so every CTA does the same work (per row: two reads and three
// writes of a row's size).  Index arithmetic
// is per row (token -> (h, w)); inside a row the lanes step through 32-bit
// chunk indices, and when every chunk a lane touches holds the same rotation
// pairs (32 is a multiple of the chunks per head row) their cos/sin are looked
// up once per row.  grid = (ceil(Tf / rows per CTA), nl * nr * F).
constexpr int kCopyThreads = 256;
constexpr int kCopyVecs = 16;  // 16-byte vectors per thread of the reset kernel
constexpr int kCommitWarps = kCopyThreads / 32;
constexpr int kCommitRowsPerWarp = 8;
constexpr int kCommitRowsPerCta = kCommitWarps * kCommitRowsPerWarp;
constexpr int kCommitBatch = 8;  // chunks per lane and tensor in flight

template <typename Elem, bool kFixedPairs>
__global__ void __launch_bounds__(kCopyThreads, 2)
    commit_copy_kernel(CacheView c, CommitParams p) {
  constexpr int kPer = 16 / sizeof(Elem);  // elements per 16-byte chunk
  constexpr int kPairs = kPer / 2;         // rotation pairs per chunk
  const int job = blockIdx.y;
  const int f = job % c.F;
  const int ri = (job / c.F) % p.nr;
  const int li = job / c.F / p.nr;
  if (f >= p.frames[ri]) return;
  const int l = p.layer0 + li, r = p.rollout0 + ri;
  const size_t lr = (size_t)l * c.R + r;
  const int n = c.count[lr];
  const int gslot = slot_of(n + f, c.S, c.W);
  if (gslot % c.N != c.shard) return;  // another shard stores this frame
  const int slot = gslot / c.N;          // local slot
  const uint32_t cpr = (uint32_t)c.d / kPer;      // chunks per head row
  const uint32_t row_chunks = cpr * (uint32_t)c.Hkv;  // chunks per token row
  const uint64_t src_off = ((uint64_t)r * c.F + f) * c.frame_bytes;
  const uint64_t dst_off = (lr * c.slots + slot) * c.frame_bytes;
  const uint4* ksrc = reinterpret_cast<const uint4*>(p.k[li] + src_off);
  const uint4* vsrc = reinterpret_cast<const uint4*>(p.v[li] + src_off);
  uint4* kdst = reinterpret_cast<uint4*>(c.k + dst_off);
  uint4* vdst = reinterpret_cast<uint4*>(c.v + dst_off);
  uint4* rdst = reinterpret_cast<uint4*>(c.krot + dst_off);
  // the ttab row slots + f holds frame n + f (the next block's frame f)
  const float2* tt_row = c.ttab + (lr * (c.slots + c.F) + c.slots + f) * c.pt;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  // kFixedPairs: 32 % cpr == 0 (chosen by the host)
  constexpr int kBatch = kFixedPairs ? kCommitBatch : kCommitBatch / 2;
  const int row_end = min(c.Tf, (int)(blockIdx.x + 1) * kCommitRowsPerCta);
  for (int tok = blockIdx.x * kCommitRowsPerCta + warp; tok < row_end; tok += kCommitWarps) {
    int hh = 0, ww = 0;
    if (tok < c.T) {
      const int tv = tok % c.Tv;  // position inside the token's view
      hh = tv / c.gw;
      ww = tv - hh * c.gw;
    }
    const uint64_t row = (uint64_t)tok * row_chunks;
    const uint4* ks = ksrc + row;
    const uint4* vs = vsrc + row;
    uint4* kd = kdst + row;
    uint4* vd = vdst + row;
    uint4* rd = rdst + row;
    float2 cs[kPairs];
    if (kFixedPairs) rope_cs(cs, (int)(lane % cpr) * kPairs, c, tt_row, hh, ww);
    for (uint32_t c0 = lane; c0 < row_chunks; c0 += 32 * kBatch) {
      uint4 kb[kBatch], vb[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const uint32_t ci = c0 + 32 * i;
        if (ci < row_chunks) {
          kb[i] = __ldcs(ks + ci);
          vb[i] = __ldcs(vs + ci);
        }
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const uint32_t ci = c0 + 32 * i;
        if (ci < row_chunks) {
          kd[ci] = kb[i];
          vd[ci] = vb[i];
          rd[ci] = kFixedPairs
                       ? rotate16_cs<Elem>(kb[i], cs)
                       : rotate16<Elem>(kb[i], (int)(ci % cpr) * kPairs, c, tt_row, hh, ww);
        }
      }
    }
  }
}

// After the copy: slot positions, counter and t table of every (layer, rollout).
__global__ void commit_meta_kernel(CacheView c, CommitParams p) {
  const int li = blockIdx.x / p.nr, ri = blockIdx.x % p.nr;
  const int l = p.layer0 + li, r = p.rollout0 + ri;
  const size_t lr = (size_t)l * c.R + r;
  int32_t* pos = c.pos + lr * c.slots;
  const int n = c.count[lr];
  const int nf = p.frames[ri];
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int f = 0; f < nf; ++f) {
      const int gslot = slot_of(n + f, c.S, c.W);
      if (gslot % c.N == c.shard) pos[gslot / c.N] = n + f;
    }
    c.count[lr] = n + nf;
  }
  __syncthreads();
  fill_ttab(c, l, r, n + nf, pos);
}

// Zero the K, V and rotated K of the listed rollouts in every layer.
// grid = (chunks per (layer, rollout) region, L * n * 3)
__global__ void __launch_bounds__(kCopyThreads)
    reset_zero_kernel(CacheView c, ResetParams p) {
  const int job = blockIdx.y;
  const int kv = job % 3;
  const int id = (job / 3) % p.n;
  const int l = (job / 3) / p.n;
  const int r = p.ids[id];
  const uint64_t region = (uint64_t)c.slots * c.frame_bytes;
  uint8_t* tensor = kv == 0 ? c.k : (kv == 1 ? c.v : c.krot);
  uint8_t* base = tensor + ((uint64_t)l * c.R + r) * region;
  uint4* dst = reinterpret_cast<uint4*>(base);
  const uint64_t nvec = region / 16;
  const uint64_t v0 = (uint64_t)blockIdx.x * kCopyThreads * kCopyVecs + threadIdx.x;
  const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int i = 0; i < kCopyVecs; ++i) {
    const uint64_t vi = v0 + (uint64_t)i * kCopyThreads;
    if (vi < nvec) dst[vi] = z;
  }
}

__global__ void reset_meta_kernel(CacheView c, ResetParams p) {
  const int l = blockIdx.x / p.n;
  const int r = p.ids[blockIdx.x % p.n];
  const size_t lr = (size_t)l * c.R + r;
  int32_t* pos = c.pos + lr * c.slots;
  for (int s = threadIdx.x; s < c.slots; s += blockDim.x) pos[s] = -1;
  if (threadIdx.x == 0) c.count[lr] = 0;
  __syncthreads();
  fill_ttab(c, l, r, 0, pos);
}

// 3D RoPE of up to two block tensors [R][F][Tx][heads][d] (e.g. the block's
// queries and keys of one call, in one launch): token row i of rollout r and
// frame f sits at t = n_r + f (t-row slots + f of the rollout's table).  The
// rows of tensor 0 come first, then those of tensor 1; one warp per token
// row; out may equal in (in place).
template <typename Elem>
struct RopeJob {
  const Elem* in;
  Elem* out;
  int Tx, heads;
  uint32_t rows;  // n_rollouts * F * Tx
};

template <typename Elem>
__global__ void __launch_bounds__(256)
    rope3d_kernel(CacheView c, int layer, RopeJob<Elem> j0, RopeJob<Elem> j1) {
  constexpr int kPer = 16 / sizeof(Elem);  // elements per 16-byte chunk
  // the attention kernel that follows may take multiprocessors this grid has
  // left (it waits for this grid's completion before reading its rows)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t cpr = c.d / kPer;         // chunks per head row
  const uint32_t rows_all = j0.rows + j1.rows;
  const uint32_t warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (uint32_t row_all = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row_all < rows_all; row_all += warps) {
    const bool second = row_all >= j0.rows;
    const RopeJob<Elem>& jb = second ? j1 : j0;
    const uint32_t row = second ? row_all - j0.rows : row_all;
    const int Tx = jb.Tx;
    const uint32_t row_chunks = cpr * jb.heads;  // chunks per token row
    const uint32_t r = row / (c.F * Tx);
    const uint32_t rem = row - r * (c.F * Tx);
    const int f = (int)(rem / Tx);
    const int tok = (int)(rem - f * Tx);
    const float2* tt = c.ttab + (((size_t)layer * c.R + r) * (c.slots + c.F) +
                                 c.slots + f) * c.pt;
    const int tv = tok % c.Tv;  // position inside the token's view
    const int hh = tok < c.T ? tv / c.gw : 0;
    const int ww = tok < c.T ? tv - hh * c.gw : 0;
    const uint4* src = reinterpret_cast<const uint4*>(jb.in) + (size_t)row * row_chunks;
    uint4* dst = reinterpret_cast<uint4*>(jb.out) + (size_t)row * row_chunks;
    if (32 % cpr == 0) {
      // every chunk a lane touches holds the same pairs (lane % cpr of each
      // head row): their cos/sin are looked up once per token row, and up to
      // 8 chunks per lane are loaded before any is rotated and stored
      constexpr int kPairs = kPer / 2;
      float2 cs[kPairs];
      rope_cs(cs, (int)(lane % cpr) * kPairs, c, tt, hh, ww);
      for (uint32_t base = lane; base < row_chunks; base += 32 * 8) {
        uint4 buf[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (base + 32 * i < row_chunks) buf[i] = src[base + 32 * i];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (base + 32 * i < row_chunks) dst[base + 32 * i] = rotate16_cs<Elem>(buf[i], cs);
      }
      continue;
    }
    for (uint32_t ci = lane; ci < row_chunks; ci += 32) {
      const int pair0 = (int)(ci % cpr) * (kPer / 2);
      dst[ci] = rotate16<Elem>(src[ci], pair0, c, tt, hh, ww);
    }
  }
}

template <typename Elem>
cudaError_t launch_rope_rows(const CacheView& c, int layer, int n_rollouts,
                             const void* in0, void* out0, int Tx0, int heads0,
                             const void* in1, void* out1, int Tx1, int heads1,
                             cudaStream_t s) {
  RopeJob<Elem> j0{static_cast<const Elem*>(in0), static_cast<Elem*>(out0), Tx0, heads0,
                   (uint32_t)((uint64_t)n_rollouts * c.F * Tx0)};
  RopeJob<Elem> j1{static_cast<const Elem*>(in1), static_cast<Elem*>(out1), Tx1, heads1,
                   in1 != nullptr ? (uint32_t)((uint64_t)n_rollouts * c.F * Tx1) : 0u};
  const uint64_t rows = (uint64_t)j0.rows + j1.rows;
  const uint64_t blocks_needed = (rows + 7) / 8;  // 8 warps per block
  const unsigned blocks = (unsigned)(blocks_needed < 148ull * 8 ? blocks_needed : 148ull * 8);
  rope3d_kernel<Elem><<<blocks, 256, 0, s>>>(c, layer, j0, j1);
  count_launch(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cache_init(const CacheView& c, cudaStream_t s) {
  cache_init_kernel<<<c.L * c.R + 1, 256, 0, s>>>(c);
  count_launch(1);
  return cudaGetLastError();
}

cudaError_t launch_commit(const CacheView& c, const CommitParams& p,
                          cudaStream_t s) {
  const unsigned row_blocks = (unsigned)((c.Tf + kCommitRowsPerCta - 1) / kCommitRowsPerCta);
  dim3 grid(row_blocks, (unsigned)(p.nl * p.nr * c.F));
  // whether every chunk a lane touches holds the same rotation pairs
  const bool fixed = 32 % (c.d * c.esz / 16) == 0;
  if (c.esz == 2) {
    if (fixed) commit_copy_kernel<uint16_t, true><<<grid, kCopyThreads, 0, s>>>(c, p);
    else commit_copy_kernel<uint16_t, false><<<grid, kCopyThreads, 0, s>>>(c, p);
  } else {
    if (fixed) commit_copy_kernel<float, true><<<grid, kCopyThreads, 0, s>>>(c, p);
    else commit_copy_kernel<float, false><<<grid, kCopyThreads, 0, s>>>(c, p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  commit_meta_kernel<<<p.nl * p.nr, 128, 0, s>>>(c, p);
  count_launch(2);
  return cudaGetLastError();
}

cudaError_t launch_reset(const CacheView& c, const ResetParams& p,
                         cudaStream_t s) {
  const uint64_t nvec = (uint64_t)c.slots * c.frame_bytes / 16;
  const uint64_t chunks = (nvec + kCopyThreads * kCopyVecs - 1) /
                          (kCopyThreads * kCopyVecs);
  dim3 grid((unsigned)chunks, (unsigned)(c.L * p.n * 3));
  reset_zero_kernel<<<grid, kCopyThreads, 0, s>>>(c, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  reset_meta_kernel<<<c.L * p.n, 128, 0, s>>>(c, p);
  count_launch(2);
  return cudaGetLastError();
}

cudaError_t launch_rope3d(const CacheView& c, int layer, int n_rollouts,
                          void* x, int Tx, int heads, cudaStream_t s) {
  if (c.esz == 2)
    return launch_rope_rows<uint16_t>(c, layer, n_rollouts, x, x, Tx, heads, nullptr,
                                      nullptr, 0, 0, s);
  return launch_rope_rows<float>(c, layer, n_rollouts, x, x, Tx, heads, nullptr, nullptr, 0,
                                 0, s);
}

cudaError_t launch_rope_block(const CacheView& c, int layer, int n_rollouts,
                              const void* q, void* q_out, const void* k, void* k_out,
                              cudaStream_t s) {
  if (c.esz != 2) return cudaErrorInvalidValue;  // the tensor-core path is bf16
  return launch_rope_rows<uint16_t>(c, layer, n_rollouts, q, q_out, c.T, c.H, k, k_out,
                                    c.Tf, c.Hkv, s);
}

}  // namespace fd
