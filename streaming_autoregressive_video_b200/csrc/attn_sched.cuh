// Schedule of the persistent tensor-core attention kernel, shared by that
// kernel and the kernel that folds the query-tile pairs it splits between
// CTAs (both must agree on which CTA holds which piece of which unit).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fd_internal.h"

namespace fd {
namespace attn {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile

struct TileCounts {
  int n1, n2, nt1, nt;
};

__device__ __forceinline__ TileCounts tile_counts(const AttnParams& p, int r) {
  TileCounts t;
  const int nv = valid_slots_local(valid_slots_global(p.count[r], p.S, p.W), p.N, p.shard);
  t.n1 = nv * p.Tf;
  t.n2 = p.shard == 0 ? p.F * p.Tf : 0;  // the block's keys belong to shard 0
  t.nt1 = (t.n1 + kBN - 1) / kBN;
  t.nt = t.nt1 + (t.n2 + kBN - 1) / kBN;
  return t;
}

// ---------------------------------------------------------------- schedule
// Work unit u = (rollout, head, pair) in that order; unit u has nt(rollout)
// KV iterations.  With U units and G CTAs, the first W = floor(U / G) waves
// run whole units (CTA c takes units c, c + G, ...: the CTAs of one head
// stream the same K/V tiles at the same time, so most of them come from L2);
// the iterations of the remaining U - W*G units, laid end to end, are cut
// into G equal ranges, one per CTA (its range starts at the SK iteration
// sk0 + c * I2 / G of the call's iteration space).  The host bounds the
// call's iterations so that iterations x G < 2^31: all of this is 32-bit.
struct Sched {
  int W;    // whole-unit waves
  int sk0;  // first iteration of the split part
  int I2;   // iterations of the split part
};

__device__ __forceinline__ Sched make_sched(const AttnParams& p) {
  const int per_r = p.H * p.nb;
  Sched s;
  s.W = p.n_rollouts * per_r / p.G;
  const int D = s.W * p.G;  // units run whole
  int total = 0, below = 0;
  for (int r = 0; r < p.n_rollouts; ++r) {
    const int nt = tile_counts(p, r).nt;
    total += per_r * nt;
    below += min(max(D - r * per_r, 0), per_r) * nt;
  }
  s.sk0 = below;
  s.I2 = total - below;
  return s;
}

// First iteration of CTA c's split range.
__device__ __forceinline__ int cta_begin(int c, const Sched& s, int G) {
  return s.sk0 + c * s.I2 / G;
}

// The (non-empty) CTA whose split range holds iteration x.
__device__ __forceinline__ int cta_of(int x, const Sched& s, int G) {
  return ((x - s.sk0 + 1) * G - 1) / s.I2;
}

// One unit's share of a CTA's work: KV tiles [kv0, kv1) of query-tile pair
// b of (rollout r, head h); the unit's iterations start at U0.
struct Piece {
  int r, h, b, kv0, kv1, unit, U0;
  TileCounts tc;
};

struct Cursor {
  int w;        // next whole-unit wave
  int it, end;  // next iteration, end of this CTA's split range
  int base;     // first iteration of rollout r
  int r;
  TileCounts tc;
};

__device__ __forceinline__ Cursor cursor_init(const AttnParams& p, const Sched& s) {
  Cursor c;
  c.w = 0;
  c.it = cta_begin(blockIdx.x, s, p.G);
  c.end = cta_begin(blockIdx.x + 1, s, p.G);
  c.base = 0;
  c.r = 0;
  c.tc = tile_counts(p, 0);
  return c;
}

// Next piece of this CTA's work, or false at its end.
__device__ __forceinline__ bool next_piece(const AttnParams& p, const Sched& s,
                                           Cursor& c, Piece& pc) {
  const int per_r = p.H * p.nb;
  while (c.w < s.W) {  // a whole unit
    const int unit = c.w * p.G + blockIdx.x;
    ++c.w;
    pc.r = unit / per_r;
    const int u = unit - pc.r * per_r;
    pc.tc = tile_counts(p, pc.r);
    if (pc.tc.nt == 0) continue;  // a shard with no key of this rollout
    pc.h = u / p.nb;
    pc.b = u - pc.h * p.nb;
    pc.kv0 = 0;
    pc.kv1 = pc.tc.nt;
    pc.unit = unit;
    pc.U0 = -1;  // not used by whole units
    return true;
  }
  if (c.it >= c.end) return false;
  int span = per_r * c.tc.nt;
  while (c.it >= c.base + span && c.r + 1 < p.n_rollouts) {
    c.base += span;
    ++c.r;
    c.tc = tile_counts(p, c.r);
    span = per_r * c.tc.nt;
  }
  const int rel = c.it - c.base;
  const int u = rel / c.tc.nt;
  pc.r = c.r;
  pc.tc = c.tc;
  pc.h = u / p.nb;
  pc.b = u - pc.h * p.nb;
  pc.U0 = c.base + u * c.tc.nt;
  pc.kv0 = c.it - pc.U0;
  pc.kv1 = min(c.tc.nt, c.end - pc.U0);
  pc.unit = c.r * per_r + u;
  c.it = pc.U0 + pc.kv1;
  return true;
}

// Partial-result slot of CTA c's piece of the split unit starting at U0:
// slot 0 when the piece opens the CTA's split range, slot 1 when it closes it.
__device__ __forceinline__ const float* part_slot(const AttnParams& p, int c,
                                                  int U0, const Sched& s) {
  const int slot = cta_begin(c, s, p.G) >= U0 ? 0 : 1;
  return p.part + ((size_t)c * 2 + slot) * kPartSlotFloats;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 r = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&r);
}

}  // namespace attn
}  // namespace fd
