// bf16 block-causal chunk attention on sm_100a tensor cores.
//
// What it computes (the behaviour is described on the pages; the formulas are
// the readings stated in include/fd.h): for every query of the current block
// of a rollout, softmax(q' k'^T / sqrt(d)) v over the rollout's valid cache
// tokens (sink frames + rolling window, "NVIDIA FlashDreams ...", Bounded
// Memory for Infinite Rollouts) and all tokens of the block itself, which
// attend to each other bidirectionally ("Cosmos3-H-Dreams" model card, Model
// Architecture: block-causal student with a KV cache; AlpaDreams GTC 2026
// write-up, section VII).  q' and k' carry 3D (t,h,w) RoPE and arrive rotated:
// cache keys were rotated once when their frame was committed, the block's
// queries and keys once per call by a pass over the block before this kernel
// (every query tile of a head reads the same keys, and a rotated query tile
// can be copied straight into the tensor core's operand layout).
//
// Schedule (persistent, G = one CTA per multiprocessor): a work unit is one
// 256-row query-tile pair of one (rollout, head) against all of the
// rollout's KV tiles.  The first floor(U / G) waves run whole units (CTA c
// takes units c, c + G, ...: the CTAs of one head stream the same K/V tiles
// together); the KV iterations of the remaining units, laid end to end
// (rollout, head, pair, KV tile), are cut into G equal ranges, one per CTA,
// so no SM idles through a partly filled last wave (attn_sched.cuh).  A unit
// cut by a range boundary is computed in pieces; every piece leaves its
// unnormalised rows (column-chunk-major), row maxima and row sums (fp32) in
// the work set's partial-result area, and a fold kernel launched right after
// this one (fold.cu) combines the pieces of each split unit in a fixed order
// and writes its rows.  No CTA ever waits for another.
//
// Roles (all warps walk the same sequence of pieces):
//   warp 0        TMA producer: each piece's two Q tiles (once the previous
//                 piece's last S product has read the old ones), then K and V
//                 tiles through 2-stage K and V shared-memory rings, walking
//                 the valid slot prefix of the cache and then the block; the
//                 ring's wraparound needs no gather because attention does
//                 not depend on key order.  No cluster multicast.
//   warp 1        MMA issuer (one thread): S = Q K^T and O += P V on tcgen05
//                 (kind::f16, bf16 operands, fp32 accumulators in TMEM); the
//                 two query tiles ping-pong so one tile's softmax overlaps the
//                 other tile's matrix products.
//   warp 2        TMEM allocator (512 columns: S0, S1, O0, O1).
//   warps 4-7     no role (their registers go to the softmax warpgroups).
//   warps 8-15    softmax: warpgroup x owns query tile x, one thread per
//                 query row (TMEM lane), all 128 columns: row max, exp2, row
//                 sum, P rounded to bf16 and written back into the S columns
//                 of TMEM as the A operand of the PV product; the
//                 O rescale is skipped unless the running max grows by more
//                 than 2^8, which keeps P <= 256 and the result exact up to
//                 rounding.  The epilogue divides by the row sum and writes
//                 bf16 rows staged through shared memory (and the optional
//                 log-sum-exp), or hands a split unit's piece over as
//                 described above.
// Every mbarrier wait is bounded: a wait that gives up raises a CTA-wide
// abort flag and the device error word, in-flight copies and MMAs are
// drained with bounded waits, TMEM is released and the CTA exits.
#include <cuda.h>
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

constexpr int kThreads = 512;
// one 64-column, 128-byte-swizzled half of a tile: 128 rows x 128 bytes
constexpr uint32_t kHalf = kBM * 64 * 2;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8
// Every kPolyEvery-th pair of exponentials on the FMA pipe (0: all on MUFU).
// At D = 128 the polynomial's extra instructions cost more than the MUFU time
// they free (measured: 505 us per 480p call all on MUFU, 521 us with every
// second pair on the FMA pipe).  At D = 64 the tensor work per tile halves
// while the exponentials stay, so MUFU is the limit and every third pair on
// the FMA pipe pays (0.805 -> 0.763 ms per 24-head 480p call; every second
// pair 0.859, every fourth 0.773).
template <int D>
constexpr int kPolyEvery = D == 64 ? 3 : 0;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s

// TMEM columns: S0 at 0, S1 at 128 (128 keys each), O0 at 256, O1 at 256 + D
constexpr uint32_t kColS0 = 0, kColO0 = 256;

constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false);

struct Shared {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full, o_empty, drain;
  uint32_t tmem_base;
  int32_t abort;
};

static_assert(sizeof(Shared) <= 256, "barrier block");
constexpr uint32_t kSmemMax = 232448;  // per-block opt-in limit on sm_100

// Shared-memory layout and per-head-size constants of the kernel for head
// size D (64 or 128): Q (two tiles), K and V stages of 128 rows x D bf16, each
// tile stored as D/64 column halves of 128 rows x 128 bytes (one 128-byte
// swizzle atom per row), then the barriers and the piece ring.
template <int D>
struct Geo {
  static_assert(D == 64 || D == 128, "head size of the tensor-core kernel");
  static constexpr uint32_t kTile = kBM * D * 2;  // 32 KB (D = 128) or 16 KB
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = 2 * kTile;
  static constexpr uint32_t kOffV = kOffK + kKStages * kTile;
  static constexpr uint32_t kOffShared = kOffV + kVStages * kTile;
  static constexpr uint32_t kOffMeta = kOffShared + 256;  // struct Meta
  // epilogue staging: 4 KB per softmax warp (32 rows x 64 bf16 columns)
  static constexpr uint32_t kOffStage = kOffMeta + 256;
  static constexpr uint32_t kStageWarp = 32 * 64 * 2;
  static constexpr uint32_t kSmemFixed = kOffStage + 8 * kStageWarp + 1024;  // + alignment slack
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, true);
};
static_assert(Geo<128>::kSmemFixed <= kSmemMax, "shared memory of the d = 128 kernel");

// Site codes for the device error word.
enum : int { kSiteProducer = 1, kSiteMma = 3, kSiteSoftmax = 4,
             kSiteSelftest = 5 };

// Bounded wait.  kSpin (MMA issuer, softmax: the critical path) polls, so
// the waiter resumes as soon as the phase completes; the other roles sleep
// between polls and leave issue slots to the working warps.
template <bool kSpin>
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity,
                                             int32_t* abort, int32_t* err,
                                             int site, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!(kSpin ? mbar_try_wait(bar, parity) : mbar_try_wait_sleep(bar, parity))) {
    if (*reinterpret_cast<volatile int32_t*>(abort)) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *reinterpret_cast<volatile int32_t*>(abort) = 1;
      atomicCAS(err, 0, kDevErrTimeout | (site << 8));
      return false;
    }
  }
  return true;
}

template <bool kSpin = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity,
                                         Shared* sh, int32_t* err, int site) {
  return bounded_wait<kSpin>(bar, parity, &sh->abort, err, site, kWaitLimitNs);
}

// Bounded wait used only while tearing down after an abort.
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// What every role needs to know about a piece.  The producer walks the
// schedule and publishes each piece in a 4-entry ring in shared memory
// (entry k & 3, `seq` = k written last); the other roles read the entry
// after their first wait for that piece, so only the producer holds the
// schedule's cursor in registers.  A piece's entry is overwritten four
// pieces later, long after every role has finished with it.
struct PieceInfo {
  int r, h, b, kv0, kv1, unit, U0, nt, nt1, n1, n2;
  int seq;
};

struct Meta {
  PieceInfo ring[4];
  int n_pieces;   // pieces of this CTA
  int my_begin;   // first iteration of this CTA's split range
  Sched sd;
};
static_assert(sizeof(Meta) <= 256, "meta block");

// End of every role branch: all 512 threads meet on named barrier 1 (each
// warp arrives from its own branch), then warp 2 releases the TMEM columns.
__device__ __forceinline__ void teardown(int warp, uint32_t tmem) {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}


// Reads ring entry k once the producer has published it (bounded wait).
__device__ __forceinline__ bool read_piece(const Meta* meta, int k, PieceInfo& pi,
                                           Shared* sh, int32_t* err, int site) {
  const volatile PieceInfo* e = &meta->ring[k & 3];
  if (e->seq != k) {
    const uint64_t t0 = globaltimer_ns();
    while (e->seq != k) {
      if (*reinterpret_cast<volatile int32_t*>(&sh->abort)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *reinterpret_cast<volatile int32_t*>(&sh->abort) = 1;
        atomicCAS(err, 0, kDevErrTimeout | (site << 8));
        return false;
      }
    }
  }
  __threadfence_block();
  pi.r = e->r;
  pi.h = e->h;
  pi.b = e->b;
  pi.kv0 = e->kv0;
  pi.kv1 = e->kv1;
  pi.unit = e->unit;
  pi.U0 = e->U0;
  pi.nt = e->nt;
  pi.nt1 = e->nt1;
  pi.n1 = e->n1;
  pi.n2 = e->n2;
  pi.seq = k;
  return true;
}

// Whether query tile 1 of pair b holds any query row (the last pair of a
// head may end inside tile 0: tile 1 is then skipped altogether).
__device__ __forceinline__ bool tile1_used(const AttnParams& p, int b) {
  return b * 2 * kBM + kBM < p.Mq;
}

// KV iterations of ring entry k and whether its tile 1 is used (what the MMA
// issuer needs of a piece).
__device__ __forceinline__ bool read_piece_len(const Meta* meta, int k, int& n, bool& two,
                                               const AttnParams& p, Shared* sh, int32_t* err,
                                               int site) {
  const volatile PieceInfo* e = &meta->ring[k & 3];
  if (e->seq != k) {
    const uint64_t t0 = globaltimer_ns();
    while (e->seq != k) {
      if (*reinterpret_cast<volatile int32_t*>(&sh->abort)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *reinterpret_cast<volatile int32_t*>(&sh->abort) = 1;
        atomicCAS(err, 0, kDevErrTimeout | (site << 8));
        return false;
      }
    }
  }
  __threadfence_block();
  n = e->kv1 - e->kv0;
  two = tile1_used(p, e->b);
  return true;
}

template <int D>
__device__ __forceinline__ void attn_body(const CUtensorMap& tm_q, const CUtensorMap& tm_kc,
                                          const CUtensorMap& tm_vc, const CUtensorMap& tm_kb,
                                          const CUtensorMap& tm_vb, const AttnParams& p) {
  using G = Geo<D>;
  constexpr uint32_t kTile = G::kTile;
  constexpr uint32_t kOffQ = G::kOffQ, kOffK = G::kOffK, kOffV = G::kOffV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + G::kOffShared);
  Meta* meta = reinterpret_cast<Meta*>(smem + G::kOffMeta);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    mbar_init(&sh->q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sh->s_full[x], 1);
      mbar_init(&sh->p_full[x], 128);
    }
    mbar_init(&sh->o_full, 1);
    mbar_init(&sh->o_empty, 256);
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_mbarrier_init();
    // the CTA's schedule: how many pieces, where its split range starts
    const Sched sd = make_sched(p);
    Cursor c = cursor_init(p, sd);
    meta->sd = sd;
    meta->my_begin = c.it;
    int n = 0;
    Piece pc;
    while (next_piece(p, sd, c, pc)) ++n;
    meta->n_pieces = n;
    for (int i = 0; i < 4; ++i) meta->ring[i].seq = -1;
  }
  if (warp == 2) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int n_pieces = meta->n_pieces;
  // launched as a programmatic dependent of the pass that rotates the
  // block's queries and keys: wait for it before any copy, then let the fold
  // kernel that follows start on multiprocessors this grid leaves
  griddep_wait();
  griddep_launch_dependents();

  // Register split (launch: 512 threads x 128): the producer/MMA warpgroup and
  // the idle warpgroup 1 give registers to the two softmax warpgroups, which
  // keep a whole 128-column S row in registers.  88 + 72 + 176 + 176 = 4 x 128.
  // Each warpgroup changes its count exactly once, at the top of its branch,
  // and never takes registers back: a later increase could claim registers a
  // softmax warpgroup is still waiting for.  Each branch ends in its own
  // teardown (block-wide named barrier, then TMEM release) and returns, so no
  // code runs after the branches join.  Inside a branch, groups of warps
  // synchronise only through bounded mbarrier waits (a warp that gives up
  // must not leave the others blocked on a named barrier).
  if (warp < 4) {
    regs_dec<88>();
    if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      prefetch_tmap(&tm_kb);
      prefetch_tmap(&tm_vb);
      const Sched sd = meta->sd;
      Cursor cur = cursor_init(p, sd);
      Piece pc;
      int g = 0, issued_k = 0, issued_v = 0;  // KV iterations of the CTA
      int issued_q = 0;                       // pieces of the CTA
      bool ok = true;
      for (int k = 0; ok && next_piece(p, sd, cur, pc); ++k) {
        // the Q tiles are reused once the previous piece's S products are done
        if (k > 0 && !wait_bar(&sh->q_empty, (k - 1) & 1, sh, p.err, kSiteProducer)) {
          ok = false;
          break;
        }
        volatile PieceInfo* e = &meta->ring[k & 3];
        e->r = pc.r;
        e->h = pc.h;
        e->b = pc.b;
        e->kv0 = pc.kv0;
        e->kv1 = pc.kv1;
        e->unit = pc.unit;
        e->U0 = pc.U0;
        e->nt = pc.tc.nt;
        e->nt1 = pc.tc.nt1;
        e->n1 = pc.tc.n1;
        e->n2 = pc.tc.n2;
        __threadfence_block();
        e->seq = k;
        mbar_arrive_expect_tx(&sh->q_full, 2 * kTile);
        for (int t = 0; t < 2; ++t)
          for (int hf = 0; hf < G::kHalves; ++hf)
            tma_load_4d(smem + kOffQ + t * kTile + hf * kHalf, &tm_q, &sh->q_full,
                        hf * 64, pc.h, pc.b * 2 * kBM + t * kBM, pc.r);
        issued_q = k + 1;
        // keys: rotated cache keys or the block keys rotated for this call,
        // both batched by (layer, rollout); values: cache (layer, rollout)
        // or the caller's block values (rollout); head: the query head's
        // key/value head (grouped-query attention)
        const int hkv = pc.h / p.kv_group;
        for (int j = pc.kv0; j < pc.kv1; ++j, ++g) {
          const bool seg1 = j < pc.tc.nt1;
          const int key0 = seg1 ? j * kBN : (j - pc.tc.nt1) * kBN;
          const CUtensorMap* mk = seg1 ? &tm_kc : &tm_kb;
          const CUtensorMap* mv = seg1 ? &tm_vc : &tm_vb;
          const int ck3 = seg1 ? p.map_row0 + pc.r : p.kb_row0 + pc.r;
          const int cv3 = seg1 ? p.map_row0 + pc.r : pc.r;
          const int ks = g % kKStages;
          if (g >= kKStages &&
              !wait_bar(&sh->k_empty[ks], ((g / kKStages) - 1) & 1, sh, p.err,
                        kSiteProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sh->k_full[ks], kTile);
          for (int hf = 0; hf < G::kHalves; ++hf)
            tma_load_4d(smem + kOffK + ks * kTile + hf * kHalf, mk,
                        &sh->k_full[ks], hf * 64, hkv, key0, ck3);
          issued_k = g + 1;
          const int vs = g % kVStages;
          if (g >= kVStages &&
              !wait_bar(&sh->v_empty[vs], ((g / kVStages) - 1) & 1, sh, p.err,
                        kSiteProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sh->v_full[vs], kTile);
          for (int hf = 0; hf < G::kHalves; ++hf)
            tma_load_4d(smem + kOffV + vs * kTile + hf * kHalf, mv,
                        &sh->v_full[vs], hf * 64, hkv, key0, cv3);
          issued_v = g + 1;
        }
      }
      if (*reinterpret_cast<volatile int32_t*>(&sh->abort)) {
        // let every copy still in flight land before the CTA exits
        if (issued_q > 0) drain_bar(&sh->q_full, (issued_q - 1) & 1);
        for (int j = max(0, issued_k - kKStages); j < issued_k; ++j)
          drain_bar(&sh->k_full[j % kKStages], (j / kKStages) & 1);
        for (int j = max(0, issued_v - kVStages); j < issued_v; ++j)
          drain_bar(&sh->v_full[j % kVStages], (j / kVStages) & 1);
      }
    }
    __syncwarp();
    } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Shared-memory descriptors as (lo, hi) halves: hi (stride 1024 B,
      // version 1, 128-byte swizzle) is common to all tiles; lo is the tile's
      // address >> 4 with the leading-byte offset (16 B for the K-major Q and
      // K tiles, one 64-column half for the MN-major V tile), and a k-step
      // inside the tile adds its byte offset >> 4.  The bases are made opaque
      // per call so the compiler adds the step offsets as it issues instead
      // of keeping every (tile, step) descriptor live across the loop.
      constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
      const uint32_t q_lo = ((smem_addr(smem + kOffQ) & 0x3FFFFu) >> 4) | (1u << 16);
      const uint32_t k_lo = ((smem_addr(smem + kOffK) & 0x3FFFFu) >> 4) | (1u << 16);
      const uint32_t v_lo = ((smem_addr(smem + kOffV) & 0x3FFFFu) >> 4) | ((kHalf >> 4) << 16);
      const uint32_t desc_hi = kDescHi;
      auto issue_s = [&](int x, int ks) {
        uint32_t a = q_lo + x * (kTile >> 4), b = k_lo + ks * (kTile >> 4);
        asm volatile("" : "+r"(a), "+r"(b));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t step = (kk >> 2) * (kHalf >> 4) + (kk & 3) * 2;  // 32 B per k-step
          mma_ss_lo(tmem + kColS0 + x * 128, a + step, b + step, desc_hi, kIdescQK, kk > 0);
        }
      };
      auto issue_pv = [&](int x, int vs, bool acc) {
        uint32_t b = v_lo + vs * (kTile >> 4);
        asm volatile("" : "+r"(b));
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          mma_ts_lo(tmem + kColO0 + x * D, tmem + kColS0 + x * 128 + kk * 8,
                    b + kk * (2048 >> 4), desc_hi, G::kIdescPV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // K tiles arrive rotated (cache keys at commit, block keys once per
      // call), so a K tile is ready as soon as its copy has landed.
      auto wait_k = [&](int g) -> bool {
        return wait_bar<true>(&sh->k_full[g % kKStages], (g / kKStages) & 1, sh, p.err,
                              kSiteMma);
      };
      // g counts the CTA's KV iterations (the K/V rings and tile 0's
      // barriers), g1 only those of pieces whose tile 1 is used (its barriers)
      int g = 0, g1 = 0;
      bool ok = true;
      for (int k = 0; k < n_pieces && ok; ++k) {
        int n = 0;
        bool two = true;
        ok = wait_bar<true>(&sh->q_full, k & 1, sh, p.err, kSiteMma) &&
             read_piece_len(meta, k, n, two, p, sh, p.err, kSiteMma) && wait_k(g);
        if (!ok) break;
        tc_fence_after();
        const int ks0 = g % kKStages;
        issue_s(0, ks0);
        mma_commit(&sh->s_full[0]);
        if (two) {
          issue_s(1, ks0);
          mma_commit(&sh->s_full[1]);
        }
        mma_commit(&sh->k_empty[ks0]);
        if (n == 1) mma_commit(&sh->q_empty);
        for (int jj = 0; jj < n; ++jj) {
          const int gj = g + jj, g1j = g1 + jj;
          const int vs = gj % kVStages;
          ok = wait_bar<true>(&sh->v_full[vs], (gj / kVStages) & 1, sh, p.err, kSiteMma) &&
               wait_bar<true>(&sh->p_full[0], gj & 1, sh, p.err, kSiteMma);
          // the first products of a piece overwrite O: the previous piece's
          // epilogue must have read it
          if (ok && jj == 0 && k > 0)
            ok = wait_bar<true>(&sh->o_empty, (k - 1) & 1, sh, p.err, kSiteMma);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, vs, jj > 0);
          const bool more = jj + 1 < n;
          const int ks = (gj + 1) % kKStages;
          if (more) {
            ok = wait_k(gj + 1);
            if (!ok) break;
            tc_fence_after();
            issue_s(0, ks);
            mma_commit(&sh->s_full[0]);
          }
          if (two) {
            ok = wait_bar<true>(&sh->p_full[1], g1j & 1, sh, p.err, kSiteMma);
            if (!ok) break;
            tc_fence_after();
            issue_pv(1, vs, jj > 0);
          }
          mma_commit(&sh->v_empty[vs]);
          if (more) {
            if (two) {
              issue_s(1, ks);
              mma_commit(&sh->s_full[1]);
            }
            mma_commit(&sh->k_empty[ks]);
            if (jj + 2 == n) mma_commit(&sh->q_empty);  // last S products of the piece
          }
        }
        if (!ok) break;
        mma_commit(&sh->o_full);
        g += n;
        if (two) g1 += n;
      }
      if (!ok) {
        // wait for the tensor core to finish what was issued
        mma_commit(&sh->drain);
        drain_bar(&sh->drain, 0);
      }
    }
    __syncwarp();
    }
    teardown(warp, tmem);
    return;
  } else if (warp < 8) {
    // warpgroup 1 has no role: the queries arrive rotated (a pass before
    // this kernel rotates the block's queries and keys)
    regs_dec<72>();
    teardown(warp, tmem);
    return;
  } else {
    regs_inc<176>();
    // ------------------------------------------------------------ softmax
    // Warpgroup x (warps 8-11: x = 0, warps 12-15: x = 1) owns query tile x:
    // one thread per query row (TMEM lane), all 128 columns, so no row data
    // is exchanged.  The MMA ping-pong keeps the two warpgroups half a period
    // apart: while one waits for its S tile or TMEM traffic, the other
    // computes on the same SMSPs.
    const int x = (warp - 8) >> 2;     // tile of this warpgroup
    const int wq = warp & 3;           // lane quarter
    const int row_t = wq * 32 + lane;  // row within the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS0 + x * 128;
    const uint32_t tO = tmem + lane_off + kColO0 + x * D;
    const float sl2 = p.scale_log2;
    int g = 0;  // KV iterations this warpgroup's tile has run (its barriers' phases)
    bool ok = true;
    uint32_t sa[64], sb[64];
    for (int k = 0; k < n_pieces && ok; ++k) {
      int n, kv0, nt1, n1, n2;
      {
        PieceInfo pi;
        ok = __all_sync(0xffffffffu, read_piece(meta, k, pi, sh, p.err, kSiteSoftmax));
        if (!ok) break;
        // tile 1 of a head's last pair may hold no query row: the tensor core
        // computes nothing for it and this warpgroup skips the piece's loop
        const bool used = x == 0 || tile1_used(p, pi.b);
        n = used ? pi.kv1 - pi.kv0 : 0;
        kv0 = pi.kv0;
        nt1 = pi.nt1;
        n1 = pi.n1;
        n2 = pi.n2;
      }
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < n && ok; ++jj) {
        const int gj = g + jj;
        const int j = kv0 + jj;
        const int valid = j < nt1 ? min(kBN, n1 - j * kBN) : min(kBN, n2 - (j - nt1) * kBN);
        ok = __all_sync(0xffffffffu, wait_bar<true>(&sh->s_full[x], gj & 1, sh, p.err,
                                                    kSiteSoftmax));
        if (!ok) break;
        tc_fence_after();
        tmem_ld64(tS, sa);
        tmem_ld64(tS + 64, sb);
        if (valid < kBN) {  // last tile of a segment: keys past its end weigh 0
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            if (i >= valid) sa[i] = 0xFF800000u;
            if (64 + i >= valid) sb[i] = 0xFF800000u;
          }
        }
        // row max: three-input max, eight independent chains, two new
        // columns per step
        auto col = [&](int c) {
          return __uint_as_float(c < 64 ? sa[c] : sb[c - 64]);
        };
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmax3(col(i), col(i + 8), col(i + 16));
#pragma unroll
        for (int c = 24; c < 128; c += 2)
          m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], col(c), col(c + 1));
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
        const float m_tile = mx * sl2;
        const bool need = m_tile > m + kRescaleThreshold;
        if (jj > 0 && __any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m - m_tile) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t r16[16];
            tmem_ld16(tO + c * 16, r16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              r16[i] = __float_as_uint(__uint_as_float(r16[i]) * alpha);
            tmem_st16(tO + c * 16, r16);
          }
          tmem_wait_st();
        }
        if (need) {
          l = (jj > 0) ? l * ex2_approx(m - m_tile) : 0.f;
          m = m_tile;
        }
        // P = 2^(s * log2(e)/sqrt(d) - m), two columns per packed
        // instruction.  In full tiles every kPolyEvery-th pair of
        // exponentials runs on the FMA pipe (exp2_poly2) to share the load of
        // the MUFU unit; partial tiles (masked columns at -inf) use MUFU
        // throughout so masked weights are exactly 0.  Row sums accumulate
        // in packed pairs.
        const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
        uint64_t ls2 = 0;  // two packed +0.0f
        uint32_t pk[32];
        auto exps = [&](const uint32_t* sv, bool full) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint64_t x2 = f2_fma(
                f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sc2, nm2);
            uint64_t e2;
            constexpr int kEvery = kPolyEvery<D> > 0 ? kPolyEvery<D> : 1;
            if (kPolyEvery<D> > 0 && full && (i % kEvery) == kEvery - 1) {
              e2 = exp2_poly2(x2);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            ls2 = f2_add(ls2, e2);
            float p0, p1;
            f2_unpack(e2, p0, p1);
            pk[i] = pack_bf16(p0, p1);
          }
        };
        // bf16 P of columns 0-63 goes to TMEM columns 0-31, of columns
        // 64-127 to columns 32-63 (S columns 64-127 are already in registers)
        // with every exponential on MUFU, a partial tile's masked columns
        // give exactly 0 and one copy of the loop serves all tiles; with
        // the FMA-pipe share (d = 64) full and partial tiles get their own
        if constexpr (kPolyEvery<D> > 0) {
          if (valid == kBN) exps(sa, true); else exps(sa, false);
        } else {
          exps(sa, true);
        }
        tmem_st32(tS, pk);
        if constexpr (kPolyEvery<D> > 0) {
          if (valid == kBN) exps(sb, true); else exps(sb, false);
        } else {
          exps(sb, true);
        }
        tmem_st32(tS + 32, pk);
        {
          float la, lb;
          f2_unpack(ls2, la, lb);
          l += la + lb;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh->p_full[x]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu,
                      wait_bar(&sh->o_full, k & 1, sh, p.err, kSiteSoftmax));
      if (!ok) break;
      tc_fence_after();
      // the piece again, from its ring entry (not kept in registers above)
      PieceInfo pi;
      ok = __all_sync(0xffffffffu, read_piece(meta, k, pi, sh, p.err, kSiteSoftmax));
      if (!ok) break;
      const int row = x * kBM + row_t;  // row within the pair
      const bool whole = pi.kv0 == 0 && pi.kv1 == pi.nt;
      const int qrow = pi.b * 2 * kBM + row;
      if (!whole) {
        // a piece of a unit split between CTAs: hand it over (unnormalised
        // row, running max, row sum) to the fold that runs after this kernel
        float* part = p.part + ((size_t)blockIdx.x * 2 +
                                (pi.U0 + pi.kv0 == meta->my_begin ? 0 : 1)) * kPartSlotFloats;
        // O in column-chunk-major order ([D/4][256 rows][4 columns]): the
        // 32 lanes of a warp hold consecutive rows, so each store of a warp
        // covers 512 contiguous bytes
        uint32_t rr[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tO + c * 32, rr);
          float4* dst = reinterpret_cast<float4*>(part) + (size_t)c * 8 * 2 * kBM + row;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i * 2 * kBM] =
                make_float4(__uint_as_float(rr[4 * i]), __uint_as_float(rr[4 * i + 1]),
                            __uint_as_float(rr[4 * i + 2]), __uint_as_float(rr[4 * i + 3]));
        }
        part[2 * kBM * D + row] = m;
        part[2 * kBM * D + 2 * kBM + row] = l;
      } else {
        // a whole unit: O / l in bf16 (and the log-sum-exp).  Each warp
        // stages its 32 rows 64 columns at a time in shared memory (16-byte
        // chunks XOR-swizzled by row) and writes them back four rows per
        // store, 128 contiguous bytes a row, instead of one row per lane.
        const float inv_l = 1.f / l;
        uint8_t* stage = smem + G::kOffStage + (warp - 8) * G::kStageWarp;
        const int qrow_w = pi.b * 2 * kBM + x * kBM + wq * 32;  // the warp's first row
        uint32_t rr[32];
#pragma unroll 1
        for (int hf = 0; hf < D / 64; ++hf) {
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            tmem_ld32(tO + hf * 64 + c2 * 32, rr);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 v = make_uint4(
                  pack_bf16(__uint_as_float(rr[8 * i]) * inv_l, __uint_as_float(rr[8 * i + 1]) * inv_l),
                  pack_bf16(__uint_as_float(rr[8 * i + 2]) * inv_l, __uint_as_float(rr[8 * i + 3]) * inv_l),
                  pack_bf16(__uint_as_float(rr[8 * i + 4]) * inv_l, __uint_as_float(rr[8 * i + 5]) * inv_l),
                  pack_bf16(__uint_as_float(rr[8 * i + 6]) * inv_l, __uint_as_float(rr[8 * i + 7]) * inv_l));
              const int chunk = c2 * 4 + i;
              *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = v;
            }
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rw = i * 4 + (lane >> 3), cc = lane & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(stage + rw * 128 + ((cc ^ (rw & 7)) << 4));
            const int qr = qrow_w + rw;
            if (qr < p.Mq)
              *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) +
                                        (((size_t)pi.r * p.Mq + qr) * p.H + pi.h) * D + hf * 64 +
                                        cc * 8) = v;
          }
          __syncwarp();
        }
        if (p.lse != nullptr && qrow < p.Mq)
          p.lse[((size_t)pi.r * p.H + pi.h) * p.Mq + qrow] =
              (m + log2f(l)) * 0.69314718055994530942f;
      }
      // O may now be overwritten by the next piece
      tc_fence_before();
      mbar_arrive(&sh->o_empty);
      g += n;
    }
    teardown(warp, tmem);
    return;
  }
}

// The kernels for head sizes 128 and 64 (the same body, instantiated).
__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_d128_sm100(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_kc,
                         const __grid_constant__ CUtensorMap tm_vc,
                         const __grid_constant__ CUtensorMap tm_kb,
                         const __grid_constant__ CUtensorMap tm_vb,
                         const __grid_constant__ AttnParams p) {
  attn_body<128>(tm_q, tm_kc, tm_vc, tm_kb, tm_vb, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_d64_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_kc,
                        const __grid_constant__ CUtensorMap tm_vc,
                        const __grid_constant__ CUtensorMap tm_kb,
                        const __grid_constant__ CUtensorMap tm_vb,
                        const __grid_constant__ AttnParams p) {
  attn_body<64>(tm_q, tm_kc, tm_vc, tm_kb, tm_vb, p);
}

using AttnKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap, const CUtensorMap, const AttnParams);

// The warpgroup register split (setmaxnreg) assumes the block launches with
// exactly 128 registers per thread; refuse to launch otherwise, as the
// increase would wait forever for registers that do not exist.
cudaError_t prepare_kernel(AttnKernel k) {
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, k);
  if (err != cudaSuccess) return err;
  if (fa.numRegs != 128) return cudaErrorNotSupported;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kSmemMax);
}

}  // namespace

size_t attn_bf16_smem_bytes(const AttnParams& p) {
  if (p.d != 64 && p.d != 128) return 0;
  const size_t smem = p.d == 128 ? Geo<128>::kSmemFixed : Geo<64>::kSmemFixed;
  return smem > kSmemMax ? 0 : smem;
}

cudaError_t launch_attn_bf16_sm100(const CUtensorMap& tm_q,
                                   const CUtensorMap& tm_kc,
                                   const CUtensorMap& tm_vc,
                                   const CUtensorMap& tm_kb,
                                   const CUtensorMap& tm_vb,
                                   const AttnParams& p, cudaStream_t s) {
  static PerDeviceOnce attr;
  cudaError_t e = once_per_device(attr, [] {
    cudaError_t err = prepare_kernel(attn_bf16_d128_sm100);
    return err == cudaSuccess ? prepare_kernel(attn_bf16_d64_sm100) : err;
  });
  if (e != cudaSuccess) return e;
  const size_t smem = attn_bf16_smem_bytes(p);
  if (smem == 0) return cudaErrorNotSupported;
  if (p.G < 1 || p.G > kAttnMaxCtas) return cudaErrorInvalidValue;
  // launched as a programmatic dependent of the kernel before it on the
  // stream (the RoPE pass): it waits for that kernel on the device before
  // reading its rows; the fold that follows is launched the same way
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  cudaError_t e2 = cudaLaunchKernelEx(&cfg, p.d == 128 ? attn_bf16_d128_sm100 : attn_bf16_d64_sm100,
                                      tm_q, tm_kc, tm_vc, tm_kb, tm_vb, p);
  count_launch(1);
  if (e2 != cudaSuccess) return e2;
  // the units past the whole-unit waves may be split between CTAs: fold them
  const int64_t units = (int64_t)p.n_rollouts * p.H * p.nb;
  const int64_t split = units - units / p.G * p.G;
  if (split == 0) return cudaSuccess;
  e2 = launch_fold_split_units(p, (uint64_t)split, s);
  count_launch(1);
  return e2;
}

}  // namespace fd

namespace fd {
namespace {

__global__ void exp2_selfcheck_kernel(const float* x, float* y, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    float a, b;
    sm100::f2_unpack(sm100::exp2_poly2(sm100::f2_pack(v, v)), a, b);
    y[3 * i] = a;
    y[3 * i + 1] = sm100::ex2_approx(v);
    y[3 * i + 2] = exp2f(v);
  }
}

}  // namespace

namespace {
// One thread waits on an mbarrier that nothing ever arrives at, through the
// same bounded wait the attention kernel uses, with a short limit: the wait
// gives up, records (timeout, site 5) in the error word and the kernel
// returns normally, so the context stays usable.
__global__ void bounded_wait_selftest_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    bounded_wait<false>(&bar, 0, &abort, err, kSiteSelftest, limit_ns);
}
}  // namespace

cudaError_t launch_bounded_wait_selftest(int32_t* err, uint64_t limit_ns,
                                         cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  count_launch(1);
  return cudaGetLastError();
}

cudaError_t launch_exp2_selfcheck(const float* x, float* y, int64_t n,
                                  cudaStream_t s) {
  const int64_t blocks = (n + 255) / 256;
  exp2_selfcheck_kernel<<<(unsigned)(blocks < 1184 ? (blocks > 0 ? blocks : 1) : 1184),
                          256, 0, s>>>(x, y, n);
  count_launch(1);
  return cudaGetLastError();
}

}  // namespace fd
