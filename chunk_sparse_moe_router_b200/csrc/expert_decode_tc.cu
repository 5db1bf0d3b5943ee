// Sparse expert kernel of the BlockFFN chunk layer for decode chunks (L <= 32) on the 5th-generation
// tensor cores: one launch per chunk, router included.  It takes chunks of 9 to 32 tokens, where the
// mma.sync kernel of expert_decode.cu is bound by its warp MMAs (this one streams the weights 1.2 to
// 4.8 times faster), and chunks of any length when one expert's W1 and W2 hold 4 MiB or more
// (decode_on_tc); the mma.sync kernel keeps small chunks of smaller experts, where its lower fixed
// cost wins.
//
// Router and prologue (decode_router.cuh): s = x Wr + b split over the CTAs, a grid barrier, then in
// every CTA the ReLU / RMSNorm statistics, the masks and the chunk's union of active experts
// (lsdiaocha.cn BlockFFN article, sections 2 and 4).
//
// Body: the union is evaluated for all L tokens as one batch (article, section 7); each (token, expert)
// term is weighted by the router output r, zero for the pairs the mask removes.  Only the W1/W2 rows of
// experts in the union are read, each once:
//  * one warp issues TMA tensor-box copies of weight rows (boxes of 8..128 rows x 64 columns, summed to
//    a block's height) and x tiles into a ring of shared-memory stages guarded by mbarriers; one warp
//    copies the h tiles of the down-projection;
//  * one thread issues tcgen05.mma (bf16 in, fp32 accumulators in tensor memory) with the weight rows as
//    the M = 128 operand and the tokens as the N operand, and hands each stage back with
//    tcgen05.commit; four warps drain the accumulators (tcgen05.ld) and run the epilogues;
//  * stream-K work split: each projection is a grid of cells (block of at most 128 rows) x (64-wide
//    step of the contraction); CTA g owns a contiguous, balanced range of cells, so every CTA issues
//    the same number of MMAs to within one cell.  A block split between CTAs is summed from their
//    partial accumulators, in CTA order, by the CTA that finishes its part last, so the result does
//    not depend on timing.
// Up-projection: blocks of (active expert, 128 of its de rows), steps over d; epilogue h = r Swish(u),
//   Swish(u) = u / (1 + e^-u) (article, section 2), stored as bf16 hi + lo parts in the 128-byte-
//   swizzled tiles the down-projection copies.  A grid barrier publishes h.
// Down-projection: blocks of 128 rows of y, steps over (active expert, 64 of its de); y[t, k] =
//   sum_a sum_j W2[e_a, k, j] (h_hi + h_lo)[a, t, j], written once per element in a fixed order: y is
//   bit-reproducible run to run.
#include "blockffn_internal.cuh"
#include "decode_router.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace bffn {
namespace tcdec {
namespace {

constexpr int kEpiWarps = 4;
constexpr int kWarpW = 0;     // weight (and x) copies
constexpr int kWarpH = 1;     // h copies of the down-projection
constexpr int kWarpMma = 2;   // tensor-memory owner, MMA issue
constexpr int kWarpEpi = 3;   // first of the kEpiWarps epilogue warps (tensor-memory lane quarters 3, 0, 1, 2)
constexpr int kThreads = (3 + kEpiWarps) * 32;
constexpr int kBlockRows = 128;                 // MMA M
constexpr int kGuardBytes = 128 * 128;          // an M = 128 operand read: 128 rows of 128 bytes
constexpr int kMaxSpan = 16;                    // experts a CTA's up-projection rows touch (<= E / G + 2)
constexpr uint64_t kWaitNs = 2000000000ull;

struct Smem {
  uint8_t* ring;              // S slots
  volatile int* abort_flag;
  uint64_t* fullW;            // [S] weight (and x) tiles landed
  uint64_t* fullH;            // [S] h tiles landed (down-projection stages)
  uint64_t* empty;            // [S] the stage's MMAs completed
  uint64_t* accA_full;        // [2] up-projection accumulator complete
  uint64_t* accA_free;        // [2] its epilogue has read it
  uint64_t* accB_full;        // [2] down-projection accumulator complete
  uint64_t* accB_free;        // [2] its epilogue has read it
  volatile int* red_flag;     // this CTA arrived last at a split block
  uint64_t* drain;            // every MMA issued has completed
  uint32_t* tmem_base;
  int32_t* act;               // [E] active experts, ascending
  int* n_act;                 // [1]
  float* rms;                 // [32] per-token sqrt(mean relu(s)^2)
  uint32_t* maskw;            // [32][32] per-token active bits
  float* pre_s;               // [kMaxSpan][32] s of the experts of this CTA's up-projection rows
  float* pre_g;               // [kMaxSpan]
};

// The CTA's abort flag, read and written with explicit shared-memory instructions.
__device__ __forceinline__ bool aborted(const Smem& sm) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void*)sm.abort_flag)) : "memory");
  return v != 0;
}
__device__ __forceinline__ void set_abort(const Smem& sm) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_u32((const void*)sm.abort_flag)), "r"(1u) : "memory");
}

__device__ __forceinline__ void set_error(const Params& p, const Smem& sm, uint32_t bit, uint32_t info) {
  atomicOr(&p.hdr->err, bit);
  p.hdr->err_info = info;
  set_abort(sm);
}

// A bounded wait that records a timeout and marks the CTA aborted; once aborted, waits fail at once.
__device__ __noinline__ bool wait_slow(const Params& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                       uint32_t where) {
  if (aborted(sm)) return false;
  if (mbar_wait_bounded(bar, parity, kWaitNs)) return true;
  set_error(p, sm, kErrRingWait, where);
  return false;
}
__device__ __forceinline__ bool wait(const Params& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                     uint32_t where) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(p, sm, bar, parity, where);
}

// ------------------------------------------------------------------------------------- work split
// Stream-K: each phase is a grid of cells, (block of at most 128 rows) x (64-wide step of the
// contraction), in block-major order.  CTA g owns the contiguous cells [C g / G, C (g + 1) / G) (floor),
// so every CTA issues the same number of MMAs to within one cell.  Its range cut at block boundaries
// gives its segments: a middle segment covers a whole block; the first and the last may cover part of
// one.  A block split between CTAs is summed from their partial accumulators, in CTA order, by the
// CTA that finishes its part last.
//   Up-projection:   blocks (active expert position a, rows [bi HA, + HA) of its de), steps = 64-column
//                    chunks of d.
//   Down-projection: blocks of y rows [rb HB, + HB), steps = (active expert position a, 64-wide chunk
//                    of its de) in expert-major order.
struct Range {
  int x0, x1;  // this CTA's cells
  int nK;      // cells per block
};
// Cell counts C stay below 2^20 (E <= 1024 experts x 2 blocks x 256 chunks; 128 row blocks x 1024 x 4
// steps) and grids below 2^9, so C * g fits 32 bits.
__device__ __forceinline__ int cell_start(int C, int g) { return int(uint32_t(C) * uint32_t(g) / gridDim.x); }
__device__ __forceinline__ Range cta_range(int C, int nK) {
  Range r;
  r.x0 = cell_start(C, blockIdx.x);
  r.x1 = cell_start(C, blockIdx.x + 1);
  r.nK = nK;
  return r;
}
__device__ __forceinline__ bool range_nonempty(int C, int g) { return cell_start(C, g + 1) > cell_start(C, g); }
// the CTA whose range holds cell x
__device__ __forceinline__ int cell_owner(int C, int x) {
  return int((uint32_t(x + 1) * gridDim.x + uint32_t(C) - 1u) / uint32_t(C)) - 1;
}

struct Seg {
  int blk, k0, k1;  // block, steps [k0, k1) of its contraction
  int idx;          // index of the segment in the CTA's range
  bool last;        // last segment of the CTA's range
};
struct SegIter {
  Range r;
  int x;
  int idx = 0;
  __device__ __forceinline__ explicit SegIter(const Range& rr) : r(rr), x(rr.x0) {}
  __device__ __forceinline__ bool next(Seg& s) {
    if (x >= r.x1) return false;
    s.blk = x / r.nK;
    s.k0 = x - s.blk * r.nK;
    s.k1 = min(r.nK, s.k0 + (r.x1 - x));
    s.idx = idx++;
    x += s.k1 - s.k0;
    s.last = x >= r.x1;
    return true;
  }
};
// Partial-accumulator slot of a split segment: 0 for the CTA's first segment, 1 for its last one
// (when it has two or more).  The CTAs sharing block blk are those of g0..g1 whose ranges are not
// empty (with fewer cells than CTAs some are); g0 uses slot 1 when its range starts in an earlier block.
__device__ __forceinline__ int seg_slot(const Seg& s) { return (s.idx > 0 && s.last) ? 1 : 0; }
__device__ __forceinline__ int owner_slot(int C, int nK, int blk, int g, int g0) {
  return (g == g0 && cell_start(C, g0) < blk * nK) ? 1 : 0;
}

struct Work {
  int CA, CB;        // cells of the up- and down-projection
  int nKA, nKB;      // cells per block
  int n_act;
  int rZ0, rZ1;      // y rows this CTA zeroes when no expert is active (multiples of 8)
};
__device__ __forceinline__ Work make_work(const Params& p, int n_act) {
  Work w;
  w.n_act = n_act;
  w.nKA = p.nck;
  w.nKB = n_act * p.nJc;
  w.CA = n_act * p.nbpe * w.nKA;
  w.CB = p.nrb * w.nKB;
  const long long ub = p.d / 8;
  w.rZ0 = int(ub * blockIdx.x / gridDim.x) * 8;
  w.rZ1 = int(ub * (blockIdx.x + 1) / gridDim.x) * 8;
  return w;
}

// Ring position: stage i of the CTA's stage sequence sits in slot i mod S; ph = (i / S) & 1.
struct RingPos {
  int i = 0, slot = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int S) {
    ++i;
    if (++slot == S) slot = 0, ph ^= 1u;
  }
};

// Geometry of an up-projection block: expert position a, rows [j0, j0 + rows) of its de, ks chunks per
// stage (W1 tiles [ks][rows][128 B], then x tiles [ks][LB][128 B]).
struct GeoA {
  int a, j0, rows, ks;
};
__device__ __forceinline__ GeoA geo_a(const Params& p, int blk) {
  GeoA g;
  g.a = blk / p.nbpe;
  g.j0 = (blk - g.a * p.nbpe) * p.HA;
  g.rows = min(p.HA, p.de - g.j0);
  g.ks = p.slot_bytes / ((g.rows + p.LB) * 128);
  return g;
}
// Geometry of a down-projection block: y rows [k0, k0 + rows), kq steps per stage (W2 tiles
// [kq][rows][128 B], then h tiles [kq][HT]).
struct GeoB {
  int k0, rows, kq;
};
__device__ __forceinline__ GeoB geo_b(const Params& p, int blk) {
  GeoB g;
  g.k0 = blk * p.HB;
  g.rows = min(p.HB, p.d - g.k0);
  g.kq = p.slot_bytes / (g.rows * 128 + p.HT);
  return g;
}

// Active-expert positions [first_expert, first_expert + span) that this CTA's up-projection cells touch
// (span 0 without cells).
__device__ __forceinline__ int first_expert(const Params& p, const Work& w) {
  const Range r = cta_range(w.CA, w.nKA);
  return r.x0 < r.x1 ? (r.x0 / w.nKA) / p.nbpe : 0;
}
__device__ __forceinline__ int expert_span(const Params& p, const Work& w) {
  const Range r = cta_range(w.CA, w.nKA);
  return r.x0 < r.x1 ? ((r.x1 - 1) / w.nKA) / p.nbpe - (r.x0 / w.nKA) / p.nbpe + 1 : 0;
}

__device__ __forceinline__ int stages_a(const Params& p, const Work& w) {
  int n = 0;
  SegIter it(cta_range(w.CA, w.nKA));
  Seg s;
  while (it.next(s)) {
    const int ks = geo_a(p, s.blk).ks;
    n += (s.k1 - s.k0 + ks - 1) / ks;
  }
  return n;
}

// ------------------------------------------------------------------------------ router and prologue
// (decode_router.cuh, instantiated for this kernel's kThreads)
using decode_router::RouterStage;
using decode_router::cp_async4;

// ------------------------------------------------------------------------------------- copies
// `rows` (a multiple of 8, <= 128) rows starting at row `r0` of the 3-D weight tensor (x = column,
// y = row, z = expert), 64 columns from column `col`, as boxes of 128, 64, 32, 16 and 8 rows into
// consecutive 128-byte rows at `dst`.
__device__ __forceinline__ void load_rows(uint8_t* dst, const CUtensorMap* maps, int col, int r0, int e, int rows,
                                          uint64_t* bar, uint64_t pol) {
  int ro = 0;
#pragma unroll
  for (int k = 4; k >= 0; --k) {
    const int hh = 8 << k;
    if (rows - ro >= hh) {
      tma_load_3d(dst + ro * 128, &maps[k], col, r0 + ro, e, bar, pol);
      ro += hh;
    }
  }
}

// Weight copy warp (lane 0): W1 rows with the matching x columns, then W2 rows, in stage order.
// Returns the number of stages issued.
__device__ int produce_w(const Params& p, const Maps& tm, const Smem& sm, const Work& w) {
  // weights stream through once (evict first), unless the caller expects the next call to reuse them
  const uint64_t pol_w = p.keep_l2 ? policy_evict_last() : policy_evict_first(), pol_x = policy_evict_last();
  RingPos rp;
  Seg sg;
  for (SegIter it(cta_range(w.CA, w.nKA)); it.next(sg);) {
    const GeoA g = geo_a(p, sg.blk);
    const int e = sm.act[g.a];
    for (int c0 = sg.k0; c0 < sg.k1; c0 += g.ks, rp.next(p.S)) {
      if (rp.i >= p.S && !wait(p, sm, &sm.empty[rp.slot], rp.ph ^ 1u, 1)) return rp.i;
      const int nc = min(g.ks, sg.k1 - c0);
      uint8_t* st = sm.ring + size_t(rp.slot) * p.slot_bytes;
      uint8_t* xt = st + g.ks * g.rows * 128;
      mbar_arrive_expect_tx(&sm.fullW[rp.slot], uint32_t(nc * (g.rows + p.LB) * 128));
      for (int c = 0; c < nc; ++c) {
        load_rows(st + c * g.rows * 128, tm.w1, (c0 + c) * 64, g.j0, e, g.rows, &sm.fullW[rp.slot], pol_w);
        tma_load_2d(xt + c * p.LB * 128, &tm.x, (c0 + c) * 64, 0, &sm.fullW[rp.slot], pol_x);
      }
    }
  }
  for (SegIter it(cta_range(w.CB, w.nKB)); it.next(sg);) {
    const GeoB g = geo_b(p, sg.blk);
    for (int k = sg.k0; k < sg.k1; k += g.kq, rp.next(p.S)) {
      if (rp.i >= p.S && !wait(p, sm, &sm.empty[rp.slot], rp.ph ^ 1u, 2)) return rp.i;
      const int nq = min(g.kq, sg.k1 - k);
      uint8_t* st = sm.ring + size_t(rp.slot) * p.slot_bytes;
      mbar_arrive_expect_tx(&sm.fullW[rp.slot], uint32_t(nq * g.rows * 128));
      for (int q = 0; q < nq; ++q) {
        const int a = (k + q) / p.nJc, c = (k + q) - a * p.nJc;
        load_rows(st + q * g.rows * 128, tm.w2, c * 64, g.k0, sm.act[a], g.rows, &sm.fullW[rp.slot], pol_w);
      }
    }
  }
  return rp.i;
}

// h copy warp (lane 0): after every CTA's up-projection is published, the down-projection stages' h
// tiles (one bulk copy of 2 LC rows x 128 bytes per step).  Returns the per-slot parity of the next h
// phase; `used` gets the slots it filled.
__device__ uint32_t produce_h(const Params& p, const Smem& sm, const Work& w, uint32_t* used) {
  RingPos rp;
  const int nA = stages_a(p, w);
  for (int k = 0; k < nA; ++k) rp.next(p.S);
  uint32_t hph = 0;  // per slot: parity of its next h-tile phase
  *used = 0;
  const Range rB = cta_range(w.CB, w.nKB);
  if (rB.x0 >= rB.x1) return hph;
  {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(&p.hdr->grid_bar) < gridDim.x) {
      if (aborted(sm)) return hph;
      if (globaltimer_ns() - t0 > kWaitNs) {
        set_error(p, sm, kErrGridBarrier, uint32_t(blockIdx.x));
        return hph;
      }
      __nanosleep(64);
    }
    fence_proxy_async_global();  // h was written with generic stores; the bulk copies read it
  }
  const uint64_t pol_h = policy_evict_last();
  const uint32_t tile = uint32_t(p.HT);  // 2 LC rows of 128 bytes, the same in the image and in the stage
  Seg sg;
  for (SegIter it(rB); it.next(sg);) {
    const GeoB g = geo_b(p, sg.blk);
    for (int k = sg.k0; k < sg.k1; k += g.kq, rp.next(p.S)) {
      // the slot is free once its previous stage's MMAs completed (the weight warp waits for the same)
      if (rp.i >= p.S && !wait(p, sm, &sm.empty[rp.slot], rp.ph ^ 1u, 3)) return hph;
      const int nq = min(g.kq, sg.k1 - k);
      uint8_t* ht = sm.ring + size_t(rp.slot) * p.slot_bytes + g.kq * g.rows * 128;
      mbar_arrive_expect_tx(&sm.fullH[rp.slot], uint32_t(nq) * tile);
      for (int q = 0; q < nq; ++q) {
        const int a = (k + q) / p.nJc, c = (k + q) - a * p.nJc;
        bulk_g2s(ht + q * p.HT, p.h + size_t(a) * p.h_expert_bytes + size_t(c) * tile, tile, &sm.fullH[rp.slot],
                 pol_h);
      }
      hph ^= 1u << rp.slot;
      *used |= 1u << rp.slot;
    }
  }
  return hph;
}

// Before the CTA exits: wait (briefly, bounded) for the copies of the last issued stages, so that no
// copy into this CTA's shared memory is in flight when it leaves (only ever pending after an abort).
// Weight stages: the last `S` of `issued`; h stages: the last phase of every slot used.
__device__ void drain_w(uint64_t* full, int issued, int S) {
  for (int i = max(0, issued - S); i < issued; ++i) mbar_wait_bounded(&full[i % S], uint32_t(i / S) & 1u, kWaitNs / 10);
}
__device__ void drain_h(uint64_t* full, uint32_t hph, uint32_t used, int S) {
  for (int s = 0; s < S; ++s)
    if ((used >> s) & 1u) mbar_wait_bounded(&full[s], ((hph >> s) & 1u) ^ 1u, kWaitNs / 10);
}

// ------------------------------------------------------------------------------------- MMA issue
// One thread.  Up-projection segment i accumulates in tensor-memory columns [(i & 1) NA, + NA),
// down-projection segment i in [2 NA + (i & 1) NB, + NB).  Each stage is handed back to the copy warps
// by a commit to its empty barrier; each accumulator to the epilogue by a commit to its full barrier.
// A descriptor's address field counts 16-byte units, so one K step of 16 (32 bytes) adds 2 and one
// tile of n rows of 128 bytes adds 8 n; shared-memory addresses stay below 2^18, so these adds never
// carry out of the field.
__device__ void mma_issue(const Params& p, const Smem& sm, const Work& w, uint32_t tmem) {
  const uint32_t idA = tc::idesc_bf16_f32(kBlockRows, p.NA), idB = tc::idesc_bf16_f32(kBlockRows, p.NB);
  const uint32_t ring = smem_u32(sm.ring);
  const int S = p.S, slot_bytes = p.slot_bytes, LB = p.LB, HT = p.HT;
  RingPos rp;
  Seg sg;
  for (SegIter it(cta_range(w.CA, w.nKA)); it.next(sg);) {
    const GeoA g = geo_a(p, sg.blk);
    const int buf = sg.idx & 1;
    if (sg.idx >= 2 && !wait(p, sm, &sm.accA_free[buf], uint32_t((sg.idx >> 1) - 1) & 1u, 4)) return;
    tc::fence_after_sync();
    const uint32_t d = tmem + uint32_t(buf * p.NA);
    const uint64_t wstep = uint64_t(g.rows) * 8, xstep = uint64_t(LB) * 8;
    uint32_t acc = 0;
    for (int c0 = sg.k0; c0 < sg.k1; c0 += g.ks, rp.next(S)) {
      if (!wait(p, sm, &sm.fullW[rp.slot], rp.ph, 5)) return;
      tc::fence_after_sync();
      const int nc = min(g.ks, sg.k1 - c0);
      const uint32_t st = ring + uint32_t(rp.slot * slot_bytes);
      uint64_t da = tc::smem_desc_k128(st);
      uint64_t db = tc::smem_desc_k128(st + uint32_t(g.ks * g.rows * 128));
      for (int c = 0; c < nc; ++c, da += wstep, db += xstep) {
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          tc::mma_bf16(d, da + 2 * k16, db + 2 * k16, idA, acc);
          acc = 1;
        }
      }
      tc::commit(&sm.empty[rp.slot]);
    }
    tc::commit(&sm.accA_full[buf]);
  }
  uint32_t hph = 0;  // per slot: parity of its next h-tile phase (fullH completes on down-projection stages only)
  for (SegIter it(cta_range(w.CB, w.nKB)); it.next(sg);) {
    const GeoB g = geo_b(p, sg.blk);
    const int buf = sg.idx & 1;
    if (sg.idx >= 2 && !wait(p, sm, &sm.accB_free[buf], uint32_t((sg.idx >> 1) - 1) & 1u, 6)) return;
    tc::fence_after_sync();
    const uint32_t d = tmem + uint32_t(2 * p.NA + buf * p.NB);
    const uint64_t wstep = uint64_t(g.rows) * 8, hstep = uint64_t(HT) >> 4;
    uint32_t acc = 0;
    for (int k = sg.k0; k < sg.k1; k += g.kq, rp.next(S)) {
      if (!wait(p, sm, &sm.fullW[rp.slot], rp.ph, 7)) return;
      if (!wait(p, sm, &sm.fullH[rp.slot], (hph >> rp.slot) & 1u, 8)) return;
      hph ^= 1u << rp.slot;
      tc::fence_after_sync();
      const int nq = min(g.kq, sg.k1 - k);
      const uint32_t st = ring + uint32_t(rp.slot * slot_bytes);
      uint64_t da = tc::smem_desc_k128(st);
      uint64_t db = tc::smem_desc_k128(st + uint32_t(g.kq * g.rows * 128));
      for (int q = 0; q < nq; ++q, da += wstep, db += hstep) {
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          tc::mma_bf16(d, da + 2 * k16, db + 2 * k16, idB, acc);
          acc = 1;
        }
      }
      tc::commit(&sm.empty[rp.slot]);
    }
    tc::commit(&sm.accB_full[buf]);
  }
}

// ------------------------------------------------------------------------------------- epilogues
// N (16, 32 or 64) accumulator columns of this thread's tensor-memory lane.
template <int N>
__device__ __forceinline__ void tmem_cols(uint32_t taddr, float (&v)[64]) {
  if constexpr (N == 16) {
    tc::ld_32x32b_x16(taddr, v);
  } else {
    tc::ld_32x32b_x32(taddr, *reinterpret_cast<float(*)[32]>(v));
    if constexpr (N == 64) tc::ld_32x32b_x32(taddr + 32, *reinterpret_cast<float(*)[32]>(v + 32));
  }
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// A segment that covers part of its block (all kEpiWarps warps call it together): row m of this CTA's
// partial accumulator (LC values, `row_ok` rows only) goes to its workspace slot, the block's counter
// counts the arrival, and the CTA that arrives last sums every partial of the block in CTA order into
// `acc` (its own from registers) and returns true.  (Every call zeroes the counters before its router
// barrier.)
template <int LC>
__device__ bool split_reduce(const Params& p, const Smem& sm, int C, int nK, const Seg& sg,
                             uint32_t* cnt, int m, bool row_ok, float (&acc)[LC]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (row_ok) {
    float4* dst = reinterpret_cast<float4*>(p.part + ((size_t(blockIdx.x) * 2 + seg_slot(sg)) * 128 + m) * LC);
#pragma unroll
    for (int i = 0; i < LC / 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
  }
  __threadfence();
  named_bar_sync(1, kEpiWarps * 32);
  const int g0 = cell_owner(C, sg.blk * nK), g1 = cell_owner(C, (sg.blk + 1) * nK - 1);
  if (warp == kWarpEpi && lane == 0) {
    uint32_t nparts = 0;
    for (int g = g0; g <= g1; ++g) nparts += range_nonempty(C, g) ? 1u : 0u;
    *sm.red_flag = atom_add_acq_rel_gpu(&cnt[sg.blk], 1u) == nparts - 1u ? 1 : 0;
  }
  named_bar_sync(1, kEpiWarps * 32);
  if (*sm.red_flag == 0) return false;
  if (row_ok) {
    float own[LC];
#pragma unroll
    for (int t = 0; t < LC; ++t) own[t] = acc[t], acc[t] = 0.f;
    // the other parts' rows, loaded PB parts at a time, added in CTA order
    constexpr int PB = LC <= 8 ? 4 : 1;
    for (int gb = g0; gb <= g1; gb += PB) {
      float4 f[PB][LC / 4];
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int g = gb + u;
        if (g <= g1 && g != int(blockIdx.x) && range_nonempty(C, g)) {
          const float4* src = reinterpret_cast<const float4*>(
              p.part + ((size_t(g) * 2 + owner_slot(C, nK, sg.blk, g, g0)) * 128 + m) * LC);
#pragma unroll
          for (int i = 0; i < LC / 4; ++i) f[u][i] = __ldcg(src + i);
        }
      }
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int g = gb + u;
        if (g > g1) break;
        if (g == int(blockIdx.x)) {
#pragma unroll
          for (int t = 0; t < LC; ++t) acc[t] += own[t];
        } else if (range_nonempty(C, g)) {
#pragma unroll
          for (int i = 0; i < LC / 4; ++i)
            acc[4 * i] += f[u][i].x, acc[4 * i + 1] += f[u][i].y, acc[4 * i + 2] += f[u][i].z, acc[4 * i + 3] += f[u][i].w;
        }
      }
    }
  }
  return true;
}

// Four warps; warp q (= warp index mod 4) reads tensor-memory lanes [32 q, 32 q + 32), i.e. rows
// 32 q + lane of a block.  LC = L rounded up to 8, 16 or 32: the up-projection accumulator has
// NA = max(16, LC) columns (token t in column t), the down-projection's 2 LC (hi part of token t in
// column t, lo part in column LC + t), matching h tiles of 2 LC rows.
template <int LC>
__device__ void epilogue(const Params& p, const Smem& sm, const Work& w, uint32_t tmem) {
  constexpr int NA = LC < 16 ? 16 : LC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = warp & 3;
  const int m = 32 * q + lane;
  const uint32_t lane_off = uint32_t(32 * q) << 16;
  float v[64];
  float acc[LC];
  bool ok = true;
  const int a_first = first_expert(p, w);
  Seg sg;
  for (SegIter it(cta_range(w.CA, w.nKA)); it.next(sg);) {
    const GeoA g = geo_a(p, sg.blk);
    const int buf = sg.idx & 1;
    ok = wait(p, sm, &sm.accA_full[buf], uint32_t(sg.idx >> 1) & 1u, 9);
    if (!ok) break;
    tc::fence_after_sync();
    const bool have = 32 * q < g.rows;
    if (have) tmem_cols<NA>(tmem + lane_off + uint32_t(buf * NA), v);
#pragma unroll
    for (int t = 0; t < LC; ++t) acc[t] = v[t];
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.accA_free[buf]);
    const bool row_ok = have && m < g.rows;
    bool done = true;
    if (sg.k0 != 0 || sg.k1 != w.nKA) done = split_reduce<LC>(p, sm, w.CA, w.nKA, sg, p.cntA, m, row_ok, acc);
    if (done && row_ok) {
      // h = r Swish(u) with r = g relu(s) / rms, as bf16 hi + lo in the h image of expert position a
      const int j = g.j0 + m, col = j & 63;
      const float gg = sm.pre_g[g.a - a_first];
      const float* ps = sm.pre_s + (g.a - a_first) * 32;
      uint8_t* himg = p.h + size_t(g.a) * p.h_expert_bytes + size_t(j >> 6) * (2 * LC * 128) + (col & 7) * 2;
#pragma unroll
      for (int t = 0; t < LC; ++t) {
        if (t < p.L) {
          const float rms = sm.rms[t];
          const float rr = (rms > 0.f) ? (gg * fmaxf(ps[t], 0.f)) / rms : 0.f;
          const float u = acc[t];
          const float hv = rr * (u / (1.f + expf(-u)));
          const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
          const __nv_bfloat16 lo = __float2bfloat16_rn(hv - __bfloat162float(hi));
          const int R0 = t, R1 = LC + t;
          *reinterpret_cast<__nv_bfloat16*>(himg + R0 * 128 + (((col >> 3) ^ (R0 & 7)) << 4)) = hi;
          *reinterpret_cast<__nv_bfloat16*>(himg + R1 * 128 + (((col >> 3) ^ (R1 & 7)) << 4)) = lo;
        }
      }
      // Columns [de, 64 nJc) of the expert's last h tile face the zero columns the W2 boxes read past
      // de, but the workspace may hold any bytes there (possibly a NaN pattern, and 0 * NaN is NaN):
      // the thread of the expert's last row zeroes them (whole 16-byte pieces: de is a multiple of 8).
      if (j == p.de - 1) {
        uint8_t* tile = himg - (col & 7) * 2;
        for (int t = 0; t < p.L; ++t)
          for (int c8 = (p.de & 63) >> 3; c8 != 0 && c8 < 8; ++c8) {
            const int R0 = t, R1 = LC + t;
            *reinterpret_cast<uint4*>(tile + R0 * 128 + ((c8 ^ (R0 & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(tile + R1 * 128 + ((c8 ^ (R1 & 7)) << 4)) = make_uint4(0, 0, 0, 0);
          }
      }
    }
  }
  // publish this CTA's h before any CTA reads it (every CTA arrives, also after an abort)
  __threadfence();
  named_bar_sync(1, kEpiWarps * 32);
  if (warp == kWarpEpi && lane == 0) {
    fence_proxy_async_global();
    red_release_gpu_add(&p.hdr->grid_bar, 1u);
    pdl_launch_dependents();
  }
  if (!ok || aborted(sm)) return;

  if (w.n_act == 0) {  // no expert is active: y = 0
    const int nb = w.rZ1 - w.rZ0;
    for (int o = threadIdx.x - kWarpEpi * 32; o < p.L * nb; o += kEpiWarps * 32)
      p.y[size_t(o / nb) * p.d + w.rZ0 + o % nb] = 0.f;
    return;
  }
  for (SegIter it(cta_range(w.CB, w.nKB)); it.next(sg);) {
    const GeoB g = geo_b(p, sg.blk);
    const int buf = sg.idx & 1;
    if (!wait(p, sm, &sm.accB_full[buf], uint32_t(sg.idx >> 1) & 1u, 10)) return;
    tc::fence_after_sync();
    const bool have = 32 * q < g.rows;
    if (have) tmem_cols<2 * LC>(tmem + lane_off + uint32_t(2 * NA + buf * 2 * LC), v);
#pragma unroll
    for (int t = 0; t < LC; ++t) acc[t] = v[t] + v[LC + t];
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.accB_free[buf]);
    const bool row_ok = have && m < g.rows;
    bool done = true;
    if (sg.k0 != 0 || sg.k1 != w.nKB) done = split_reduce<LC>(p, sm, w.CB, w.nKB, sg, p.cntB, m, row_ok, acc);
    if (done && row_ok) {
#pragma unroll
      for (int t = 0; t < LC; ++t)
        if (t < p.L) p.y[size_t(t) * p.d + g.k0 + m] = acc[t];
    }
  }
}

// ------------------------------------------------------------------------------------- kernel
template <int LC>
__global__ void __launch_bounds__(kThreads, 1)
    expert_decode_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ Maps tm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem sm;
  sm.ring = base;
  uint8_t* tail = base + p.pre_bytes;
  sm.abort_flag = reinterpret_cast<volatile int*>(tail);
  sm.red_flag = reinterpret_cast<volatile int*>(tail + 8);
  sm.tmem_base = reinterpret_cast<uint32_t*>(tail + 16);
  sm.fullW = reinterpret_cast<uint64_t*>(tail + 32);
  sm.fullH = sm.fullW + p.S;
  sm.empty = sm.fullH + p.S;
  sm.accA_full = sm.empty + p.S;
  sm.accA_free = sm.accA_full + 2;
  sm.accB_full = sm.accA_free + 2;
  sm.accB_free = sm.accB_full + 2;
  sm.drain = sm.accB_free + 2;
  sm.act = reinterpret_cast<int32_t*>(sm.drain + 1);
  sm.n_act = sm.act + ((p.E + 3) & ~3);
  sm.rms = reinterpret_cast<float*>(sm.n_act + 4);
  sm.maskw = reinterpret_cast<uint32_t*>(sm.rms + 32);
  sm.pre_s = reinterpret_cast<float*>(sm.maskw + 32 * 32);
  sm.pre_g = sm.pre_s + kMaxSpan * 32;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&sm.fullW[s], 1);
      mbar_init(&sm.fullH[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.accA_full[b], 1);
      mbar_init(&sm.accA_free[b], kEpiWarps);
      mbar_init(&sm.accB_full[b], 1);
      mbar_init(&sm.accB_free[b], kEpiWarps);
    }
    mbar_init(sm.drain, 1);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpW && lane == 0) {
    for (int k = 0; k < 5; ++k) {
      prefetch_tensormap(&tm.w1[k]);
      prefetch_tensormap(&tm.w2[k]);
    }
    prefetch_tensormap(&tm.x);
  }
  if (warp == kWarpMma) tc::tmem_alloc(sm.tmem_base, uint32_t(p.tmem_cols));
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *sm.tmem_base;

  // ---- router: this CTA's units, then every CTA's partials
  const RouterStage rs = decode_router::router_stage<kThreads>(p, base);
  {
    const int U = p.rq * p.rcb;
    for (int e = tid; e < p.E; e += kThreads) {
      cp_async4(rs.g + e, p.g + e);
      if (p.br) cp_async4(rs.b + e, p.br + e);
    }
    if (int(blockIdx.x) < U) decode_router::router_copy_w<kThreads>(p, rs.W, blockIdx.x);
    asm volatile("cp.async.commit_group;" ::: "memory");
    // x may come from the previous kernel in the stream, and the workspace is shared with it
    pdl_wait();
    for (int u = blockIdx.x; u < U; u += gridDim.x) {
      if (u != int(blockIdx.x)) {
        decode_router::router_copy_w<kThreads>(p, rs.W, u);
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      decode_router::router_load_x<kThreads>(p, rs.X, u);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
      decode_router::router_unit<kThreads>(p, rs, u);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // split-block counters start at 0: the workspace may have held other data (another shape's h or
    // partials); no CTA counts an arrival before this barrier
    {
      const int ncnt = p.E * p.nbpe + p.nrb;
      for (int o = int(blockIdx.x) * kThreads + tid; o < ncnt; o += int(gridDim.x) * kThreads) p.cntA[o] = 0u;
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      red_release_gpu_add(&p.hdr->router_bar, 1u);
      const uint64_t t0 = globaltimer_ns();
      const uint32_t need = gridDim.x + (p.inject_timeout ? 1u : 0u);
      const uint64_t limit = p.inject_timeout ? kInjectedWaitNs : kWaitNs;
      while (ld_acquire_gpu(&p.hdr->router_bar) < need) {
        if (globaltimer_ns() - t0 > limit) {
          set_error(p, sm, kErrRouterBarrier, uint32_t(blockIdx.x));
          break;
        }
        __nanosleep(32);
      }
    }
    __syncthreads();
  }
  int issuedW = 0;
  uint32_t hph = 0, hused = 0;
  if (!aborted(sm)) {
    float* sbuf = rs.W;  // [L][E], over the router's staging
    decode_router::prologue_router_stats<kThreads>(p, sm, rs, sbuf);
    __syncthreads();
    const Work w = make_work(p, *sm.n_act);
    {  // s and g of every expert this CTA's up-projection cells touch
      const int a_first = first_expert(p, w), span = expert_span(p, w);
      for (int o = tid; o < span * p.L; o += kThreads) {
        const int aa = o / p.L, t = o - aa * p.L;
        sm.pre_s[aa * 32 + t] = sbuf[size_t(t) * p.E + sm.act[a_first + aa]];
      }
      for (int aa = tid; aa < span; aa += kThreads) sm.pre_g[aa] = rs.g[sm.act[a_first + aa]];
    }
    fence_proxy_async_smem();  // the ring held generic data before bulk copies write into it
    __syncthreads();

    if (warp == kWarpW) {
      if (lane == 0) issuedW = produce_w(p, tm, sm, w);
    } else if (warp == kWarpH) {
      if (lane == 0) hph = produce_h(p, sm, w, &hused);
    } else if (warp == kWarpMma) {
      if (lane == 0) {
        mma_issue(p, sm, w, tmem);
        tc::commit(sm.drain);  // completes once every MMA issued above has
        mbar_wait_bounded(sm.drain, 0, kWaitNs);
      }
    } else {
      epilogue<LC>(p, sm, w, tmem);
    }
  }
  __syncthreads();
  if (aborted(sm)) {  // no copy into this CTA's shared memory may be in flight when it leaves
    if (warp == kWarpW && lane == 0) drain_w(sm.fullW, issuedW, p.S);
    if (warp == kWarpH && lane == 0) drain_h(sm.fullH, hph, hused, p.S);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kWarpMma) tc::tmem_dealloc(tmem, uint32_t(p.tmem_cols));
  // the last CTA out sets the grid's counters back for the next call on this workspace
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.hdr->exit_ctr, 1u) == gridDim.x - 1) {
      p.hdr->router_bar = 0u;
      p.hdr->grid_bar = 0u;
      p.hdr->exit_ctr = 0u;
    }
  }
}

template <int LC>
cudaError_t launch_lc(const Params& p, const Maps& tm, const Launch& plan, cudaStream_t st,
                      bool pdl) {
  auto kfn = expert_decode_tc_kernel<LC>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kfn, p, tm);
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

}  // namespace


bool plan(int L, int d, int E, int de, int grid, int max_smem, Params* p, Launch* out) {
  if (L < 1 || L > kDecodeMaxL || d % 8 != 0 || de % 8 != 0 || E < 1 || E > kMaxE) return false;
  const int G = grid;
  if (G < 1) return false;
  if ((E + G - 1) / G + 2 > kMaxSpan) return false;  // experts one CTA's up-projection rows touch
  const int lc = lc_of(L);
  p->nck = (d + 63) / 64;
  p->nJc = (de + 63) / 64;
  p->LB = round_up(L, 8);
  p->NA = lc;
  p->NB = 2 * lc;
  p->HT = 2 * lc * 128;
  p->h_expert_bytes = p->nJc * p->HT;
  // a stage: two steps of a full 128-row block (W1 and x tiles, or W2 and h tiles)
  {
    const int sa = 2 * (kBlockRows + p->LB) * 128, sb = 2 * (kBlockRows * 128 + p->HT);
    p->slot_bytes = round_up(sa > sb ? sa : sb, 1024);
  }
  const int cols = 2 * p->NA + 2 * p->NB;
  p->tmem_cols = cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : 256;
  if (G > kTcMaxGrid) return false;  // two partial-accumulator slots per CTA in the workspace
  p->nbpe = (de + kBlockRows - 1) / kBlockRows;
  p->HA = round_up((de + p->nbpe - 1) / p->nbpe, 8);
  p->nrb = (d + kBlockRows - 1) / kBlockRows;
  p->HB = round_up((d + p->nrb - 1) / p->nrb, 8);
  {
    // stream-K cell arithmetic in 32 bits: cells x grid < 2^32
    const unsigned long long ca = 1ull * E * p->nbpe * p->nck, cb = 1ull * p->nrb * E * p->nJc;
    if ((ca > cb ? ca : cb) * kTcMaxGrid >= (1ull << 32)) return false;
  }
  // router units, and the staging they and the chunk's s need at the ring's start
  p->rrows = decode_router_rows(d);
  p->rq = decode_router_parts(d);
  p->rcb = (E + 31) / 32;
  const size_t gb = size_t(2) * ((E + 3) & ~3) * 4;  // g and b
  const size_t router_need = size_t(p->rrows) * 128 + size_t(L) * p->rrows * 4 + size_t(kThreads / 32) * 8 * 32 * 4;
  const size_t s_need = size_t(L) * E * 4;
  const size_t pre_need = gb + (router_need > s_need ? router_need : s_need);
  // barriers, tmem address and the per-CTA tables after the ring
  const size_t tail = 32 + size_t(3 * 32 + 9) * 8 + size_t(((E + 3) & ~3) + 4) * 4 + 32 * 4 + 32 * 32 * 4 +
                      size_t(kMaxSpan) * 33 * 4 + 64;
  for (int S = 32; S >= 2; --S) {
    size_t pre = size_t(S) * p->slot_bytes;
    if (pre < pre_need) pre = size_t(round_up(int(pre_need), 1024));
    // an M = 128 operand read starting in the last slot may reach kGuardBytes past the ring's end
    const size_t reach = size_t(S) * p->slot_bytes + kGuardBytes;
    const size_t tail_alloc = pre + tail >= reach ? tail : reach - pre;
    const size_t smem = 1024 + pre + tail_alloc;
    if (smem + 256 <= size_t(max_smem)) {  // + the kernel's static shared variables
      p->S = S;
      p->pre_bytes = int(pre);
      p->tail_bytes = int(tail_alloc);
      out->grid = G;
      out->smem = smem;
      return true;
    }
  }
  return false;
}

template <int LC>
cudaError_t occupancy_lc(size_t smem, int* ctas) {
  auto kfn = expert_decode_tc_kernel<LC>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
  if (err != cudaSuccess) return err;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, kfn, kThreads, smem);
}

cudaError_t occupancy(int L, size_t smem, int* ctas_per_sm) {
  if (L <= 16) return occupancy_lc<16>(smem, ctas_per_sm);
  return occupancy_lc<32>(smem, ctas_per_sm);
}

cudaError_t launch(const Params& p, const Maps& tm, const Launch& plan, cudaStream_t st, bool pdl) {
  if (p.L <= 16) return launch_lc<16>(p, tm, plan, st, pdl);
  return launch_lc<32>(p, tm, plan, st, pdl);
}

}  // namespace tcdec
}  // namespace bffn
