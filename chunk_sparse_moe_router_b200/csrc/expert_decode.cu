// Sparse expert kernel of the BlockFFN chunk layer for chunks of up to 8 tokens of experts under 4 MiB
// (decode_on_tc false): one launch per chunk, router included.  (Other decode shapes take the tcgen05
// kernel of expert_decode_tc.cu.)
//
// Router (lsdiaocha.cn BlockFFN article, section 2: the router's linear map s = x Wr + b, before its
// ReLU and RMSNorm): d is cut into parts of at most 256 rows and E into blocks of 32 experts; each
// (part, block) unit runs on one CTA, which stages its Wr rows (copied before the dependent-launch
// wait: weights never depend on the previous kernel in the stream) and its x columns in shared
// memory and writes a partial projection.  After a grid-wide barrier (bounded wait) every CTA adds
// the parts in part order.  The split depends on d only, so s is the same bits for every grid size.
//
// Prologue (every CTA): ReLU and RMSNorm statistics per token (one warp per token, shuffle
// reduction), the per-token active masks with __ballot_sync, and the chunk's union of active experts
// as an ascending list built with __popc and a warp scan (article, sections 2 and 4).  CTA 0 also
// writes the active list, n_active, the sparsity counts and the optional masks / router outputs.
//
// Body: the union is evaluated for all L tokens as one batch, outer loop over active experts and
// inner batched product (article, section 7); each (token, expert) term is weighted by the router
// output r, which is zero for the pairs the mask removes.  Only the W1/W2 rows of experts in the
// union are read.  The kernel is HBM-bound (2L flop per bf16 weight), so everything serves the
// memory stream:
//  * one persistent CTA per SM; each phase's rows are split over the CTAs in contiguous ranges
//    balanced to within one row, so every SM streams the same number of bytes;
//  * weights are read in long contiguous runs, as HBM wants them: the up-projection streams whole
//    W1 rows (a CTA's rows of one expert are one contiguous block), the down-projection whole
//    blocks of consecutive W2 rows; copies are TMA bulk copies / tensor boxes of several KB issued
//    from several lanes into a ring of shared-memory stages guarded by mbarriers;
//  * 8 consumer warps run mma.sync m16n8k16 (bf16 in, fp32 accumulate) with tokens as M and weight
//    rows as N, reading operands with conflict-free ldmatrix (padded rows / 128-byte swizzle).
//
// Phase A (up-projection): the CTA owns rows [rA0, rA1) of the flattened (active expert, j) space,
//   taken in groups of RS rows, one group per stage; a consumer warp owns whole groups and computes
//   u = W1[e, j, :] . x_t over all of K (x stays resident in shared memory, in K passes when it is
//   large), then h = r[t, e] * Swish(u), Swish(u) = u / (1 + e^-u) (article, section 2).  h goes to
//   the workspace as a high and a low bf16 part (so the bf16 down-projection keeps about 16 mantissa
//   bits of h), already in the swizzled tile layout the down-projection loads.
// Grid barrier: all h are written before any CTA reads h (bounded wait).  W2 tiles keep streaming
//   in while it is pending; only the h tiles wait for it.
// Phase B (down-projection): the CTA owns output rows [rB0, rB1) of y and sums over every active
//   expert, y[t, k] = sum_a sum_j W2[e_a, k, j] (h_hi + h_lo)[a, t, j], with the hi and lo parts as
//   two stacks of L rows of the MMA's M dimension.  Each y element is written exactly once, in a
//   fixed summation order, so y is bit-reproducible run to run.
#include "blockffn_internal.cuh"
#include "decode_router.cuh"
#include "ptx.cuh"

namespace bffn {
namespace {

constexpr int NCW = 8;                      // consumer warps
constexpr int kThreads = (NCW + 2) * 32;    // + weight producer warp + x / h producer warp
constexpr int GPW = 2;                      // row groups per consumer warp per row-block (x in smem)
constexpr int GB = NCW * GPW;               // row groups per row-block (x in smem)
constexpr int kMaxSpan = 16;                // experts a CTA's up-projection rows touch (<= E / G + 2)
constexpr int kXregChunks = 4;              // 64-column chunks of x one warp keeps in registers
constexpr uint64_t kWaitNs = 2000000000ull;
// 16-row n groups of a down-projection row block: up to 48 rows (with 8 tokens a row block of W2 then
// fills a 32 KB stage with the h tiles), 32 for the longer token classes (accumulator registers)
template <int LC>
constexpr int kNP2 = LC == 8 ? 3 : 2;
constexpr int np2_of(int lc) { return lc == 8 ? 3 : 2; }

// ------------------------------------------------------------------------------------- smem
struct Smem {
  uint8_t* xbuf;       // resident x part [L][PX]
  uint8_t* ring;       // S slots
  float* red;          // [NCW][MT][4][32][4] phase-B cross-warp partials (aliases xbuf when it fits)
  uint8_t* zero;       // 16 zero bytes
  volatile int* abort_flag;
  uint64_t* fullW;     // [S]
  uint64_t* fullH;     // [S]
  uint64_t* empty;     // [S]
  uint64_t* xfull;     // x part landed
  uint64_t* xfree;     // consumers done with the x part
  int32_t* act;        // [E] active experts, ascending
  int* n_act;          // [1]
  float* rms;          // [32] per-token sqrt(mean relu(s)^2)
  uint32_t* maskw;     // [32][32] per-token active bits
  float* pre_s;        // [kMaxSpan][32] s of the experts of this CTA's up-projection rows
  float* pre_g;        // [kMaxSpan]
  float* red_s;        // [S][NCW][32][2] per-stage partial sums (K split)
  uint64_t* rbar;      // [S] partial sums of a stage written (NCW arrivals)
  float* ustage;       // [ustage_units][L][8] up-projection sums u of a block of rows until its epilogue (K split)
};

__device__ __forceinline__ uint32_t swz(int row, int chunk16) {
  return uint32_t(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

// The CTA's abort flag, read and written with explicit shared-memory instructions.
__device__ __forceinline__ bool aborted(const Smem& sm) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void*)sm.abort_flag)) : "memory");
  return v != 0;
}
__device__ __forceinline__ void set_abort(const Smem& sm) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_u32((const void*)sm.abort_flag)), "r"(1u) : "memory");
}

__device__ __forceinline__ void set_error(const DecodeParams& p, const Smem& sm, uint32_t bit, uint32_t info) {
  atomicOr(&p.hdr->err, bit);
  p.hdr->err_info = info;
  set_abort(sm);
}

// A wait that records a timeout and marks the CTA aborted; once aborted, waits are skipped (callers
// skip the work) so that every warp still reaches the same named barriers and the CTA can finish.
// The first try is inline, the rest out of line.
__device__ __noinline__ bool ring_wait_slow(const DecodeParams& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                            uint32_t where) {
  if (aborted(sm)) return false;
  if (mbar_wait_slow(bar, parity, kWaitNs)) return true;
  if ((threadIdx.x & 31) == 0) set_error(p, sm, kErrRingWait, where);
  set_abort(sm);
  return false;
}

__device__ __forceinline__ bool ring_wait(const DecodeParams& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                          uint32_t where) {
  if (mbar_try_wait(bar, parity) && !aborted(sm)) return true;
  return ring_wait_slow(p, sm, bar, parity, where);
}

// ------------------------------------------------------------------------------------- work split
struct Work {
  int rA0, rA1;        // phase-A rows (flattened over active experts)
  int rB0, nB;         // phase-B rows of y
  int nRBB;            // phase-B row-blocks of RBB rows
  int nEg;             // phase-B expert groups of NEB
  int nJs;             // phase-B j-stages per expert group
  int n_act;
};

__device__ __forceinline__ Work make_work(const DecodeParams& p, int n_act) {
  Work w;
  const int G = gridDim.x, c = blockIdx.x;
  // in units of 8 rows, so a 16-byte piece of the h image (8 consecutive j) belongs to one CTA
  const long long RA8 = (long long)n_act * p.de / 8;
  w.rA0 = int(RA8 * c / G) * 8;
  w.rA1 = int(RA8 * (c + 1) / G) * 8;
  w.rB0 = int((long long)p.d * c / G);
  w.nB = int((long long)p.d * (c + 1) / G) - w.rB0;
  w.nRBB = (w.nB + p.RBB - 1) / p.RBB;
  w.nEg = (n_act + p.NEB - 1) / p.NEB;
  w.nJs = (p.nJc + p.KWB - 1) / p.KWB;
  w.n_act = n_act;
  return w;
}

// Phase-A row group: h (a power of two <= RSM) adjacent rows of one expert, starting at flattened row
// r.  Groups never cross an expert or the CTA's range, so one box fetches exactly the group.
struct Group {
  int a, j0, h;
};

__device__ __forceinline__ Group group_at(const DecodeParams& p, int r, int r_end) {
  Group gr;
  gr.a = r / p.de;
  gr.j0 = r - gr.a * p.de;
  const int room = min(p.de - gr.j0, r_end - r);
  int h = p.RSM;
  while (h > room) h >>= 1;
  gr.h = h;
  return gr;
}

// Groups [g_begin, g_begin + GB) of the CTA, walking from cursor r: the first group's row, their
// count, and the cursor after them.
__device__ __forceinline__ int rowblock_walk(const DecodeParams& p, int r, int r_end, int* ngroups) {
  int n = 0;
  while (r < r_end && n < GB) {
    r += group_at(p, r, r_end).h;
    ++n;
  }
  *ngroups = n;
  return r;
}

// The k-th group of the row-block starting at cursor r (k < number of groups).
__device__ __forceinline__ Group group_k(const DecodeParams& p, int r, int r_end, int k, int* row0) {
  Group gr = group_at(p, r, r_end);
  for (int q = 0; q < k; ++q) {
    r += gr.h;
    gr = group_at(p, r, r_end);
  }
  *row0 = r;
  return gr;
}

__device__ __forceinline__ bool stage_is_chunked(int c0, int nc, int nfull) { return c0 + nc <= nfull; }

// Position in the stage ring: stage index, its slot, and the parity of the slot's barrier phase that
// the stage uses (advanced incrementally: no division per stage).
struct RingPos {
  int i = 0, slot = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int S) {
    ++i;
    if (++slot == S) slot = 0, ph ^= 1u;
  }
  __device__ __forceinline__ void seek(int k, int S) {
    i = k;
    slot = k % S;
    ph = uint32_t(k / S) & 1u;
  }
};

// ------------------------------------------------------------------------------------- producers
// Weight producer (one warp): W1 row groups, then W2 expert tiles, in stage order.
template <bool KSPLIT>
__device__ void produce_weights(const DecodeParams& p, const TensorMaps& tm, const Smem& sm, const Work& w) {
  const int lane = threadIdx.x & 31;
  // weights stream through once (evict first), unless the caller expects the next call to reuse them
  const uint64_t pol_w = p.keep_l2 ? policy_evict_last() : policy_evict_first();
  RingPos rp;
  bool ok = true;
  // ---- phase A: stage = one box of a group's whole rows over the pass's columns
  const int KC = p.nKf / p.KP;                 // full chunks per pass
  const bool tail = p.nKc > p.nKf;             // only with one pass
  if constexpr (KSPLIT) {
    // one pass, and every group is RSM adjacent rows of one expert (the CTA's rows are whole multiples
    // of 8): stage s holds rows [rA0 + s RSM, + RSM)
    const int h = p.RSM, hsel = __ffs(h) - 1;
    for (int r = w.rA0; r < w.rA1; r += h, rp.next(p.S)) {
      if (aborted(sm)) { ok = false; break; }
      const int slot = rp.slot;
      if (rp.i >= p.S && !mbar_wait_bounded(&sm.empty[slot], rp.ph ^ 1u, kWaitNs)) {
        if (lane == 0) set_error(p, sm, kErrRingWait, 1);
        ok = false;
        break;
      }
      if (lane == 0) {
        const int a = r / p.de, j0 = r - a * p.de, e = sm.act[a];
        uint8_t* dst = sm.ring + size_t(slot) * p.slot_bytes;
        mbar_arrive_expect_tx(&sm.fullW[slot], uint32_t(KC + (tail ? 1 : 0)) * h * 128);
        if (KC > 0) tma_load_4d(dst, &tm.w1_ch[hsel], 0, j0, 0, e, &sm.fullW[slot], pol_w);
        if (tail) tma_load_3d(dst + p.w1_tail_off, &tm.w1_3d[hsel], p.nKf * 64, j0, e, &sm.fullW[slot], pol_w);
      }
      __syncwarp();
    }
  } else
  for (int r = w.rA0; r < w.rA1 && ok;) {
    int ngr;
    const int r_next = rowblock_walk(p, r, w.rA1, &ngr);
    int row0 = 0;
    const Group mine = group_k(p, r, w.rA1, lane < ngr ? lane : 0, &row0);  // lane k: group k
    const int hsel = __ffs(mine.h) - 1;
    const int e = sm.act[mine.a];
    for (int ps = 0; ps < p.KP && ok; ++ps) {
      for (int gl = 0; gl < ngr; ++gl, rp.next(p.S)) {
        if (aborted(sm)) { ok = false; break; }
        const int slot = rp.slot;
        if (rp.i >= p.S && !mbar_wait_bounded(&sm.empty[slot], rp.ph ^ 1u, kWaitNs)) {
          if (lane == 0) set_error(p, sm, kErrRingWait, 1);
          ok = false;
          break;
        }
        const int h = __shfl_sync(0xffffffffu, mine.h, gl);
        if (lane == 0) mbar_arrive_expect_tx(&sm.fullW[slot], uint32_t(KC + (tail ? 1 : 0)) * h * 128);
        __syncwarp();
        if (lane == gl) {
          uint8_t* dst = sm.ring + size_t(slot) * p.slot_bytes;
          if (KC > 0) tma_load_4d(dst, &tm.w1_ch[hsel], 0, mine.j0, ps * KC, e, &sm.fullW[slot], pol_w);
          if (tail)
            tma_load_3d(dst + p.w1_tail_off, &tm.w1_3d[hsel], p.nKf * 64, mine.j0, e, &sm.fullW[slot], pol_w);
        }
        __syncwarp();
      }
    }
    r = r_next;
  }
  // ---- phase B: stage = NEB experts x KWB chunks of W2 rows [k0, k0 + RBB)
  for (int rb = 0; rb < w.nRBB && ok; ++rb) {
    const int k0 = w.rB0 + rb * p.RBB;
    for (int eg = 0; eg < w.nEg && ok; ++eg) {
      const int a0 = eg * p.NEB, nq = min(p.NEB, w.n_act - a0);
      for (int js = 0; js < w.nJs; ++js, rp.next(p.S)) {
        if (aborted(sm)) { ok = false; break; }
        const int slot = rp.slot;
        if (rp.i >= p.S && !mbar_wait_bounded(&sm.empty[slot], rp.ph ^ 1u, kWaitNs)) {
          if (lane == 0) set_error(p, sm, kErrRingWait, 2);
          ok = false;
          break;
        }
        const int c0 = js * p.KWB, nc = min(p.KWB, p.nJc - c0);
        const bool chunked = stage_is_chunked(c0, nc, p.nJf);
        if (lane == 0) mbar_arrive_expect_tx(&sm.fullW[slot], uint32_t(nq) * (chunked ? p.KWB : nc) * p.RBB * 128);
        __syncwarp();
        if (lane < nq) {
          uint8_t* dst = sm.ring + size_t(slot) * p.slot_bytes + size_t(lane) * p.eB;
          const int e = sm.act[a0 + lane];
          if (chunked) {
            tma_load_4d(dst, &tm.w2_ch, 0, k0, c0, e, &sm.fullW[slot], pol_w);
          } else {
            for (int c = 0; c < nc; ++c)
              tma_load_3d(dst + size_t(c) * p.RBB * 128, &tm.w2_3d, (c0 + c) * 64, k0, e, &sm.fullW[slot], pol_w);
          }
        }
        __syncwarp();
      }
    }
  }
  // every copy this warp issued lands before the CTA may exit
  for (int k = max(0, rp.i - p.S); k < rp.i; ++k) mbar_wait_bounded(&sm.fullW[k % p.S], (k / p.S) & 1, kWaitNs / 10);
}

// x / h producer (one warp): the resident x parts of phase A, then (after the grid barrier) the h
// tiles of phase B.
template <bool KSPLIT>
__device__ void produce_x_h(const DecodeParams& p, const TensorMaps& tm, const Smem& sm, const Work& w) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol_x = policy_evict_last();
  // ---- x parts: once, or once per (row-block, pass) when K is split in passes
  const int KC = p.nKf / p.KP;
  const bool tail = p.nKc > p.nKf;
  int nrb = 0;
  if constexpr (KSPLIT) {
    nrb = w.rA0 < w.rA1 ? 1 : 0;  // one pass: x is loaded once
  } else {
    for (int r = w.rA0; r < w.rA1; ++nrb) {
      int ngr;
      r = rowblock_walk(p, r, w.rA1, &ngr);
    }
  }
  int xloads = 0;
  const int nparts = (p.KP > 1) ? nrb * p.KP : (nrb > 0 ? 1 : 0);
  for (int part = 0; part < nparts; ++part) {
    if (aborted(sm)) break;
    if (xloads > 0 && !mbar_wait_bounded(sm.xfree, (xloads - 1) & 1, kWaitNs)) {
      if (lane == 0) set_error(p, sm, kErrRingWait, 8);
      break;
    }
    const int ps = part % p.KP;
    if (lane == 0) {
      mbar_arrive_expect_tx(sm.xfull, uint32_t(KC + (tail ? 1 : 0)) * p.LB * 128);
      if (KC > 0) tma_load_3d(sm.xbuf, &tm.x_ch, 0, 0, ps * KC, sm.xfull, pol_x);
      if (tail) tma_load_2d(sm.xbuf + size_t(KC) * p.LB * 128, &tm.x_2d, p.nKf * 64, 0, sm.xfull, pol_x);
    }
    __syncwarp();
    ++xloads;
  }
  if (xloads > 0) mbar_wait_bounded(sm.xfull, (xloads - 1) & 1, kWaitNs / 10);  // the last x copies landed

  // ---- h tiles after the grid barrier
  int nG = 0;
  if constexpr (KSPLIT) {
    nG = (w.rA1 - w.rA0) / p.RSM;
  } else {
    for (int r = w.rA0; r < w.rA1; ++nG) r += group_at(p, r, w.rA1).h;
  }
  const int stagesA = p.KP * nG;
  const int stagesB = w.nRBB * w.nEg * w.nJs;
  if (stagesB == 0) return;
  {
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (ld_acquire_gpu(&p.hdr->grid_bar) < gridDim.x) {
      if (aborted(sm) || globaltimer_ns() - t0 > kWaitNs) { ok = false; break; }
      __nanosleep(32);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) set_error(p, sm, kErrGridBarrier, uint32_t(blockIdx.x));
      return;
    }
    fence_proxy_async_global();
  }
  const uint64_t pol_h = policy_evict_last();
  uint32_t hphase = 0;
  int issued = 0;
  int eg = 0, js = 0;
  RingPos rp;
  rp.seek(stagesA, p.S);
  for (int jb = 0; jb < stagesB; ++jb, rp.next(p.S)) {
    if (aborted(sm)) break;
    const int slot = rp.slot;
    if (rp.i >= p.S && !mbar_wait_bounded(&sm.empty[slot], rp.ph ^ 1u, kWaitNs)) {
      if (lane == 0) set_error(p, sm, kErrRingWait, 6);
      break;
    }
    const int a0 = eg * p.NEB, nq = min(p.NEB, w.n_act - a0);
    const int c0 = js * p.KWB, nc = min(p.KWB, p.nJc - c0);
    const uint32_t bytes = uint32_t(nc) * p.HR * 128;
    if (lane == 0) mbar_arrive_expect_tx(&sm.fullH[slot], bytes * nq);
    __syncwarp();
    if (lane < nq)
      bulk_g2s(sm.ring + size_t(slot) * p.slot_bytes + size_t(lane) * p.eB + p.hoff,
               p.h + size_t(a0 + lane) * p.h_expert_bytes + size_t(c0) * p.HR * 128, bytes, &sm.fullH[slot], pol_h);
    __syncwarp();
    hphase ^= 1u << slot;
    ++issued;
    if (++js == w.nJs) {
      js = 0;
      if (++eg == w.nEg) eg = 0;
    }
  }
  uint32_t ph = hphase;
  for (int k = issued - 1; k >= 0 && k >= issued - p.S; --k) {
    const int slot = (stagesA + k) % p.S;
    ph ^= 1u << slot;
    mbar_wait_bounded(&sm.fullH[slot], (ph >> slot) & 1u, kWaitNs / 10);
  }
}

// ------------------------------------------------------------------------------------- consumers
// Columns [de, 64 nJc) of an expert's last h tile face the zero columns the W2 boxes read past de, but
// the workspace may hold any bytes there (another shape's data, possibly a NaN pattern, and 0 * NaN is
// NaN): whoever writes the expert's last row of token t also zeroes that tail in rows t and L + t.  de
// is a multiple of 8, so the tail is whole 16-byte pieces.  `img` is the start of the tile.
__device__ __forceinline__ void zero_h_tail(const DecodeParams& p, uint8_t* img, int t) {
  for (int c8 = (p.de & 63) >> 3; c8 != 0 && c8 < 8; ++c8) {
    *reinterpret_cast<uint4*>(img + swz(t, c8)) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(img + swz(p.L + t, c8)) = make_uint4(0, 0, 0, 0);
  }
}

// The epilogue of one up-projection value: h = r * Swish(u), stored as bf16 hi and lo parts in the
// down-projection's tile layout.
__device__ __forceinline__ void store_h(const DecodeParams& p, const Smem& sm, int a_first, int a, int j, int t,
                                        float u) {
  const float sv = sm.pre_s[(a - a_first) * 32 + t];
  const float rms = sm.rms[t];
  const float rr = (rms > 0.f) ? (sm.pre_g[a - a_first] * fmaxf(sv, 0.f)) / rms : 0.f;
  const float hv = rr * (u / (1.f + expf(-u)));
  const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
  const __nv_bfloat16 lo = __float2bfloat16_rn(hv - __bfloat162float(hi));
  uint8_t* himg = p.h + size_t(a) * p.h_expert_bytes + size_t(j >> 6) * p.HR * 128;
  const int col = j & 63;
  *reinterpret_cast<__nv_bfloat16*>(himg + swz(t, col >> 3) + (col & 7) * 2) = hi;
  *reinterpret_cast<__nv_bfloat16*>(himg + swz(p.L + t, col >> 3) + (col & 7) * 2) = lo;
  if (j == p.de - 1) zero_h_tail(p, himg, t);
}

// Epilogue of a block of the CTA's up-projection rows [r0, r1) (multiples of 8): h = r Swish(u) with
// r = g relu(s) / rms, split into bf16 hi and lo parts and written to the global h image as 16-byte
// pieces of 8 consecutive j (one expert each: row blocks and de are multiples of 8).  u of
// row r0 + i waits in unit i / 8 of the staging buffer.
__device__ void flush_u(const DecodeParams& p, const Smem& sm, int a_first, int r0, int r1) {
  const int units = (r1 - r0) >> 3;
  for (int o = threadIdx.x; o < units * p.L; o += NCW * 32) {
    const int u = o / p.L, t = o - u * p.L;
    const int row = r0 + u * 8;
    const int a = row / p.de, j = row - a * p.de;
    const float rms = sm.rms[t];
    const float sv = sm.pre_s[(a - a_first) * 32 + t];
    const float rr = (rms > 0.f) ? (sm.pre_g[a - a_first] * fmaxf(sv, 0.f)) / rms : 0.f;
    const float4* us = reinterpret_cast<const float4*>(sm.ustage + (u * p.L + t) * 8);
    const float4 ua = us[0], ub = us[1];
    const float uv[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float h0 = rr * (uv[2 * k] / (1.f + expf(-uv[2 * k])));
      const float h1 = rr * (uv[2 * k + 1] / (1.f + expf(-uv[2 * k + 1])));
      const __nv_bfloat162 hh = __floats2bfloat162_rn(h0, h1);
      const __nv_bfloat162 ll = __floats2bfloat162_rn(h0 - __low2float(hh), h1 - __high2float(hh));
      hi[k] = *reinterpret_cast<const uint32_t*>(&hh);
      lo[k] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    uint8_t* img = p.h + size_t(a) * p.h_expert_bytes + size_t(j >> 6) * p.HR * 128;
    *reinterpret_cast<uint4*>(img + swz(t, (j & 63) >> 3)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(img + swz(p.L + t, (j & 63) >> 3)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    if (j + 8 == p.de) zero_h_tail(p, img, t);
  }
}

// Up-projection split over K (L <= 8, one pass): every consumer warp works on every stage over its
// own 64-column chunks c = cw + NCW q and writes its partial sums; then each warp adds the NCW
// partials of one token in warp order and frees the slot.  The x fragments of the
// first kXregChunks chunks of a warp stay in registers; further chunks read them from shared memory.
// Only tokens 0-7 are real rows of the MMA (rows 8-15 are zero).  Every group has RSM rows (the CTA's
// rows are whole multiples of 8 and RSM <= 8), so a warp's operand offsets inside a stage are the
// same for every stage and are computed once; chunks past the end read a zero row, so loads and
// MMAs run unconditionally.
__device__ void phase_a_ksplit(const DecodeParams& p, const Smem& sm, const Work& w, int a_first, RingPos& rp) {
  const int cw = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int KC = p.nKf;
  const int nck = p.nKc;
  const int h = p.RSM;
  const uint32_t xb = smem_u32(sm.xbuf), zaddr = smem_u32(sm.zero);
  const int lrow = lane & 7, lhalf = (lane >> 3) & 1;  // ldmatrix .x2 addressing: rows 0-7, two k halves
  if (w.rA0 >= w.rA1) return;  // no up-projection rows: x is not loaded
  // the offset inside a stage of this lane's 16-byte piece for chunk c, k16 = 0 (k16 adds 32 bytes
  // before the swizzle: the swizzled chunk index is (2 k16 + lhalf) ^ (row & 7))
  auto w_row = [&](int c) { return (c < KC ? c * h : (p.w1_tail_off >> 7)) + (lrow < h ? lrow : 0); };
  ring_wait(p, sm, sm.xfull, 0, 7);
  uint32_t xf[kXregChunks][4][2];
  int wrow[kXregChunks];
#pragma unroll
  for (int q = 0; q < kXregChunks; ++q) {
    const int c = cw + q * NCW;
    wrow[q] = c < nck ? w_row(c) : -1;
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16) {
      const uint32_t ad = c < nck ? xb + swz(c * p.LB + lrow, k16 * 2 + lhalf) : zaddr;
      ldmatrix_x2(ad, xf[q][k16][0], xf[q][k16][1]);
    }
  }
  const int blk_rows = p.ustage_units * 8;  // rows whose u fit the staging buffer
  int blk0 = w.rA0;
  for (int r = w.rA0; r < w.rA1; r += h, rp.next(p.S)) {
    const int slot = rp.slot;
    if (ring_wait(p, sm, &sm.fullW[slot], rp.ph, 3)) {
      const uint32_t wb = smem_u32(sm.ring + size_t(slot) * p.slot_bytes);
      // all fragment loads of a batch first, then its MMAs: one k16 chain per accumulator
      float ak[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int v = 0; v < 4; ++v) ak[k][v] = 0.f;
#pragma unroll
      for (int q0 = 0; q0 < kXregChunks; q0 += 2) {  // two chunks per batch
        uint32_t wf[2][4][2];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const int wr = wrow[q0 + q];
            const uint32_t ad = wr >= 0 ? wb + swz(wr, k16 * 2 + lhalf) : zaddr;
            ldmatrix_x2(ad, wf[q][k16][0], wf[q][k16][1]);
          }
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint32_t a[4] = {xf[q0 + q][k16][0], 0u, xf[q0 + q][k16][1], 0u};
            mma_bf16_16816(ak[k16], a, wf[q][k16][0], wf[q][k16][1]);
          }
      }
      for (int c = cw + kXregChunks * NCW; c < nck; c += NCW) {  // chunks whose x stays in smem
        const int wr = w_row(c);
        uint32_t wf[4][2], xs[4][2];
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          ldmatrix_x2(wb + swz(wr, k16 * 2 + lhalf), wf[k16][0], wf[k16][1]);
          ldmatrix_x2(xb + swz(c * p.LB + lrow, k16 * 2 + lhalf), xs[k16][0], xs[k16][1]);
        }
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          const uint32_t a[4] = {xs[k16][0], 0u, xs[k16][1], 0u};
          mma_bf16_16816(ak[k16], a, wf[k16][0], wf[k16][1]);
        }
      }
      float2* red = reinterpret_cast<float2*>(sm.red_s) + size_t(slot) * NCW * 32;
      red[cw * 32 + lane] = make_float2((ak[0][0] + ak[1][0]) + (ak[2][0] + ak[3][0]),
                                        (ak[0][1] + ak[1][1]) + (ak[2][1] + ak[3][1]));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.rbar[slot]);
    // Every warp finishes one token of the stage: the MMA fragment's lanes 4 cw .. 4 cw + 3 hold token
    // cw (rows 2 (lane & 3) and + 1), so lanes 0-3 of warp cw add the NCW partial sums of those lanes in
    // warp order.  All warps run this every stage, then release the slot (NCW arrivals).
    {
      const bool ok = ring_wait(p, sm, &sm.rbar[slot], rp.ph, 9);
      float u0 = 0.f, u1 = 0.f;
      const int src = cw * 4 + (lane & 3);
      if (ok && lane < 4) {
        const float2* red = reinterpret_cast<const float2*>(sm.red_s) + size_t(slot) * NCW * 32;
#pragma unroll
        for (int ww = 0; ww < NCW; ++ww) {
          const float2 v = red[ww * 32 + src];
          u0 += v.x;
          u1 += v.y;
        }
      }
      // the slot and its partial sums are free once read; u waits in shared memory for the epilogue
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      const int t = cw, loc = r - blk0 + lane * 2;  // rows loc, loc + 1 of the block (loc even)
      if (ok && lane < 4 && t < p.L && lane * 2 < h)
        *reinterpret_cast<float2*>(sm.ustage + ((loc >> 3) * p.L + t) * 8 + (loc & 7)) = make_float2(u0, u1);
    }
    if (r + h - blk0 == blk_rows || r + h >= w.rA1) {  // the block is full, or the CTA's rows end
      named_bar_sync(1, NCW * 32);  // every u of the block is staged
      flush_u(p, sm, a_first, blk0, r + h);
      named_bar_sync(1, NCW * 32);  // the staging buffer is free for the next block
      blk0 = r + h;
    }
  }
}

// Up-projection with x resident in shared memory (any L, K in passes): a consumer warp owns whole
// row groups (gl = cw + NCW q within a row-block of GB groups) over all of K.
template <int MTA>
__device__ void phase_a_smem(const DecodeParams& p, const Smem& sm, const Work& w, int a_first, RingPos& rp) {
  const int cw = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int mtA = (p.L + 15) / 16;
  const uint32_t zaddr = smem_u32(sm.zero);
  const int KC = p.nKf / p.KP;
  const int nck = KC + (p.nKc > p.nKf ? 1 : 0);
  const int tail_q = p.w1_tail_off >> 7;
  int xloads = 0;
  for (int r = w.rA0; r < w.rA1;) {
    int ngr;
    const int r_next = rowblock_walk(p, r, w.rA1, &ngr);
    Group gq[GPW];
    int grow[GPW];
#pragma unroll
    for (int q = 0; q < GPW; ++q) {
      const int gl = cw + q * NCW;
      gq[q] = group_k(p, r, w.rA1, gl < ngr ? gl : 0, &grow[q]);
    }
    float acc[GPW][MTA][4];
#pragma unroll
    for (int q = 0; q < GPW; ++q)
#pragma unroll
      for (int a = 0; a < MTA; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[q][a][c] = 0.f;
    for (int ps = 0; ps < p.KP; ++ps) {
      if (p.KP > 1 || xloads == 0) {
        ring_wait(p, sm, sm.xfull, xloads & 1, 7);
        ++xloads;
      }
      const uint32_t xb = smem_u32(sm.xbuf);
      // every warp waits for and releases every stage in order (one barrier phase at a time, so the
      // parity of a wait is never ambiguous whatever S is); only the stage's owner computes
      for (int gl = 0; gl < ngr; ++gl, rp.next(p.S)) {
        const int slot = rp.slot;
        const int q = gl / NCW;
        if (ring_wait(p, sm, &sm.fullW[slot], rp.ph, 3) && (gl % NCW) == cw) {
          int h = gq[0].h;
#pragma unroll
          for (int qq = 1; qq < GPW; ++qq)
            if (qq == q) h = gq[qq].h;
          const uint32_t wb = smem_u32(sm.ring + size_t(slot) * p.slot_bytes);
          const int brow = (lane & 7) < h ? (lane & 7) : 0;  // rows past the group: never used
          float ak[4][MTA][4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int mt = 0; mt < MTA; ++mt)
#pragma unroll
              for (int v = 0; v < 4; ++v) ak[k][mt][v] = 0.f;
          for (int c = 0; c < nck; ++c) {
            const int wq = (c < KC ? c * h : tail_q) + brow;
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16) {
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4(wb + swz(wq, k16 * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
#pragma unroll
              for (int mt = 0; mt < MTA; ++mt) {
                if (mt < mtA) {
                  uint32_t a[4];
                  const int row = mt * 16 + (lane & 15);
                  const uint32_t ad = row < p.L ? xb + swz(c * p.LB + row, k16 * 2 + (lane >> 4)) : zaddr;
                  ldmatrix_x4(ad, a[0], a[1], a[2], a[3]);
                  mma_bf16_16816(ak[k16][mt], a, b0, b1);
                }
              }
            }
          }
#pragma unroll
          for (int qq = 0; qq < GPW; ++qq)
            if (qq == q)
#pragma unroll
              for (int mt = 0; mt < MTA; ++mt)
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  acc[qq][mt][v] += (ak[0][mt][v] + ak[1][mt][v]) + (ak[2][mt][v] + ak[3][mt][v]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
      }
      if (p.KP > 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.xfree);  // this warp is done with the x part
      }
    }
#pragma unroll
    for (int qq = 0; qq < GPW; ++qq) {
      const int gl = qq * NCW + cw;
      if (gl >= ngr) continue;
#pragma unroll
      for (int mt = 0; mt < MTA; ++mt) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int t = mt * 16 + gid + (v >> 1) * 8;
          const int n = tig * 2 + (v & 1);
          if (t >= p.L || n >= gq[qq].h) continue;
          store_h(p, sm, a_first, gq[qq].a, gq[qq].j0 + n, t, acc[qq][mt][v]);
        }
      }
    }
    r = r_next;
  }
}

template <int LC, bool KSPLIT>
__device__ void consume(const DecodeParams& p, const Smem& sm, const Work& w) {
  constexpr int MTA = (LC + 15) / 16;
  constexpr int MT = (2 * LC + 15) / 16;
  const int ctid = threadIdx.x;
  const int cw = ctid >> 5, lane = ctid & 31;
  const uint32_t zaddr = smem_u32(sm.zero);
  RingPos rp;

  const int a_first = w.rA0 / p.de;  // pre_s / pre_g hold s and g of experts a_first ..

  // ---------------- phase A
  if constexpr (KSPLIT) {
    phase_a_ksplit(p, sm, w, a_first, rp);
  } else {
    phase_a_smem<MTA>(p, sm, w, a_first, rp);
  }
  // publish this CTA's h before any CTA reads h
  __threadfence();
  named_bar_sync(1, NCW * 32);
  if (ctid == 0) {
    fence_proxy_async_global();
    red_release_gpu_add(&p.hdr->grid_bar, 1u);
    pdl_launch_dependents();
  }

  // ---------------- phase B
  // A stage holds nq <= NEB experts x nc <= KWB chunks of 64 j; its k-steps (16 j each) in
  // expert-major order g = qe * 4 KWB + kk go to warp g % NCW, at most kKS per warp (the plan keeps
  // NEB KWB <= 8).  The offsets of a warp's k-steps inside a stage are the same for every stage, so
  // they are computed once; a k-step outside the stage, or an operand row outside the tile, reads the
  // zero row, and loads and MMAs run unconditionally (zero fragments add nothing).
  constexpr int kKS = 4;
  constexpr int KB = MT == 1 ? 4 : 2;  // k-steps per batch: all loads of a batch, then its MMAs
  constexpr int NP2 = kNP2<LC>;        // 16-row n groups of a row block (RBB <= 16 NP2)
  constexpr int NSET = 1;
  int ks_qe[kKS], ks_c[kKS], offA[kKS][MT], offB[kKS][NP2];
#pragma unroll
  for (int b = 0; b < kKS; ++b) {
    const int g = cw + NCW * b;
    const int qe = g / (4 * p.KWB), kk = g - qe * 4 * p.KWB;
    const int c = kk >> 2, k16 = kk & 3;
    ks_qe[b] = qe;
    ks_c[b] = c;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int row = mt * 16 + (lane & 15);
      offA[b][mt] = row < p.HR ? qe * p.eB + p.hoff + c * p.HR * 128 + int(swz(row, k16 * 2 + (lane >> 4))) : -1;
    }
#pragma unroll
    for (int np2 = 0; np2 < NP2; ++np2) {
      const int row = np2 * 16 + (lane & 7) + (lane >> 4) * 8;
      offB[b][np2] = row < p.RBB ? qe * p.eB + int(swz(c * p.RBB + row, k16 * 2 + ((lane >> 3) & 1))) : -1;
    }
  }
  uint32_t hphase = 0;
  for (int rb = 0; rb < w.nRBB; ++rb) {
    float acc[NSET][MT][2 * NP2][4];
#pragma unroll
    for (int e = 0; e < NSET; ++e)
#pragma unroll
      for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < 2 * NP2; ++b)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[e][a][b][c] = 0.f;
    int eg = 0, js = 0;
    for (int s = 0; s < w.nEg * w.nJs; ++s, rp.next(p.S)) {
      const int slot = rp.slot;
      const bool okW = ring_wait(p, sm, &sm.fullW[slot], rp.ph, 4);
      const bool okH = okW && ring_wait(p, sm, &sm.fullH[slot], (hphase >> slot) & 1u, 5);
      hphase ^= 1u << slot;
      if (okH) {
        const int nq = min(p.NEB, w.n_act - eg * p.NEB);
        const int nc = min(p.KWB, p.nJc - js * p.KWB);
        const uint32_t sb = smem_u32(sm.ring + size_t(slot) * p.slot_bytes);
#pragma unroll
        for (int b0 = 0; b0 < kKS; b0 += KB) {
          uint32_t af[KB][MT][4], bf[KB][NP2][4];
#pragma unroll
          for (int b = 0; b < KB; ++b) {
            const bool in = ks_qe[b0 + b] < nq && ks_c[b0 + b] < nc;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const int o = offA[b0 + b][mt];
              ldmatrix_x4(in && o >= 0 ? sb + uint32_t(o) : zaddr, af[b][mt][0], af[b][mt][1], af[b][mt][2],
                          af[b][mt][3]);
            }
#pragma unroll
            for (int np2 = 0; np2 < NP2; ++np2) {
              const int o = offB[b0 + b][np2];
              ldmatrix_x4(in && o >= 0 ? sb + uint32_t(o) : zaddr, bf[b][np2][0], bf[b][np2][1], bf[b][np2][2],
                          bf[b][np2][3]);
            }
          }
#pragma unroll
          for (int b = 0; b < KB; ++b)
#pragma unroll
            for (int np2 = 0; np2 < NP2; ++np2)
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                mma_bf16_16816(acc[b % NSET][mt][np2 * 2], af[b][mt], bf[b][np2][0], bf[b][np2][1]);
                mma_bf16_16816(acc[b % NSET][mt][np2 * 2 + 1], af[b][mt], bf[b][np2][2], bf[b][np2][3]);
              }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      if (++js == w.nJs) js = 0, ++eg;
    }
#pragma unroll
    for (int e = 1; e < NSET; ++e)
#pragma unroll
      for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < 2 * NP2; ++b)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[0][a][b][c] += acc[e][a][b][c];
    // sum the warps' partials in a fixed order; y = (hi part) + (lo part)
    constexpr int NT8 = 2 * NP2;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT8; ++nt)
        *reinterpret_cast<float4*>(sm.red + ((((cw * MT + mt) * NT8 + nt) * 32 + lane) * 4)) =
            make_float4(acc[0][mt][nt][0], acc[0][mt][nt][1], acc[0][mt][nt][2], acc[0][mt][nt][3]);
    named_bar_sync(1, NCW * 32);
    const int k0 = w.rB0 + rb * p.RBB, nrows = min(p.RBB, w.nB - rb * p.RBB);
    for (int o = ctid; o < p.L * nrows; o += NCW * 32) {
      const int t = o / nrows, c = o - t * nrows;
      float v = 0.f;
      for (int half = 0; half < 2; ++half) {
        const int row = half * p.L + t;
        const int mt = row >> 4, r16 = row & 15;
        const int ln = (r16 & 7) * 4 + ((c & 7) >> 1);
        const int reg = (r16 >> 3) * 2 + (c & 1);
        const int nt = c >> 3;
#pragma unroll
        for (int ww = 0; ww < NCW; ++ww) v += sm.red[((((ww * MT + mt) * NT8 + nt) * 32 + ln) * 4) + reg];
      }
      p.y[size_t(t) * p.d + k0 + c] = v;
    }
    named_bar_sync(1, NCW * 32);
  }
}

// ------------------------------------------------------------------------------ router and prologue
// (decode_router.cuh, instantiated for this kernel's kThreads)
using decode_router::RouterStage;
using decode_router::cp_async4;

template <int LC, bool KSPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    expert_decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ TensorMaps tm) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int MT = (2 * LC + 15) / 16;
  constexpr int kRedBytes = NCW * MT * 2 * kNP2<LC> * 32 * 4 * 4;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem sm;
  sm.xbuf = base;
  sm.ring = base + p.xbuf_bytes;
  uint8_t* after_ring = base + p.pre_bytes;  // >= the ring's end
  const bool red_alias = p.xbuf_bytes >= kRedBytes;  // x is no longer needed in phase B
  sm.red = reinterpret_cast<float*>(red_alias ? sm.xbuf : after_ring);
  uint8_t* tail = red_alias ? after_ring : after_ring + kRedBytes;
  sm.zero = tail;
  sm.abort_flag = reinterpret_cast<volatile int*>(tail + 16);
  sm.fullW = reinterpret_cast<uint64_t*>(tail + 32);
  sm.fullH = sm.fullW + p.S;
  sm.empty = sm.fullH + p.S;
  sm.xfull = sm.empty + p.S;
  sm.xfree = sm.xfull + 1;
  sm.act = reinterpret_cast<int32_t*>(sm.xfree + 1);
  sm.n_act = sm.act + kMaxE;
  sm.rms = reinterpret_cast<float*>(sm.n_act + 4);
  sm.maskw = reinterpret_cast<uint32_t*>(sm.rms + 32);
  sm.pre_s = reinterpret_cast<float*>(sm.maskw + 32 * 32);
  sm.pre_g = sm.pre_s + kMaxSpan * 32;
  sm.red_s = reinterpret_cast<float*>(reinterpret_cast<uintptr_t>(sm.pre_g + kMaxSpan + 3) & ~uintptr_t(15));
  sm.rbar = reinterpret_cast<uint64_t*>(sm.red_s + (p.ksplit ? size_t(p.S) * NCW * 32 * 2 : 0));
  sm.ustage = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(sm.rbar + p.S) + 15) & ~uintptr_t(15));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&sm.fullW[s], 1);
      mbar_init(&sm.fullH[s], 1);
      mbar_init(&sm.empty[s], NCW);
    }
    mbar_init(sm.xfull, 1);
    mbar_init(sm.xfree, NCW);
    for (int s2 = 0; s2 < p.S; ++s2) mbar_init(&sm.rbar[s2], NCW);
    *reinterpret_cast<uint4*>(sm.zero) = make_uint4(0, 0, 0, 0);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == NCW && lane == 0) {
    for (int k = 0; k < 4; ++k) {
      prefetch_tensormap(&tm.w1_ch[k]);
      prefetch_tensormap(&tm.w1_3d[k]);
    }
    prefetch_tensormap(&tm.w2_ch);
    prefetch_tensormap(&tm.w2_3d);
    prefetch_tensormap(&tm.x_ch);
    prefetch_tensormap(&tm.x_2d);
  }
  __syncthreads();

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
  if (!aborted(sm)) {
    float* sbuf = rs.W;  // [L][E], over the router's staging
    decode_router::prologue_router_stats<kThreads>(p, sm, rs, sbuf);
    __syncthreads();
    const int n_act = *sm.n_act;
    const Work w = make_work(p, n_act);
    if (w.rA0 < w.rA1) {  // s and g of every expert this CTA's up-projection rows touch
      const int a_first = w.rA0 / p.de, span = (w.rA1 - 1) / p.de - a_first + 1;
      for (int o = tid; o < span * p.L; o += kThreads) {
        const int aa = o / p.L, t = o - aa * p.L;
        sm.pre_s[aa * 32 + t] = sbuf[size_t(t) * p.E + sm.act[a_first + aa]];
      }
      for (int aa = tid; aa < span; aa += kThreads) sm.pre_g[aa] = rs.g[sm.act[a_first + aa]];
    }
    fence_proxy_async_smem();  // the ring held generic data before bulk copies write into it
    __syncthreads();

    if (warp < NCW) {
      consume<LC, KSPLIT>(p, sm, w);
    } else if (warp == NCW) {
      produce_weights<KSPLIT>(p, tm, sm, w);
    } else {
      produce_x_h<KSPLIT>(p, tm, sm, w);
    }
  }
  // the last CTA out sets the grid's counters back for the next call on this workspace
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.hdr->exit_ctr, 1u) == gridDim.x - 1) {
      p.hdr->router_bar = 0u;
      p.hdr->grid_bar = 0u;
      p.hdr->exit_ctr = 0u;
    }
  }
}

template <int LC, bool KSPLIT>
cudaError_t launch_lc(const DecodeParams& p, const TensorMaps& tm, const DecodeLaunch& plan, cudaStream_t st,
                      bool pdl) {
  auto kfn = expert_decode_kernel<LC, KSPLIT>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
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

size_t decode_h_bytes(int L, int E, int de) { return size_t(E) * ((de + 63) / 64) * size_t(2 * L) * 128; }

bool expert_decode_plan(int L, int d, int E, int de, int num_sms, int max_smem, DecodeParams* p,
                        DecodeLaunch* out) {
  if (L < 1 || L > kTcSmallL || d % 8 != 0 || de % 8 != 0 || E < 1 || E > kMaxE) return false;
  const int lc = 8;
  const int mt = (2 * lc + 15) / 16;
  const int G = num_sms;
  if (d > 256 * 64) return false;  // a box spans at most 256 chunks
  if ((E + G - 1) / G + 2 > kMaxSpan) return false;  // experts one CTA's up-projection rows touch
  // up-projection: x resident per pass of KC full 64-column chunks (plus the ragged chunk, which
  // needs a single pass); stages of one box of up to RSM whole rows
  p->nKf = d / 64;
  p->nKc = (d + 63) / 64;
  p->LB = round_up(L, 8);
  const int xbudget = 100 * 1024;
  p->KP = 1;
  if (p->nKc > p->nKf) {
    if (size_t(p->nKc) * p->LB * 128 > size_t(xbudget)) return false;
  } else {
    while (size_t(p->nKf / p->KP) * p->LB * 128 > size_t(xbudget) || p->nKf % p->KP != 0) {
      if (++p->KP > p->nKf) return false;
    }
  }
  const int KC = p->nKf / p->KP;
  const int nck = KC + (p->nKc > p->nKf ? 1 : 0);
  p->Kp = KC * 64;
  p->xbuf_bytes = round_up(nck * p->LB * 128, 1024);
  p->ksplit = (L <= 8 && p->KP == 1) ? 1 : 0;
  const int target = 32 * 1024;
  p->RSM = 8;
  while (p->RSM > 1 && p->RSM * nck * 128 > target) p->RSM >>= 1;
  // the ragged chunk's tile sits at a 1024-byte aligned offset after the full chunks
  p->w1_tail_off = round_up(KC * p->RSM * 128, 1024);
  const int slotA = round_up(nck > KC ? p->w1_tail_off + p->RSM * 128 : KC * p->RSM * 128, 1024);
  // down-projection: W2 boxes of RBB rows x KWB chunks per expert, NEB experts per stage
  p->HR = 2 * L;
  p->nJc = (de + 63) / 64;
  p->nJf = de / 64;
  p->h_expert_bytes = p->nJc * p->HR * 128;
  const int rbmax = (d + G - 1) / G;
  const int rbb_cap = 16 * np2_of(lc);
  p->RBB = round_up(rbmax < 1 ? 1 : (rbmax > rbb_cap ? rbb_cap : rbmax), 8);
  auto part_bytes = [&](int kwb) {
    const int w2 = p->RBB * kwb * 128;  // multiple of 1024
    return round_up(w2 + round_up(p->HR * kwb * 128, 16), 1024);
  };
  p->KWB = p->nJc;
  if (p->nJf >= 1 && p->KWB > p->nJf) p->KWB = p->nJf;
  const int slot_cap = slotA > 8192 ? slotA : 8192;
  while (p->RBB > 32 && part_bytes(p->KWB) > slot_cap) p->RBB -= 8;  // keep the stage at the A size
  while (p->KWB > 1 && part_bytes(p->KWB) > slot_cap) --p->KWB;
  p->hoff = p->RBB * p->KWB * 128;
  p->eB = part_bytes(p->KWB);
  const int slot = round_up(slotA > p->eB ? slotA : p->eB, 1024);
  p->NEB = slot / p->eB;
  if (p->NEB < 1) p->NEB = 1;
  while (p->NEB > 1 && p->NEB * p->KWB > 8) --p->NEB;  // a stage has at most 32 k-steps of 16 j
  p->slot_bytes = slot;
  const size_t red = size_t(NCW) * mt * 2 * np2_of(lc) * 32 * 4 * 4;
  const size_t red_extra = size_t(p->xbuf_bytes) >= red ? 0 : red;
  const size_t tail = 32 + 3 * 8 * 32 + 16 + size_t(kMaxE + 4) * 4 + 32 * 4 + 32 * 32 * 4 + (kMaxSpan * 33) * 4 + 16;
  const size_t per_slot = (p->ksplit ? size_t(NCW) * 32 * 2 * 4 : 0) + 16;  // red_s and rbar of one slot
  // staged u: blocks of ustage_units units of 8 rows, L tokens x 8 floats each
  {
    const int worst = int((size_t(E) * de / 8 + G - 1) / G);  // units of 8 rows a CTA may get
    const int cap = 8192 / (L * 32) > 0 ? 8192 / (L * 32) : 1;   // about 8 KB of staging
    p->ustage_units = p->ksplit ? (worst < cap ? worst : cap) : 0;
    p->ustage_bytes = p->ustage_units * L * 32;
  }
  // router units, and the shared memory the router's staging and the chunk's s need before the ring
  // is filled: at the start of the region of x and the ring, which is made at least that large
  p->rrows = decode_router_rows(d);
  p->rq = decode_router_parts(d);
  p->rcb = (E + 31) / 32;
  const size_t gb = size_t(2) * ((E + 3) & ~3) * 4;  // g and b
  const size_t router_need = size_t(p->rrows) * 128 + size_t(L) * p->rrows * 4 + size_t(kThreads / 32) * 8 * 32 * 4;
  const size_t s_need = size_t(L) * E * 4;
  const size_t pre_need = gb + (router_need > s_need ? router_need : s_need);
  const size_t fixed = 1024 + red_extra + tail + size_t(p->ustage_bytes);
  if (fixed + pre_need >= size_t(max_smem)) return false;
  int S = int((size_t(max_smem) - fixed - size_t(p->xbuf_bytes)) / (size_t(p->slot_bytes) + per_slot));
  if (S > 32) S = 32;
  for (;; --S) {
    if (S < 2) return false;
    size_t pre = size_t(p->xbuf_bytes) + size_t(S) * p->slot_bytes;
    if (pre < pre_need) pre = round_up(int(pre_need), 1024);
    const size_t smem = fixed + pre + size_t(S) * per_slot;
    if (smem <= size_t(max_smem)) {
      p->S = S;
      p->pre_bytes = int(pre);
      out->smem = smem;
      break;
    }
  }
  out->grid = G;
  out->lclass = lc;
  return true;
}

cudaError_t expert_decode_occupancy(const DecodeParams& p, size_t smem, int* ctas_per_sm) {
  auto kfn = p.ksplit ? expert_decode_kernel<8, true> : expert_decode_kernel<8, false>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, kfn, kThreads, smem);
}

cudaError_t expert_decode_launch(const DecodeParams& p, const TensorMaps& tm, const DecodeLaunch& plan,
                                 cudaStream_t st, bool pdl) {
  // other decode shapes (decode_on_tc) take the tcgen05 kernel (expert_decode_tc.cu)
  if (plan.lclass != 8) return cudaErrorInvalidValue;
  return p.ksplit ? launch_lc<8, true>(p, tm, plan, st, pdl) : launch_lc<8, false>(p, tm, plan, st, pdl);
}

}  // namespace bffn
