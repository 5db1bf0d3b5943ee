// Batched decode path of the BlockFFN chunk layer: many independent chunks of up to 8 tokens (one per
// sequence of a serving step, or one per layer of a stacked model) in two launches.
//
// Router kernel (one CTA per group of up to 64 tokens of one layer): s = x Wr + b in fp32, then ReLU, the
// RMSNorm statistics over the
// E router entries, the per-token active bits with __ballot_sync, the chunk's union of active experts
// as an ascending list built with __popc and a warp scan, the sparsity counts, and
// r = g relu(s) / rms for the expert kernel (lsdiaocha.cn BlockFFN article, sections 2 and 4; BlockFFN
// abstract: a ReLU router followed by RMSNorm, chunk-level sparsity as the union of the chunk's
// activated experts).
//
// Expert kernel (persistent, one CTA per SM): the CTAs form `teams` teams of T; team k takes chunks
// k, k + teams, k + 2 teams, ... in order.  Per chunk the union is evaluated for all its tokens as one
// batch, outer loop over the active experts and inner batched product (article, section 7), and only
// the union's W1 / W2 rows are read, each exactly once:
//  * up-projection: the chunk's (active expert, j) rows are split over the team's CTAs in 8-row units;
//    a CTA walks its rows in groups of at most 128 rows of one expert and streams each group over d
//    in stages of about 32 KB (128 columns of a full group, more of a short one; TMA tensor boxes into
//    a ring of shared-memory stages guarded by mbarriers).  Consumer warp w owns rows [16 w, 16 w + 16) of the group: mma.sync m16n8k16 with the
//    weight rows as M (16), the chunk's tokens as N (8) and x read from shared memory as the B operand,
//    accumulated over all of d in registers.  The epilogue h = r Swish(u), Swish(u) = u / (1 + e^-u)
//    (article, section 2), goes to the team's h image as bf16 hi + lo parts (about 16 mantissa bits).
//  * a team barrier (one arrival counter per chunk) publishes h.  Each role walks the schedule A(0),
//    A(1), B(0), A(2), B(1), ...: a chunk's down-projection follows the next chunk's up-projection, so
//    the barrier has a whole phase of slack and the weight stream practically never waits on it.
//  * one warp issues every copy into the ring in stage order (W1 boxes, W2 boxes with the stage's h
//    tiles on the same barrier), another the x tiles; eight consumer warps run the MMAs.  Each ring
//    barrier keeps one parity bit, so every waiter on it stays within one pass of the ring: the copy
//    warp waits for each slot's release in turn and the consumers for each stage in turn.
//  * down-projection: y rows are split over the team's CTAs in 8-row units; a stage holds one active
//    expert's W2 rows of this CTA for one or more 64-wide j chunks, plus the matching h tiles.  Warp w
//    owns m-tiles w and w + 8 of the CTA's rows for the whole chunk (output-stationary: no cross-warp
//    reduction), with separate accumulators for the hi and lo parts of h, added once at the end.
//    Every y element has one writer and a fixed summation order: y is bit-reproducible.
//  The ring runs on across chunks and phases, so no SM idles between chunks.
#include "blockffn.h"
#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace batch {
namespace {

constexpr int NCW = 8;                     // consumer warps
constexpr int kWarpW = NCW;                // copies into the ring: W1, W2 and the h tiles
constexpr int kWarpX = NCW + 1;            // x tiles of the up-projection
constexpr int kThreads = (NCW + 2) * 32;
constexpr int kGroupRows = 128;            // up-projection rows of one group (8 m-tiles)
constexpr int kStageA = kStageABytes;      // bytes of an up-projection stage (at most)
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kRouterThreads = 256;

__device__ __forceinline__ uint32_t swz(int row, int chunk16) {
  return uint32_t(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}
__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

__device__ __forceinline__ int layer_of(const Params& p, int c) { return p.layer ? p.layer[c] : c % p.n_layers; }
__device__ __forceinline__ bool layer_ok(const Params& p, int l) { return l >= 0 && l < p.n_layers; }

// ===================================================================================== router kernel
// One CTA routes a group of up to 64 tokens (kRouterTokens): G = 64 / L chunks that use the same layer
// (chunks l, l + n_layers, l + 2 n_layers, ... when there is no layer array; one chunk per CTA when
// there is one).  s = x Wr (+ b) is a small GEMM of the group's tokens against the layer's Wr: tiles of
// 32 rows of d x 64 experts staged in shared memory, each thread a 4 x 4 register tile of (token,
// expert) sums accumulated over d in increasing order, so s does not depend on timing.  s goes to
// r's place in the workspace; then one warp per token takes the RMS of relu(s) over the E experts and
// the active bits (__ballot_sync), one warp per chunk the union (__popc and a warp scan) and counts, and
// r = g relu(s) / rms overwrites s (rms: the RMS of the ReLU outputs, or their sum for the ReMoE router).
constexpr int kRouterTokens = 64;
constexpr int kRtK = 32;   // rows of d per tile
constexpr int kRtE = 64;   // experts per tile

__device__ __forceinline__ int router_group_size(const Params& p) {
  return p.layer ? 1 : max(1, kRouterTokens / p.L);
}
// Chunk of slot j of router CTA b (or -1): without a layer array, CTA b takes layer b % n_layers and
// that layer's chunks [G (b / n_layers), + G) in its own order.
__device__ __forceinline__ int router_chunk(const Params& p, int b, int j) {
  if (p.layer) return j == 0 ? b : -1;
  const int G = router_group_size(p), l = b % p.n_layers, q = b / p.n_layers;
  const long long c = (long long)l + (long long)p.n_layers * (G * q + j);
  return c < p.C ? int(c) : -1;
}

__global__ void __launch_bounds__(kRouterThreads) batch_router_kernel(const Params p) {
  __shared__ __align__(16) float Xs[kRtK][kRouterTokens];
  __shared__ __align__(16) float Ws[kRtK][kRtE];
  __shared__ uint32_t maskw[kRouterTokens][32];
  __shared__ float rms[kRouterTokens];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = p.L, d = p.d, E = p.E, nW = (E + 31) >> 5;
  const int G = router_group_size(p);
  const int c0 = router_chunk(p, blockIdx.x, 0);
  if (c0 < 0) return;
  const int layer = layer_of(p, c0);
  int nchunks = 0;
  while (nchunks < G && router_chunk(p, blockIdx.x, nchunks) >= 0) ++nchunks;
  const int M = nchunks * L;  // tokens of the group
  if (tid < nchunks) p.chunk_bar[router_chunk(p, blockIdx.x, tid)] = 0u;  // the expert kernel's counters
  if (!layer_ok(p, layer)) {  // an invalid layer index: the chunk is left empty and the error recorded
    if (tid == 0) {
      atomicOr(&p.hdr->err, kErrBadLayer);
      p.hdr->err_info = uint32_t(c0);
      p.n_active[c0] = 0;
      if (p.counts) p.counts[2 * c0] = L * E, p.counts[2 * c0 + 1] = E;
    }
    if (p.tok_mask)
      for (int o = tid; o < L * nW; o += kRouterThreads) p.tok_mask[size_t(c0) * L * nW + o] = 0u;
    return;
  }
  const float* Wr = p.Wr + size_t(layer) * d * E;
  const float* g = p.g + size_t(layer) * E;
  const float* br = p.br ? p.br + size_t(layer) * E : nullptr;
  // token m of the group: chunk router_chunk(m / L), row m % L
  auto token_row = [&](int m) -> const __nv_bfloat16* {
    return p.x + (size_t(router_chunk(p, blockIdx.x, m / L)) * L + (m % L)) * d;
  };
  auto s_row = [&](int m) -> float* {  // s (then r) of token m, in r's place in the workspace
    return p.r + (size_t(router_chunk(p, blockIdx.x, m / L)) * L + (m % L)) * E;
  };

  // ---- s = x Wr + b
  const int ty = tid >> 4, tx = tid & 15;  // tokens 4 ty .. 4 ty + 3, experts 4 tx .. 4 tx + 3 of the tile
  for (int eb = 0; eb < E; eb += kRtE) {
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += kRtK) {
      {  // x: 64 tokens x 32 columns (bf16 -> fp32, transposed), 8 columns per thread
        const int m = tid >> 2, k8 = (tid & 3) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && k0 + k8 < d) v = *reinterpret_cast<const uint4*>(token_row(m) + k0 + k8);
        const __nv_bfloat16* hv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
        for (int i = 0; i < 8; ++i) Xs[k8 + i][m] = __bfloat162float(hv[i]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // Wr: 32 rows x 64 experts, 4 per thread and pass
        const int o = tid + h * kRouterThreads, k = o >> 4, e4 = (o & 15) * 4;
        float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k0 + k < d) {
          const float* src = Wr + size_t(k0 + k) * E + eb + e4;
          if ((E & 3) == 0 && eb + e4 + 3 < E) {
            w = *reinterpret_cast<const float4*>(src);
          } else {
            if (eb + e4 + 0 < E) w.x = src[0];
            if (eb + e4 + 1 < E) w.y = src[1];
            if (eb + e4 + 2 < E) w.z = src[2];
            if (eb + e4 + 3 < E) w.w = src[3];
          }
        }
        *reinterpret_cast<float4*>(&Ws[k][e4]) = w;
      }
      __syncthreads();
#pragma unroll 8
      for (int k = 0; k < kRtK; ++k) {
        const float4 a = *reinterpret_cast<const float4*>(&Xs[k][ty * 4]);
        const float4 b = *reinterpret_cast<const float4*>(&Ws[k][tx * 4]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = ty * 4 + i;
      if (m >= M) continue;
      float* sr = s_row(m);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = eb + tx * 4 + j;
        if (e < E) sr[e] = acc[i][j] + (br ? br[e] : 0.f);
      }
    }
  }
  __syncthreads();  // s of every token is written (global memory, this CTA)

  // ---- per token (one warp each): the RMS of relu(s) over the E experts and the active bits
  for (int m = warp; m < M; m += kRouterThreads / 32) {
    const float* sr = s_row(m);
    float sumsq = 0.f, sum = 0.f;
    for (int ww = 0; ww < nW; ++ww) {
      const int e = ww * 32 + lane;
      const float sv = e < E ? sr[e] : -1.f;
      const float a = fmaxf(sv, 0.f);
      sumsq = fmaf(a, a, sumsq);
      sum += a;
      const uint32_t bits = __ballot_sync(0xffffffffu, sv > 0.f);
      if (lane == 0) maskw[m][ww] = bits;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    if (lane == 0) rms[m] = router_norm(p.sum_norm, sum, sumsq, E);  // the normaliser: RMS or sum
  }
  __syncthreads();
  // ---- per chunk (one warp each): the union, ascending (lane w holds word w of the OR of the masks)
  for (int j = warp; j < nchunks; j += kRouterThreads / 32) {
    const int c = router_chunk(p, blockIdx.x, j);
    uint32_t u = 0;
    int tok_active = 0;
    if (lane < nW)
      for (int t = 0; t < L; ++t) {
        const uint32_t mw = maskw[j * L + t][lane];
        u |= mw;
        tok_active += __popc(mw);
      }
    const int cnt = __popc(u);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - cnt;
    uint32_t rest = u;
    int32_t* out = p.active_idx + size_t(c) * E;
    while (rest) {
      const int b = __ffs(rest) - 1;
      rest &= rest - 1;
      out[pos++] = lane * 32 + b;
    }
    int act_sum = tok_active;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) act_sum += __shfl_xor_sync(0xffffffffu, act_sum, o);
    if (lane == 0) {
      p.n_active[c] = total;
      if (p.counts) {
        p.counts[2 * c] = L * E - act_sum;
        p.counts[2 * c + 1] = E - total;
      }
    }
    if (p.tok_mask)
      for (int o = lane; o < L * nW; o += 32) p.tok_mask[size_t(c) * L * nW + o] = maskw[j * L + o / nW][o % nW];
  }
  // ---- r = g relu(s) / rms over s (0 for a token with no active expert); each thread its own elements
  for (int o = tid; o < M * E; o += kRouterThreads) {
    const int m = o / E, e = o - m * E;
    float* sr = s_row(m);
    const float rm = rms[m];
    sr[e] = rm > 0.f ? (g[e] * fmaxf(sr[e], 0.f)) / rm : 0.f;
  }
}

// ===================================================================================== expert kernel
struct Smem {
  uint8_t* xbuf;        // x of the current chunk: [nKc][8 rows][128 B], 128-byte swizzled
  uint8_t* ring;        // S slots
  uint64_t* fullW;      // [S] the stage's tiles landed (weights; and h for down-projection stages)
  uint64_t* empty;      // [S] every consumer warp is done with the slot (NCW arrivals)
  uint64_t* xfull;      // x of the chunk landed
  uint64_t* xfree;      // every consumer warp is done with x (NCW arrivals)
  volatile int* abort_flag;
};

__device__ __forceinline__ bool aborted(const Smem& sm) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void*)sm.abort_flag)) : "memory");
  return v != 0;
}
__device__ __forceinline__ void set_abort(const Smem& sm) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_u32((const void*)sm.abort_flag)), "r"(1u) : "memory");
}
// The first error of a launch keeps its record: err_info = where (bits 0-7) | CTA (bits 8-15) | ring
// stage index, low 16 bits (bits 16-31).
__device__ __forceinline__ void set_error(const Params& p, const Smem& sm, uint32_t bit, uint32_t info) {
  if (atomicOr(&p.hdr->err, bit) == 0u) p.hdr->err_info = info;
  set_abort(sm);
}
__device__ __forceinline__ uint32_t site(uint32_t where, int stage) {
  return where | (uint32_t(blockIdx.x & 255) << 8) | (uint32_t(stage) << 16);
}

// A bounded wait: on timeout it records the error and marks the CTA aborted; once the CTA is aborted,
// waits fail at once (every role then skips its work and the CTA can finish).
__device__ __noinline__ bool wait_slow(const Params& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                       uint32_t where) {
  if (aborted(sm)) return false;
  if (mbar_wait_slow(bar, parity, kWaitNs)) return true;
  if ((threadIdx.x & 31) == 0) set_error(p, sm, kErrRingWait, where);
  set_abort(sm);
  return false;
}
__device__ __forceinline__ bool wait(const Params& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                     uint32_t where) {
  if (mbar_try_wait(bar, parity) && !aborted(sm)) return true;
  return wait_slow(p, sm, bar, parity, where);
}

struct RingPos {
  int i = 0, slot = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int S) {
    ++i;
    if (++slot == S) slot = 0, ph ^= 1u;
  }
};

// This CTA's share of one chunk.
struct Work {
  int c;            // chunk
  int eb;           // first row of the chunk's layer in the stacked expert dimension (layer E)
  int n_act;
  int rA0, rA1;     // up-projection rows, flattened over (active expert position, j)
  int rB0, nB;      // down-projection: y rows [rB0, rB0 + nB)
};
__device__ __forceinline__ Work make_work(const Params& p, int c, int gi) {
  Work w;
  w.c = c;
  const int layer = layer_of(p, c);
  w.eb = layer_ok(p, layer) ? layer * p.E : 0;
  w.n_act = layer_ok(p, layer) ? __ldg(p.n_active + c) : 0;
  const long long R8 = (long long)w.n_act * p.de / 8;
  w.rA0 = int(R8 * gi / p.T) * 8;
  w.rA1 = int(R8 * (gi + 1) / p.T) * 8;
  const long long D8 = p.d / 8;
  w.rB0 = int(D8 * gi / p.T) * 8;
  w.nB = int(D8 * (gi + 1) / p.T) * 8 - w.rB0;
  return w;
}

// Up-projection group starting at flattened row r: rows [j0, j0 + rows) of active expert position a.
struct Group {
  int a, j0, rows;
};
__device__ __forceinline__ Group group_at(const Params& p, int r, int r_end) {
  Group g;
  g.a = r / p.de;
  g.j0 = r - g.a * p.de;
  g.rows = min(kGroupRows, min(p.de - g.j0, r_end - r));
  return g;
}
// 64-column chunks of d per up-projection stage of a group of `rows` rows: about kStageA bytes, so that
// a short group (a CTA's rows often start or end a few rows into an expert) still moves its weights in
// a few large stages rather than many small ones.
__device__ __forceinline__ int chunks_per_stage(const Params& p, int rows) { return chunks_per_stage_a(rows, p.nKc); }
__device__ __forceinline__ int stages_of_group(const Params& p, int rows) {
  const int ks = chunks_per_stage(p, rows);
  return (p.nKc + ks - 1) / ks;
}
__device__ __forceinline__ int stages_b_per_expert(const Params& p) { return (p.nJc + p.KWB - 1) / p.KWB; }
__device__ __forceinline__ int stages_a(const Params& p, const Work& w) {
  int n = 0;
  for (int r = w.rA0; r < w.rA1;) {
    const int rows = group_at(p, r, w.rA1).rows;
    n += stages_of_group(p, rows);
    r += rows;
  }
  return n;
}

// Box `bi` of the split of `rows` (a multiple of 8, at most 256) into tensor boxes of 128, 128, 64, 32,
// 16 and 8 rows: its row offset and map index (height 8 << k).  False past the last box.
__device__ __forceinline__ bool box_of(int rows, int bi, int* ro, int* k) {
  int off = 0, n = 0;
  for (int q = 0; q < 2 && rows - off >= 128; ++q) {
    if (n++ == bi) { *ro = off, *k = 4; return true; }
    off += 128;
  }
  for (int kk = 3; kk >= 0; --kk) {
    const int hh = 8 << kk;
    if (rows - off >= hh) {
      if (n++ == bi) { *ro = off, *k = kk; return true; }
      off += hh;
    }
  }
  return false;
}
__device__ __forceinline__ int boxes_of(int rows) {
  int n = 0, ro, k;
  while (box_of(rows, n, &ro, &k)) ++n;
  return n;
}

__device__ __forceinline__ uint8_t* h_image(const Params& p, int team, int i) {
  return p.h + (size_t(team) * kHImagesPerTeam + (i % kHImagesPerTeam)) * size_t(p.E) * p.nJc * kHTile;
}

// ------------------------------------------------------------------------------------- producers
// Every role walks the same schedule of the team's chunks i = 0 .. n-1 (chunk team + i teams):
//   A(0), A(1), B(0), A(2), B(1), ..., A(n-1), B(n-2), B(n-1)
// (step s runs A(s), then B(s-1)).  The down-projection of a chunk thus comes one up-projection
// later than the chunk's own up-projection, so the team barrier that publishes its h has a whole
// phase of slack and the ring of weight stages never waits on it.  h images: four per team, chunk i
// using image i % kHImagesPerTeam = 4 (a CTA may write h of chunk i + 1 while another still reads h
// of chunk i - 2).

__device__ __forceinline__ int team_chunks(const Params& p, int team) {
  return team < p.C ? (p.C - team + p.teams - 1) / p.teams : 0;
}

// Weight copy warp: W1 of the up-projection groups and W2 of the down-projection stages, in schedule
// order.  Lane q issues box q of a stage (at most 16).  Returns the number of stages issued.
__device__ int produce_w(const Params& p, const Maps& tm, const Smem& sm, int team, int gi) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_first();  // weights stream through once
  RingPos rp;
  const int nsB = stages_b_per_expert(p), n = team_chunks(p, team);
  bool ok = true;
  for (int st_i = 0; st_i <= n && ok; ++st_i) {
    if (st_i < n) {  // A(st_i)
      const int c = team + st_i * p.teams;
      const Work w = make_work(p, c, gi);
      for (int r = w.rA0; r < w.rA1 && ok;) {
        const Group g = group_at(p, r, w.rA1);
        const int e = w.eb + __ldg(p.active_idx + size_t(c) * p.E + g.a);
        const int nb = boxes_of(g.rows);
        const int KS = chunks_per_stage(p, g.rows), nsA = stages_of_group(p, g.rows);
        for (int ks = 0; ks < nsA; ++ks, rp.next(p.S)) {
          if (rp.i >= p.S && !wait(p, sm, &sm.empty[rp.slot], rp.ph ^ 1u, site(1, rp.i))) { ok = false; break; }
          const int nc = min(KS, p.nKc - ks * KS);
          uint8_t* st = sm.ring + size_t(rp.slot) * p.slot_bytes;
          if (ks * KS + nc <= p.nKf) {  // one box of the chunked view (chunks past the last read as zeros)
            if (lane == 0) {
              mbar_arrive_expect_tx(&sm.fullW[rp.slot], uint32_t(KS * g.rows * 128));
              tma_load_4d(st, &tm.w1c[(g.rows >> 3) - 1], 0, g.j0, ks * KS, e, &sm.fullW[rp.slot], pol);
            }
          } else {  // the stage holds the ragged last chunk of d: per-chunk boxes of the plain view
            if (lane == 0) mbar_arrive_expect_tx(&sm.fullW[rp.slot], uint32_t(nc * g.rows * 128));
            __syncwarp();
            int ro, k;
            if (lane < nc * nb && box_of(g.rows, lane % nb, &ro, &k)) {
              const int cc = lane / nb;
              tma_load_3d(st + (cc * g.rows + ro) * 128, &tm.w1[k], (ks * KS + cc) * 64, g.j0 + ro, e,
                          &sm.fullW[rp.slot], pol);
            }
          }
          __syncwarp();
        }
        r += g.rows;
      }
    }
    if (st_i >= 1 && ok) {  // B(st_i - 1)
      const int i = st_i - 1, c = team + i * p.teams;
      const Work w = make_work(p, c, gi);
      if (w.nB > 0 && w.n_act > 0) {
        {  // every CTA of the team has published its h of chunk i (normally long since: a phase of slack)
          const uint64_t t0 = globaltimer_ns();
          bool passed = true;
          while (ld_acquire_gpu(&p.chunk_bar[c]) < uint32_t(p.T)) {
            if (aborted(sm) || globaltimer_ns() - t0 > kWaitNs) { passed = false; break; }
            __nanosleep(64);
          }
          passed = __all_sync(0xffffffffu, passed);
          if (!passed) {
            if (lane == 0 && !aborted(sm)) set_error(p, sm, kErrTeamBarrier, site(11, i));
            return rp.i;
          }
          fence_proxy_async_global();  // h was written with generic stores; the bulk copies read it
        }
        const uint8_t* himg = h_image(p, team, i);
        const int nb = boxes_of(w.nB), rp16 = round16(w.nB);
        for (int a = 0; a < w.n_act && ok; ++a) {
          const int e = w.eb + __ldg(p.active_idx + size_t(c) * p.E + a);
          for (int jb = 0; jb < nsB; ++jb, rp.next(p.S)) {
            if (rp.i >= p.S && !wait(p, sm, &sm.empty[rp.slot], rp.ph ^ 1u, site(2, rp.i))) { ok = false; break; }
            const int nc = min(p.KWB, p.nJc - jb * p.KWB);
            uint8_t* st = sm.ring + size_t(rp.slot) * p.slot_bytes;
            const uint32_t hbytes = uint32_t(nc * kHTile);
            const bool chunked = jb * p.KWB + nc <= p.nJf;
            if (lane == 0) {
              mbar_arrive_expect_tx(&sm.fullW[rp.slot], uint32_t((chunked ? p.KWB : nc) * w.nB * 128) + hbytes);
              // the h tiles of the stage: one bulk copy of nc tiles after the W2 rows
              bulk_g2s(st + size_t(p.KWB) * rp16 * 128, himg + (size_t(a) * p.nJc + jb * p.KWB) * kHTile, hbytes,
                       &sm.fullW[rp.slot], pol);
              // one box of the chunked view (chunks past the last read as zeros)
              if (chunked)
                tma_load_4d(st, &tm.w2c[w.nB == p.hB[0] ? 0 : 1], 0, w.rB0, jb * p.KWB, e, &sm.fullW[rp.slot], pol);
            }
            __syncwarp();
            int ro, k;  // the stage holds the ragged last chunk of de: per-chunk boxes of the plain view
            if (!chunked && lane < nc * nb && box_of(w.nB, lane % nb, &ro, &k)) {
              const int cc = lane / nb;
              tma_load_3d(st + (cc * w.nB + ro) * 128, &tm.w2[k], (jb * p.KWB + cc) * 64, w.rB0 + ro, e,
                          &sm.fullW[rp.slot], pol);
            }
            __syncwarp();
          }
        }
      }
    }
  }
  return rp.i;
}

// x copy warp: x of each chunk into xbuf once the consumers are done with the previous chunk's.
// Returns the number of x loads issued.
__device__ int produce_x(const Params& p, const Maps& tm, const Smem& sm, int team) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_first();
  int i = 0;
  for (int c = team; c < p.C; ++i, c += p.teams) {
    if (i > 0 && !wait(p, sm, sm.xfree, uint32_t(i - 1) & 1u, site(4, i))) break;
    if (lane == 0) mbar_arrive_expect_tx(sm.xfull, uint32_t(p.nKc) * 1024);
    __syncwarp();
    for (int k = lane; k < p.nKc; k += 32) tma_load_3d(sm.xbuf + k * 1024, &tm.x, k * 64, 0, c, sm.xfull, pol);
    __syncwarp();
  }
  return i;
}

// ------------------------------------------------------------------------------------- consumers
// Every CTA of the team has published its h of chunk c (lane 0 polls, bounded; the whole warp gets the
// answer).
__device__ __noinline__ bool team_passed(const Params& p, const Smem& sm, int c) {
  const int lane = threadIdx.x & 31;
  bool ok = true;
  if (lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(&p.chunk_bar[c]) < uint32_t(p.T)) {
      if (aborted(sm)) { ok = false; break; }
      if (globaltimer_ns() - t0 > kWaitNs) {
        set_error(p, sm, kErrTeamBarrier, site(12, c));
        ok = false;
        break;
      }
      __nanosleep(64);
    }
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ void prefetch_l1(const void* ptr) { asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr)); }

// The lines of chunk c's metadata that this CTA reads (n_active, the union list, r) into L1 ahead of use.
__device__ __forceinline__ void prefetch_chunk(const Params& p, int c, int lane) {
  if (c >= p.C) return;
  const int act_lines = (p.E * 4 + 127) / 128, r_lines = (p.L * p.E * 4 + 127) / 128;
  if (lane == 0) prefetch_l1(p.n_active + c);
  for (int q = lane; q < act_lines + r_lines; q += 32)
    prefetch_l1(q < act_lines ? reinterpret_cast<const char*>(p.active_idx + size_t(c) * p.E) + q * 128
                              : reinterpret_cast<const char*>(p.r + size_t(c) * p.L * p.E) + (q - act_lines) * 128);
}

__device__ void consume(const Params& p, const Smem& sm, int team, int gi) {
  const int cw = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const uint32_t xb = smem_u32(sm.xbuf);
  const int nsB = stages_b_per_expert(p);
  RingPos rp;
  // ldmatrix lane addressing: A (x4) rows lane & 15, k half lane >> 4; B (x2) rows lane & 7, k half (lane >> 3) & 1
  const int arow = lane & 15, ahalf = lane >> 4, brow = lane & 7, bhalf = (lane >> 3) & 1;
  const int n = team_chunks(p, team);
  if (cw == 0) prefetch_chunk(p, team, lane);
  for (int st_i = 0; st_i <= n; ++st_i) {
    if (cw == 0) prefetch_chunk(p, team + (st_i + 1) * p.teams, lane);  // the next step's chunk
   if (st_i < n) {
    // ---------------- up-projection of chunk i = st_i
    const int i = st_i, c = team + i * p.teams;
    const Work w = make_work(p, c, gi);
    uint8_t* himg = h_image(p, team, i);
    const bool xok = wait(p, sm, sm.xfull, uint32_t(i) & 1u, site(5, i));
    for (int r = w.rA0; r < w.rA1;) {
      const Group g = group_at(p, r, w.rA1);
      const int KS = chunks_per_stage(p, g.rows), nsA = stages_of_group(p, g.rows);
      const bool mine = 16 * cw < g.rows;
      // the router outputs this lane's epilogue needs, loaded now so that their latency overlaps the stages
      const int e = __ldg(p.active_idx + size_t(c) * p.E + g.a);
      float rr[2] = {0.f, 0.f};
      if (mine)
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (2 * tig + q < p.L) rr[q] = __ldg(p.r + (size_t(c) * p.L + 2 * tig + q) * p.E + e);
      float acc[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[k][v] = 0.f;
      for (int ks = 0; ks < nsA; ++ks, rp.next(p.S)) {
        const int slot = rp.slot;
        if (wait(p, sm, &sm.fullW[slot], rp.ph, site(6, rp.i)) && xok && mine) {
          const int nc = min(KS, p.nKc - ks * KS);
          const uint32_t sb = smem_u32(sm.ring + size_t(slot) * p.slot_bytes);
          for (int cc = 0; cc < nc; ++cc) {
            const uint32_t wbase = sb + cc * g.rows * 128, xbase = xb + (ks * KS + cc) * 1024;
            // all fragments of the 64-column chunk, then its four MMAs into four accumulators
            uint32_t a[4][4], b[4][2];
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16) {
              ldmatrix_x4(wbase + swz(16 * cw + arow, 2 * k16 + ahalf), a[k16][0], a[k16][1], a[k16][2], a[k16][3]);
              ldmatrix_x2(xbase + swz(brow, 2 * k16 + bhalf), b[k16][0], b[k16][1]);
            }
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16) mma_bf16_16816(acc[k16], a[k16], b[k16][0], b[k16][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
      }
      if (mine && !aborted(sm)) {
        // h = r Swish(u) for rows 16 cw + gid (+ 8) and tokens 2 tig (+ 1), into the h image as bf16 hi / lo
        uint8_t* ex = himg + size_t(g.a) * p.nJc * kHTile;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int row = 16 * cw + gid + (v >> 1) * 8, t = 2 * tig + (v & 1);
          if (row < g.rows && t < p.L) {
            const int j = g.j0 + row, col = j & 63;
            const float u = (acc[0][v] + acc[1][v]) + (acc[2][v] + acc[3][v]);
            const float hv = rr[v & 1] * (u / (1.f + expf(-u)));
            const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
            const __nv_bfloat16 lo = __float2bfloat16_rn(hv - __bfloat162float(hi));
            uint8_t* tile = ex + size_t(j >> 6) * kHTile;
            *reinterpret_cast<__nv_bfloat16*>(tile + swz(t, col >> 3) + (col & 7) * 2) = hi;
            *reinterpret_cast<__nv_bfloat16*>(tile + swz(8 + t, col >> 3) + (col & 7) * 2) = lo;
            // the columns past de of the expert's last tile face the zero columns the W2 boxes read
            // past de, but the image may hold any bytes there (0 * NaN is NaN): zero them
            if (j == p.de - 1)
              for (int c8 = (p.de & 63) >> 3; c8 != 0 && c8 < 8; ++c8) {
                *reinterpret_cast<uint4*>(tile + swz(t, c8)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(tile + swz(8 + t, c8)) = make_uint4(0, 0, 0, 0);
              }
          }
        }
      }
      r += g.rows;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.xfree);
    // publish this CTA's h of the chunk (every CTA arrives, also after an abort)
    __threadfence();
    named_bar_sync(1, NCW * 32);
    if (cw == 0 && lane == 0) {
      fence_proxy_async_global();
      red_release_gpu_add(&p.chunk_bar[c], 1u);
    }
   }
   if (st_i >= 1) {
    // ---------------- down-projection of chunk i = st_i - 1 (after an abort every warp still walks the
    // same stages and named barriers, skipping the work, so that no warp waits at a barrier another
    // warp has left)
    const int i = st_i - 1, c = team + i * p.teams;
    const Work w = make_work(p, c, gi);
    const bool has_b = w.nB > 0 && w.n_act > 0;
    // A CTA with down-projection stages learns that every CTA of the team published h of chunk i from
    // the h tiles (the copy warp waited for that before copying them); one without stages waits for the
    // chunk's counter itself, so that no CTA runs further ahead of the h images others still read than
    // the schedule allows.
    const bool tok = has_b || team_passed(p, sm, c);
    float acc[2][2][2][4];  // [m-tile][hi, lo][even, odd k16]
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[m][q][k][v] = 0.f;
    const int MB = (w.nB + 15) >> 4, rp16 = round16(w.nB);
    const bool m0 = cw < MB, m1 = cw + 8 < MB;
    if (w.nB > 0) {
      for (int a = 0; a < w.n_act; ++a) {
        for (int jb = 0; jb < nsB; ++jb, rp.next(p.S)) {
          const int slot = rp.slot;
          const bool okW = tok && wait(p, sm, &sm.fullW[slot], rp.ph, site(8, rp.i));
          if (okW && m0) {
            const int nc = min(p.KWB, p.nJc - jb * p.KWB);
            const uint32_t sb = smem_u32(sm.ring + size_t(slot) * p.slot_bytes);
            const uint32_t hb = sb + uint32_t(p.KWB * rp16 * 128);
            for (int cc = 0; cc < nc; ++cc) {
              const uint32_t wbase = sb + cc * w.nB * 128, hbase = hb + cc * kHTile;
              // all fragments of the 64-wide j chunk first, then the MMAs into the even / odd accumulators
              uint32_t bh[4][2], bl[4][2], a0[4][4];
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16) {
                ldmatrix_x2(hbase + swz(brow, 2 * k16 + bhalf), bh[k16][0], bh[k16][1]);
                ldmatrix_x2(hbase + swz(8 + brow, 2 * k16 + bhalf), bl[k16][0], bl[k16][1]);
                ldmatrix_x4(wbase + swz(16 * cw + arow, 2 * k16 + ahalf), a0[k16][0], a0[k16][1], a0[k16][2],
                            a0[k16][3]);
              }
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16) {
                mma_bf16_16816(acc[0][0][k16 & 1], a0[k16], bh[k16][0], bh[k16][1]);
                mma_bf16_16816(acc[0][1][k16 & 1], a0[k16], bl[k16][0], bl[k16][1]);
              }
              if (m1) {
                uint32_t a1[4][4];
#pragma unroll
                for (int k16 = 0; k16 < 4; ++k16)
                  ldmatrix_x4(wbase + swz(16 * (cw + 8) + arow, 2 * k16 + ahalf), a1[k16][0], a1[k16][1], a1[k16][2],
                              a1[k16][3]);
#pragma unroll
                for (int k16 = 0; k16 < 4; ++k16) {
                  mma_bf16_16816(acc[1][0][k16 & 1], a1[k16], bh[k16][0], bh[k16][1]);
                  mma_bf16_16816(acc[1][1][k16 & 1], a1[k16], bl[k16][0], bl[k16][1]);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
      }
      float* yc = p.y + size_t(c) * p.L * p.d + w.rB0;
      const bool ok = tok && !aborted(sm);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (!ok || !(m == 0 ? m0 : m1)) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int row = 16 * (cw + 8 * m) + gid + (v >> 1) * 8, t = 2 * tig + (v & 1);
          if (row < w.nB && t < p.L)
            yc[size_t(t) * p.d + row] = (acc[m][0][0][v] + acc[m][0][1][v]) + (acc[m][1][0][v] + acc[m][1][1][v]);
        }
      }
    }
   }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    batch_expert_kernel(const __grid_constant__ Params p, const __grid_constant__ Maps tm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem sm;
  sm.xbuf = base;
  sm.ring = base + p.xbuf_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm.ring + size_t(p.S) * p.slot_bytes);
  sm.fullW = bars;
  sm.empty = bars + p.S;
  sm.xfull = bars + 2 * p.S;
  sm.xfree = sm.xfull + 1;
  sm.abort_flag = reinterpret_cast<volatile int*>(sm.xfull + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&sm.fullW[s], 1);
      mbar_init(&sm.empty[s], NCW);
    }
    mbar_init(sm.xfull, 1);
    mbar_init(sm.xfree, NCW);
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
  __syncthreads();
  // everything below reads what the router kernel wrote (union, r, the zeroed team counters)
  pdl_wait();
  const int team = blockIdx.x / p.T, gi = blockIdx.x - team * p.T;
  int issuedW = 0, issuedX = 0;
  if (warp < NCW) {
    consume(p, sm, team, gi);
  } else if (warp == kWarpW) {
    issuedW = produce_w(p, tm, sm, team, gi);
  } else {
    issuedX = produce_x(p, tm, sm, team);
  }
  __syncthreads();
  if (aborted(sm) && lane == 0) {  // no copy into this CTA's shared memory may be in flight when it leaves
    if (warp == kWarpW)
      for (int k = max(0, issuedW - p.S); k < issuedW; ++k)
        mbar_wait_bounded(&sm.fullW[k % p.S], uint32_t(k / p.S) & 1u, kWaitNs / 10);
    if (warp == kWarpX && issuedX > 0) mbar_wait_bounded(sm.xfull, uint32_t(issuedX - 1) & 1u, kWaitNs / 10);
  }
}

}  // namespace

// ===================================================================================== host side
bool plan(int C, int L, int d, int E, int de, int teams, int num_sms, int max_smem, Params* p, Launch* out) {
  if (C < 1 || L < 1 || L > kMaxL || d % 8 != 0 || de % 8 != 0 || E < 1 || E > kMaxE) return false;
  if (teams < 1 || teams > kMaxTeams || teams > num_sms) return false;
  const int T = num_sms / teams;
  const int nB_max = ((d / 8 + T - 1) / T) * 8;
  if (nB_max > kMaxRowsB) return false;
  p->teams = teams;
  p->T = T;
  p->nKc = (d + 63) / 64;
  p->nJc = (de + 63) / 64;
  p->nKf = d / 64;
  p->nJf = de / 64;
  p->hB[0] = 8 * ((d / 8) / T);
  p->hB[1] = p->hB[0] + 8;
  p->xbuf_bytes = p->nKc * 1024;
  if (p->xbuf_bytes > 96 * 1024) return false;
  const int rp16 = (nB_max + 15) & ~15;
  const int bchunk = rp16 * 128 + kHTile;
  int kwb = (36 * 1024) / bchunk;
  if (kwb < 1) kwb = 1;
  if (kwb > p->nJc) kwb = p->nJc;
  p->KWB = kwb;
  const int stage_a = kStageA;  // an up-projection stage holds at most kStageA bytes
  int slot = stage_a > kwb * bchunk ? stage_a : kwb * bchunk;
  slot = (slot + 1023) & ~1023;
  p->slot_bytes = slot;
  const size_t fixed = 1024 + 256;  // alignment slack; barriers and the abort flag
  long long S = ((long long)max_smem - (long long)fixed - p->xbuf_bytes) / slot;
  if (S > 8) S = 8;
  if (S < 2) return false;
  p->S = int(S);
  out->grid = teams * T;
  out->smem = fixed + size_t(p->xbuf_bytes) + size_t(p->S) * slot;
  return true;
}

cudaError_t occupancy(size_t smem, int* ctas_per_sm) {
  cudaError_t err = cudaFuncSetAttribute(batch_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, batch_expert_kernel, kThreads, smem);
}

cudaError_t launch_router(const Params& p, cudaStream_t st) {
  // router CTAs: one per chunk with a layer array, else ceil(chunks of a layer / G) per layer
  int ctas = p.C;
  if (!p.layer) {
    const int G = kRouterTokens / p.L < 1 ? 1 : kRouterTokens / p.L;
    const int per_layer = (p.C + p.n_layers - 1) / p.n_layers;
    ctas = p.n_layers * ((per_layer + G - 1) / G);
  }
  batch_router_kernel<<<ctas, kRouterThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch(const Params& p, const Maps& m, const Launch& plan, cudaStream_t st) {
  cudaError_t err;
  if ((err = launch_router(p, st)) != cudaSuccess) return err;
  err = cudaFuncSetAttribute(batch_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
  if (err != cudaSuccess) return err;
  // programmatic dependent launch: the expert kernel's set-up overlaps the router kernel's tail; it
  // reads the router's outputs only after griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, batch_expert_kernel, p, m);
}

}  // namespace batch
}  // namespace bffn
