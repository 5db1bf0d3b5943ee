// Prefill variant of the BlockFFN chunk layer (L in the hundreds to thousands of tokens).
//
// At this size the layer is a dense contraction per expert, so it runs as grouped GEMMs on the
// tcgen05 tensor cores (lsdiaocha.cn BlockFFN article, sections 2 and 4: the same router and experts;
// the tokens of the chunk are grouped per active expert instead of evaluated as one batch):
//   P1 router       x Wr on the warp tensor cores with Wr as bf16 hi + lo pairs (cls_losses.cu): the
//                   error, at most 2^-18 sum_k |x_k Wr_k| plus fp32 rounding, stays below the 1e-3 margin
//                   of the workloads' pre-activations, so the mask decisions match fp32 and fp64
//   P2 stats        per token: RMS of relu(s), active bits, optional r and masks
//   P3 grouping     per expert: its tokens in ascending order with r_{t,e}, 128-row tiles
//   P4 GEMM1        per (expert, 128-token tile): U = X[T_e] W1_e^T on tcgen05 (the A rows gathered by
//                   four loader warps with coalesced cp.async), h = r Swish(U) split into bf16 hi + lo parts
//   P5 GEMM2        per (expert tile, 256 columns of d): Y[T_e] += (H_hi + H_lo) W2_e^T on tcgen05,
//                   added into y with vector reductions
#include <cuda_bf16.h>

#include "blockffn_internal.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace bffn {
namespace {

constexpr uint64_t kPWaitNs = 2000000000ull;

// ---------------------------------------------------------------------------------- P2 stats
// One warp per token: RMS over the E router entries of relu(s), the active bits, r if asked for.
__global__ void __launch_bounds__(256) prefill_stats_kernel(PrefillParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int t = warp;
  if (t >= p.L) return;
  float* st = p.s + size_t(t) * p.E;
  for (int e = lane; e < p.E; e += 32) {  // s = the projection's parts in order, plus the bias
    float v = 0.f;
    for (int k = 0; k < p.ksplit; ++k) v += p.s_part[(size_t(k) * p.L + t) * p.E + e];
    st[e] = v + (p.br ? p.br[e] : 0.f);
  }
  __syncwarp();
  float sumsq = 0.f, sum = 0.f;
  int n_pos = 0;
  for (int w = 0; w < p.W; ++w) {
    const int e = w * 32 + lane;
    const float sv = e < p.E ? st[e] : -1.f;
    const float a = fmaxf(sv, 0.f);
    sumsq = fmaf(a, a, sumsq);
    sum += a;
    const uint32_t bits = __ballot_sync(0xffffffffu, sv > 0.f);
    if (lane == 0) {
      p.mask[size_t(t) * p.W + w] = bits;
      if (p.tok_mask) p.tok_mask[size_t(t) * p.W + w] = bits;
    }
    n_pos += __popc(bits);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  const float rms = router_norm(p.sum_norm, sum, sumsq, p.E);  // the normaliser: RMS or sum
  if (lane == 0) {
    p.rms[t] = rms;
    atomicAdd(p.n_pos, n_pos);  // an integer sum: the same in any order
  }
  if (p.r_out)
    for (int e = lane; e < p.E; e += 32)
      p.r_out[size_t(t) * p.E + e] = rms > 0.f ? (p.g[e] * fmaxf(st[e], 0.f)) / rms : 0.f;
}

// ---------------------------------------------------------------------------------- P3 grouping
__device__ __forceinline__ bool active_bit(const PrefillParams& p, int t, int e) {
  return t < p.L && ((p.mask[size_t(t) * p.W + (e >> 5)] >> (e & 31)) & 1u);
}

// Tokens [t0, t1) of warp w when 8 warps split L tokens into 32-token groups.
__device__ __forceinline__ void warp_token_range(int L, int w, int* t0, int* t1) {
  const int groups = (L + 31) / 32, per = (groups + 7) / 8;
  *t0 = min(L, w * per * 32);
  *t1 = min(L, (w + 1) * per * 32);
}

// One CTA per expert: the number of its tokens (8 warps count a share each).
__global__ void __launch_bounds__(256) prefill_count_kernel(PrefillParams p) {
  __shared__ int wc[8];
  const int e = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int t0, t1;
  warp_token_range(p.L, warp, &t0, &t1);
  int n = 0;
#pragma unroll 4
  for (int t = t0; t < t1; t += 32) n += __popc(__ballot_sync(0xffffffffu, active_bit(p, t + lane, e)));
  if (lane == 0) wc[warp] = n;
  __syncthreads();
  if (threadIdx.x == 0) p.cnt[e] = wc[0] + wc[1] + wc[2] + wc[3] + wc[4] + wc[5] + wc[6] + wc[7];
}

// Pair and tile offsets of every expert, the union (active experts ascending), n_active and the
// counts: one warp.
__global__ void __launch_bounds__(32) prefill_scan_kernel(PrefillParams p) {
  const int lane = threadIdx.x;
  int pairs = 0, tiles = 0, nact = 0;
  for (int e0 = 0; e0 < p.E; e0 += 32) {
    const int ee = e0 + lane;
    const int c = ee < p.E ? p.cnt[ee] : 0;
    const int mt = (c + 127) >> 7;
    int ic = c, im = mt, ia = c > 0 ? 1 : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xffffffffu, ic, o), vm = __shfl_up_sync(0xffffffffu, im, o),
                va = __shfl_up_sync(0xffffffffu, ia, o);
      if (lane >= o) ic += vc, im += vm, ia += va;
    }
    if (ee < p.E) {
      p.off[ee] = pairs + ic - c;
      p.toff[ee] = tiles + im - mt;
      if (c > 0) p.active_idx[nact + ia - 1] = ee;
    }
    pairs += __shfl_sync(0xffffffffu, ic, 31);
    tiles += __shfl_sync(0xffffffffu, im, 31);
    nact += __shfl_sync(0xffffffffu, ia, 31);
  }
  if (lane == 0) {
    p.off[p.E] = pairs;
    p.toff[p.E] = tiles;
    *p.n_active = nact;
    if (p.counts) {
      p.counts[0] = p.L * p.E - *p.n_pos;
      p.counts[1] = p.E - nact;
    }
  }
}

// One CTA per expert: its token list (ascending) and r values at its pair offset.  8 warps take a
// share of the tokens each; a warp's position is the expert's offset plus the lower warps' counts.
__global__ void __launch_bounds__(256) prefill_fill_kernel(PrefillParams p) {
  __shared__ int wc[8];
  const int e = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int t0, t1;
  warp_token_range(p.L, warp, &t0, &t1);
  int n = 0;
#pragma unroll 4
  for (int t = t0; t < t1; t += 32) n += __popc(__ballot_sync(0xffffffffu, active_bit(p, t + lane, e)));
  if (lane == 0) wc[warp] = n;
  __syncthreads();
  int base = p.off[e];
  for (int w = 0; w < warp; ++w) base += wc[w];
  const float ge = p.g[e];
  for (int t = t0; t < t1; t += 32) {
    const int tt = t + lane;
    const bool on = active_bit(p, tt, e);
    const uint32_t b = __ballot_sync(0xffffffffu, on);
    if (on) {
      const int pos = base + __popc(b & ((1u << lane) - 1u));
      p.tok[pos] = tt;
      p.rv[pos] = (ge * p.s[size_t(tt) * p.E + e]) / p.rms[tt];  // s > 0, so relu(s) = s and rms > 0
    }
    base += __popc(b);
  }
}

}  // namespace

namespace {

// ---------------------------------------------------------------------------------- P4/P5 GEMMs
constexpr int kG1Threads = 320;  // GEMM1: warp 0 TMA producer, warp 1 MMA issuer (owns TMEM), warps 2-5
                                 // epilogue, warps 6-9 the gathered A rows (one token row per thread)
constexpr int kG2EpWarps = 8;    // GEMM2 epilogue warps: a multiple of 4 (each lane quarter gets kG2EpWarps / 4)
constexpr int kG2Threads = 64 + 32 * kG2EpWarps;  // GEMM2: warps 0, 1 as in GEMM1, then the epilogue
constexpr int kTileM = 128;
constexpr int kPf1 = 12;  // GEMM1: W1 rows are prefetched into L2 this many stages ahead
constexpr int kEpBlock = 32 * 32;  // GEMM2 epilogue: a warp's 32 x 32 fp32 block, 16-byte pieces swizzled by row

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// y[0..3] += v, a reduction performed at L2; the line is marked to stay in L2 (y takes every pair's
// contribution while W2 streams past).
__device__ __forceinline__ void red_add_v4(float* y, float a, float b, float c, float d, uint64_t policy) {
  asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(y), "f"(a), "f"(b), "f"(c),
               "f"(d), "l"(policy)
               : "memory");
}

struct GemmSmem {
  uint8_t* stages;
  uint64_t* full;   // [S] operands of a stage landed
  uint64_t* empty;  // [S] MMAs of a stage done reading it
  uint64_t* accf;   // [2] accumulator buffer complete
  uint64_t* acce;   // [2] accumulator buffer drained by the epilogue warps
  uint64_t* drain;  // every MMA of this CTA complete (before TMEM is freed)
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  int* toff;        // [E+1] copies of the per-expert tile offsets, pair offsets and token counts
  int* off;         // [E+1]
  int* cnt;         // [E]
  float* ep_buf;    // GEMM2: per epilogue warp a 32 x 32 fp32 block (kEpBlock floats)
};

__device__ __forceinline__ GemmSmem carve(uint8_t* raw, int S, uint32_t stage_bytes, int E) {
  GemmSmem g;
  g.stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  g.full = reinterpret_cast<uint64_t*>(g.stages + size_t(S) * stage_bytes);
  g.empty = g.full + S;
  g.accf = g.empty + S;
  g.acce = g.accf + 2;
  g.drain = g.acce + 2;
  g.tmem_slot = reinterpret_cast<uint32_t*>(g.drain + 1);
  g.abort_flag = reinterpret_cast<volatile int*>(g.tmem_slot + 1);
  g.toff = reinterpret_cast<int*>(g.tmem_slot + 4);
  g.off = g.toff + (E + 1);
  g.cnt = g.off + (E + 1);
  g.ep_buf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(g.cnt + E) + 15) & ~uintptr_t(15));
  return g;
}

__device__ __forceinline__ bool g_aborted(const GemmSmem& g) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void*)g.abort_flag)) : "memory");
  return v != 0;
}

// A bounded wait; on timeout the CTA records the error and stops (every role then skips its work).
__device__ __noinline__ bool g_wait_slow(const PrefillParams& p, const GemmSmem& g, uint64_t* bar, uint32_t parity,
                                         uint32_t where) {
  if (g_aborted(g)) return false;
  if (mbar_wait_slow(bar, parity, kPWaitNs)) return true;
  if ((threadIdx.x & 31) == 0) {
    atomicOr(&p.hdr->err, kErrPrefillWait);
    p.hdr->err_info = where;
  }
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_u32((const void*)g.abort_flag)), "r"(1u) : "memory");
  return false;
}
__device__ __forceinline__ bool g_wait(const PrefillParams& p, const GemmSmem& g, uint64_t* bar, uint32_t parity,
                                       uint32_t where) {
  if (mbar_try_wait(bar, parity) && !g_aborted(g)) return true;
  return g_wait_slow(p, g, bar, parity, where);
}

struct Ring {
  int i = 0, slot = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int S) {
    ++i;
    if (++slot == S) slot = 0, ph ^= 1u;
  }
};

// The expert owning 128-row tile `tile`: the largest e with toff[e] <= tile (experts without tokens
// share their successor's offset, so the expert found has at least one tile).
__device__ __forceinline__ int tile_expert(const int32_t* toff, int E, int tile) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (toff[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// GEMM2 tile -> (N tile jn, expert e, 128-row tile of the expert).  The d / N column slices of y form
// groups of G; a group's tiles come before the next group's, expert-major inside it, and an expert's
// tiles in a group are N-tile-major.  So the CTAs working on one W2_e slice at a time share it in L2
// and it comes from HBM once; an expert's H rows repeat from L2 over the group's G slices; and the y
// elements the tiles add into are those of one group's columns (L x G N fp32, 32 MiB at L = 4096,
// G N = 2048), which stay in L2 through the ~E_t additions each takes.  H is read from HBM once per
// group.
struct Tile2 {
  int e, jn, m0;
};
__device__ __forceinline__ int slice_group(int NT) {
  int G = NT < 8 ? NT : 8;
  while (NT % G != 0) --G;
  return G;
}
__device__ __forceinline__ Tile2 tile2_at(const GemmSmem& g, int E, int NT, int tile) {
  const int G = slice_group(NT), T1 = g.toff[E];
  const int grp = tile / (T1 * G), rem = tile - grp * (T1 * G);
  Tile2 t;
  t.e = tile_expert(g.toff, E, rem / G);  // the expert's tiles in the group are [toff[e] G, toff[e+1] G)
  const int nm = g.toff[t.e + 1] - g.toff[t.e];
  const int li = rem - g.toff[t.e] * G;
  t.jn = grp * G + li / nm;
  t.m0 = (li - (li / nm) * nm) * kTileM;
  return t;
}

__device__ __forceinline__ uint32_t tmem_cols(int n) {
  uint32_t c = 32;
  while (c < uint32_t(2 * n)) c <<= 1;
  return c;
}

__device__ void gemm_setup(const PrefillParams& p, const GemmSmem& g, int S, int N, int full_count,
                           int epilogue_warps) {
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i <= p.E; i += blockDim.x) {  // the tables every tile lookup reads
    g.toff[i] = p.toff[i];
    g.off[i] = p.off[i];
    if (i < p.E) g.cnt[i] = p.cnt[i];
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&g.full[s], full_count);
      mbar_init(&g.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&g.accf[b], 1);
      mbar_init(&g.acce[b], epilogue_warps);
    }
    mbar_init(g.drain, 1);
    *g.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(g.tmem_slot, tmem_cols(N));
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
}

__device__ void gemm_teardown(const PrefillParams& p, const GemmSmem& g, int N) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 1) {  // every MMA issued by this CTA has completed before the columns are freed
    if (lane == 0) tc::commit(g.drain);
    __syncwarp();
    mbar_wait_bounded(g.drain, 0, kPWaitNs / 10);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(*g.tmem_slot, tmem_cols(N));
  (void)p;
}

// The producer's copies land before the CTA may exit.
__device__ void producer_drain(const GemmSmem& g, const Ring& rp, int S) {
  for (int k = rp.i - S > 0 ? rp.i - S : 0; k < rp.i; ++k)
    mbar_wait_bounded(&g.full[k % S], uint32_t(k / S) & 1u, kPWaitNs / 10);
}

// GEMM1: per tile of 128 pairs of expert e, U = X[tokens] W1_e^T (N = de), then h = r Swish(U) as
// bf16 hi and lo parts into H[pair][0, de) and H[pair][de, 2 de).
__global__ void __launch_bounds__(kG1Threads, 1)
    prefill_gemm1_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps m) {
  extern __shared__ uint8_t smem_raw[];
  const int N = p.N1, S = p.S1;
  const uint32_t a_bytes = kTileM * 128, stage_bytes = a_bytes + uint32_t(N) * 128;
  const GemmSmem g = carve(smem_raw, S, stage_bytes, p.E);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) prefetch_tensormap(&m.w1);
  gemm_setup(p, g, S, N, 1 + kTileM, 4);  // the W1 box (expect_tx) and one row-copy arrival per A row
  const uint32_t tmem = *g.tmem_slot;
  const int T = g.toff[p.E];
  const int KB = p.d / 64;

  if (warp == 0) {
    const uint64_t pol_w = policy_evict_first();  // W1 streams through once
    Ring rp;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
      const int e = tile_expert(g.toff, p.E, tile);
      for (int kb = 0; kb < KB; ++kb, rp.next(S)) {
        if (rp.i >= S && !g_wait(p, g, &g.empty[rp.slot], rp.ph ^ 1u, 21)) { ok = false; break; }
        uint8_t* st = g.stages + size_t(rp.slot) * stage_bytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&g.full[rp.slot], uint32_t(N) * 128);
          tma_load_2d(st + a_bytes, &m.w1, kb * 64, e * p.de, &g.full[rp.slot], pol_w);
        }
        __syncwarp();
      }
    }
    producer_drain(g, rp, S);
  } else if (warp >= 6) {
    // A rows: lanes 8q..8q+7 of a loader warp copy the eight 16-byte pieces of one token row (128
    // bytes: 64 bf16 of the K block), so a warp-wide copy covers 4 whole rows; loader warp w takes rows
    // 32w..32w+31 in 8 such steps.  Pieces land in the 128-byte-swizzled layout; a thread's arrival on
    // the stage barrier fires when its copies complete.
    const int lw = warp - 6, c = lane & 7, rq = lane >> 3;
    const int tpr = threadIdx.x - 6 * 32;  // W1 L2 prefetch: rows 2 tpr, 2 tpr + 1 of a future stage
    Ring rp;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
      const int e = tile_expert(g.toff, p.E, tile);
      const int m0 = (tile - g.toff[e]) * kTileM, ne = g.cnt[e];
      const __nv_bfloat16* src[8];
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int r = lw * 32 + it * 4 + rq;
        const int tok = p.tok[g.off[e] + m0 + (m0 + r < ne ? r : 0)];  // rows past the expert repeat row 0
        src[it] = p.x + size_t(tok) * p.d + c * 8;
      }
      const int tile_nx = tile + int(gridDim.x);
      const int e_nx = tile_nx < T ? tile_expert(g.toff, p.E, tile_nx) : -1;
      for (int kb = 0; kb < KB; ++kb, rp.next(S)) {
        if (rp.i >= S && !g_wait(p, g, &g.empty[rp.slot], rp.ph ^ 1u, 25)) { ok = false; break; }
        const uint32_t st = smem_u32(g.stages + size_t(rp.slot) * stage_bytes);
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int r = lw * 32 + it * 4 + rq;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(st + uint32_t(r * 128 + ((c ^ (r & 7)) << 4))),
                       "l"(src[it] + kb * 64)
                       : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&g.full[rp.slot]))
                     : "memory");
        // the W1 lines of the stage kPf1 ahead into L2
        const int kf = kb + kPf1;
        const int ef = kf < KB ? e : e_nx, kbf = kf < KB ? kf : kf - KB;
        if (ef >= 0 && kbf < KB)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (2 * tpr + h < N) prefetch_l2(p.W1 + (size_t(ef) * p.de + 2 * tpr + h) * p.d + kbf * 64);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // every row copy has landed before the CTA may exit
  } else if (warp == 1) {
    const uint32_t idesc = tc::idesc_bf16_f32(kTileM, N);
    Ring rp;
    int tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x, ++tcount) {
      const int ab = tcount & 1;
      if (tcount >= 2 && !g_wait(p, g, &g.acce[ab], uint32_t((tcount >> 1) - 1) & 1u, 22)) { ok = false; break; }
      tc::fence_after_sync();
      for (int kb = 0; kb < KB; ++kb, rp.next(S)) {
        if (!g_wait(p, g, &g.full[rp.slot], rp.ph, 23)) { ok = false; break; }
        tc::fence_after_sync();
        fence_proxy_async_smem();  // the A rows were written by ordinary (non-bulk) copies
        if (lane == 0) {
          const uint32_t sa = smem_u32(g.stages + size_t(rp.slot) * stage_bytes);
          const uint64_t ad = tc::smem_desc_k128(sa), bd = tc::smem_desc_k128(sa + a_bytes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16(tmem + uint32_t(ab * N), ad + 2 * k, bd + 2 * k, idesc, uint32_t(kb | k));
          tc::commit(&g.empty[rp.slot]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc::commit(&g.accf[ab]);
      __syncwarp();
    }
  } else {
    const int q = warp & 3;  // this warp's quarter of the tensor-memory lanes (rows)
    int tcount = 0;
    for (int tile = blockIdx.x; tile < T; tile += gridDim.x, ++tcount) {
      const int ab = tcount & 1;
      if (!g_wait(p, g, &g.accf[ab], uint32_t(tcount >> 1) & 1u, 24)) break;
      tc::fence_after_sync();
      const int e = tile_expert(g.toff, p.E, tile);
      const int m0 = (tile - g.toff[e]) * kTileM, ne = g.cnt[e];
      const int row = q * 32 + lane;
      const bool valid = m0 + row < ne;
      const size_t pair = size_t(g.off[e] + m0 + row);
      const float r = valid ? p.rv[pair] : 0.f;
      __nv_bfloat16* hrow = p.H + pair * size_t(2 * p.de);
      for (int c0 = 0; c0 < N; c0 += 32) {
        float v[32];
        tc::ld_32x32b_x32(tmem + (uint32_t(q * 32) << 16) + uint32_t(ab * N + c0), v);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = r * (v[2 * i] / (1.f + expf(-v[2 * i])));
          const float h1 = r * (v[2 * i + 1] / (1.f + expf(-v[2 * i + 1])));
          const __nv_bfloat162 hh = __floats2bfloat162_rn(h0, h1);
          const __nv_bfloat162 ll = __floats2bfloat162_rn(h0 - __low2float(hh), h1 - __high2float(hh));
          hi[i] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[i] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        if (valid) {
          uint4* dh = reinterpret_cast<uint4*>(hrow + c0);
          uint4* dl = reinterpret_cast<uint4*>(hrow + p.de + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            dh[k] = make_uint4(hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
            dl[k] = make_uint4(lo[4 * k], lo[4 * k + 1], lo[4 * k + 2], lo[4 * k + 3]);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&g.acce[ab]);
    }
  }
  gemm_teardown(p, g, N);
}

// GEMM2: per tile of 128 pairs of expert e and N2 columns of d, Y = H_hi W2_e^T + H_lo W2_e^T, added
// into y[token] with vector reductions (every pair's row goes to its token's row).
__global__ void __launch_bounds__(kG2Threads, 1)
    prefill_gemm2_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps m) {
  extern __shared__ uint8_t smem_raw[];
  const int N = p.N2, S = p.S2;
  const uint32_t a_bytes = kTileM * 128, stage_bytes = 2 * a_bytes + uint32_t(N) * 128;
  const GemmSmem g = carve(smem_raw, S, stage_bytes, p.E);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tensormap(&m.h);
    prefetch_tensormap(&m.w2);
  }
  gemm_setup(p, g, S, N, 1, kG2EpWarps);
  const uint32_t tmem = *g.tmem_slot;
  const int NT = p.d / N;
  const int T = g.toff[p.E] * NT;
  const int KB = p.de / 64;

  if (warp == 0) {
    const uint64_t pol_h = policy_evict_normal();  // an expert's H rows repeat over its N tiles, soon
    const uint64_t pol_w = policy_evict_normal();  // W2_e[jn] is read by every row tile of e, close together
    Ring rp;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x) {
      const Tile2 tl = tile2_at(g, p.E, NT, tile);
      const int e = tl.e, jn = tl.jn;
      const int row0 = g.off[e] + tl.m0;
      for (int kb = 0; kb < KB; ++kb, rp.next(S)) {
        if (rp.i >= S && !g_wait(p, g, &g.empty[rp.slot], rp.ph ^ 1u, 31)) { ok = false; break; }
        uint8_t* st = g.stages + size_t(rp.slot) * stage_bytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&g.full[rp.slot], stage_bytes);
          tma_load_2d(st, &m.h, kb * 64, row0, &g.full[rp.slot], pol_h);
          tma_load_2d(st + a_bytes, &m.h, p.de + kb * 64, row0, &g.full[rp.slot], pol_h);
          tma_load_2d(st + 2 * a_bytes, &m.w2, kb * 64, e * p.d + jn * N, &g.full[rp.slot], pol_w);
        }
        __syncwarp();
      }
    }
    producer_drain(g, rp, S);
  } else if (warp == 1) {
    const uint32_t idesc = tc::idesc_bf16_f32(kTileM, N);
    Ring rp;
    int tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < T && ok; tile += gridDim.x, ++tcount) {
      const int ab = tcount & 1;
      if (tcount >= 2 && !g_wait(p, g, &g.acce[ab], uint32_t((tcount >> 1) - 1) & 1u, 32)) { ok = false; break; }
      tc::fence_after_sync();
      for (int kb = 0; kb < KB; ++kb, rp.next(S)) {
        if (!g_wait(p, g, &g.full[rp.slot], rp.ph, 33)) { ok = false; break; }
        tc::fence_after_sync();
        if (lane == 0) {
          const uint32_t sa = smem_u32(g.stages + size_t(rp.slot) * stage_bytes);
          const uint64_t dhi = tc::smem_desc_k128(sa), dlo = tc::smem_desc_k128(sa + a_bytes),
                         db = tc::smem_desc_k128(sa + 2 * a_bytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            tc::mma_bf16(tmem + uint32_t(ab * N), dhi + 2 * k, db + 2 * k, idesc, uint32_t(kb | k));
            tc::mma_bf16(tmem + uint32_t(ab * N), dlo + 2 * k, db + 2 * k, idesc, 1u);
          }
          tc::commit(&g.empty[rp.slot]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc::commit(&g.accf[ab]);
      __syncwarp();
    }
  } else {
    // kG2EpWarps / 4 warps per lane quarter q, taking the tile's 32-column blocks in turn.  Each block
    // leaves tensor memory one row per lane, goes through this warp's shared block, and is added into y
    // by rows: 8 lanes cover one row's 128 bytes, so a reduction instruction writes 4 whole lines of y
    // instead of 32 pieces of 32 different lines.  The block's 16-byte pieces are swizzled by row (piece
    // c of row r at c ^ (r & 7)), so both the row-per-lane writes and the 8-lanes-per-row reads are free
    // of bank conflicts.
    const int q = warp & 3, set = (warp - 2) >> 2, nsets = kG2EpWarps / 4;
    const uint64_t pol_y = policy_evict_last();
    float* blk = g.ep_buf + (warp - 2) * kEpBlock;
    float4* mine = reinterpret_cast<float4*>(blk + lane * 32);
    int tcount = 0;
    for (int tile = blockIdx.x; tile < T; tile += gridDim.x, ++tcount) {
      const int ab = tcount & 1;
      if (!g_wait(p, g, &g.accf[ab], uint32_t(tcount >> 1) & 1u, 34)) break;
      tc::fence_after_sync();
      const Tile2 tl = tile2_at(g, p.E, NT, tile);
      const int e = tl.e, jn = tl.jn, m0 = tl.m0, ne = g.cnt[e];
      const int row = q * 32 + lane;
      const int tok = m0 + row < ne ? p.tok[g.off[e] + m0 + row] : -1;  // this lane's row's token
      float* ycols = p.y + size_t(jn) * N + (lane & 7) * 4;
      for (int c0 = 32 * set; c0 < N; c0 += 32 * nsets) {
        float v[32];
        tc::ld_32x32b_x32(tmem + (uint32_t(q * 32) << 16) + uint32_t(ab * N + c0), v);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mine[k ^ (lane & 7)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3);
          const int tok_r = __shfl_sync(0xffffffffu, tok, r);
          const float4 a = reinterpret_cast<const float4*>(blk + r * 32)[(lane & 7) ^ (r & 7)];
          if (tok_r >= 0) red_add_v4(ycols + size_t(tok_r) * p.d + c0, a.x, a.y, a.z, a.w, pol_y);
        }
        __syncwarp();  // the block is read before the next one overwrites it
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&g.acce[ab]);
    }
  }
  gemm_teardown(p, g, N);
}

}  // namespace

bool prefill_plan(int L, int d, int E, int de, int num_sms, int max_smem, PrefillParams* p, PrefillLaunch* out) {
  if (L <= kDecodeMaxL || d % 64 != 0 || de % 64 != 0 || de > 256 || E < 1 || E > kMaxE) return false;
  if ((long long)L * E >= (1ll << 31) / 2) return false;  // pair indices, and H rows as TMA coordinates
  p->W = (E + 31) / 32;
  p->ksplit = cls::router_projection_parts(L, d, E, num_sms);
  p->N1 = de;
  p->N2 = d % 256 == 0 ? 256 : d % 128 == 0 ? 128 : 64;
  // alignment slack, barriers, tensor-memory slot, abort flag, the three per-expert tables
  const size_t fixed = 1024 + 256 + (3 * size_t(E) + 2) * 4;
  const size_t fixed2 = fixed + 16 + kG2EpWarps * kEpBlock * sizeof(float);  // + the epilogue blocks
  const size_t st1 = size_t(kTileM) * 128 + size_t(p->N1) * 128;
  const size_t st2 = 2 * size_t(kTileM) * 128 + size_t(p->N2) * 128;
  p->S1 = int((size_t(max_smem) - fixed) / st1);
  p->S2 = int((size_t(max_smem) - fixed2) / st2);
  if (p->S1 > 6) p->S1 = 6;
  if (p->S2 > 6) p->S2 = 6;
  if (p->S1 < 2 || p->S2 < 2) return false;
  out->grid = num_sms;
  out->smem1 = fixed + size_t(p->S1) * st1;
  out->smem2 = fixed2 + size_t(p->S2) * st2;
  return true;
}

cudaError_t prefill_launch(const PrefillParams& p, const PrefillMaps& m, const PrefillLaunch& pl, int num_sms,
                           cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(p.y, 0, size_t(p.L) * p.d * sizeof(float), st);
  if (err != cudaSuccess) return err;
  if ((err = cudaMemsetAsync(p.n_pos, 0, sizeof(int32_t), st)) != cudaSuccess) return err;
  if ((err = cls::router_projection(p.x, p.L, p.d, p.Wr, p.E, p.wsplit, p.s_part, p.ksplit, num_sms, st)) !=
      cudaSuccess)
    return err;
  prefill_stats_kernel<<<(p.L + 7) / 8, 256, 0, st>>>(p);
  prefill_count_kernel<<<p.E, 256, 0, st>>>(p);
  prefill_scan_kernel<<<1, 32, 0, st>>>(p);
  prefill_fill_kernel<<<p.E, 256, 0, st>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if ((err = cudaFuncSetAttribute(prefill_gemm1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(pl.smem1))) != cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(prefill_gemm2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(pl.smem2))) != cudaSuccess)
    return err;
  prefill_gemm1_kernel<<<pl.grid, kG1Threads, pl.smem1, st>>>(p, m);
  prefill_gemm2_kernel<<<pl.grid, kG2Threads, pl.smem2, st>>>(p, m);
  return cudaGetLastError();
}

}  // namespace bffn
