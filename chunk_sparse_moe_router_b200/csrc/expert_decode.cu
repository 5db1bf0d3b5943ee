// Sparse expert kernel of the BlockFFN chunk layer for decode-sized chunks (L <= 32).
//
// The chunk's union U of active experts (lsdiaocha.cn BlockFFN article, section 4) is evaluated for all L
// tokens as one batch, outer loop over active experts and inner batched product (article, section 7),
// and each (token, expert) term is weighted by the router output r, which is zero for the pairs
// the mask removes.  Only the rows of W1/W2 that belong to experts in U are read.
//
// The kernel is memory-bound: every weight byte is used by L tokens (2L flop per bf16 weight), so
// it is built around keeping HBM busy:
//  * one persistent CTA per SM; the work of each phase is split over the CTAs in contiguous row
//    ranges balanced to within one row, so every SM streams the same number of bytes;
//  * weights move with bulk (TMA) copies into a ring of shared-memory slots guarded by mbarriers,
//    one producer warp keeping up to S slots in flight, with an L2 evict-first hint;
//  * 4 consumer warps run mma.sync m16n8k16 (bf16 in, fp32 accumulate) with tokens as the M
//    dimension and 8 weight rows as N, reading operands from shared memory with ldmatrix.
//
// Phase A (up-projection): the CTA owns rows [rA0, rA1) of the flattened (active expert, j) space;
//   u[t, row] = W1[e, j, :] . x_t,  h = r[t, e] * Swish(u)  (Swish(u) = u / (1 + e^-u), article
//   section 2), stored to the workspace as a high and a low bf16 part so the down-projection keeps
//   ~16 mantissa bits of h on bf16 tensor cores.
// Grid barrier: every CTA's h must be visible before any down-projection (bounded wait).  The
//   producer keeps prefetching W2 tiles while the barrier is pending; only the h tiles wait for it.
// Phase B (down-projection): the CTA owns output rows [rB0, rB1) of y and sums over every active
//   expert:  y[t, k] = sum_a sum_j W2[e_a, k, j] (h_hi + h_lo)[a, t, j].  The hi and lo parts are
//   two stacks of L rows of the MMA's M dimension, added in the epilogue.  Each y element is written
//   exactly once, in a fixed summation order, so y is bit-reproducible run to run.
#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace {

constexpr int NCW = 4;                  // consumer warps
constexpr int kThreads = (NCW + 2) * 32;
constexpr int RB = 32;                  // weight rows per row-block: 4 n-tiles of 8
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxSpan = 3;             // experts a 32-row block can touch when de >= 16

struct Smem {
  uint8_t* ring;
  int32_t* act;        // [E] the chunk's active expert ids (copied once per CTA)
  float* rs;           // [kMaxSpan][L] router outputs of the experts of the current row-block
  float* red;          // [NCW][MT][4][32][4]
  uint64_t* fullW;     // [S]
  uint64_t* fullH;     // [S]
  uint64_t* empty;     // [S]
  uint8_t* zero;       // 16 zero bytes
  volatile int* abort_flag;
};

struct Work {
  int nA;              // phase A rows of this CTA
  int rA0;
  int nB;              // phase B rows of this CTA
  int rB0;
  int nRBA, nRBB;      // row-blocks
  int nKA;             // stages per phase-A row-block
  int nJB;             // j-chunks per expert in phase B
  int n_act;
  int stagesA, stagesB;
};

__device__ __forceinline__ Work make_work(const DecodeParams& p, int n_act) {
  Work w;
  const int G = gridDim.x, c = blockIdx.x;
  const long long RA = (long long)n_act * p.de;
  w.rA0 = int(RA * c / G);
  w.nA = int(RA * (c + 1) / G) - w.rA0;
  w.rB0 = int((long long)p.d * c / G);
  w.nB = int((long long)p.d * (c + 1) / G) - w.rB0;
  w.nRBA = (w.nA + RB - 1) / RB;
  w.nRBB = (w.nB + RB - 1) / RB;
  w.nKA = (p.d + p.KcA - 1) / p.KcA;
  w.nJB = (p.de + p.KcB - 1) / p.KcB;
  w.n_act = n_act;
  w.stagesA = w.nRBA * w.nKA;
  w.stagesB = w.nRBB * n_act * w.nJB;
  return w;
}

__device__ __forceinline__ void set_error(const DecodeParams& p, const Smem& sm, uint32_t bit, uint32_t info) {
  atomicOr(&p.hdr->err, bit);
  p.hdr->err_info = info;
  *sm.abort_flag = 1;
}

// ----------------------------------------------------------------------------------------- producers
// Weight producer: phase A stages (x rows + W1 rows) then phase B stages (W2 rows), in order.
__device__ void produce_weights(const DecodeParams& p, const Smem& sm, const Work& w) {
  const int lane = threadIdx.x % 32;
  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_x = policy_evict_last();
  const int total = w.stagesA + w.stagesB;
  int i = 0;
  for (; i < total; ++i) {
    if (*sm.abort_flag) break;
    const int slot = i % p.S;
    if (i >= p.S) {
      if (!mbar_wait_bounded(&sm.empty[slot], ((i / p.S) - 1) & 1, kWaitNs)) {
        if (lane == 0) set_error(p, sm, kErrRingWait, 1);
        break;
      }
    }
    uint8_t* base = sm.ring + size_t(slot) * p.slot_bytes;
    if (i < w.stagesA) {
      const int rb = i / w.nKA, kc = i % w.nKA;
      const int r0 = w.rA0 + rb * RB, nrows = min(RB, w.nA - rb * RB);
      const int k0 = kc * p.KcA, kw = min(p.KcA, p.d - k0);
      const uint32_t rowb = uint32_t(kw) * 2;
      if (lane == 0) mbar_arrive_expect_tx(&sm.fullW[slot], rowb * uint32_t(p.L + nrows));
      __syncwarp();
      for (int c = lane; c < p.L + nrows; c += 32) {
        if (c < p.L) {
          bulk_g2s(base + size_t(c) * p.pitchA, p.x + size_t(c) * p.d + k0, rowb, &sm.fullW[slot], pol_x);
        } else {
          const int row = r0 + (c - p.L);
          const int a = row / p.de, j = row % p.de;
          const int e = sm.act[a];
          const __nv_bfloat16* src = p.W1 + (size_t(e) * p.de + j) * p.d + k0;
          bulk_g2s(base + p.woff + size_t(c - p.L) * p.pitchA, src, rowb, &sm.fullW[slot], pol_w);
        }
      }
    } else {
      const int jb = i - w.stagesA;
      const int per_rb = w.n_act * w.nJB;
      const int rb = jb / per_rb, rem = jb % per_rb;
      const int a = rem / w.nJB, jc = rem % w.nJB;
      const int k0 = w.rB0 + rb * RB, nrows = min(RB, w.nB - rb * RB);
      const int j0 = jc * p.KcB, jw = min(p.KcB, p.de - j0);
      const uint32_t rowb = uint32_t(jw) * 2;
      const int e = sm.act[a];
      if (lane == 0) mbar_arrive_expect_tx(&sm.fullW[slot], rowb * uint32_t(nrows));
      __syncwarp();
      for (int c = lane; c < nrows; c += 32) {
        const __nv_bfloat16* src = p.W2 + (size_t(e) * p.d + k0 + c) * p.de + j0;
        bulk_g2s(base + p.woff + size_t(c) * p.pitchB, src, rowb, &sm.fullW[slot], pol_w);
      }
    }
    __syncwarp();
  }
  // Drain: every copy this warp issued must land before the CTA may exit.
  const int issued = i;
  for (int k = max(0, issued - p.S); k < issued; ++k) {
    mbar_wait_bounded(&sm.fullW[k % p.S], (k / p.S) & 1, kWaitNs / 10);
  }
}

// h producer: after the grid barrier, the h tiles of every phase-B stage.
__device__ void produce_h(const DecodeParams& p, const Smem& sm, const Work& w) {
  const int lane = threadIdx.x % 32;
  if (w.stagesB == 0) return;
  {
    const uint64_t t0 = globaltimer_ns();
    bool ok = true;
    while (ld_acquire_gpu(&p.hdr->grid_bar) < gridDim.x) {
      if (*sm.abort_flag || globaltimer_ns() - t0 > kWaitNs) { ok = false; break; }
      __nanosleep(64);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) set_error(p, sm, kErrGridBarrier, uint32_t(blockIdx.x));
      return;
    }
    fence_proxy_async_global();
  }
  const uint64_t pol_h = policy_evict_last();
  const int L2 = 2 * p.L;
  uint32_t hphase = 0;  // bit s = parity of the next fullH phase of slot s
  int issued = 0;
  for (int jb = 0; jb < w.stagesB; ++jb) {
    if (*sm.abort_flag) break;
    const int i = w.stagesA + jb;
    const int slot = i % p.S;
    if (i >= p.S) {
      if (!mbar_wait_bounded(&sm.empty[slot], ((i / p.S) - 1) & 1, kWaitNs)) {
        if (lane == 0) set_error(p, sm, kErrRingWait, 2);
        break;
      }
    }
    const int per_rb = w.n_act * w.nJB;
    const int rem = jb % per_rb;
    const int a = rem / w.nJB, jc = rem % w.nJB;
    const int j0 = jc * p.KcB, jw = min(p.KcB, p.de - j0);
    const uint32_t rowb = uint32_t(jw) * 2;
    uint8_t* base = sm.ring + size_t(slot) * p.slot_bytes;
    if (lane == 0) mbar_arrive_expect_tx(&sm.fullH[slot], rowb * uint32_t(L2));
    __syncwarp();
    for (int c = lane; c < L2; c += 32) {
      const __nv_bfloat16* src = p.h + (size_t(a) * L2 + c) * p.de + j0;
      bulk_g2s(base + size_t(c) * p.pitchB, src, rowb, &sm.fullH[slot], pol_h);
    }
    __syncwarp();
    hphase ^= 1u << slot;
    ++issued;
  }
  // Drain this warp's copies.
  uint32_t ph = hphase;
  for (int k = issued - 1; k >= 0 && k >= issued - p.S; --k) {
    const int slot = (w.stagesA + k) % p.S;
    ph ^= 1u << slot;  // parity of that stage's phase
    mbar_wait_bounded(&sm.fullH[slot], (ph >> slot) & 1u, kWaitNs / 10);
  }
}

// ----------------------------------------------------------------------------------------- consumers
template <int MT>
__device__ __forceinline__ void mma_stage(const uint8_t* abase, int rowsA, int pitch, const uint8_t* wbase,
                                          int kw, const uint8_t* zero, float (&acc)[MT][4][4], int mtn) {
  const int cw = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nks = kw / 16;
  const uint32_t zaddr = smem_u32(zero);
  const uint32_t abase_u = smem_u32(abase), wbase_u = smem_u32(wbase);
  for (int ks = cw; ks < nks; ks += NCW) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (mt < mtn) {
        const int row = mt * 16 + (lane & 15);
        const int kcol = ks * 16 + (lane >> 4) * 8;
        const uint32_t addr = (row < rowsA) ? abase_u + uint32_t(row * pitch + kcol * 2) : zaddr;
        ldmatrix_x4(addr, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
      }
    }
    uint32_t b[4][2];
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      const int nrow = np * 16 + (lane & 7) + (lane >> 4) * 8;
      const int kcol = ks * 16 + ((lane >> 3) & 1) * 8;
      ldmatrix_x4(wbase_u + uint32_t(nrow * pitch + kcol * 2), b[2 * np][0], b[2 * np][1], b[2 * np + 1][0],
                  b[2 * np + 1][1]);
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (mt < mtn) {
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_bf16_16816(acc[mt][nt], a[mt], b[nt][0], b[nt][1]);
      }
    }
  }
}

// Value of output (row, col) of the row-block, summed over the consumer warps' partials.
template <int MT>
__device__ __forceinline__ float red_value(const float* red, int row, int col) {
  const int mt = row >> 4, r16 = row & 15;
  const int lane = (r16 & 7) * 4 + ((col & 7) >> 1);
  const int reg = (r16 >> 3) * 2 + (col & 1);
  const int nt = col >> 3;
  float v = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) v += red[((((w * MT + mt) * 4 + nt) * 32 + lane) * 4) + reg];
  return v;
}

template <int MT>
__device__ __forceinline__ void stash(float* red, const float (&acc)[MT][4][4]) {
  const int cw = threadIdx.x / 32, lane = threadIdx.x % 32;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
      *reinterpret_cast<float4*>(red + ((((cw * MT + mt) * 4 + nt) * 32 + lane) * 4)) =
          make_float4(acc[mt][nt][0], acc[mt][nt][1], acc[mt][nt][2], acc[mt][nt][3]);
}

// Wait for a ring barrier; on timeout record the error and mark the CTA aborted.  Once aborted,
// waits are skipped (the caller skips the work) so every consumer warp still reaches the same
// named barriers and the CTA can finish.
__device__ __forceinline__ bool ring_wait(const DecodeParams& p, const Smem& sm, uint64_t* bar, uint32_t parity,
                                          uint32_t where) {
  if (*sm.abort_flag) return false;
  if (mbar_wait_bounded(bar, parity, kWaitNs)) return true;
  if ((threadIdx.x & 31) == 0) set_error(p, sm, kErrRingWait, where);
  *sm.abort_flag = 1;
  return false;
}

template <int LC>
__device__ void consume(const DecodeParams& p, const Smem& sm, const Work& w) {
  constexpr int MT = (2 * LC + 15) / 16;  // m-tiles of the down-projection (2L rows: h hi + lo)
  const int ctid = threadIdx.x;           // consumers are threads [0, NCW*32)
  const int lane = ctid % 32;
  const int mtA = (p.L + 15) / 16, mtB = (2 * p.L + 15) / 16;
  float acc[MT][4][4];
  uint32_t hphase = 0;
  int i = 0;  // global stage index, same order as the producers

  // ---------------- phase A: up-projection, Swish, router scale
  for (int rb = 0; rb < w.nRBA; ++rb) {
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;
    const int r0 = w.rA0 + rb * RB, nrows = min(RB, w.nA - rb * RB);
    const int a_first = r0 / p.de;
    {
      // r of the (at most kMaxSpan) experts this row-block touches, fetched while the stages stream
      const int a_last = (r0 + nrows - 1) / p.de;
      for (int o = ctid; o < (a_last - a_first + 1) * p.L; o += NCW * 32) {
        const int aa = o / p.L, t = o % p.L;
        const float* src = p.r + size_t(t) * p.E + sm.act[a_first + aa];
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(sm.rs + aa * p.L + t)), "l"(src)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int kc = 0; kc < w.nKA; ++kc, ++i) {
      const int slot = i % p.S;
      if (ring_wait(p, sm, &sm.fullW[slot], (i / p.S) & 1, 3)) {
        const uint8_t* base = sm.ring + size_t(slot) * p.slot_bytes;
        const int kw = min(p.KcA, p.d - kc * p.KcA);
        mma_stage<MT>(base, p.L, p.pitchA, base + p.woff, kw, sm.zero, acc, mtA);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
    stash<MT>(sm.red, acc);
    asm volatile("cp.async.wait_all;" ::: "memory");
    named_bar_sync(1, NCW * 32);
    for (int o = ctid; o < p.L * nrows; o += NCW * 32) {
      const int t = o / nrows, c = o % nrows;
      const float u = red_value<MT>(sm.red, t, c);
      const int row = r0 + c;
      const int a = row / p.de, j = row % p.de;
      const float rr = sm.rs[(a - a_first) * p.L + t];
      const float hv = rr * (u / (1.f + expf(-u)));
      const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
      const __nv_bfloat16 lo = __float2bfloat16_rn(hv - __bfloat162float(hi));
      p.h[(size_t(a) * 2 * p.L + t) * p.de + j] = hi;
      p.h[(size_t(a) * 2 * p.L + p.L + t) * p.de + j] = lo;
    }
    named_bar_sync(1, NCW * 32);
  }
  // publish this CTA's h before any CTA starts reading h
  __threadfence();
  named_bar_sync(1, NCW * 32);
  if (ctid == 0) {
    fence_proxy_async_global();
    red_release_gpu_add(&p.hdr->grid_bar, 1u);
    pdl_launch_dependents();
  }

  // ---------------- phase B: down-projection over every active expert
  for (int rb = 0; rb < w.nRBB; ++rb) {
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;
    for (int s = 0; s < w.n_act * w.nJB; ++s, ++i) {
      const int slot = i % p.S;
      const bool okW = ring_wait(p, sm, &sm.fullW[slot], (i / p.S) & 1, 4);
      const bool okH = okW && ring_wait(p, sm, &sm.fullH[slot], (hphase >> slot) & 1u, 5);
      hphase ^= 1u << slot;
      if (okH) {
        const uint8_t* base = sm.ring + size_t(slot) * p.slot_bytes;
        const int jc = s % w.nJB;
        const int jw = min(p.KcB, p.de - jc * p.KcB);
        mma_stage<MT>(base, 2 * p.L, p.pitchB, base + p.woff, jw, sm.zero, acc, mtB);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
    stash<MT>(sm.red, acc);
    named_bar_sync(1, NCW * 32);
    const int k0 = w.rB0 + rb * RB, nrows = min(RB, w.nB - rb * RB);
    for (int o = ctid; o < p.L * nrows; o += NCW * 32) {
      const int t = o / nrows, c = o % nrows;
      const float v = red_value<MT>(sm.red, t, c) + red_value<MT>(sm.red, p.L + t, c);
      p.y[size_t(t) * p.d + k0 + c] = v;
    }
    named_bar_sync(1, NCW * 32);
  }
}

template <int LC>
__global__ void __launch_bounds__(kThreads, 1) expert_decode_kernel(DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr int MT = (2 * LC + 15) / 16;
  Smem sm;
  sm.ring = smem_raw;
  sm.red = reinterpret_cast<float*>(smem_raw + size_t(p.S) * p.slot_bytes);
  // tail (16-byte aligned): zero block [16] | abort flag [16] | fullW[S] | fullH[S] | empty[S] |
  // act[E] | rs[kMaxSpan][L]
  uint8_t* tail = reinterpret_cast<uint8_t*>(sm.red + NCW * MT * 4 * 32 * 4);
  sm.zero = tail;
  sm.abort_flag = reinterpret_cast<volatile int*>(tail + 16);
  sm.fullW = reinterpret_cast<uint64_t*>(tail + 32);
  sm.fullH = sm.fullW + p.S;
  sm.empty = sm.fullH + p.S;
  sm.act = reinterpret_cast<int32_t*>(sm.empty + p.S);
  sm.rs = reinterpret_cast<float*>(sm.act + p.E);

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&sm.fullW[s], 1);
      mbar_init(&sm.fullH[s], 1);
      mbar_init(&sm.empty[s], NCW);
    }
    *reinterpret_cast<uint4*>(sm.zero) = make_uint4(0, 0, 0, 0);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // the router (previous kernel) wrote the active list, r and reset the grid barrier
  pdl_wait();
  // one round trip: the count and the whole list (entries past the count are not used)
  const int n_raw = *p.n_active;
  for (int a = threadIdx.x; a < p.E; a += kThreads) sm.act[a] = min(max(p.active_idx[a], 0), p.E - 1);
  const int n_act = min(max(n_raw, 0), p.E);  // never index past the active list
  __syncthreads();
  const Work w = make_work(p, n_act);

  const int warp = threadIdx.x / 32;
  if (warp < NCW) {
    consume<LC>(p, sm, w);
  } else if (warp == NCW) {
    produce_weights(p, sm, w);
  } else {
    produce_h(p, sm, w);
  }
}

template <int LC>
cudaError_t launch_lc(const DecodeParams& p, const DecodeLaunch& plan, cudaStream_t st, bool pdl) {
  auto kfn = expert_decode_kernel<LC>;
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
  return cudaLaunchKernelEx(&cfg, kfn, p);
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

}  // namespace

bool expert_decode_plan(int L, int d, int de, int num_sms, int max_smem, DecodeParams* p,
                        DecodeLaunch* out) {
  if (L < 1 || L > kDecodeMaxL) return false;
  const int lc = L <= 8 ? 8 : L <= 16 ? 16 : 32;
  const int mt = (2 * lc + 15) / 16;
  p->KcA = d < 256 ? d : 256;
  p->KcB = de < 256 ? de : 256;
  p->pitchA = round_up(p->KcA * 2, 128) + 16;
  p->pitchB = round_up(p->KcB * 2, 128) + 16;
  const int pitch_max = p->pitchA > p->pitchB ? p->pitchA : p->pitchB;
  const int areg = round_up(L * p->pitchA > 2 * L * p->pitchB ? L * p->pitchA : 2 * L * p->pitchB, 128);
  p->woff = areg;
  p->slot_bytes = round_up(areg + RB * pitch_max, 128);
  const size_t red_bytes = size_t(NCW) * mt * 4 * 32 * 4 * 4;
  const size_t extra = size_t(kMaxE) * 4 + size_t(kMaxSpan) * kDecodeMaxL * 4;  // act + rs
  const size_t fixed = red_bytes + 3 * 8 * 32 + 64 + extra;
  if (size_t(max_smem) <= fixed) return false;
  int S = int((size_t(max_smem) - fixed) / size_t(p->slot_bytes));
  if (S > 16) S = 16;
  if (S < 2) return false;
  p->S = S;
  out->grid = num_sms;
  out->lclass = lc;
  out->smem = size_t(S) * p->slot_bytes + red_bytes + 3 * 8 * size_t(S) + 64 + extra;
  return true;
}

cudaError_t expert_decode_launch(const DecodeParams& p, const DecodeLaunch& plan, cudaStream_t st,
                                 bool pdl) {
  switch (plan.lclass) {
    case 8: return launch_lc<8>(p, plan, st, pdl);
    case 16: return launch_lc<16>(p, plan, st, pdl);
    default: return launch_lc<32>(p, plan, st, pdl);
  }
}

}  // namespace bffn
