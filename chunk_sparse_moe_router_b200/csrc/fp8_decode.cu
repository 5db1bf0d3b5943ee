// Low-bit expert weights for the batched decode path: fp8 e4m3 codes with power-of-two scales (the
// intelliparadigm survey, section 4.1, lists low-bit quantisation of MoE expert weights; the BlockFFN
// layer itself is unchanged: lsdiaocha.cn BlockFFN article, sections 2 and 4).
//
// Format (per layer l with experts e = l E .. l E + E - 1):
//   W1[e][j][k] = s1[e][j] q1[e][j][k]          a power-of-two scale per row j of W1
//   W2[e][k][j] = t2[l] s2[e][j] q2[e][k][j]    a power-of-two scale per column j of W2 (t2 the layer's largest,
//                                               s2 <= 1 the ratio)
// The scale of a row (column) is the smallest 2^m with 448 2^m >= its largest |w|; a code is w / 2^m rounded
// to the nearest e4m3 value (ties to even).  Both scales are indexed by (e, j), so both fold into the
// up-projection's epilogue:
//   u_j = s1_j sum_k q1_jk x_k,  h''_j = s2_j r Swish(u_j),  y_k = t2 sum_{e, j} q2_kj h''_j
// and the expert weights stream from HBM at one byte each.
//
// Kernels of a forward call: the batched router (decode_batch.cu), x to f16, a scan of the per-chunk
// up-projection items, then per wave of chunks an up-projection and a down-projection kernel.  Both
// stream kernels take 64 weight rows per item through a ring of stages (64 rows x 256 bytes of codes as
// two TMA boxes, plus the matching f16 activations by cp.async), filled by one producer warp; eight
// consumer warps own 16 rows and half of a stage's k each: ldmatrix brings four fp8 codes per thread, cvt
// turns each pair into its exact f16 values, and mma.sync f16 (fp32 accumulate) contracts them with the
// activations in f16, read in the same order of k (a thread's pair of A slots 2c, 2c+1 holds codes 4c,
// 4c+1 and slots 2c+8, 2c+9 codes 4c+2, 4c+3, so its B fragment is the activations at 4c .. 4c+3).  The
// activations are x (bf16 values, exact in f16 in the normal range) and h'' as an f16 hi + lo pair (h''
// rounded once to f16 would put y's largest errors on the decode layer at 9.4e-4 rms(y), 0.75 of the
// per-element tolerance 2e-2 |y| + 1e-3 rms(y): too little margin).
// Every sum runs in a fixed order: y is bit-reproducible.
#include <algorithm>
#include <cuda_fp16.h>

#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace fp8 {
namespace {

constexpr int kCT = 256;            // consumer threads: 8 warps = 4 groups of 16 weight rows x 2 halves of k
constexpr int kT = kCT + 32;        // + one producer warp: the code boxes (TMA) and activations (cp.async)
constexpr int kRows = 64;           // weight rows per item
constexpr int kKB = 256;            // code bytes (k values) of a row per stage
constexpr int kWSub = kRows * 128;  // one tensor box: 64 rows x 128 codes, 128-byte swizzle (8 KB)
constexpr int kWBytes = 2 * kWSub;  // a stage's codes: two boxes side by side along k
constexpr int kAPitch = 2 * kKB + 32;  // 544 B rows of 256 f16 activations: conflict-free 8-byte loads
constexpr int kStages = 4;
constexpr int kXBytes = 8 * kAPitch;                                      // 4352 (8 token rows)
constexpr int kUpStage = (kWBytes + kXBytes + 1023) / 1024 * 1024;       // 21504: boxes stay 1024-aligned
constexpr int kDownStage = (kWBytes + 2 * kXBytes + 1023) / 1024 * 1024;  // 25600 (h'' hi and lo planes)
constexpr int kUpSmem = kStages * kUpStage + 1024;                       // + alignment slack
constexpr int kDownSmem = kStages * kDownStage + 1024;
constexpr uint64_t kFp8WaitNs = 2000000000ull;

__device__ __forceinline__ int layer_of(const Fp8Params& p, int c) { return p.layer ? p.layer[c] : c % p.n_layers; }

// The mbarrier receives one arrival once every cp.async this thread issued before has landed (its
// expected count includes these arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Barrier `id` (1 .. 15) among `n` threads (whole warps).
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}


// The smallest m with 448 2^m >= amax (0 for amax == 0), in exact fp32 comparisons.
__device__ __forceinline__ int pow2_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int ex;
  frexpf(amax, &ex);
  int m = ex - 9;
  while (ldexpf(448.f, m) < amax) ++m;
  while (ldexpf(448.f, m - 1) >= amax) --m;
  return m;
}

// ------------------------------------------------------------------------------------ quantisation
// One warp per row of W1: the row's largest |w|, its scale, its codes.
__global__ void __launch_bounds__(256) quant_w1_kernel(const __nv_bfloat16* __restrict__ W1, long long rows, int d,
                                                       uint8_t* __restrict__ q1, float* __restrict__ s1) {
  const long long row = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* w = W1 + row * d;
  float amax = 0.f;
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 v = *reinterpret_cast<const uint4*>(w + k);
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__bfloat162float(b[i])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int m = pow2_exponent(amax);
  if (lane == 0) s1[row] = ldexpf(1.f, m);
  for (int k = lane * 8; k < d; k += 256) {
    const uint4 v = *reinterpret_cast<const uint4*>(w + k);
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      c[i] = f32x2_to_e4m3x2(ldexpf(__bfloat162float(b[2 * i]), -m), ldexpf(__bfloat162float(b[2 * i + 1]), -m));
    *reinterpret_cast<uint2*>(q1 + row * d + k) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  }
}

// Per column (e, j) of W2: the exponent of its scale, kept as an int in s2's place for now, and the
// layer's largest exponent (an integer maximum: the same in any order).
__global__ void __launch_bounds__(256) colmax_w2_kernel(const __nv_bfloat16* __restrict__ W2, int NE, int E, int d,
                                                        int de, int* __restrict__ m2, int* __restrict__ mlayer) {
  const long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (q >= (long long)NE * de) return;
  const int e = int(q / de), j = int(q % de);
  const __nv_bfloat16* col = W2 + size_t(e) * d * de + j;
  float amax = 0.f;
#pragma unroll 8
  for (int k = 0; k < d; ++k) amax = fmaxf(amax, fabsf(__bfloat162float(col[size_t(k) * de])));
  const int m = pow2_exponent(amax);
  m2[q] = m;
  atomicMax(mlayer + e / E, m);
}

__global__ void __launch_bounds__(256) fill_int_kernel(int* __restrict__ v, int n, int value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = value;
}

// The codes of W2, two adjacent columns at a time (each with its own scale).
__global__ void __launch_bounds__(256) quant_w2_kernel(const __nv_bfloat16* __restrict__ W2, long long n_pairs, int d,
                                                       int de, const int* __restrict__ m2, uint8_t* __restrict__ q2) {
  const long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (q >= n_pairs) return;
  const long long i = 2 * q;  // element index in [NE][d][de]; de is even
  const int j = int(i % de);
  const int e = int(i / (size_t(d) * de));
  const int ma = m2[size_t(e) * de + j], mb = m2[size_t(e) * de + j + 1];
  const __nv_bfloat162 w = *reinterpret_cast<const __nv_bfloat162*>(W2 + i);
  *reinterpret_cast<uint16_t*>(q2 + i) =
      uint16_t(f32x2_to_e4m3x2(ldexpf(__low2float(w), -ma), ldexpf(__high2float(w), -mb)));
}

// s2 = 2^(m2 - M_layer) over the ints (each element read and written by its own thread).
__global__ void __launch_bounds__(256) finish_s2_kernel(int NE, int E, int de, const int* __restrict__ mlayer,
                                                        float* __restrict__ s2) {
  const long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (q >= (long long)NE * de) return;
  const int m = reinterpret_cast<const int*>(s2)[q];
  s2[q] = ldexpf(1.f, m - mlayer[q / de / E]);
}

// t2 = 2^M_layer in place, after every s2 has read its layer's exponent.
__global__ void __launch_bounds__(256) finish_t2_kernel(int n_layers, float* __restrict__ t2) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l < n_layers) t2[l] = ldexpf(1.f, reinterpret_cast<const int*>(t2)[l]);
}

// ------------------------------------------------------------------------------------ forward helpers
// x -> f16 rows, 8 per chunk (rows past L are zero).
__global__ void __launch_bounds__(256) x_to_f16_kernel(const __nv_bfloat16* __restrict__ x, int C, int L, int d,
                                                       __half* __restrict__ xh) {
  const long long n8 = (long long)C * 8 * d / 8;  // 8 values per thread
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n8; q += (long long)gridDim.x * blockDim.x) {
    const long long i = q * 8;
    const long long row = i / d;  // c * 8 + t
    const int t = int(row % 8), k = int(i % d);
    const long long c = row / 8;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (t < L) {
      const uint4 v = *reinterpret_cast<const uint4*>(x + (c * L + t) * d + k);
      const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
      __half2* o = reinterpret_cast<__half2*>(&out);
#pragma unroll
      for (int u = 0; u < 4; ++u) o[u] = __floats2half2_rn(__bfloat162float(b[2 * u]), __bfloat162float(b[2 * u + 1]));
    }
    *reinterpret_cast<uint4*>(xh + i) = out;
  }
}

// offs[c] = sum over earlier chunks of n_active x ceil(de / 64): the up-projection items before chunk c.
__global__ void __launch_bounds__(1024) scan_items_kernel(const int32_t* __restrict__ n_active, int C, int JB,
                                                          int32_t* __restrict__ offs) {
  __shared__ int part[1024];
  const int tid = threadIdx.x;
  const int per = (C + 1023) / 1024, b = tid * per, e = min(C, b + per);
  int sum = 0;
  for (int c = b; c < e; ++c) sum += max(n_active[c], 0) * JB;
  part[tid] = sum;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan (Hillis-Steele), integers: order-independent
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = tid > 0 ? part[tid - 1] : 0;
  for (int c = b; c < e; ++c) {
    offs[c] = run;
    run += max(n_active[c], 0) * JB;
  }
  if (tid == 1023) offs[C] = part[1023];
}

// The chunk whose items contain `item` (offs ascending over [c0, c1]).
__device__ __forceinline__ int chunk_of_item(const int32_t* offs, int c0, int c1, int item) {
  int lo = c0, hi = c1 - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offs[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// A's fragments of 32-code block kb (0 .. 7) of a stage for warp rows 16 w .. 16 w + 15 (see the file
// comment): the stage holds two boxes of 64 rows x 128 codes, 16-byte pieces swizzled by the row.
__device__ __forceinline__ void load_a(uint32_t wbase, int warp, int lane, int kb, uint32_t (&a0)[4],
                                       uint32_t (&a1)[4]) {
  const int row = 16 * warp + (lane & 15), piece = ((kb & 3) << 1) | (lane >> 4);
  const uint32_t addr = wbase + (kb >> 2) * kWSub + row * 128 + ((piece ^ (row & 7)) << 4);
  uint32_t r0, r1, r2, r3;
  ldmatrix_x4(addr, r0, r1, r2, r3);
  a0[0] = e4m3x2_to_f16x2(r0);
  a0[1] = e4m3x2_to_f16x2(r1);
  a0[2] = e4m3x2_to_f16x2(r0 >> 16);
  a0[3] = e4m3x2_to_f16x2(r1 >> 16);
  a1[0] = e4m3x2_to_f16x2(r2);
  a1[1] = e4m3x2_to_f16x2(r3);
  a1[2] = e4m3x2_to_f16x2(r2 >> 16);
  a1[3] = e4m3x2_to_f16x2(r3 >> 16);
}

// Up-projection items of chunks [c0, c1) -> descriptors {chunk, active slot, row block, global expert},
// one thread per item (the items of a wave are offs[c0] .. offs[c1] - 1).
__global__ void __launch_bounds__(256) decode_items_kernel(const Fp8Params p, int c0, int c1, int4* __restrict__ desc) {
  const int item0 = p.offs[c0], n = p.offs[c1] - item0;
  const int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= n) return;
  const int c = chunk_of_item(p.offs, c0, c1, item0 + q);
  const int rem = item0 + q - p.offs[c];
  const int a = rem / p.JB;
  desc[q] = make_int4(c, a, rem - a * p.JB, layer_of(p, c) * p.E + p.active_idx[size_t(c) * p.E + a]);
}

// ------------------------------------------------------------------------------------ up-projection
// Items of chunks [c0, c1): (chunk, active expert, 64-row block of de), described by desc[].  A CTA walks
// items blockIdx.x, + gridDim.x, ...; each item is ns = ceil(d / 256) stages of 64 rows x 256 codes of W1
// and 8 x 256 f16 of x.  Warp 8 produces: it waits until the 8 consumer warps have released a ring slot
// (empty[s]), then issues the slot's two code boxes (TMA, transaction bytes on full[s]) and the x rows
// (cp.async, one arrival per lane on full[s] once its copies land).  The consumers wait on full[s] only,
// so no CTA-wide barrier sits between stages.  At an item's end the two k-halves of a row group meet at a
// barrier of their own; the epilogue writes h'' = s2 r Swish(s1 u) as f16 hi + lo into
// h[chunk - c0][a][plane][t][j].
__global__ void __launch_bounds__(kT) up_kernel(const Fp8Params p, const __grid_constant__ Maps mp, int c0, int c1,
                                               const int4* __restrict__ desc) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float4 xchg[2][4 * 32];  // the k-half 1 warps' partial sums at an item's end (by item parity)
  __shared__ __align__(8) uint64_t full[kStages];   // a stage's code boxes and x rows landed
  __shared__ __align__(8) uint64_t empty[kStages];  // the 8 consumer warps are done reading a stage
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int n_items = p.offs[c1] - p.offs[c0];
  const int G = int(gridDim.x), b = int(blockIdx.x);
  const int mine = n_items > b ? (n_items - b + G - 1) / G : 0;
  const int ns = (p.d + kKB - 1) / kKB;
  const int total = mine * ns;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023) & ~1023u;
  uint8_t* const sgen = smem_raw + (sbase - smem_u32(smem_raw));
  if (tid == 0) {
    prefetch_tensormap(&mp.w1);
    for (int q = 0; q < kStages; ++q) {
      mbar_init(&full[q], 1 + 32);
      mbar_init(&empty[q], kCT / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (wid == kCT / 32) {  // producer
    const uint64_t pol = policy_evict_first();  // the codes stream through once
    int4 dl = make_int4(0, 0, 0, 0), dn = make_int4(0, 0, 0, 0);  // the item being loaded, the next one
    if (mine > 0) dl = desc[b];
    if (mine > 1) dn = desc[b + G];
    int ml = 0;
    for (int i = 0; i < total; ++i) {
      const int m = i / ns, ks = i - m * ns;
      if (m != ml) {  // next item: its descriptor arrived long ago; fetch the one after
        ml = m;
        dl = dn;
        if (m + 1 < mine) dn = desc[b + (m + 1) * G];
      }
      const int slot = i % kStages;
      if (i >= kStages && !mbar_wait_bounded(&empty[slot], uint32_t(i / kStages - 1) & 1u, kFp8WaitNs))
        atomicOr(&p.hdr->err, uint32_t(kErrRingWait));  // recorded; the CTA goes on without hanging
      const int k0 = ks * kKB;
      if (lane == 0) {  // W1 codes: two boxes (rows past de belong to the next expert: their u is never
                        // stored; columns past d and rows past the last expert read as zeros)
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[slot], kWBytes);
        uint8_t* dst = sgen + slot * kUpStage;
        tma_load_2d(dst, &mp.w1, k0, dl.w * p.de + dl.z * kRows, &full[slot], pol);
        tma_load_2d(dst + kWSub, &mp.w1, k0 + 128, dl.w * p.de + dl.z * kRows, &full[slot], pol);
      }
      const int k = k0 + lane * 8;  // x in f16: 8 rows, this lane's 16-byte piece of each
      const bool ok = k < p.d;
      const uint32_t xs = sbase + slot * kUpStage + kWBytes + lane * 16;
#pragma unroll
      for (int t = 0; t < 8; ++t)
        cp_async16(xs + t * kAPitch, ok ? p.xh + (size_t(dl.x) * 8 + t) * p.d + k : p.xh, ok ? 16 : 0);
      cp_async_arrive_noinc(&full[slot]);
    }
    cp_async_wait_all();
    return;
  }

  // consumers: warp rows 16 w .. 16 w + 15 of the item, k-half wk of each stage
  const int g = lane >> 2, cq = lane & 3, warp = wid & 3, wk = wid >> 2;
  int4 dc = make_int4(0, 0, 0, 0);  // the current item; the epilogue's inputs fetched at its first stages
  float ep_r[2] = {0.f, 0.f}, ep_s1[2] = {0.f, 0.f}, ep_s2[2] = {0.f, 0.f};
  auto fetch_epilogue = [&]() {
    const int el = dc.w % p.E;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = dc.z * kRows + 16 * warp + g + 8 * h, t = 2 * cq + h;
      ep_r[h] = t < p.L ? p.r[(size_t(dc.x) * p.L + t) * p.E + el] : 0.f;  // token 2 cq + h
      ep_s1[h] = j < p.de ? p.s1[size_t(dc.w) * p.de + j] : 0.f;  // row g + 8 h
      ep_s2[h] = j < p.de ? p.s2[size_t(dc.w) * p.de + j] : 0.f;
    }
  };
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i = 0; i < total; ++i) {
    const int mc = i / ns, ks = i - mc * ns;
    if (ks == 0) dc = desc[b + mc * G];
    if (ks == (ns > 1 ? 1 : 0)) fetch_epilogue();
    const int slot = i % kStages;
    if (!mbar_wait_bounded(&full[slot], uint32_t(i / kStages) & 1u, kFp8WaitNs))
      atomicOr(&p.hdr->err, uint32_t(kErrRingWait));
    const uint32_t ws = sbase + slot * kUpStage, xs = ws + kWBytes;
    const uint32_t brow = xs + g * kAPitch + cq * 8;
#pragma unroll
    for (int kq = 0; kq < kKB / 64; ++kq) {
      const int kb = wk * (kKB / 64) + kq;
      uint32_t a0[4], a1[4];
      load_a(ws, warp, lane, kb, a0, a1);
      uint32_t b00, b01, b10, b11;
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b00), "=r"(b01) : "r"(brow + kb * 64));
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b10), "=r"(b11) : "r"(brow + kb * 64 + 32));
      mma_f16_16816(acc, a0, b00, b01);
      mma_f16_16816(acc, a1, b10, b11);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (ks == ns - 1) {  // the item's epilogue: the two halves of k added, then h'' by the k-half 0 warp
      float4* xc = xchg[mc & 1];
      if (wk == 1) xc[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      named_sync(1 + warp, 64);
      if (wk == 0) {
        const float4 o = xc[warp * 32 + lane];
        const float sum[4] = {acc[0] + o.x, acc[1] + o.y, acc[2] + o.z, acc[3] + o.w};
        __half* hb = p.h + (size_t(dc.x - c0) * p.E + dc.y) * 2 * 8 * p.de;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int h = v >> 1, t = 2 * cq + (v & 1);  // row g + 8 h, token t
          const int j = dc.z * kRows + 16 * warp + g + 8 * h;
          if (j >= p.de) continue;
          const float uu = ep_s1[h] * sum[v];
          const float r = (v & 1) ? ep_r[1] : ep_r[0];
          const float hh = t < p.L ? ep_s2[h] * (r * (uu / (1.f + expf(-uu)))) : 0.f;
          const __half hi = __float2half_rn(hh);
          hb[size_t(t) * p.de + j] = hi;
          hb[(8 + size_t(t)) * p.de + j] = __float2half_rn(hh - __half2float(hi));
        }
      }
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    }
  }
}

// ------------------------------------------------------------------------------------ down-projection
// Items of chunks [c0, c1): (chunk, 64-row block of d), output-stationary.  An item's stages run over the
// chunk's active experts a and 256-wide blocks jk of de: 64 rows x 256 codes of W2 and the h'' hi and lo
// planes (8 x 256 f16 each).  A chunk without active experts still takes one (empty) stage and writes zeros.  The CTA's
// items are taken in groups of kItemTab: a group's per-item stage counts and layers go to shared memory
// first (the one CTA-wide barrier pair per group); the producer warp then walks the group's stages,
// fetching the expert of the stage after the one it loads one stage early, while the consumers contract.
// y[c][t][k] = t2 acc (one writer per element, a fixed order of terms).
constexpr int kItemTab = 256;
__global__ void __launch_bounds__(kT) down_kernel(const Fp8Params p, const __grid_constant__ Maps mp, int c0, int c1) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int2 itab[kItemTab];  // per item of the group: {stages, layer (-1: none active)}
  __shared__ float4 xchg[2][4 * 32];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int RB = (p.d + kRows - 1) / kRows, JK = (p.de + kKB - 1) / kKB;
  const int G = int(gridDim.x), b = int(blockIdx.x);
  const int n_items = (c1 - c0) * RB;
  const int mine = n_items > b ? (n_items - b + G - 1) / G : 0;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023) & ~1023u;
  uint8_t* const sgen = smem_raw + (sbase - smem_u32(smem_raw));
  if (tid == 0) {
    prefetch_tensormap(&mp.w2);
    for (int q = 0; q < kStages; ++q) {
      mbar_init(&full[q], 1 + 32);
      mbar_init(&empty[q], kCT / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const bool producer = wid == kCT / 32;
  const uint64_t pol = policy_evict_first();
  int base_use = 0;  // stages of earlier item groups: stage u of the CTA uses slot u % kStages, phase u / kStages
  int items_done = 0;  // items finished by the consumers (the exchange buffer's parity)
  auto chunk_of = [&](int m) { return c0 + (b + m * G) / RB; };
  auto rb_of = [&](int m) { return (b + m * G) % RB; };

  for (int gb = 0; gb < mine; gb += kItemTab) {
    const int gn = min(kItemTab, mine - gb);
    __syncthreads();  // the previous group's table is no longer read
    for (int k = tid; k < gn; k += kT) {
      const int c = chunk_of(gb + k), l = layer_of(p, c);
      const bool ok = l >= 0 && l < p.n_layers;
      const int na = ok ? max(p.n_active[c], 0) : 0;
      itab[k] = make_int2(max(1, na * JK), na > 0 ? l : -1);
    }
    __syncthreads();
    int total = 0;
    for (int k = 0; k < gn; ++k) total += itab[k].x;

    if (producer) {
      // the expert of stage s of group item k (0 when the item has no active expert)
      auto expert_of = [&](int k, int s) -> int {
        const int2 t = itab[k];
        if (t.y < 0) return 0;
        return t.y * p.E + p.active_idx[size_t(chunk_of(gb + k)) * p.E + s / JK];
      };
      auto next_of = [&](int k, int s, int& kn, int& sn) {
        if (s + 1 < itab[k].x) kn = k, sn = s + 1;
        else kn = k + 1, sn = 0;
      };
      // cursor: item k_l, stage s_l of it; e_l its expert, e_n the next stage's (in flight)
      int k_l = 0, s_l = 0, k_n, s_n;
      int e_l = expert_of(0, 0);
      next_of(0, 0, k_n, s_n);
      int e_n = k_n < gn ? expert_of(k_n, s_n) : 0;
      for (int i = 0; i < total; ++i) {
        const int u = base_use + i, slot = u % kStages;
        if (u >= kStages && !mbar_wait_bounded(&empty[slot], uint32_t(u / kStages - 1) & 1u, kFp8WaitNs))
          atomicOr(&p.hdr->err, uint32_t(kErrRingWait));
        const int c = chunk_of(gb + k_l), rb = rb_of(gb + k_l);
        const bool any = itab[k_l].y >= 0;
        const int a = s_l / JK, j0 = (s_l - a * JK) * kKB;
        if (lane == 0) {  // W2 codes: two boxes (an empty item's boxes come from expert 0 and meet zero h)
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&full[slot], kWBytes);
          uint8_t* dst = sgen + slot * kDownStage;
          tma_load_2d(dst, &mp.w2, j0, e_l * p.d + rb * kRows, &full[slot], pol);
          tma_load_2d(dst + kWSub, &mp.w2, j0 + 128, e_l * p.d + rb * kRows, &full[slot], pol);
        }
        const int j = j0 + lane * 8;  // h'' hi and lo planes: 16 rows x this lane's 16-byte piece
        const bool ok = any && j < p.de;
        const __half* hsrc = p.h + (size_t(c - c0) * p.E + a) * 2 * 8 * p.de + j;
        const uint32_t hs = sbase + slot * kDownStage + kWBytes + lane * 16;
#pragma unroll
        for (int t = 0; t < 16; ++t) cp_async16(hs + t * kAPitch, ok ? hsrc + size_t(t) * p.de : p.h, ok ? 16 : 0);
        cp_async_arrive_noinc(&full[slot]);
        // advance: the next stage's expert is in flight already; start fetching the one after it
        k_l = k_n;
        s_l = s_n;
        e_l = e_n;
        if (k_l < gn) {
          next_of(k_l, s_l, k_n, s_n);
          e_n = k_n < gn ? expert_of(k_n, s_n) : 0;
        }
      }
    } else {
      const int g = lane >> 2, cq = lane & 3, warp = wid & 3, wk = wid >> 2;
      int k_c = 0, s_c = 0;  // consumer cursor
      float t2c = 0.f;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < total; ++i) {
        const int u = base_use + i, slot = u % kStages;
        if (s_c == 0) t2c = itab[k_c].y >= 0 ? p.t2[itab[k_c].y] : 0.f;  // used at the item's last stage
        if (!mbar_wait_bounded(&full[slot], uint32_t(u / kStages) & 1u, kFp8WaitNs))
          atomicOr(&p.hdr->err, uint32_t(kErrRingWait));
        const uint32_t ws = sbase + slot * kDownStage, hs = ws + kWBytes;
        const uint32_t brow_hi = hs + g * kAPitch + cq * 8, brow_lo = brow_hi + 8 * kAPitch;
        const bool work = itab[k_c].y >= 0;  // an empty item's stage is only waited for
#pragma unroll
        for (int kq = 0; kq < kKB / 64; ++kq) {
          if (!work) break;
          const int kb = wk * (kKB / 64) + kq;
          uint32_t a0[4], a1[4];
          load_a(ws, warp, lane, kb, a0, a1);
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(h0), "=r"(h1) : "r"(brow_hi + kb * 64));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(h2), "=r"(h3) : "r"(brow_hi + kb * 64 + 32));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(l0), "=r"(l1) : "r"(brow_lo + kb * 64));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(l2), "=r"(l3) : "r"(brow_lo + kb * 64 + 32));
          mma_f16_16816(acc, a0, h0, h1);
          mma_f16_16816(acc, a0, l0, l1);
          mma_f16_16816(acc, a1, h2, h3);
          mma_f16_16816(acc, a1, l2, l3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (s_c + 1 == itab[k_c].x) {  // the item's last stage: the two halves of k added, then y rows
          float4* xc = xchg[items_done & 1];
          if (wk == 1) xc[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
          named_sync(1 + warp, 64);
          const int c = chunk_of(gb + k_c), rb = rb_of(gb + k_c);
          if (wk == 0) {
            const float4 o = xc[warp * 32 + lane];
            const float sum[4] = {acc[0] + o.x, acc[1] + o.y, acc[2] + o.z, acc[3] + o.w};
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int k = rb * kRows + 16 * warp + g + (v >> 1) * 8, t = 2 * cq + (v & 1);
              if (k < p.d && t < p.L) p.y[(size_t(c) * p.L + t) * p.d + k] = t2c * sum[v];
            }
          }
          acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
          ++items_done;
          ++k_c;
          s_c = 0;
        } else {
          ++s_c;
        }
      }
    }
    base_use += total;
  }
  if (producer) cp_async_wait_all();
}

}  // namespace

size_t workspace_bytes(int C, int L, int d, int E, int de) {
  const Fp8Layout l = layout(C, L, d, E, de);
  return l.total;
}

Fp8Layout layout(int C, int L, int d, int E, int de) {
  Fp8Layout l;
  l.r_off = sizeof(WsHeader);
  l.bar_off = l.r_off + align256(size_t(C) * L * E * 4);
  l.offs_off = l.bar_off + align256(size_t(C) * 4);
  l.xh_off = l.offs_off + align256(size_t(C + 1) * 4);
  l.h_off = l.xh_off + align256(size_t(C) * 8 * d * 2);
  const size_t per_chunk = size_t(E) * 2 * 8 * de * 2;  // f16 h'' hi and lo rows of every active slot
  l.wave = int(std::max<size_t>(1, std::min<size_t>(size_t(C), kHBufBytes / per_chunk)));
  l.desc_off = l.h_off + align256(size_t(l.wave) * per_chunk);
  l.total = l.desc_off + align256(size_t(l.wave) * E * ((de + 63) / 64) * 16);
  return l;
}

cudaError_t quantize(const __nv_bfloat16* W1, const __nv_bfloat16* W2, int n_layers, int E, int d, int de,
                     uint8_t* q1, uint8_t* q2, float* s1, float* s2, float* t2, cudaStream_t st) {
  const int NE = n_layers * E;
  const long long rows = (long long)NE * de;
  quant_w1_kernel<<<unsigned((rows * 32 + 255) / 256), 256, 0, st>>>(W1, rows, d, q1, s1);
  // t2 holds the layers' largest exponents (ints) until the last kernel
  int* mlayer = reinterpret_cast<int*>(t2);
  int* m2 = reinterpret_cast<int*>(s2);
  fill_int_kernel<<<(n_layers + 255) / 256, 256, 0, st>>>(mlayer, n_layers, -(1 << 30));
  colmax_w2_kernel<<<unsigned((rows + 255) / 256), 256, 0, st>>>(W2, NE, E, d, de, m2, mlayer);
  const long long pairs = (long long)NE * d * de / 2;
  quant_w2_kernel<<<unsigned((pairs + 255) / 256), 256, 0, st>>>(W2, pairs, d, de, m2, q2);
  finish_s2_kernel<<<unsigned((rows + 255) / 256), 256, 0, st>>>(NE, E, de, mlayer, s2);
  finish_t2_kernel<<<(n_layers + 255) / 256, 256, 0, st>>>(n_layers, t2);
  return cudaGetLastError();
}

cudaError_t forward(const Fp8Params& p, const Maps& m, const batch::Params& rp, int num_sms, cudaStream_t st) {
  cudaError_t err;
  if ((err = batch::launch_router(rp, st)) != cudaSuccess) return err;
  {
    const long long n8 = (long long)p.C * p.d;  // C * 8 * d / 8
    const unsigned grid = unsigned(std::min<long long>((n8 + 255) / 256, (long long)num_sms * 16));
    x_to_f16_kernel<<<grid, 256, 0, st>>>(rp.x, p.C, p.L, p.d, p.xh);
  }
  scan_items_kernel<<<1, 1024, 0, st>>>(p.n_active, p.C, p.JB, p.offs);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if ((err = cudaFuncSetAttribute(up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUpSmem)) != cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDownSmem)) !=
      cudaSuccess)
    return err;
  const int grid = 2 * num_sms;
  const long long max_items = (long long)p.wave * p.E * p.JB;  // a wave's items when every expert is active
  for (int c0 = 0; c0 < p.C; c0 += p.wave) {
    const int c1 = std::min(p.C, c0 + p.wave);
    decode_items_kernel<<<unsigned((max_items + 255) / 256), 256, 0, st>>>(p, c0, c1, p.desc);
    up_kernel<<<grid, kT, kUpSmem, st>>>(p, m, c0, c1, p.desc);
    down_kernel<<<grid, kT, kDownSmem, st>>>(p, m, c0, c1);
  }
  return cudaGetLastError();
}

}  // namespace fp8
}  // namespace bffn
