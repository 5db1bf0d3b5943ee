// The CLS-aware training objectives of BlockFFN and their backward through the router (lsdiaocha.cn
// BlockFFN article, section 3: an activation-locality loss, a binary cross-entropy between adjacent
// tokens' activation patterns compared through LeftShift and approximated by a sharp sigmoid, and a
// chunk-sparsification loss, the probability that an expert is activated by at least one token of a
// chunk of L consecutive tokens).  The pages print no formulas; the readings taken:
//   p_{t,i} = sigmoid(alpha s_{t,i}),  s = x Wr + b
//   L_AL = mean over the (L-1) E adjacent pairs of each chunk of BCE(p_t; q = p_{t+1})
//          with BCE(p; q) = -(q log p + (1 - q) log(1 - p)), gradient through both sides
//   L_CS = mean over chunks and experts of 1 - prod_t (1 - p_t)
//   J = w_al L_AL + w_cs L_CS;  outputs L_AL, L_CS, dS = dJ/ds, dWr = x^T dS, db = sum_t dS, dx = dS Wr^T.
//
// Six kernels, all deterministic (fixed-order sums, no atomics):
//   split_wr     Wr (fp32) -> hi + lo bf16 pair, experts padded to a multiple of 64 with zeros
//   router_gemm  s = x (Wr_hi + Wr_lo) + b on the warp tensor cores (fp32 accumulate; the pair carries
//                Wr to about 2^-17 relative), written into the dS buffer
//   chunk_terms  per (chunk, expert): the two losses' partial sums, dS in place of s, and the hi + lo
//                bf16 split of dS
//   dx           dx = (dS_hi + dS_lo)(Wr_hi + Wr_lo)^T without the lo*lo product, fp32 out
//   dwr          per token split: x^T (dS_hi + dS_lo) into fp32 partials, and partial sums of db
//   reduce       the partials of dWr, db and the losses, in a fixed order
// The GEMMs are skinny (one side is E = 64 experts wide) and HBM-bound: x is read twice (router GEMM and
// dWr) and dx written once; bf16 pairs let the bf16 warp MMAs carry the fp32 operands.
#include <algorithm>

#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace cls {
namespace {

constexpr int kThreads = 256;
constexpr int kGemmThreads = 128;     // router GEMM and dWr: 4 warps, each a 64 x 32 tile of the output
constexpr int kTokTile = 128;         // router GEMM and dx: tokens per CTA
constexpr int kNTile = 64;            // experts per CTA
constexpr int kKTile = 64;            // reduction slice per pipeline stage
constexpr int kStages = 3;
constexpr int kPitch = kKTile + 8;    // bf16 pitch of 64-wide tiles: 144 B, so 8 ldmatrix rows hit 32 banks
constexpr int kDTile = 128;           // dWr: rows of Wr per CTA; dx: columns of x per slice
constexpr int kPitchWide = kDTile + 8;  // 272 B
constexpr int kSplitTok = 64;         // dWr: tokens per pipeline stage
constexpr int kDxSlices = 4;          // dx: column slices per CTA (the CTA's dS tile is loaded once)
constexpr int kDxMaxEp = 128;         // dx keeps its dS tile resident up to this many (padded) experts
constexpr int kChunksPerTile = 4;     // chunk_terms: chunks per CTA tile (x 64 experts = 256 threads)
constexpr int kReduceThreads = 1024;

constexpr int kRouterStage = (kTokTile + 2 * kKTile) * kPitch * 2;            // 36864 B
constexpr int kRouterSmem = kStages * kRouterStage;                           // 110592 B
constexpr int kDwrStage = kSplitTok * kPitchWide * 2 + 2 * kSplitTok * kPitch * 2;  // 35840 B
constexpr int kDwrSmem = kStages * kDwrStage;                                 // 107520 B
constexpr int kDxWideSmem = 2 * (kTokTile + kDTile) * kPitch * 2;             // 73728 B (any Ep, one slice)
__host__ __device__ constexpr int dx_smem(int Ep) { return 6 * kTokTile * (Ep + 8) * 2; }  // tile + 2 slices

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *hi = h;
  *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

// log sigmoid(z) and log sigmoid(-z) = log(1 - sigmoid(z)), both without cancellation.
__device__ __forceinline__ void log_sigmoids(float z, float& lsp, float& lsn) {
  const float m = log1pf(expf(-fabsf(z)));
  lsp = -(fmaxf(-z, 0.f) + m);
  lsn = -(fmaxf(z, 0.f) + m);
}

// acc[mt][nt] += A[mt] (B_hi + B_lo) for a warp's 4 x 4 grid of 16 x 8 tiles, B given as two 16 x 16
// halves (n-pairs) of hi and lo fragments.
__device__ __forceinline__ void mma_pair(float (&acc)[4][4][4], const uint32_t (&a)[4][4], int np, uint32_t h0,
                                         uint32_t h1, uint32_t h2, uint32_t h3, uint32_t l0, uint32_t l1, uint32_t l2,
                                         uint32_t l3) {
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    mma_bf16_16816(acc[mt][2 * np], a[mt], h0, h1);
    mma_bf16_16816(acc[mt][2 * np], a[mt], l0, l1);
    mma_bf16_16816(acc[mt][2 * np + 1], a[mt], h2, h3);
    mma_bf16_16816(acc[mt][2 * np + 1], a[mt], l2, l3);
  }
}

__global__ void __launch_bounds__(kThreads) split_wr_kernel(const float* __restrict__ Wr, int d, int E, int Ep,
                                                            __nv_bfloat16* __restrict__ hi,
                                                            __nv_bfloat16* __restrict__ lo) {
  const size_t n = size_t(d) * Ep;
  for (size_t q = blockIdx.x * size_t(blockDim.x) + threadIdx.x; q < n; q += size_t(gridDim.x) * blockDim.x) {
    const int k = int(q / Ep), e = int(q % Ep);
    split_bf16(e < E ? Wr[size_t(k) * E + e] : 0.f, hi + q, lo + q);
  }
}

// s[t0 .. t0+128, e0 .. e0+64] = x W + b.  Warp w owns tokens 64 (w & 1) .. +63 and experts
// 32 (w >> 1) .. +31: each operand fragment it loads from shared memory feeds four MMAs.  With a K split
// (gridDim.z > 1) CTA z takes columns [z kper, (z+1) kper) of x and writes its partial product to
// s + z T E (b, if any, goes to part 0).
__global__ void __launch_bounds__(kGemmThreads) router_gemm_kernel(const __nv_bfloat16* __restrict__ x, int T,
                                                                   int d, const __nv_bfloat16* __restrict__ wh,
                                                                   const __nv_bfloat16* __restrict__ wl, int Ep,
                                                                   const float* __restrict__ br, int E,
                                                                   float* __restrict__ s, int kper) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kXBytes = kTokTile * kPitch * 2, kWBytes = kKTile * kPitch * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wm = warp & 1, wn = warp >> 1;
  const int t0 = blockIdx.x * kTokTile, e0 = blockIdx.y * kNTile;
  const int kbeg = blockIdx.z * kper, kend = min(d, kbeg + kper);
  const int nk = (kend - kbeg + kKTile - 1) / kKTile;
  const uint32_t sbase = smem_u32(smem);
  if (blockIdx.z > 0) br = nullptr;
  s += size_t(blockIdx.z) * T * E;

  auto load = [&](int kt) {
    const uint32_t st = sbase + (kt % kStages) * kRouterStage;
    const int k0 = kbeg + kt * kKTile;
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // x: 128 rows x 8 pieces of 16 B
      const int idx = tid + j * kGemmThreads, row = idx >> 3, ch = idx & 7;
      const int gt = t0 + row, gk = k0 + ch * 8;
      const bool ok = gt < T && gk < kend;
      cp_async16(st + (row * kPitch + ch * 8) * 2, ok ? x + size_t(gt) * d + gk : x, ok ? 16 : 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // Wr hi and lo: 64 rows x 8 pieces each
      const int idx = tid + j * kGemmThreads, row = idx >> 3, ch = idx & 7;
      const int gk = k0 + row;
      const bool ok = gk < kend;
      const size_t off = ok ? size_t(gk) * Ep + e0 + ch * 8 : 0;
      cp_async16(st + kXBytes + (row * kPitch + ch * 8) * 2, wh + off, ok ? 16 : 0);
      cp_async16(st + kXBytes + kWBytes + (row * kPitch + ch * 8) * 2, wl + off, ok ? 16 : 0);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 4; ++n) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < kStages - 1; ++kt) {
    if (kt < nk) load(kt);
    cp_async_commit();
  }
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<kStages - 2>();
    __syncthreads();  // stage kt landed for every thread; stage kt-1 is no longer read
    if (kt + kStages - 1 < nk) load(kt + kStages - 1);
    cp_async_commit();
    const uint32_t xs = sbase + (kt % kStages) * kRouterStage, whs = xs + kXBytes, wls = whs + kWBytes;
#pragma unroll
    for (int kk = 0; kk < kKTile / 16; ++kk) {
      uint32_t a[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        ldmatrix_x4(xs + ((wm * 64 + mt * 16 + (lane & 15)) * kPitch + kk * 16 + (lane >> 4) * 8) * 2, a[mt][0],
                    a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const uint32_t off = ((kk * 16 + (lane & 15)) * kPitch + wn * 32 + np * 16 + (lane >> 4) * 8) * 2;
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        ldmatrix_x4_trans(whs + off, h0, h1, h2, h3);
        ldmatrix_x4_trans(wls + off, l0, l1, l2, l3);
        mma_pair(acc, a, np, h0, h1, h2, h3, l0, l1, l2, l3);
      }
    }
  }
  cp_async_wait<0>();
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int e = e0 + wn * 32 + nt * 8 + 2 * c;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + wm * 64 + mt * 16 + g + 8 * h;
        if (t >= T) continue;
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (e + q < E) s[size_t(t) * E + e + q] = acc[mt][nt][2 * h + q] + (br != nullptr ? br[e + q] : 0.f);
      }
    }
}

// Per (chunk, expert): the loss terms and dS.  A CTA takes tiles of 4 chunks x 64 experts: the tile's
// s values are staged in shared memory with coalesced loads, thread (chunk ty, expert tx) walks its
// column of L values twice (losses and the chunk product K; then dS), and dS goes back over s.
__global__ void __launch_bounds__(kThreads) chunk_terms_kernel(float* __restrict__ sd, int C, int L, int E, int Ep,
                                                               float alpha, float f_al, float f_cs,
                                                               __nv_bfloat16* __restrict__ dsh,
                                                               __nv_bfloat16* __restrict__ dsl,
                                                               double* __restrict__ loss_part) {
  extern __shared__ __align__(16) float tile[];  // [4 L][64]
  __shared__ double red[2][kThreads / 32];
  const int tid = threadIdx.x, tx = tid & 63, ty = tid >> 6;
  const int e0 = blockIdx.x * 64, i = e0 + tx;
  const int rows = kChunksPerTile * L;
  double al = 0.0, cs = 0.0;
  for (long long grp = blockIdx.y; grp * kChunksPerTile < C; grp += gridDim.y) {
    const long long c_first = grp * kChunksPerTile;
    const long long t_first = c_first * L;
    const int chunks = C - c_first < kChunksPerTile ? int(C - c_first) : kChunksPerTile;
    const int nrows = chunks * L;
    __syncthreads();  // the previous tile is fully read
    for (int q = tid; q < rows * 64; q += kThreads) {
      const int r = q >> 6, col = q & 63;
      const int e = e0 + col;
      tile[q] = (r < nrows && e < E) ? sd[size_t(t_first + r) * E + e] : 0.f;
    }
    __syncthreads();
    if (ty < chunks && i < E) {
      const float* col = tile + ty * L * 64 + tx;
      float log_keep = 0.f, al_c = 0.f, lsp_prev = 0.f, lsn_prev = 0.f;
      for (int t = 0; t < L; ++t) {
        float lsp, lsn;
        log_sigmoids(alpha * col[t * 64], lsp, lsn);
        if (t > 0) al_c -= expf(lsp) * lsp_prev + expf(lsn) * lsn_prev;  // BCE(p_{t-1}; q = p_t)
        log_keep += lsn;
        lsp_prev = lsp;
        lsn_prev = lsn;
      }
      al += double(al_c);
      cs += double(-expm1f(log_keep));  // 1 - prod_t (1 - p_t)
      const float K = expf(log_keep);
      float z_prev = 0.f, z = alpha * col[0];
      for (int t = 0; t < L; ++t) {
        const float z_next = t + 1 < L ? alpha * col[(t + 1) * 64] : 0.f;
        float lsp, lsn;
        log_sigmoids(z, lsp, lsn);
        const float p = expf(lsp), pq = expf(lsp + lsn);  // p and p (1 - p)
        float g_al = 0.f;
        if (t + 1 < L) {
          float lsp_n, lsn_n;
          log_sigmoids(z_next, lsp_n, lsn_n);
          g_al += p - expf(lsp_n);  // the predicting side: p_t - p_{t+1}
        }
        if (t > 0) g_al -= z_prev * pq;  // the target side of the pair (t-1, t)
        const float ds = f_al * g_al + f_cs * p * K;
        const size_t o = size_t(t_first + ty * L + t);
        sd[o * E + i] = ds;
        split_bf16(ds, dsh + o * Ep + i, dsl + o * Ep + i);
        z_prev = z;
        z = z_next;
      }
    } else if (ty < chunks) {  // padding experts of the split copy are zero
      for (int t = 0; t < L; ++t) {
        const size_t o = size_t(t_first + ty * L + t);
        dsh[o * Ep + i] = __float2bfloat16_rn(0.f);
        dsl[o * Ep + i] = __float2bfloat16_rn(0.f);
      }
    }
  }
  // fixed-order block sums
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    al += __shfl_xor_sync(0xffffffffu, al, o);
    cs += __shfl_xor_sync(0xffffffffu, cs, o);
  }
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = al;
    red[1][tid >> 5] = cs;
  }
  __syncthreads();
  if (tid == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) {
      a += red[0][w];
      b += red[1][w];
    }
    const size_t cta = size_t(blockIdx.y) * gridDim.x + blockIdx.x;
    loss_part[2 * cta] = a;
    loss_part[2 * cta + 1] = b;
  }
}

// dx = dS Wr^T for Ep <= 128: the CTA's 128 tokens of dS (hi and lo) stay in shared memory while up to
// 4 slices of 128 columns of Wr stream through two buffers.  Warp w owns tokens 32 (w & 3) .. +31 and
// columns 64 (w >> 2) .. +63 of each slice; dx is written with streaming stores (it is not read again).
__global__ void __launch_bounds__(kThreads, 2) dx_kernel(const __nv_bfloat16* __restrict__ dsh,
                                                         const __nv_bfloat16* __restrict__ dsl, int T, int Ep,
                                                         const __nv_bfloat16* __restrict__ wh,
                                                         const __nv_bfloat16* __restrict__ wl, int d,
                                                         float* __restrict__ dx) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wt = warp & 3, wc = warp >> 2;
  const int pitch = Ep + 8, chunks = Ep >> 3;
  const uint32_t tile_bytes = kTokTile * pitch * 2;
  const uint32_t ah = smem_u32(smem), al = ah + tile_bytes, wbuf = al + tile_bytes;  // wbuf: [2][hi, lo]
  const int t0 = blockIdx.x * kTokTile;
  const int n_slices_all = (d + kDTile - 1) / kDTile, s_first = blockIdx.y * kDxSlices;
  const int ns = min(kDxSlices, n_slices_all - s_first);

  for (int idx = tid; idx < kTokTile * chunks; idx += kThreads) {
    const int row = idx / chunks, ch = idx % chunks;
    const int gt = t0 + row;
    const bool ok = gt < T;
    const size_t off = ok ? size_t(gt) * Ep + ch * 8 : 0;
    cp_async16(ah + (row * pitch + ch * 8) * 2, dsh + off, ok ? 16 : 0);
    cp_async16(al + (row * pitch + ch * 8) * 2, dsl + off, ok ? 16 : 0);
  }
  auto load_w = [&](int j) {
    const uint32_t bh = wbuf + (j & 1) * 2 * tile_bytes, bl = bh + tile_bytes;
    const int k0 = (s_first + j) * kDTile;
    for (int idx = tid; idx < kDTile * chunks; idx += kThreads) {
      const int row = idx / chunks, ch = idx % chunks;
      const int gk = k0 + row;
      const bool ok = gk < d;
      const size_t off = ok ? size_t(gk) * Ep + ch * 8 : 0;
      cp_async16(bh + (row * pitch + ch * 8) * 2, wh + off, ok ? 16 : 0);
      cp_async16(bl + (row * pitch + ch * 8) * 2, wl + off, ok ? 16 : 0);
    }
  };
  load_w(0);
  cp_async_commit();  // group 0: the dS tile and slice 0
  if (ns > 1) load_w(1);
  cp_async_commit();  // group 1: slice 1 (possibly empty)
  const int g = lane >> 2, c = lane & 3;
  for (int j = 0; j < ns; ++j) {
    cp_async_wait<1>();  // groups 0 .. j are complete
    __syncthreads();
    const uint32_t bh = wbuf + (j & 1) * 2 * tile_bytes, bl = bh + tile_bytes;
    float acc[2][8][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int n = 0; n < 8; ++n) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
    for (int kk = 0; kk < Ep / 16; ++kk) {
      uint32_t a_h[2][4], a_l[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t ao = ((wt * 32 + mt * 16 + (lane & 15)) * pitch + kk * 16 + (lane >> 4) * 8) * 2;
        ldmatrix_x4(ah + ao, a_h[mt][0], a_h[mt][1], a_h[mt][2], a_h[mt][3]);
        ldmatrix_x4(al + ao, a_l[mt][0], a_l[mt][1], a_l[mt][2], a_l[mt][3]);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const uint32_t bo =
            ((wc * 64 + np * 16 + (lane & 7) + ((lane >> 4) << 3)) * pitch + kk * 16 + ((lane >> 3) & 1) * 8) * 2;
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        ldmatrix_x4(bh + bo, h0, h1, h2, h3);
        ldmatrix_x4(bl + bo, l0, l1, l2, l3);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma_bf16_16816(acc[mt][2 * np], a_h[mt], h0, h1);
          mma_bf16_16816(acc[mt][2 * np], a_h[mt], l0, l1);
          mma_bf16_16816(acc[mt][2 * np], a_l[mt], h0, h1);
          mma_bf16_16816(acc[mt][2 * np + 1], a_h[mt], h2, h3);
          mma_bf16_16816(acc[mt][2 * np + 1], a_h[mt], l2, l3);
          mma_bf16_16816(acc[mt][2 * np + 1], a_l[mt], h2, h3);
        }
      }
    }
    const int k0 = (s_first + j) * kDTile + wc * 64;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int k = k0 + nt * 8 + 2 * c;
        if (k >= d) continue;  // d % 8 == 0: the pair (k, k+1) is whole
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = t0 + wt * 32 + mt * 16 + g + 8 * h;
          if (t < T)
            __stcs(reinterpret_cast<float2*>(dx + size_t(t) * d + k), make_float2(acc[mt][nt][2 * h], acc[mt][nt][2 * h + 1]));
        }
      }
    __syncthreads();  // buffer j & 1 is no longer read
    if (j + 2 < ns) load_w(j + 2);
    cp_async_commit();
  }
  cp_async_wait<0>();
}

// dx for any Ep (wider expert sets): one 128 x 128 tile per CTA, the experts in slices of 64.  Warp w
// owns tokens 16w .. 16w+15 and all 128 columns.
__global__ void __launch_bounds__(kThreads) dx_wide_kernel(const __nv_bfloat16* __restrict__ dsh,
                                                           const __nv_bfloat16* __restrict__ dsl, int T, int Ep,
                                                           const __nv_bfloat16* __restrict__ wh,
                                                           const __nv_bfloat16* __restrict__ wl, int d,
                                                           float* __restrict__ dx) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kABytes = kTokTile * kPitch * 2, kBBytes = kDTile * kPitch * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kTokTile, k0 = blockIdx.y * kDTile;
  const uint32_t ah = smem_u32(smem), al = ah + kABytes, bh = al + kABytes, bl = bh + kBBytes;
  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  for (int e0 = 0; e0 < Ep; e0 += kKTile) {
    if (e0 > 0) __syncthreads();  // the previous slice is no longer read
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int idx = tid + j * kThreads, row = idx >> 3, ch = idx & 7;
      const uint32_t so = (row * kPitch + ch * 8) * 2;
      const int gt = t0 + row, gk = k0 + row;
      const bool okt = gt < T, okk = gk < d;
      const size_t ot = okt ? size_t(gt) * Ep + e0 + ch * 8 : 0, ok_ = okk ? size_t(gk) * Ep + e0 + ch * 8 : 0;
      cp_async16(ah + so, dsh + ot, okt ? 16 : 0);
      cp_async16(al + so, dsl + ot, okt ? 16 : 0);
      cp_async16(bh + so, wh + ok_, okk ? 16 : 0);
      cp_async16(bl + so, wl + ok_, okk ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kKTile / 16; ++kk) {
      uint32_t a_h[4], a_l[4];
      const uint32_t ao = ((warp * 16 + (lane & 15)) * kPitch + kk * 16 + (lane >> 4) * 8) * 2;
      ldmatrix_x4(ah + ao, a_h[0], a_h[1], a_h[2], a_h[3]);
      ldmatrix_x4(al + ao, a_l[0], a_l[1], a_l[2], a_l[3]);
#pragma unroll
      for (int np = 0; np < kDTile / 16; ++np) {
        const uint32_t bo = ((np * 16 + (lane & 7) + ((lane >> 4) << 3)) * kPitch + kk * 16 + ((lane >> 3) & 1) * 8) * 2;
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        ldmatrix_x4(bh + bo, h0, h1, h2, h3);
        ldmatrix_x4(bl + bo, l0, l1, l2, l3);
        mma_bf16_16816(acc[2 * np], a_h, h0, h1);
        mma_bf16_16816(acc[2 * np], a_h, l0, l1);
        mma_bf16_16816(acc[2 * np], a_l, h0, h1);
        mma_bf16_16816(acc[2 * np + 1], a_h, h2, h3);
        mma_bf16_16816(acc[2 * np + 1], a_h, l2, l3);
        mma_bf16_16816(acc[2 * np + 1], a_l, h2, h3);
      }
    }
  }
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int k = k0 + nt * 8 + 2 * c;
    if (k >= d) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = t0 + warp * 16 + g + 8 * h;
      if (t < T) __stcs(reinterpret_cast<float2*>(dx + size_t(t) * d + k), make_float2(acc[nt][2 * h], acc[nt][2 * h + 1]));
    }
  }
}

// part[split, k0 .. k0+128, e0 .. e0+64] = x[split]^T dS[split].  Warp w owns rows 64 (w & 1) .. +63 of
// Wr and experts 32 (w >> 1) .. +31.  The CTAs of one split share its db: the CTA in column x of the grid
// adds up the dS of the pipeline stages kt with kt % gridDim.x == x (64 tokens each) into
// db_part[split, x].
__global__ void __launch_bounds__(kGemmThreads) dwr_kernel(const __nv_bfloat16* __restrict__ x, int T, int d,
                                                           const __nv_bfloat16* __restrict__ dsh,
                                                           const __nv_bfloat16* __restrict__ dsl, int Ep,
                                                           int tok_per_split, float* __restrict__ part,
                                                           float* __restrict__ db_part) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float sdb[2][64];
  constexpr int kXBytes = kSplitTok * kPitchWide * 2, kDBytes = kSplitTok * kPitch * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wm = warp & 1, wn = warp >> 1;
  const int k0 = blockIdx.x * kDTile, e0 = blockIdx.z * kNTile;
  const int ts = blockIdx.y * tok_per_split, te = min(T, ts + tok_per_split);
  const int nt = (te - ts + kSplitTok - 1) / kSplitTok;
  const uint32_t sbase = smem_u32(smem);

  auto load = [&](int kt) {
    const uint32_t st = sbase + (kt % kStages) * kDwrStage;
    const int tok0 = ts + kt * kSplitTok;
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // x: 64 tokens x 16 pieces of 16 B
      const int idx = tid + j * kGemmThreads, row = idx >> 4, ch = idx & 15;
      const int gt = tok0 + row, gk = k0 + ch * 8;
      const bool ok = gt < te && gk < d;
      cp_async16(st + (row * kPitchWide + ch * 8) * 2, ok ? x + size_t(gt) * d + gk : x, ok ? 16 : 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // dS hi and lo: 64 tokens x 8 pieces each
      const int idx = tid + j * kGemmThreads, row = idx >> 3, ch = idx & 7;
      const int gt = tok0 + row;
      const bool ok = gt < te;
      const size_t off = ok ? size_t(gt) * Ep + e0 + ch * 8 : 0;
      cp_async16(st + kXBytes + (row * kPitch + ch * 8) * 2, dsh + off, ok ? 16 : 0);
      cp_async16(st + kXBytes + kDBytes + (row * kPitch + ch * 8) * 2, dsl + off, ok ? 16 : 0);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 4; ++n) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
  float dbacc = 0.f;
#pragma unroll
  for (int kt = 0; kt < kStages - 1; ++kt) {
    if (kt < nt) load(kt);
    cp_async_commit();
  }
  for (int kt = 0; kt < nt; ++kt) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (kt + kStages - 1 < nt) load(kt + kStages - 1);
    cp_async_commit();
    const uint32_t xs = sbase + (kt % kStages) * kDwrStage, dhs = xs + kXBytes, dls = dhs + kDBytes;
    if (kt % int(gridDim.x) == int(blockIdx.x)) {  // this CTA's share of db: thread (half, expert)
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(smem + (dhs - sbase));
      const __nv_bfloat16* l = reinterpret_cast<const __nv_bfloat16*>(smem + (dls - sbase));
      const int e = tid & 63, r0 = (tid >> 6) * 32;
      for (int r = r0; r < r0 + 32; ++r)
        dbacc += __bfloat162float(h[r * kPitch + e]) + __bfloat162float(l[r * kPitch + e]);
    }
#pragma unroll
    for (int kk = 0; kk < kSplitTok / 16; ++kk) {
      uint32_t a[4][4];  // A = x^T: rows are Wr rows (columns of x), k runs over tokens
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        ldmatrix_x4_trans(xs + ((kk * 16 + (lane & 7) + ((lane >> 4) << 3)) * kPitchWide + wm * 64 + mt * 16 +
                                ((lane >> 3) & 1) * 8) * 2,
                          a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const uint32_t off = ((kk * 16 + (lane & 15)) * kPitch + wn * 32 + np * 16 + (lane >> 4) * 8) * 2;
        uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
        ldmatrix_x4_trans(dhs + off, h0, h1, h2, h3);
        ldmatrix_x4_trans(dls + off, l0, l1, l2, l3);
        mma_pair(acc, a, np, h0, h1, h2, h3, l0, l1, l2, l3);
      }
    }
  }
  cp_async_wait<0>();
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int e = e0 + wn * 32 + n * 8 + 2 * c;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = k0 + wm * 64 + mt * 16 + g + 8 * h;
        if (k < d)
          *reinterpret_cast<float2*>(part + (size_t(blockIdx.y) * d + k) * Ep + e) =
              make_float2(acc[mt][n][2 * h], acc[mt][n][2 * h + 1]);
      }
    }
  sdb[tid >> 6][tid & 63] = dbacc;
  __syncthreads();
  if (tid < 64)
    db_part[(size_t(blockIdx.y) * gridDim.x + blockIdx.x) * Ep + e0 + tid] = sdb[0][tid] + sdb[1][tid];
}

// CTA 0: the losses; CTAs [1, 1 + n_eg): db for experts 64 (b-1) .. +63; the rest: dWr, one element per
// thread.  Every sum runs in a fixed order.
__global__ void __launch_bounds__(kReduceThreads) reduce_kernel(const float* __restrict__ part, int splits, int d,
                                                                int E, int Ep, float* __restrict__ dWr,
                                                                const float* __restrict__ db_part, int db_rows,
                                                                float* __restrict__ db,
                                                                const double* __restrict__ loss_part, int n_loss,
                                                                double inv_al, double inv_cs,
                                                                float* __restrict__ loss) {
  const int tid = threadIdx.x;
  const int n_eg = Ep / 64;
  if (blockIdx.x == 0) {
    __shared__ double sl[2][kReduceThreads / 32];
    double a = 0.0, b = 0.0;
    for (int q = tid; q < n_loss; q += kReduceThreads) {
      a += loss_part[2 * q];
      b += loss_part[2 * q + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if ((tid & 31) == 0) {
      sl[0][tid >> 5] = a;
      sl[1][tid >> 5] = b;
    }
    __syncthreads();
    if (tid == 0) {
      double sa = 0.0, sb = 0.0;
      for (int w = 0; w < kReduceThreads / 32; ++w) {
        sa += sl[0][w];
        sb += sl[1][w];
      }
      loss[0] = float(sa * inv_al);
      loss[1] = float(sb * inv_cs);
    }
    return;
  }
  if (int(blockIdx.x) <= n_eg) {
    if (db == nullptr) return;
    __shared__ float sdb[16][64];
    const int e = (blockIdx.x - 1) * 64 + (tid & 63), rg = tid >> 6;  // 16 row groups
    float acc = 0.f;
#pragma unroll 4
    for (int r = rg; r < db_rows; r += 16) acc += db_part[size_t(r) * Ep + e];
    sdb[rg][tid & 63] = acc;
    __syncthreads();
    if (tid < 64 && e < E) {
      float v = 0.f;
      for (int q = 0; q < 16; ++q) v += sdb[q][tid];
      db[e] = v;
    }
    return;
  }
  if (dWr == nullptr) return;
  const size_t q = size_t(blockIdx.x - 1 - n_eg) * kReduceThreads + tid;
  if (q >= size_t(d) * E) return;
  const int k = int(q / E), e = int(q % E);
  float v = 0.f;
#pragma unroll 6
  for (int sp = 0; sp < splits; ++sp) v += part[(size_t(sp) * d + k) * Ep + e];
  dWr[q] = v;
}

}  // namespace

Plan plan(int C, int L, int d, int E) {
  Plan p{};
  const long long T = 1ll * C * L;
  p.T = int(T);
  p.Ep = (E + 63) / 64 * 64;
  const int n_eg = p.Ep / 64;
  p.dtiles = (d + kDTile - 1) / kDTile;
  const int target = std::max(1, kTargetCtas / (p.dtiles * n_eg));
  const long long per = (T + target - 1) / target;
  p.tok_per_split = int((per + kSplitTok - 1) / kSplitTok * kSplitTok);
  p.splits = int((T + p.tok_per_split - 1) / p.tok_per_split);
  const long long groups = (C + kChunksPerTile - 1) / kChunksPerTile;
  p.b_rows = int(std::min<long long>(groups, std::max(1, kTargetCtasTerms / n_eg)));
  size_t off = 0;
  p.wr_off = off;
  off = align256(off + 2 * size_t(d) * p.Ep * 2);
  p.ds_off = off;
  off = align256(off + 2 * size_t(T) * p.Ep * 2);
  p.part_off = off;
  off = align256(off + size_t(p.splits) * d * p.Ep * 4);
  p.loss_off = off;
  off = align256(off + size_t(p.b_rows) * n_eg * 2 * sizeof(double));
  p.db_off = off;
  off = align256(off + size_t(p.splits) * p.dtiles * p.Ep * 4);
  p.total = off;
  return p;
}

bool chunk_fits(int L) { return size_t(kChunksPerTile) * L * 64 * 4 <= size_t(kMaxChunkTileBytes); }

cudaError_t launch(const void* x, int C, int L, int d, const float* Wr, const float* br, int E, float alpha,
                   float w_al, float w_cs, float* loss, float* dS, float* dWr, float* db, float* dx, void* ws,
                   int num_sms, cudaStream_t st) {
  const Plan p = plan(C, L, d, E);
  const bool dx_tile = p.Ep <= kDxMaxEp;
  cudaError_t err;
  if ((err = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouterSmem)) !=
      cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(dx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dx_smem(kDxMaxEp))) !=
      cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(dx_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDxWideSmem)) !=
      cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(dwr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDwrSmem)) != cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(chunk_terms_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kMaxChunkTileBytes)) != cudaSuccess)
    return err;
  uint8_t* base = static_cast<uint8_t*>(ws);
  __nv_bfloat16* wh = reinterpret_cast<__nv_bfloat16*>(base + p.wr_off);
  __nv_bfloat16* wl = wh + size_t(d) * p.Ep;
  __nv_bfloat16* dsh = reinterpret_cast<__nv_bfloat16*>(base + p.ds_off);
  __nv_bfloat16* dsl = dsh + size_t(p.T) * p.Ep;
  float* part = reinterpret_cast<float*>(base + p.part_off);
  double* loss_part = reinterpret_cast<double*>(base + p.loss_off);
  float* db_part = reinterpret_cast<float*>(base + p.db_off);
  const int n_eg = p.Ep / 64;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const unsigned tok_tiles = unsigned((p.T + kTokTile - 1) / kTokTile);

  const size_t nw = size_t(d) * p.Ep;
  split_wr_kernel<<<unsigned(std::min<size_t>((nw + kThreads - 1) / kThreads, size_t(num_sms) * 8)), kThreads, 0,
                    st>>>(Wr, d, E, p.Ep, wh, wl);
  router_gemm_kernel<<<dim3(tok_tiles, n_eg), kGemmThreads, kRouterSmem, st>>>(xb, p.T, d, wh, wl, p.Ep, br, E, dS,
                                                                             d);
  const double n_al = double(C) * (L - 1) * E, n_cs = double(C) * E;
  const float f_al = L > 1 ? float(double(w_al) * alpha / n_al) : 0.f;
  const float f_cs = float(double(w_cs) * alpha / n_cs);
  chunk_terms_kernel<<<dim3(n_eg, p.b_rows), kThreads, size_t(kChunksPerTile) * L * 64 * 4, st>>>(
      dS, C, L, E, p.Ep, alpha, f_al, f_cs, dsh, dsl, loss_part);
  if (dx != nullptr) {
    if (dx_tile)
      dx_kernel<<<dim3(tok_tiles, (p.dtiles + kDxSlices - 1) / kDxSlices), kThreads, dx_smem(p.Ep), st>>>(
          dsh, dsl, p.T, p.Ep, wh, wl, d, dx);
    else
      dx_wide_kernel<<<dim3(tok_tiles, p.dtiles), kThreads, kDxWideSmem, st>>>(dsh, dsl, p.T, p.Ep, wh, wl, d, dx);
  }
  if (dWr != nullptr || db != nullptr)
    dwr_kernel<<<dim3(p.dtiles, p.splits, n_eg), kGemmThreads, kDwrSmem, st>>>(xb, p.T, d, dsh, dsl, p.Ep,
                                                                               p.tok_per_split, part, db_part);
  const size_t n_dwr = dWr != nullptr ? size_t(d) * E : 0;
  const unsigned grid_r = unsigned(1 + n_eg + (n_dwr + kReduceThreads - 1) / kReduceThreads);
  reduce_kernel<<<grid_r, kReduceThreads, 0, st>>>(part, p.splits, d, E, p.Ep, dWr, db_part, p.splits * p.dtiles, db,
                                                    loss_part, p.b_rows * n_eg, L > 1 ? 1.0 / n_al : 0.0,
                                                    1.0 / n_cs, loss);
  return cudaGetLastError();
}

int router_projection_parts(int T, int d, int E, int num_sms) {
  const long long tiles = 1ll * ((T + kTokTile - 1) / kTokTile) * ((E + 63) / 64);
  const int kt = (d + kKTile - 1) / kKTile;  // 64-column slices of x
  long long parts = (2ll * num_sms + tiles - 1) / tiles;
  if (parts > kMaxRouterParts) parts = kMaxRouterParts;
  if (parts > kt) parts = kt;
  const int per = (kt + int(parts) - 1) / int(parts);  // slices per part
  return (kt + per - 1) / per;
}

cudaError_t router_projection(const __nv_bfloat16* x, int T, int d, const float* Wr, int E, __nv_bfloat16* wsplit,
                              float* s, int parts, int num_sms, cudaStream_t st) {
  cudaError_t err =
      cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouterSmem);
  if (err != cudaSuccess) return err;
  const int Ep = (E + 63) / 64 * 64;
  const size_t nw = size_t(d) * Ep;
  __nv_bfloat16* wh = wsplit;
  __nv_bfloat16* wl = wsplit + nw;
  const int kt = (d + kKTile - 1) / kKTile, kper = (kt + parts - 1) / parts * kKTile;
  split_wr_kernel<<<unsigned(std::min<size_t>((nw + kThreads - 1) / kThreads, size_t(num_sms) * 8)), kThreads, 0,
                    st>>>(Wr, d, E, Ep, wh, wl);
  router_gemm_kernel<<<dim3(unsigned((T + kTokTile - 1) / kTokTile), Ep / 64, parts), kGemmThreads, kRouterSmem,
                       st>>>(x, T, d, wh, wl, Ep, nullptr, E, s, kper);
  return cudaGetLastError();
}

}  // namespace cls
}  // namespace bffn
