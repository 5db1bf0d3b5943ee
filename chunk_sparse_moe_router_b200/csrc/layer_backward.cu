// The BlockFFN layer's backward (the training side of the layer of lsdiaocha.cn BlockFFN article, section 2:
// ReLU + RMSNorm router, non-gated Swish experts weighted by r).  The pages print no backward; this is the
// chain rule through the forward, for upstream gradient dy.  Only the (token, expert) pairs with s > 0 (the
// ReLU active) take part: every other pair has a = 0 and r = 0, so its terms below are exact zeros (and its
// dr is multiplied by a = 0 or masked by [s > 0] in the router backward).  Per expert e with active tokens
// T_e (grouped by expert, ascending token order within an expert):
//   U_e = X[T_e] W1_e^T,  Q_e = dY[T_e] W2_e                  (pair rows, [|T_e|, de])
//   h = Swish(U), dr_te = sum_j h Q, RH = r h, DU = r Q Swish'(U)
//   dW2_e = dY[T_e]^T RH_e,  dW1_e = DU_e^T X[T_e],  dX[t] = sum_{e: t in T_e} DU_e[t] W1_e
//   router: r = g a / rho, a = relu(s), rho = rms(a):  dg = sum_t dr a / rho,
//           da = g dr / rho - a sum_i(dr g a) / (E rho^3),  dS = da [s > 0]
//   dWr = X^T dS,  db = sum_t dS,  dX += dS Wr^T
// Every contraction runs through one tiled GEMM on the warp tensor cores (mma.sync bf16, fp32
// accumulate), grouped over the experts where a dimension is the expert's pairs (rows gathered through the
// pair -> token list); fp32 operands (dy, RH, DU, dS, Wr) are carried as bf16 hi + lo pairs (about 2^-17
// relative) and the lo x lo product is dropped.  dX's expert terms are written per pair and added per
// token in expert order.  Every sum runs in a fixed order: results are bit-reproducible.
#include <algorithm>

#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace bwd {
namespace {

constexpr int kT = 256;          // GEMM: 8 warps, each a 64 x 32 tile of the 128 x 128 CTA tile
constexpr int kBM = 128, kBN = 128, kBK = 32;
constexpr int kStages = 3;
constexpr int kKPitch = kBK + 8;        // K-major tiles: rows of 32 k (80 B): 8 ldmatrix rows on 32 banks
constexpr int kMPitch = kBM + 8;        // M/N-major tiles: rows of 128 (272 B)
constexpr int kPart = 10240;            // bytes of one operand part of a stage (the larger layout, 128 x 80 B)

struct GemmArgs {
  const __nv_bfloat16 *a_hi, *a_lo, *b_hi, *b_lo;
  float* c;
  int M, N, K;
  long long lda, ldb, ldc;          // elements between consecutive stored rows
  long long sa, sb, sc;             // batch strides (blockIdx.z) of operands that are not grouped
  const int* goff;                  // grouped GEMMs: batch z owns pairs goff[z] .. goff[z + 1] - 1
  const int* tok;                   // pair -> token
};

// Stored-row modes of an operand: kPlain (row r of the batch's matrix, at z times its batch stride),
// kPairs (row goff[z] + r of a pair-major array), kTokens (row tok[goff[z] + r] of a token-major array).
constexpr int kPlain = 0, kPairs = 1, kTokens = 2;
// Grouping: none; M is batch z's pair count (C rows are pair rows); K is batch z's pair count.
constexpr int kNoGroup = 0, kGroupM = 1, kGroupK = 2;

// C[m][n] = sum_k A[m][k] B[k][n].  A K-major: A[m][k] = a[m lda + k]; else A[k][m] = a[k lda + m].
// B K-major: B[k][n] = b[n ldb + k]; else b[k ldb + n].  ASPLIT / BSPLIT: the operand is hi + lo.  The stored
// row (m or n of a K-major operand, k otherwise) goes through the operand's mode AMODE / BMODE.
template <bool AK, bool ASPLIT, bool BK, bool BSPLIT, int AMODE, int BMODE, int GRP>
__global__ void __launch_bounds__(kT) gemm_kernel(const GemmArgs g) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kParts = (ASPLIT ? 2 : 1) + (BSPLIT ? 2 : 1);
  constexpr int kStage = kParts * kPart;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wm = warp & 1, wn = warp >> 1;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN, z = blockIdx.z;
  int base = 0, Mz = g.M, Kz = g.K;
  if (GRP != kNoGroup) {
    base = g.goff[z];
    const int cnt = g.goff[z + 1] - base;
    if (GRP == kGroupM) Mz = cnt;
    else Kz = cnt;
  }
  if (m0 >= Mz) return;  // a row tile past this batch's pairs (the grid covers the largest batch)
  const long long za = AMODE == kPlain ? z * g.sa : 0, zb = BMODE == kPlain ? z * g.sb : 0;
  const __nv_bfloat16* A[2] = {g.a_hi + za, ASPLIT ? g.a_lo + za : nullptr};
  const __nv_bfloat16* B[2] = {g.b_hi + zb, BSPLIT ? g.b_lo + zb : nullptr};
  float* C = g.c + (GRP == kGroupM ? 0 : z * g.sc);
  const int nk = (Kz + kBK - 1) / kBK;
  const uint32_t sbase = smem_u32(smem);

  // the stored row of local row r (r already checked against its bound)
  auto stored_row = [&](int mode, int r) -> long long {
    if (mode == kPairs) return (long long)base + r;
    if (mode == kTokens) return g.tok[base + r];
    return r;
  };
  auto load_tile = [&](uint32_t dst, const __nv_bfloat16* src, bool kmajor, int mode, int outer0, int outer_n,
                       long long ld, int k0) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {  // 512 pieces of 16 B
      const int idx = tid + q * kT;
      if (kmajor) {  // [128 outer][32 k]: 4 pieces per row
        const int row = idx >> 2, ch = idx & 3;
        const int o = outer0 + row, k = k0 + ch * 8;
        const bool ok = o < outer_n && k < Kz;
        cp_async16(dst + (row * kKPitch + ch * 8) * 2, ok ? src + stored_row(mode, o) * ld + k : src, ok ? 16 : 0);
      } else {  // [32 k][128 outer]: 16 pieces per row
        const int row = idx >> 4, ch = idx & 15;
        const int k = k0 + row, o = outer0 + ch * 8;
        const bool ok = k < Kz && o < outer_n;
        cp_async16(dst + (row * kMPitch + ch * 8) * 2, ok ? src + stored_row(mode, k) * ld + o : src, ok ? 16 : 0);
      }
    }
  };
  auto load = [&](int kt) {
    const uint32_t st = sbase + (kt % kStages) * kStage;
    const int k0 = kt * kBK;
    load_tile(st, A[0], AK, AMODE, m0, Mz, g.lda, k0);
    if (ASPLIT) load_tile(st + kPart, A[1], AK, AMODE, m0, Mz, g.lda, k0);
    const uint32_t sb = st + (ASPLIT ? 2 : 1) * kPart;
    load_tile(sb, B[0], BK, BMODE, n0, g.N, g.ldb, k0);
    if (BSPLIT) load_tile(sb + kPart, B[1], BK, BMODE, n0, g.N, g.ldb, k0);
  };

  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = acc[a][b][2] = acc[a][b][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < kStages - 1; ++kt) {
    if (kt < nk) load(kt);
    cp_async_commit();
  }
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (kt + kStages - 1 < nk) load(kt + kStages - 1);
    cp_async_commit();
    const uint32_t st = sbase + (kt % kStages) * kStage;
    const uint32_t sa[2] = {st, st + kPart};
    const uint32_t sbb = st + (ASPLIT ? 2 : 1) * kPart;
    const uint32_t sb[2] = {sbb, sbb + kPart};
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk) {
      uint32_t a[2][4][4];  // [part][m-tile][reg]
#pragma unroll
      for (int pa = 0; pa < (ASPLIT ? 2 : 1); ++pa)
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int mb = wm * 64 + mt * 16;
          if (AK)
            ldmatrix_x4(sa[pa] + ((mb + (lane & 15)) * kKPitch + kk * 16 + (lane >> 4) * 8) * 2, a[pa][mt][0],
                        a[pa][mt][1], a[pa][mt][2], a[pa][mt][3]);
          else
            ldmatrix_x4_trans(
                sa[pa] + ((kk * 16 + (lane & 7) + ((lane >> 4) << 3)) * kMPitch + mb + ((lane >> 3) & 1) * 8) * 2,
                a[pa][mt][0], a[pa][mt][1], a[pa][mt][2], a[pa][mt][3]);
        }
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int nb = wn * 32 + np * 16;
        uint32_t b[2][4];  // [part]: (b0, b1) of n-tile 2 np, (b2, b3) of 2 np + 1
#pragma unroll
        for (int pb = 0; pb < (BSPLIT ? 2 : 1); ++pb) {
          if (BK)
            ldmatrix_x4(sb[pb] + ((nb + (lane & 7) + ((lane >> 4) << 3)) * kKPitch + kk * 16 + ((lane >> 3) & 1) * 8) * 2,
                        b[pb][0], b[pb][1], b[pb][2], b[pb][3]);
          else
            ldmatrix_x4_trans(sb[pb] + ((kk * 16 + (lane & 15)) * kMPitch + nb + (lane >> 4) * 8) * 2, b[pb][0],
                              b[pb][1], b[pb][2], b[pb][3]);
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float* d = acc[mt][2 * np + h];
            mma_bf16_16816(d, a[0][mt], b[0][2 * h], b[0][2 * h + 1]);
            if (BSPLIT) mma_bf16_16816(d, a[0][mt], b[1][2 * h], b[1][2 * h + 1]);
            if (ASPLIT) mma_bf16_16816(d, a[1][mt], b[0][2 * h], b[0][2 * h + 1]);
          }
      }
    }
  }
  cp_async_wait<0>();
  const int gq = lane >> 2, cq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int n = n0 + wn * 32 + nt * 8 + 2 * cq;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + wm * 64 + mt * 16 + gq + 8 * h;
        if (m >= Mz) continue;
        const long long crow = GRP == kGroupM ? (long long)base + m : m;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (n + q >= g.N) continue;
          float* p = C + crow * g.ldc + n + q;
          *p = acc[mt][nt][2 * h + q];
        }
      }
    }
}

// M (for kGroupM: the largest batch's pair count, at most T) sets the grid's row tiles.
template <bool AK, bool ASPLIT, bool BK, bool BSPLIT, int AMODE = kPlain, int BMODE = kPlain,
          int GRP = kNoGroup>
cudaError_t gemm(const GemmArgs& g, int batch, cudaStream_t st) {
  constexpr int kParts = (ASPLIT ? 2 : 1) + (BSPLIT ? 2 : 1);
  const int smem = kStages * kParts * kPart;
  auto fn = gemm_kernel<AK, ASPLIT, BK, BSPLIT, AMODE, BMODE, GRP>;
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  fn<<<dim3((g.N + kBN - 1) / kBN, (g.M + kBM - 1) / kBM, batch), kT, smem, st>>>(g);
  return cudaGetLastError();
}

__device__ __forceinline__ void split2(float v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *hi = h;
  *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

// src [rows][cols] fp32 (row stride cols) -> hi, lo [rows][ld] bf16, columns cols .. ld-1 zero.
__global__ void __launch_bounds__(256) split_kernel(const float* __restrict__ src, long long rows, int cols, int ld,
                                                    __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  const long long n = rows * ld;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n; q += (long long)gridDim.x * blockDim.x) {
    const long long r = q / ld;
    const int c = int(q - r * ld);
    split2(c < cols ? src[r * cols + c] : 0.f, hi + q, lo + q);
  }
}

// Per token (one warp): s = the router parts in order + b; a = relu(s); rho; r = g a / rho (0 when rho = 0).
__global__ void __launch_bounds__(256) router_fwd_kernel(const float* __restrict__ parts, int P, int T, int E,
                                                         const float* __restrict__ br, const float* __restrict__ g,
                                                         float* __restrict__ s, float* __restrict__ r,
                                                         float* __restrict__ rho) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (t >= T) return;
  float sumsq = 0.f;
  for (int i = lane; i < E; i += 32) {
    float v = 0.f;
    for (int k = 0; k < P; ++k) v += parts[(size_t(k) * T + t) * E + i];
    v += br ? br[i] : 0.f;
    s[size_t(t) * E + i] = v;
    const float a = fmaxf(v, 0.f);
    sumsq = fmaf(a, a, sumsq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
  const float rh = sqrtf(sumsq / float(E));
  if (lane == 0) rho[t] = rh;
  for (int i = lane; i < E; i += 32) {
    const float a = fmaxf(s[size_t(t) * E + i], 0.f);
    r[size_t(t) * E + i] = rh > 0.f ? g[i] * a / rh : 0.f;
  }
}

// Grouping of the active pairs (s > 0) by expert, in ascending token order within an expert.
// cnt[e]: one CTA per expert counts its active tokens.
__global__ void __launch_bounds__(256) group_count_kernel(const float* __restrict__ s, int T, int E,
                                                          int* __restrict__ cnt) {
  __shared__ int part[8];
  const int e = blockIdx.x;
  int c = 0;
  for (int t = threadIdx.x; t < T; t += 256) c += s[size_t(t) * E + e] > 0.f ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int sum = 0;
    for (int w = 0; w < 8; ++w) sum += part[w];
    cnt[e] = sum;
  }
}

// goff[e] = sum of cnt over experts before e (goff[E] = the pair count); one thread, E <= 1024 steps.
__global__ void group_scan_kernel(const int* __restrict__ cnt, int E, int* __restrict__ goff) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int run = 0;
  for (int e = 0; e < E; ++e) {
    goff[e] = run;
    run += cnt[e];
  }
  goff[E] = run;
}

// One CTA per expert walks the tokens in order, 256 at a time: the active ones get consecutive pair indices
// from goff[e]: tok[pair] = t, pexp[pair] = e, pidx[t][e] = pair (-1 for an inactive pair).
__global__ void __launch_bounds__(256) group_fill_kernel(const float* __restrict__ s, int T, int E,
                                                         const int* __restrict__ goff, int* __restrict__ tok,
                                                         int* __restrict__ pexp, int* __restrict__ pidx) {
  __shared__ int wsum[8];
  const int e = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int run = goff[e];
  for (int t0 = 0; t0 < T; t0 += 256) {
    const int t = t0 + threadIdx.x;
    const bool on = t < T && s[size_t(t) * E + e] > 0.f;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (lane == 0) wsum[w] = __popc(bal);
    __syncthreads();
    int before = run;
    for (int q = 0; q < w; ++q) before += wsum[q];
    int total = 0;
    for (int q = 0; q < 8; ++q) total += wsum[q];
    const int pos = before + __popc(bal & ((1u << lane) - 1u));
    if (t < T) {
      pidx[size_t(t) * E + e] = on ? pos : -1;
      if (on) {
        tok[pos] = t;
        pexp[pos] = e;
      }
    }
    run += total;
    __syncthreads();  // wsum is rewritten by the next block of tokens
  }
}

// Per active pair (one warp): h = Swish(u), dr_te = sum_j h q, RH = r h and DU = r q Swish'(u) as hi + lo,
// all pair-major ([pair][de]).
__global__ void __launch_bounds__(256) expert_pointwise_kernel(const float* __restrict__ U, const float* __restrict__ Q,
                                                               const float* __restrict__ r, const int* __restrict__ tok,
                                                               const int* __restrict__ pexp,
                                                               const int* __restrict__ goff, int E, int de,
                                                               float* __restrict__ dr, __nv_bfloat16* __restrict__ rh_hi,
                                                               __nv_bfloat16* __restrict__ rh_lo,
                                                               __nv_bfloat16* __restrict__ du_hi,
                                                               __nv_bfloat16* __restrict__ du_lo) {
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= goff[E]) return;
  const int t = tok[w], e = pexp[w];
  const float re = r[size_t(t) * E + e];
  const size_t base = size_t(w) * de;
  float acc = 0.f;
  for (int j = lane; j < de; j += 32) {
    const float u = U[base + j], q = Q[base + j];
    const float sg = 1.f / (1.f + expf(-u));
    const float h = u * sg;
    acc = fmaf(h, q, acc);
    split2(re * h, rh_hi + base + j, rh_lo + base + j);
    split2(re * q * (sg * (1.f + u * (1.f - sg))), du_hi + base + j, du_lo + base + j);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) dr[size_t(t) * E + e] = acc;
}

// dx[t] += the expert terms of token t's pairs, in expert order (one CTA per token).
__global__ void __launch_bounds__(256) pair_reduce_kernel(const float* __restrict__ xp, const int* __restrict__ pidx,
                                                          int T, int E, int d, float* __restrict__ dx) {
  extern __shared__ int plist[];  // the token's pair indices, ascending expert
  __shared__ int np;
  const int t = blockIdx.x;
  if (t >= T) return;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int e = 0; e < E; ++e) {
      const int q = pidx[size_t(t) * E + e];
      if (q >= 0) plist[n++] = q;
    }
    np = n;
  }
  __syncthreads();
  const int n = np;
  float* out = dx + size_t(t) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = out[c];
    for (int i = 0; i < n; ++i) acc += xp[size_t(plist[i]) * d + c];
    out[c] = acc;
  }
}

// Per token (one warp): the RMSNorm / ReLU backward: dS (fp32 [T, E] and hi + lo [T, Ep], padding zero) and
// the token's share of dg (dr a / rho).
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ s, const float* __restrict__ rho,
                                                         const float* __restrict__ dr, const float* __restrict__ g,
                                                         int T, int E, int Ep, float* __restrict__ ds,
                                                         float* __restrict__ dgc, __nv_bfloat16* __restrict__ ds_hi,
                                                         __nv_bfloat16* __restrict__ ds_lo) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (t >= T) return;
  const float rh = rho[t];
  float c = 0.f;  // sum_i dr_i g_i a_i
  for (int i = lane; i < E; i += 32) c = fmaf(dr[size_t(t) * E + i] * g[i], fmaxf(s[size_t(t) * E + i], 0.f), c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  for (int i = lane; i < Ep; i += 32) {
    float v = 0.f, dgv = 0.f;
    if (i < E && rh > 0.f) {
      const float sv = s[size_t(t) * E + i], a = fmaxf(sv, 0.f), d_r = dr[size_t(t) * E + i];
      dgv = d_r * a / rh;
      const float da = g[i] * d_r / rh - a * c / (float(E) * rh * rh * rh);
      v = sv > 0.f ? da : 0.f;
    }
    if (i < E) {
      ds[size_t(t) * E + i] = v;
      dgc[size_t(t) * E + i] = dgv;
    }
    split2(v, ds_hi + size_t(t) * Ep + i, ds_lo + size_t(t) * Ep + i);
  }
}

// Column sums of two [T, E] arrays in a fixed order: 32 experts x 8 row groups per CTA.
__global__ void __launch_bounds__(256) colsum2_kernel(const float* __restrict__ a, const float* __restrict__ b, int T,
                                                      int E, float* __restrict__ sa, float* __restrict__ sb) {
  __shared__ float pa[8][32], pb[8][32];
  const int i = blockIdx.x * 32 + (threadIdx.x & 31), rg = threadIdx.x >> 5;
  float x = 0.f, y = 0.f;
  if (i < E)
    for (int t = rg; t < T; t += 8) {
      x += a[size_t(t) * E + i];
      y += b[size_t(t) * E + i];
    }
  pa[rg][threadIdx.x & 31] = x;
  pb[rg][threadIdx.x & 31] = y;
  __syncthreads();
  if (rg == 0 && i < E) {
    float u = 0.f, v = 0.f;
    for (int q = 0; q < 8; ++q) {
      u += pa[q][threadIdx.x];
      v += pb[q][threadIdx.x];
    }
    if (sa) sa[i] = u;
    if (sb) sb[i] = v;
  }
}

}  // namespace

Layout layout(int T, int d, int E, int de, int num_sms) {
  Layout l;
  const size_t P = size_t(T) * E;  // the most pairs a call can have
  const size_t Ep = size_t(E + 63) / 64 * 64;
  l.parts = cls::router_projection_parts(T, d, E, num_sms);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  l.wsplit = take(2 * size_t(d) * Ep * 2);
  l.sparts = take(size_t(l.parts) * T * E * 4);
  l.s = take(size_t(T) * E * 4);
  l.r = take(size_t(T) * E * 4);
  l.rho = take(size_t(T) * 4);
  l.dyhl = take(2 * size_t(T) * d * 2);
  l.U = take(P * de * 4);
  l.Q = take(P * de * 4);
  l.rhhl = take(2 * P * de * 2);
  l.duhl = take(2 * P * de * 2);
  l.dr = take(size_t(T) * E * 4);
  l.ds = take(size_t(T) * E * 4);
  l.dgc = take(size_t(T) * E * 4);
  l.dshl = take(2 * size_t(T) * Ep * 2);
  l.cnt = take(size_t(E) * 4);
  l.goff = take(size_t(E + 1) * 4);
  l.tok = take(P * 4);
  l.pexp = take(P * 4);
  l.pidx = take(P * 4);
  l.xp = take(P * d * 4);
  l.total = off;
  return l;
}

cudaError_t launch(const __nv_bfloat16* x, int T, int d, const float* Wr, const float* br, const float* g,
                   const __nv_bfloat16* W1, const __nv_bfloat16* W2, int E, int de, const float* dy, float* dx,
                   float* dWr, float* db, float* dg, float* dW1, float* dW2, void* ws, int num_sms, cudaStream_t st) {
  const Layout l = layout(T, d, E, de, num_sms);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto F = [&](size_t o) { return reinterpret_cast<float*>(base + o); };
  auto H = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(base + o); };
  auto I = [&](size_t o) { return reinterpret_cast<int*>(base + o); };
  const int Ep = (E + 63) / 64 * 64;
  const size_t P = size_t(T) * E;
  __nv_bfloat16* wsplit = H(l.wsplit);  // [2][d][Ep]: Wr hi, lo
  __nv_bfloat16 *dy_hi = H(l.dyhl), *dy_lo = dy_hi + size_t(T) * d;
  __nv_bfloat16 *rh_hi = H(l.rhhl), *rh_lo = rh_hi + P * de;
  __nv_bfloat16 *du_hi = H(l.duhl), *du_lo = du_hi + P * de;
  __nv_bfloat16 *ds_hi = H(l.dshl), *ds_lo = ds_hi + size_t(T) * Ep;
  int *goff = I(l.goff), *tok = I(l.tok);
  cudaError_t err;
  const unsigned ew = unsigned(std::min<long long>(((long long)T * d + 255) / 256, (long long)num_sms * 16));

  // router forward (s, r, rho) and dy as hi + lo
  if ((err = cls::router_projection(x, T, d, Wr, E, wsplit, F(l.sparts), l.parts, num_sms, st)) != cudaSuccess)
    return err;
  router_fwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(F(l.sparts), l.parts, T, E, br, g, F(l.s), F(l.r), F(l.rho));
  split_kernel<<<ew, 256, 0, st>>>(dy, T, d, d, dy_hi, dy_lo);
  // the active pairs, grouped by expert; dr of the inactive pairs stays 0
  if ((err = cudaMemsetAsync(F(l.dr), 0, size_t(T) * E * 4, st)) != cudaSuccess) return err;
  group_count_kernel<<<E, 256, 0, st>>>(F(l.s), T, E, I(l.cnt));
  group_scan_kernel<<<1, 32, 0, st>>>(I(l.cnt), E, goff);
  group_fill_kernel<<<E, 256, 0, st>>>(F(l.s), T, E, goff, tok, I(l.pexp), I(l.pidx));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;

  GemmArgs a{};
  // U_e = X[T_e] W1_e^T: pair rows [|T_e|, de]; X rows gathered, W1_e [de][d] (K-major)
  a = GemmArgs{x, nullptr, W1, nullptr, F(l.U), T, de, d, d, d, de, 0, (long long)de * d, 0, goff, tok};
  if ((err = gemm<true, false, true, false, kTokens, kPlain, kGroupM>(a, E, st)) != cudaSuccess) return err;
  // Q_e = dY[T_e] W2_e: pair rows [|T_e|, de]; dY rows gathered, W2_e [d][de] (N-major)
  a = GemmArgs{dy_hi, dy_lo, W2, nullptr, F(l.Q), T, de, d, d, de, de, 0, (long long)d * de, 0, goff, tok};
  if ((err = gemm<true, true, false, false, kTokens, kPlain, kGroupM>(a, E, st)) != cudaSuccess) return err;
  // h, dr, RH, DU per pair (one warp per possible pair; the warps past the pair count return)
  expert_pointwise_kernel<<<unsigned((P * 32 + 255) / 256), 256, 0, st>>>(F(l.U), F(l.Q), F(l.r), tok, I(l.pexp),
                                                                          goff, E, de, F(l.dr), rh_hi, rh_lo, du_hi,
                                                                          du_lo);
  // dW2_e = dY[T_e]^T RH_e: [d, de]; A = dY (M-major, rows k gathered), B = RH_e (N-major pair rows)
  a = GemmArgs{dy_hi, dy_lo, rh_hi, rh_lo, dW2, d, de, 0, d, de, de, 0, 0, (long long)d * de, goff, tok};
  if ((err = gemm<false, true, false, true, kTokens, kPairs, kGroupK>(a, E, st)) != cudaSuccess) return err;
  // dW1_e = DU_e^T X[T_e]: [de, d]; A = DU_e (M-major pair rows), B = X (N-major, rows k gathered)
  a = GemmArgs{du_hi, du_lo, x, nullptr, dW1, de, d, 0, de, d, d, 0, 0, (long long)de * d, goff, tok};
  if ((err = gemm<false, true, false, false, kPairs, kTokens, kGroupK>(a, E, st)) != cudaSuccess) return err;
  // the expert terms of dX per pair: DU_e W1_e, [|T_e|, d]; A = DU_e (K-major pair rows), B = W1_e [de][d]
  a = GemmArgs{du_hi, du_lo, W1, nullptr, F(l.xp), T, d, de, de, d, d, 0, (long long)de * d, 0, goff, tok};
  if ((err = gemm<true, true, false, false, kPairs, kPlain, kGroupM>(a, E, st)) != cudaSuccess) return err;
  // router backward
  router_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(F(l.s), F(l.rho), F(l.dr), g, T, E, Ep, F(l.ds), F(l.dgc), ds_hi,
                                                 ds_lo);
  colsum2_kernel<<<(E + 31) / 32, 256, 0, st>>>(F(l.ds), F(l.dgc), T, E, db, dg);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  // dWr = X^T dS: [d, E], A = X (M-major), B = dS [T][Ep] (N-major)
  a = GemmArgs{x, nullptr, ds_hi, ds_lo, dWr, d, E, T, d, Ep, E, 0, 0, 0, nullptr, nullptr};
  if ((err = gemm<false, false, false, true>(a, 1, st)) != cudaSuccess) return err;
  // dX = dS Wr^T: [T, d], A = dS [T][Ep] (K-major), B = Wr as [d][Ep] (K-major); then the pairs' terms
  a = GemmArgs{ds_hi, ds_lo, wsplit, wsplit + size_t(d) * Ep, dx, T, d, Ep, Ep, Ep, d, 0, 0, 0, nullptr, nullptr};
  if ((err = gemm<true, true, true, true>(a, 1, st)) != cudaSuccess) return err;
  pair_reduce_kernel<<<T, 256, size_t(E) * 4, st>>>(F(l.xp), I(l.pidx), T, E, d, dx);
  return cudaGetLastError();
}

}  // namespace bwd
}  // namespace bffn
