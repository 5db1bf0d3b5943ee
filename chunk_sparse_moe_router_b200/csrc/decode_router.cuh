// Router projection and prologue of the decode kernels (BlockFFN chunk layer, L <= 32), shared by the
// expert kernels through templates on their thread count NT, parameter type P and shared-memory
// layout SM (P has x, Wr, br, g, s_part, rq, rrows, rcb, L, d, E and the output pointers; SM has act,
// n_act, rms and maskw).
//
// s = x Wr + b (lsdiaocha.cn BlockFFN article, section 2: the router's linear map, before its ReLU and
// RMSNorm).  d is cut into rq parts of rrows rows and E into blocks of 32 experts; unit u = (part
// u / rcb, block u % rcb) runs on CTA u mod G and writes a partial projection; after a grid-wide
// barrier every CTA adds the parts in part order.  The split depends on d only, so s is the same bits
// for every grid size.
#pragma once
#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace bffn {
namespace decode_router {

// Unit u = (part q = u / rcb, expert block cb = u % rcb): rows [q rrows, + rrows) of d, experts
// [32 cb, + 32).  Staging at the start of the dynamic shared memory (RouterStage): g and b [E] (copied
// before the dependent-launch wait with this CTA's first Wr rows), Wr rows [rrows][32] fp32, x columns
// [L][rrows] converted to fp32, warp sums [warps][8][32] fp32.
struct RouterStage {
  float* g;
  float* b;
  float* W;
  float* X;
  float* wsum;
};

template <int NT, class P>
__device__ __forceinline__ RouterStage router_stage(const P& p, uint8_t* base) {
  RouterStage r;
  const int E4 = (p.E + 3) & ~3;
  r.g = reinterpret_cast<float*>(base);
  r.b = r.g + E4;
  r.W = r.b + E4;
  r.X = r.W + size_t(p.rrows) * 32;
  r.wsum = r.X + size_t(p.L) * p.rrows;
  return r;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

template <int NT, class P>
__device__ void router_copy_w(const P& p, float* Ws, int u) {
  const int cb = u % p.rcb, q = u / p.rcb;
  const int k0 = q * p.rrows, nk = min(p.d - k0, p.rrows);
  const int e0 = cb * 32, Ec = min(32, p.E - e0);
  if ((p.E & 3) == 0) {  // Ec is then a multiple of 4 too
    for (int o = threadIdx.x; o < nk * 8; o += NT) {
      const int kk = o >> 3, c4 = (o & 7) * 4;
      float* dst = Ws + kk * 32 + c4;
      if (c4 < Ec)
        cp_async16(dst, p.Wr + size_t(k0 + kk) * p.E + e0 + c4);
      else
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    for (int o = threadIdx.x; o < nk * 32; o += NT) {
      const int kk = o >> 5, c = o & 31;
      if (c < Ec)
        cp_async4(Ws + kk * 32 + c, p.Wr + size_t(k0 + kk) * p.E + e0 + c);
      else
        Ws[kk * 32 + c] = 0.f;
    }
  }
}

// x columns of unit u, bf16 -> fp32 (exact)
template <int NT, class P>
__device__ void router_load_x(const P& p, float* Xs, int u) {
  const int k0 = (u / p.rcb) * p.rrows, nk = min(p.d - k0, p.rrows);
  const int q8 = nk >> 3;  // k0 and nk are multiples of 8
  for (int o = threadIdx.x; o < p.L * q8; o += NT) {
    const int t = o / q8, c8 = (o - t * q8) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(p.x + size_t(t) * p.d + k0 + c8);
    float4* dst = reinterpret_cast<float4*>(Xs + size_t(t) * p.rrows + c8);
    dst[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    dst[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                         __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
  }
}

// Partial projection of unit u from the staged operands.  Warp w takes rows [w R4, w R4 + R4) of the
// part (R4 = rrows / warps rounded up to 4), lane = expert column, 8 tokens at a time; each sum runs
// over its rows in increasing order, then the CTA adds the warps' sums in warp order.
template <int NT, class P>
__device__ void router_unit(const P& p, const RouterStage& rs, int u) {
  constexpr int kRouterWarps = NT / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = u % p.rcb, q = u / p.rcb;
  const int k0 = q * p.rrows, nk = min(p.d - k0, p.rrows);
  const int e0 = cb * 32, Ec = min(32, p.E - e0);
  const int per = ((p.rrows + kRouterWarps - 1) / kRouterWarps + 3) & ~3;
  const int r0 = min(nk, warp * per), r1 = min(nk, r0 + per);
  for (int t0 = 0; t0 < p.L; t0 += 8) {
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    for (int k = r0; k < r1; k += 4) {
      float wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wv[i] = rs.W[(k + i) * 32 + lane];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (t0 + t < p.L) {
          const float4 xv = *reinterpret_cast<const float4*>(rs.X + size_t(t0 + t) * p.rrows + k);
          acc[t] = fmaf(xv.x, wv[0], acc[t]);
          acc[t] = fmaf(xv.y, wv[1], acc[t]);
          acc[t] = fmaf(xv.z, wv[2], acc[t]);
          acc[t] = fmaf(xv.w, wv[3], acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) rs.wsum[(warp * 8 + t) * 32 + lane] = acc[t];
    __syncthreads();
    for (int o = threadIdx.x; o < 8 * 32; o += NT) {
      const int t = o >> 5, c = o & 31;
      if (t0 + t < p.L && c < Ec) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kRouterWarps; ++w) v += rs.wsum[(w * 8 + t) * 32 + c];
        p.s_part[(size_t(q) * p.L + t0 + t) * p.E + e0 + c] = v;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------- prologue
// s = the parts in part order plus b, into sbuf [L][E]; per token the RMS of relu(s) over the E
// experts and the active bits; then the union (ascending).  CTA 0 writes the chunk's outputs besides y.
template <int NT, class P, class SM>
__device__ void prologue_router_stats(const P& p, const SM& sm, const RouterStage& rs, float* sbuf) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nW = (p.E + 31) >> 5;
  const size_t qs = size_t(p.L) * p.E;
  for (int o = tid; o < p.L * p.E; o += NT) {
    const float* src = p.s_part + o;
    float v = 0.f;
    int q = 0;
    for (; q + 8 <= p.rq; q += 8) {  // written by other CTAs of this grid: L2 loads, not L1
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = __ldcg(src + (q + i) * qs);
#pragma unroll
      for (int i = 0; i < 8; ++i) v += a[i];
    }
    for (; q < p.rq; ++q) v += __ldcg(src + q * qs);
    if (p.br) v += rs.b[o % p.E];
    sbuf[o] = v;
  }
  __syncthreads();
  for (int t = warp; t < p.L; t += NT / 32) {
    const float* st = sbuf + size_t(t) * p.E;
    float sumsq = 0.f, sum = 0.f;
    for (int ww = 0; ww < nW; ++ww) {
      const int e = ww * 32 + lane;
      const float sv = e < p.E ? st[e] : -1.f;
      const float a = fmaxf(sv, 0.f);
      sumsq = fmaf(a, a, sumsq);
      sum += a;
      const uint32_t bits = __ballot_sync(0xffffffffu, sv > 0.f);
      if (lane == 0) sm.maskw[t * 32 + ww] = bits;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    if (lane == 0) sm.rms[t] = router_norm(p.sum_norm, sum, sumsq, p.E);  // the normaliser: RMS or sum
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t u = 0;
    int tok_active = 0;
    if (lane < nW)
      for (int t = 0; t < p.L; ++t) {
        const uint32_t m = sm.maskw[t * 32 + lane];
        u |= m;
        tok_active += __popc(m);
      }
    const int c = __popc(u);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int pos = incl - c;
    uint32_t rest = u;
    while (rest) {
      const int b = __ffs(rest) - 1;
      rest &= rest - 1;
      sm.act[pos++] = lane * 32 + b;
    }
    int act_sum = tok_active;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) act_sum += __shfl_xor_sync(0xffffffffu, act_sum, o);
    if (lane == 0) {
      *sm.n_act = total;
      if (blockIdx.x == 0) {
        *p.n_active = total;
        if (p.counts) {
          p.counts[0] = p.L * p.E - act_sum;
          p.counts[1] = p.E - total;
        }
      }
    }
  }
  __syncthreads();
  if (blockIdx.x == 0) {  // the chunk's outputs besides y
    for (int a = tid; a < *sm.n_act; a += NT) p.active_idx[a] = sm.act[a];
    if (p.tok_mask)
      for (int o = tid; o < p.L * nW; o += NT) p.tok_mask[o] = sm.maskw[(o / nW) * 32 + (o % nW)];
    if (p.r_out)  // r = g relu(s) / rms, the expression the up-projection epilogue uses
      for (int o = tid; o < p.L * p.E; o += NT) {
        const int t = o / p.E, e = o - t * p.E;
        const float rms = sm.rms[t];
        p.r_out[o] = rms > 0.f ? (rs.g[e] * fmaxf(sbuf[o], 0.f)) / rms : 0.f;
      }
  }
}

}  // namespace decode_router
}  // namespace bffn
