// Router of the BlockFFN chunk layer for decode-sized chunks (L <= 32), fused with the chunk union.
//
// Step 1 (lsdiaocha.cn BlockFFN article, section 2): s = x Wr + b in fp32.  The grid is a set of
// thread-block clusters: cluster `blockIdx.y` owns 32 router columns (experts), and the CTAs of a
// cluster split the d rows of Wr.  Each CTA stages its Wr slice and its x slice in shared memory
// with cp.async, accumulates 4x4 register blocks of (token, expert) outputs over a strided share of
// its rows, reduces the shares in a fixed order, and the cluster then sums its CTAs' partials
// through distributed shared memory in rank order — so s is bit-reproducible run to run.
// Step 2 (same section): ReLU, then RMSNorm over the E entries of each token, one warp per token
// with a shuffle reduction.
// Step 3 (article, section 4): the union of active experts. Per token, __ballot_sync packs
// "s > 0" into 32-bit words; OR over the chunk's tokens gives the union; __popc and a warp scan
// turn it into the ascending active-expert list, n_active and the sparsity counts.
// Steps 2-3 need all E columns, so they run in the last cluster to finish (an atomic ticket; no
// CTA ever waits for another).
#include <cooperative_groups.h>

#include <algorithm>

#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace bffn {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kCols = 32;  // experts per cluster
constexpr int kMaxCluster = 16;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Steps 2 and 3 over the full s [L,E] (one CTA); s_s is shared memory for L*E floats.
__device__ void router_finish(const RouterParams& p, float* s_s, uint32_t* mask_s /* [L][nW] */) {
  const int L = p.L, E = p.E, nW = (E + 31) / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = kRouterThreads / 32;
  // one pass over s (written by every cluster; read through L2)
  for (int o = threadIdx.x; o < L * E; o += kRouterThreads) s_s[o] = __ldcg(p.s_ws + o);
  __syncthreads();
  for (int t = warp; t < L; t += nwarps) {
    const float* st = s_s + size_t(t) * E;
    float sumsq = 0.f;
    for (int w = 0; w < nW; ++w) {
      const int e = w * 32 + lane;
      const float sv = (e < E) ? st[e] : -1.f;
      const float a = fmaxf(sv, 0.f);
      sumsq = fmaf(a, a, sumsq);
      const uint32_t bits = __ballot_sync(0xffffffffu, sv > 0.f);
      if (lane == 0) {
        mask_s[t * nW + w] = bits;
        if (p.tok_mask) p.tok_mask[size_t(t) * nW + w] = bits;
      }
    }
    sumsq = warp_sum(sumsq);
    const float ms = sumsq / float(E);
    const float rms = sqrtf(ms);
    for (int e = lane; e < E; e += 32) {
      const float a = fmaxf(st[e], 0.f);
      const float r = (ms > 0.f) ? (p.g[e] * a) / rms : 0.f;
      p.r_ws[size_t(t) * E + e] = r;
      if (p.r_out) p.r_out[size_t(t) * E + e] = r;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // one lane per 32-expert word (E <= 1024 -> nW <= 32)
    uint32_t u = 0;
    int tok_active = 0;
    if (lane < nW) {
      for (int t = 0; t < L; ++t) {
        const uint32_t m = mask_s[t * nW + lane];
        u |= m;
        tok_active += __popc(m);
      }
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
      p.active_idx[pos++] = lane * 32 + b;
    }
    int act_sum = tok_active;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) act_sum += __shfl_xor_sync(0xffffffffu, act_sum, o);
    if (lane == 0) {
      *p.n_active = total;
      if (p.counts) {
        p.counts[0] = L * E - act_sum;
        p.counts[1] = E - total;
      }
      p.hdr->grid_bar = 0u;
      p.hdr->ticket = 0u;
    }
  }
}

template <int LP>
__global__ void __launch_bounds__(kRouterThreads) router_decode_kernel(RouterParams p) {
  extern __shared__ __align__(16) float smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int q = int(cluster.block_rank());
  const int C = int(cluster.num_blocks());
  const int e0 = blockIdx.y * kCols;
  const int Ec = min(kCols, p.E - e0);
  const int k0 = q * p.Rq;
  const int nk = max(0, min(p.d, k0 + p.Rq) - k0);
  const int tid = threadIdx.x;

  float* W_s = smem;                        // [Rq][32]; reused for s [L][E] by the last cluster
  float* X_s = W_s + p.wreg_floats;         // [Rq][LP]
  float* P_s = X_s + size_t(p.Rq) * LP;     // [256][16]
  float* Cp_s = P_s + kRouterThreads * 16;  // [LP][32]
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(Cp_s + LP * kCols);  // [L][nW]
  // raw bf16 x slice [L][Rq] shares P_s (not yet in use when x is staged)
  __nv_bfloat16* Xraw = reinterpret_cast<__nv_bfloat16*>(P_s);

  // x may be written by the previous kernel in the stream, and the workspace is shared with it.
  pdl_wait();
  pdl_launch_dependents();

  // Stage the Wr slice (columns beyond Ec are zero) with cp.async.
  const bool vec = ((p.E & 3) == 0);
  if (vec) {
    const int q4 = kCols / 4;
    for (int o = tid; o < nk * q4; o += kRouterThreads) {
      const int kk = o / q4, c4 = (o % q4) * 4;
      float* dst = W_s + kk * kCols + c4;
      if (c4 < Ec) {
        const float* src = p.Wr + size_t(k0 + kk) * p.E + e0 + c4;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
      } else {
        dst[0] = dst[1] = dst[2] = dst[3] = 0.f;
      }
    }
  } else {
    for (int o = tid; o < nk * kCols; o += kRouterThreads) {
      const int kk = o / kCols, c = o % kCols;
      float* dst = W_s + kk * kCols + c;
      if (c < Ec) {
        const float* src = p.Wr + size_t(k0 + kk) * p.E + e0 + c;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
      } else {
        *dst = 0.f;
      }
    }
  }
  // x slice [L][nk] as raw bf16, 16 bytes per copy (k0 and nk are multiples of 8)
  {
    const int q8 = nk / 8;
    for (int o = tid; o < p.L * q8; o += kRouterThreads) {
      const int t = o / q8, c8 = (o % q8) * 8;
      const __nv_bfloat16* src = p.x + size_t(t) * p.d + k0 + c8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(Xraw + t * p.Rq + c8)), "l"(src)
                   : "memory");
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  // transpose to [k][t] and widen to fp32; tokens >= L are zero
  for (int o = tid; o < nk * LP; o += kRouterThreads) {
    const int kk = o / LP, t = o % LP;
    X_s[kk * LP + t] = (t < p.L) ? __bfloat162float(Xraw[t * p.Rq + kk]) : 0.f;
  }
  __syncthreads();

  // 4 tokens x 4 experts per thread; KS threads share the rows of each block.
  constexpr int TB = LP / 4, CB = kCols / 4, NB = TB * CB, KS = kRouterThreads / NB;
  static_assert(kRouterThreads % NB == 0, "block split");
  {
    const int blk = tid % NB, ks = tid / NB;
    const int tb = blk / CB, cb = blk % CB;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int kk = ks; kk < nk; kk += KS) {
      const float4 w = *reinterpret_cast<const float4*>(W_s + kk * kCols + cb * 4);
      const float4 xv = *reinterpret_cast<const float4*>(X_s + kk * LP + tb * 4);
      const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
      const float ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i * 4 + j] = fmaf(xs[i], ws[j], acc[i * 4 + j]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) P_s[tid * 16 + i] = acc[i];
  }
  __syncthreads();
  for (int o = tid; o < LP * kCols; o += kRouterThreads) {
    const int t = o / kCols, e = o % kCols;
    const int blk = (t / 4) * CB + e / 4, sub = (t % 4) * 4 + (e % 4);
    float sum = 0.f;
    for (int ks = 0; ks < KS; ++ks) sum += P_s[(ks * NB + blk) * 16 + sub];
    Cp_s[o] = sum;
  }
  cluster.sync();
  // Every rank sums a 1/C share of the (token, expert) outputs over the C partials, in rank order.
  // All remote loads of an output are issued before the first add (one DSMEM round trip).
  {
    const int n_out = p.L * Ec;
    const int per = (n_out + C - 1) / C;
    const int o0 = q * per, o1 = min(n_out, o0 + per);
    for (int o = o0 + tid; o < o1; o += kRouterThreads) {
      const int t = o / Ec, e = o % Ec;
      float part[kMaxCluster];
#pragma unroll
      for (int rk = 0; rk < kMaxCluster; ++rk)
        part[rk] = (rk < C) ? cluster.map_shared_rank(Cp_s, rk)[t * kCols + e] : 0.f;
      float sum = 0.f;
#pragma unroll
      for (int rk = 0; rk < kMaxCluster; ++rk) sum += part[rk];
      if (p.br) sum += p.br[e0 + e];
      p.s_ws[size_t(t) * p.E + e0 + e] = sum;
    }
  }
  __threadfence();
  cluster.sync();  // every share of s is written; every rank's shared memory may now be released
  if (q != 0) return;

  __shared__ int is_last;
  if (tid == 0) is_last = (atomicAdd(&p.hdr->ticket, 1u) == gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  router_finish(p, W_s, mask_s);
}

template <int LP>
cudaError_t launch_lp(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st, bool pdl) {
  auto kfn = router_decode_kernel<LP>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
  if (err != cudaSuccess) return err;
  if (plan.cluster > 8) {
    err = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.cluster, (p.E + kCols - 1) / kCols, 1);
  cfg.blockDim = dim3(kRouterThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kfn, p);
}

}  // namespace

bool router_decode_plan(int L, int d, int E, int max_smem, RouterLaunch* out, int* Rq) {
  if (L < 1 || L > kDecodeMaxL || E < 1 || E > kMaxE) return false;
  const int lp = L <= 4 ? 4 : L <= 8 ? 8 : L <= 16 ? 16 : 32;
  const int nW = (E + 31) / 32;
  for (int cluster : {8, 16}) {
    int rq = (d + cluster - 1) / cluster;
    rq = (rq + 7) & ~7;
    if (size_t(L) * rq * 2 > size_t(kRouterThreads) * 16 * 4) continue;  // x slice must fit in P_s
    const size_t wreg = std::max(size_t(rq) * kCols * 4, size_t(L) * E * 4);
    size_t smem = wreg + size_t(rq) * lp * 4 + kRouterThreads * 16 * 4 + size_t(lp) * kCols * 4 +
                  size_t(L) * nW * 4;
    if (smem <= size_t(max_smem)) {
      out->cluster = cluster;
      out->lp = lp;
      out->smem = smem;
      out->wreg_floats = int(wreg / 4);
      *Rq = rq;
      return true;
    }
  }
  return false;
}

cudaError_t router_decode_launch(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st,
                                 bool pdl) {
  switch (plan.lp) {
    case 4: return launch_lp<4>(p, plan, st, pdl);
    case 8: return launch_lp<8>(p, plan, st, pdl);
    case 16: return launch_lp<16>(p, plan, st, pdl);
    default: return launch_lp<32>(p, plan, st, pdl);
  }
}

}  // namespace bffn
