// Router projection of the BlockFFN chunk layer for decode-sized chunks (L <= 32).
//
// s = x Wr + b in fp32 (lsdiaocha.cn BlockFFN article, section 2: the router's linear map, before its
// ReLU and RMSNorm).  The work is spread over many SMs with thread-block clusters: cluster y owns 32
// router columns (experts), and its C CTAs split the d rows.  Each CTA stages its [rows x 32] slice of
// Wr (issued before the dependent-launch wait: weights never depend on the previous kernel) and its
// [L x rows] slice of x in shared memory with cp.async.  Each warp takes a contiguous share of the
// rows with one accumulator per token (lane = column), the CTA adds its warps' shares in warp order,
// and the cluster then adds the C partials through distributed shared memory in rank order, every
// rank finishing a 1/C share of the outputs with all of its remote loads in flight at once.  The
// order of every sum is fixed, so s is bit-reproducible.  The ReLU, the RMSNorm and the chunk union
// run in the expert kernel's prologue.
#include <cooperative_groups.h>

#include <algorithm>

#include "blockffn_internal.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace bffn {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kCols = 32;         // router columns per cluster
constexpr int kMaxCluster = 16;

template <int LT>
__global__ void __launch_bounds__(kRouterThreads) router_decode_kernel(RouterParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int q = int(cluster.block_rank());
  const int C = int(cluster.num_blocks());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kRouterThreads / 32;
  const int e0 = blockIdx.y * kCols;
  const int Ec = min(kCols, p.E - e0);
  const int k0 = q * p.xt;  // xt holds the rows per rank here
  const int nk = max(0, min(p.d, k0 + p.xt) - k0);

  float* W_s = reinterpret_cast<float*>(smem_raw);                                      // [rows][32]
  __nv_bfloat16* X_s = reinterpret_cast<__nv_bfloat16*>(W_s + size_t(p.xt) * kCols);   // [LT][rows]
  float* wpart = reinterpret_cast<float*>(X_s + size_t(LT) * p.xt);                     // [NW][LT][32]
  float* part = wpart + NW * LT * kCols;                                                // [LT][32]

  // The router weights do not depend on the previous kernel in the stream: start their copies first.
  if ((p.E & 3) == 0) {
    constexpr int q4 = kCols / 4;
    for (int o = tid; o < nk * q4; o += kRouterThreads) {
      const int kk = o / q4, c4 = (o - kk * q4) * 4;
      float* dst = W_s + kk * kCols + c4;
      if (c4 < Ec)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                     "l"(p.Wr + size_t(k0 + kk) * p.E + e0 + c4)
                     : "memory");
      else
        dst[0] = dst[1] = dst[2] = dst[3] = 0.f;
    }
  } else {
    for (int o = tid; o < nk * kCols; o += kRouterThreads) {
      const int kk = o / kCols, c = o - kk * kCols;
      float* dst = W_s + kk * kCols + c;
      if (c < Ec)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)),
                     "l"(p.Wr + size_t(k0 + kk) * p.E + e0 + c)
                     : "memory");
      else
        *dst = 0.f;
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // x may come from the previous kernel in the stream, and the workspace is shared with it.
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) p.hdr->grid_bar = 0u;  // expert kernel barrier
  {
    const int q8 = nk / 8;  // nk and k0 are multiples of 8
    for (int o = tid; o < p.L * q8; o += kRouterThreads) {
      const int t = o / q8, c8 = (o - t * q8) * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(X_s + size_t(t) * p.xt + c8)),
                   "l"(p.x + size_t(t) * p.d + k0 + c8)
                   : "memory");
    }
    for (int o = p.L * p.xt + tid; o < LT * p.xt; o += kRouterThreads)  // padding tokens read as 0
      X_s[o] = __float2bfloat16_rn(0.f);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // warp w takes a contiguous share of the CTA's rows for every token, lane = column: LT independent
  // accumulators per thread; x is a broadcast, W_s a conflict-free row.
  {
    const int per = (nk + NW - 1) / NW;
    const int r0 = warp * per, r1 = min(nk, r0 + per);
    float acc[LT];
#pragma unroll
    for (int t = 0; t < LT; ++t) acc[t] = 0.f;
#pragma unroll 4
    for (int kk = r0; kk < r1; ++kk) {
      const float wv = W_s[kk * kCols + lane];
#pragma unroll
      for (int t = 0; t < LT; ++t) acc[t] = fmaf(__bfloat162float(X_s[t * p.xt + kk]), wv, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < LT; ++t) wpart[(warp * LT + t) * kCols + lane] = acc[t];
  }
  __syncthreads();
  for (int o = tid; o < LT * kCols; o += kRouterThreads) {  // the warps' shares, in warp order
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += wpart[w * LT * kCols + o];
    part[o] = v;
  }
  cluster.sync();
  {
    const int n_out = p.L * Ec;
    const int per = (n_out + C - 1) / C;
    const int o0 = q * per, o1 = min(n_out, o0 + per);
    for (int o = o0 + tid; o < o1; o += kRouterThreads) {
      const int t = o / Ec, c = o - t * Ec;
      float v[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) v[r] = r < C ? cluster.map_shared_rank(part, r)[t * kCols + c] : 0.f;
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) sum += v[r];
      if (p.br) sum += p.br[e0 + c];
      p.s_ws[size_t(t) * p.E + e0 + c] = sum;
    }
  }
  cluster.sync();  // no rank leaves while another still reads its partials
}

}  // namespace

bool router_decode_plan(int L, int d, int E, int max_smem, RouterLaunch* out) {
  if (L < 1 || L > kDecodeMaxL || E < 1 || E > kMaxE || d % 8 != 0) return false;
  const int LT = L <= 8 ? 8 : L <= 16 ? 16 : 32;
  for (int cluster : {8, 16}) {
    int rows = (d + cluster - 1) / cluster;
    rows = (rows + 7) & ~7;
    const size_t smem = size_t(rows) * kCols * 4 + size_t(LT) * rows * 2 +
                        size_t(kRouterThreads / 32 + 1) * LT * kCols * 4;
    if (smem <= size_t(max_smem) && (cluster == 16 || rows <= 256)) {
      out->cluster = cluster;
      out->xt = rows;
      out->smem = smem;
      out->grid = (E + kCols - 1) / kCols;
      out->lt = LT;
      return true;
    }
  }
  return false;
}

template <int LT>
static cudaError_t launch_lt(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st, bool pdl) {
  auto kfn = router_decode_kernel<LT>;
  cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
  if (err != cudaSuccess) return err;
  if (plan.cluster > 8) {
    err = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.cluster, plan.grid, 1);
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

cudaError_t router_decode_launch(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st, bool pdl) {
  switch (plan.lt) {
    case 8: return launch_lt<8>(p, plan, st, pdl);
    case 16: return launch_lt<16>(p, plan, st, pdl);
    default: return launch_lt<32>(p, plan, st, pdl);
  }
}

}  // namespace bffn
