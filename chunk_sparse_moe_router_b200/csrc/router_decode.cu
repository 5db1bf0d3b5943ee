// Router projection of the BlockFFN chunk layer for decode-sized chunks (L <= 32).
//
// s = x Wr + b in fp32 (lsdiaocha.cn BlockFFN article, section 2: the router's linear map, before its
// ReLU and RMSNorm).  The work is spread over many SMs with thread-block clusters: cluster y owns 32
// router columns (experts), and its C CTAs split the d rows.  Each CTA stages its [rows x 32] slice of
// Wr and its [L x rows] slice of x in shared memory with cp.async (one memory round trip), computes
// its partial sums (one output per thread and token group), and the cluster then adds the C partials
// through distributed shared memory in rank order, every rank finishing a 1/C share of the outputs
// with all of its remote loads in flight at once.  The order of every sum is fixed, so s is
// bit-reproducible.  The ReLU, the RMSNorm and the chunk union run in the expert kernel's prologue.
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

__global__ void __launch_bounds__(kRouterThreads) router_decode_kernel(RouterParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int q = int(cluster.block_rank());
  const int C = int(cluster.num_blocks());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e0 = blockIdx.y * kCols;
  const int Ec = min(kCols, p.E - e0);
  const int k0 = q * p.xt;  // xt holds the rows per rank here
  const int nk = max(0, min(p.d, k0 + p.xt) - k0);
  const int LP = (p.L + 7) & ~7;

  float* W_s = reinterpret_cast<float*>(smem_raw);                                      // [rows][32]
  __nv_bfloat16* X_s = reinterpret_cast<__nv_bfloat16*>(W_s + size_t(p.xt) * kCols);   // [LP][rows]
  float* part = reinterpret_cast<float*>(X_s + size_t(LP) * p.xt);                      // [LP][32]

  // x may come from the previous kernel in the stream, and the workspace is shared with it.
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) p.hdr->grid_bar = 0u;  // expert kernel barrier

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
  {
    const int q8 = nk / 8;  // nk and k0 are multiples of 8
    for (int o = tid; o < p.L * q8; o += kRouterThreads) {
      const int t = o / q8, c8 = (o - t * q8) * 8;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(X_s + size_t(t) * p.xt + c8)),
                   "l"(p.x + size_t(t) * p.d + k0 + c8)
                   : "memory");
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // warp w handles tokens w, w+8, ...; lane = column.  x is a broadcast, Wr a conflict-free row.
  for (int t = warp; t < LP; t += kRouterThreads / 32) {
    float acc = 0.f;
    if (t < p.L) {
      const __nv_bfloat16* xr = X_s + size_t(t) * p.xt;
#pragma unroll 8
      for (int kk = 0; kk < nk; ++kk) acc = fmaf(__bfloat162float(xr[kk]), W_s[kk * kCols + lane], acc);
    }
    part[t * kCols + lane] = acc;
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
  const int LP = (L + 7) & ~7;
  for (int cluster : {8, 16}) {
    int rows = (d + cluster - 1) / cluster;
    rows = (rows + 7) & ~7;
    const size_t smem = size_t(rows) * kCols * 4 + size_t(LP) * rows * 2 + size_t(LP) * kCols * 4;
    if (smem <= size_t(max_smem) && (cluster == 16 || rows <= 256)) {
      out->cluster = cluster;
      out->xt = rows;
      out->smem = smem;
      out->grid = (E + kCols - 1) / kCols;
      return true;
    }
  }
  return false;
}

cudaError_t router_decode_launch(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st, bool pdl) {
  cudaError_t err =
      cudaFuncSetAttribute(router_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(plan.smem));
  if (err != cudaSuccess) return err;
  if (plan.cluster > 8) {
    err = cudaFuncSetAttribute(router_decode_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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
  return cudaLaunchKernelEx(&cfg, router_decode_kernel, p);
}

}  // namespace bffn
