// Cross-chunk expert reuse: for each chunk c, the number of experts in both U_a(c) and U_b(c), where the
// unions are the ascending active lists of two calls (typically the same sequence's chunk at the same
// layer in two consecutive verification steps).  The BlockFFN article (section 5) reports that more than
// 85 % of the experts active for a token are active for the next one as well; the reuse rate of a chunk
// is overlap / |U_b|.
#include "blockffn_internal.cuh"

namespace bffn {
namespace {

// One warp per chunk: U_b's bits in 32 words (E <= 1024) in registers spread over the lanes (lane w
// holds word w), then each lane tests its share of U_a against them (a shuffle fetches the word), and
// the warp adds the hits: an integer count, the same in any order.
__global__ void __launch_bounds__(256) union_overlap_kernel(const int32_t* idx_a, const int32_t* n_a,
                                                            const int32_t* idx_b, const int32_t* n_b, int C, int E,
                                                            int32_t* overlap) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (c >= C) return;
  const int nb = min(max(n_b[c], 0), E), na = min(max(n_a[c], 0), E);
  uint32_t word = 0;  // lane w: bits of experts 32 w .. 32 w + 31 in U_b
  for (int q = 0; q < nb; ++q) {
    const int e = idx_b[size_t(c) * E + q];
    if (e >= 0 && e < E && (e >> 5) == lane) word |= 1u << (e & 31);
  }
  int hits = 0;
  for (int q0 = 0; q0 < na; q0 += 32) {
    const int q = q0 + lane;
    const int e = q < na ? idx_a[size_t(c) * E + q] : -1;
    const int w = (e >= 0 && e < E) ? (e >> 5) : 0;
    const uint32_t bits = __shfl_sync(0xffffffffu, word, w);
    if (e >= 0 && e < E && ((bits >> (e & 31)) & 1u)) ++hits;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hits += __shfl_xor_sync(0xffffffffu, hits, o);
  if (lane == 0) overlap[c] = hits;
}

}  // namespace

cudaError_t union_overlap_launch(const int32_t* idx_a, const int32_t* n_a, const int32_t* idx_b, const int32_t* n_b,
                                 int C, int E, int32_t* overlap, cudaStream_t st) {
  const int warps_per_block = 8;
  union_overlap_kernel<<<(C + warps_per_block - 1) / warps_per_block, warps_per_block * 32, 0, st>>>(
      idx_a, n_a, idx_b, n_b, C, E, overlap);
  return cudaGetLastError();
}

}  // namespace bffn
