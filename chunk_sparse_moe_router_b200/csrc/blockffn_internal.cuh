// Internal declarations of the BlockFFN chunk-layer kernels: workspace layout and launch parameters.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace bffn {

constexpr int kMaxE = 1024;
constexpr int kDecodeMaxL = 32;

// Device error word bits (WsHeader::err).
enum : uint32_t {
  kErrGridBarrier = 1u,   // expert kernel: waiting for every CTA to finish the up-projection
  kErrRingWait = 2u,      // expert kernel: waiting on a shared-memory ring barrier
  kErrRouterWait = 4u,    // router: bulk-copy wait
};

// First 256 bytes of every workspace.
struct alignas(256) WsHeader {
  uint32_t ticket;     // router: E-slice clusters finished (the last one resets it)
  uint32_t grid_bar;   // expert kernel: CTAs past the up-projection (reset by the router)
  uint32_t err;        // error bits, cleared by blockffn_device_status
  uint32_t err_info;
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct WsLayout {
  size_t s_off, r_off, h_off, total;
};

// Workspace: header | s fp32 [L,E] | r fp32 [L,E] | h bf16 [E][2L][de] (decode up-projection
// output, stored as a high and a low bf16 part per value)
__host__ __device__ inline WsLayout ws_layout(int L, int d, int E, int de) {
  (void)d;
  WsLayout w;
  w.s_off = sizeof(WsHeader);
  w.r_off = w.s_off + align256(size_t(L) * E * sizeof(float));
  w.h_off = w.r_off + align256(size_t(L) * E * sizeof(float));
  size_t hrows = (L <= kDecodeMaxL) ? size_t(2) * L : 0;
  w.total = w.h_off + align256(size_t(E) * hrows * de * sizeof(__nv_bfloat16));
  return w;
}

// ------------------------------------------------------------------------------------ router
struct RouterParams {
  const __nv_bfloat16* x;   // [L,d]
  const float* Wr;          // [d,E]
  const float* br;          // [E] or null
  const float* g;           // [E]
  int L, d, E;
  int Rq;                   // router rows per cluster rank (multiple of 8)
  int wreg_floats;          // floats of the Wr-slice region (also holds s [L,E] at the end)
  float* s_ws;              // [L,E]
  float* r_ws;              // [L,E]
  float* r_out;             // [L,E] or null
  uint32_t* tok_mask;       // [L, ceil(E/32)] or null
  int32_t* counts;          // [2] or null
  int32_t* active_idx;      // [E]
  int32_t* n_active;        // [1]
  WsHeader* hdr;
};

struct RouterLaunch {
  int cluster;       // CTAs per cluster (d split)
  int lp;            // padded token count (4, 8, 16, 32)
  size_t smem;       // dynamic shared memory bytes
  int wreg_floats;   // see RouterParams::wreg_floats
};

bool router_decode_plan(int L, int d, int E, int max_smem, RouterLaunch* out, int* Rq);
cudaError_t router_decode_launch(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st,
                                 bool pdl);

// ------------------------------------------------------------------------------------ experts
struct DecodeParams {
  const __nv_bfloat16* x;    // [L,d]
  const __nv_bfloat16* W1;   // [E,de,d]
  const __nv_bfloat16* W2;   // [E,d,de]
  float* y;                  // [L,d]
  const int32_t* active_idx; // [E]
  const int32_t* n_active;   // [1]
  const float* r;            // [L,E]
  __nv_bfloat16* h;          // [E][2L][de]
  WsHeader* hdr;
  int L, d, E, de;
  int S;            // ring slots
  int slot_bytes;   // bytes per slot
  int woff;         // offset of the weight rows inside a slot
  int pitchA;       // smem row pitch (bytes) of up-projection tiles
  int pitchB;       // smem row pitch (bytes) of down-projection tiles
  int KcA;          // K elements per up-projection stage
  int KcB;          // K elements per down-projection stage
};

struct DecodeLaunch {
  int grid;
  int lclass;       // 8, 16 or 32
  size_t smem;
};

bool expert_decode_plan(int L, int d, int de, int num_sms, int max_smem, DecodeParams* p,
                        DecodeLaunch* out);
cudaError_t expert_decode_launch(const DecodeParams& p, const DecodeLaunch& plan, cudaStream_t st,
                                 bool pdl);

}  // namespace bffn
