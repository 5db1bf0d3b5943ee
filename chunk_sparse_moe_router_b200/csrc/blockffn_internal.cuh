// Internal declarations of the BlockFFN chunk-layer kernels: workspace layout and launch parameters.
#pragma once
#include <cuda.h>  // CUtensorMap (header only; driver entry points are looked up at run time)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace bffn {

constexpr int kMaxE = 1024;
constexpr int kDecodeMaxL = 32;

// Device error word bits (WsHeader::err).
enum : uint32_t {
  kErrGridBarrier = 1u,   // expert kernel: waiting for every CTA to finish the up-projection
  kErrRingWait = 2u,      // expert kernel: waiting on a shared-memory ring barrier
};

// First 256 bytes of every workspace.
struct alignas(256) WsHeader {
  uint32_t ticket;     // reserved
  uint32_t grid_bar;   // expert kernel: CTAs past the up-projection (reset by the router, per call)
  uint32_t err;        // error bits, cleared by blockffn_device_status
  uint32_t err_info;
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Decode up-projection output h: per expert, ceil(de/64) tiles of [2L rows][64 bf16] (hi rows, then
// lo rows) in the 128-byte-swizzled layout the down-projection loads.
size_t decode_h_bytes(int L, int E, int de);

struct WsLayout {
  size_t s_off, h_off, total;
};

// Workspace: header | s fp32 [L,E] (router projection) | h (decode only)
inline WsLayout ws_layout(int L, int d, int E, int de) {
  (void)d;
  WsLayout w;
  w.s_off = sizeof(WsHeader);
  w.h_off = w.s_off + align256(size_t(L) * E * sizeof(float));
  w.total = w.h_off + (L <= kDecodeMaxL ? align256(decode_h_bytes(L, E, de)) : 0);
  return w;
}

// ------------------------------------------------------------------------------------ router
struct RouterParams {
  const __nv_bfloat16* x;   // [L,d]
  const float* Wr;          // [d,E]
  const float* br;          // [E] or null
  int L, d, E;
  int xt;                   // Wr rows per cluster rank (multiple of 8)
  float* s_ws;              // [L,E] out
  WsHeader* hdr;
};

struct RouterLaunch {
  int cluster;      // CTAs per cluster (split of d)
  int grid;         // clusters (32 router columns each)
  int xt;           // d rows per CTA
  int lt;           // tokens rounded up to 8, 16 or 32 (accumulators per thread)
  size_t smem;
};

bool router_decode_plan(int L, int d, int E, int max_smem, RouterLaunch* out);
cudaError_t router_decode_launch(const RouterParams& p, const RouterLaunch& plan, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------------------------ experts
struct DecodeParams {
  const float* s;             // [L,E] router projection (workspace)
  const float* g;             // [E]
  float* y;                   // [L,d]
  int32_t* active_idx;        // [E]
  int32_t* n_active;          // [1]
  uint32_t* tok_mask;         // [L, ceil(E/32)] or null
  int32_t* counts;            // [2] or null
  float* r_out;               // [L,E] or null
  uint8_t* h;                 // decode_h_bytes(L, E, de)
  WsHeader* hdr;
  int L, d, E, de;
  int S;            // ring slots
  int slot_bytes;   // bytes per slot (multiple of 1024)
  // up-projection: one stage = one W1 box of h (1, 2, 4 or 8 <= RSM) whole adjacent rows of one
  // expert over the Kp columns of a pass; x stays resident per pass
  int RSM;          // largest box height
  int KP;           // K passes
  int Kp;           // columns per pass (multiple of 64 unless the pass is the only one)
  int nKf;          // full 64-column chunks of d
  int nKc;          // 64-column chunks of d (the last may be ragged)
  int LB;           // x tile rows (L rounded up to 8)
  int xbuf_bytes;   // resident x tiles [chunks of a pass][LB][128 B]
  int w1_tail_off;  // offset of the ragged-chunk tile in an up-projection stage (1024-aligned)
  int ustage_bytes; // shared-memory staging of a CTA's up-projection sums (K split only)
  int ksplit;       // 1: L <= 8 and one pass: the consumer warps split K inside every up-projection stage
  // down-projection: stages of NEB experts, each a W2 box of RBB rows x KWB 64-column chunks
  int NEB;
  int nJc, nJf;     // 64-column chunks of de (all / full)
  int KWB;
  int RBB;          // multiple of 8
  int HR;           // h rows: 2L
  int h_expert_bytes;
  int eB;           // bytes of one expert's part of a down-projection stage (W2 tile, then h tile)
  int hoff;         // offset of the h tile within that part
  int sbuf_floats;  // floats of the ring the prologue may use to stage s
};

// Tensor maps (128-byte swizzle, out-of-bounds elements read as zero).  The chunked views put the
// 64-column chunks of a row in a dimension of their own so that one box carries whole rows (or a
// block of rows with all of their chunks): a compact, contiguous region of memory that lands as
// 8-row x 128-byte swizzled atoms.  They cover the full chunks only; the plain views serve a ragged
// last chunk.
struct TensorMaps {
  CUtensorMap x_ch;      // [64, L, nKf]        box {64, LB, chunks per pass}
  CUtensorMap x_2d;      // [d, L]              box {64, LB}
  CUtensorMap w1_ch[4];  // [64, de, nKf, E]    box {64, 2^k, chunks per pass, 1}
  CUtensorMap w1_3d[4];  // [d, de, E]          box {64, 2^k, 1}
  CUtensorMap w2_ch;     // [64, d, nJf, E]     box {64, RBB, KWB, 1}
  CUtensorMap w2_3d;     // [de, d, E]          box {64, RBB, 1}
};

struct DecodeLaunch {
  int grid;
  int lclass;       // 8, 16 or 32
  size_t smem;
};

bool expert_decode_plan(int L, int d, int E, int de, int num_sms, int max_smem, DecodeParams* p,
                        DecodeLaunch* out);
cudaError_t expert_decode_launch(const DecodeParams& p, const TensorMaps& tm, const DecodeLaunch& plan,
                                 cudaStream_t st, bool pdl);

}  // namespace bffn
