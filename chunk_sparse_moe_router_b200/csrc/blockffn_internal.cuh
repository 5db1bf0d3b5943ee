// Internal declarations of the BlockFFN chunk-layer kernels: workspace layout and launch parameters.
#pragma once
#include <cuda.h>  // CUtensorMap (header only; driver entry points are looked up at run time)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace bffn {

constexpr int kMaxE = 1024;
constexpr int kDecodeMaxL = 32;

// A router barrier made unreachable on purpose (the fault-injection flag of blockffn_chunk_forward_ex)
// gives up after this long; every other device wait gives up after about 2 s.
constexpr uint64_t kInjectedWaitNs = 1000000ull;

// The per-token normaliser of the router's ReLU outputs a: their RMS over the E experts (BlockFFN's
// RMSNorm), or their sum (the ReMoE router).  r = g a / normaliser, and r = 0 when it is 0.
__device__ __forceinline__ float router_norm(int sum_norm, float sum, float sumsq, int E) {
  return sum_norm ? sum : sqrtf(sumsq / float(E));
}

// Device error word bits (WsHeader::err).
enum : uint32_t {
  kErrGridBarrier = 1u,   // expert kernel: waiting for every CTA to finish the up-projection
  kErrRingWait = 2u,      // expert kernel: waiting on a shared-memory ring barrier
  kErrPrefillWait = 4u,   // prefill GEMMs: waiting on a shared-memory barrier
  kErrRouterBarrier = 8u, // expert kernel: waiting for every CTA's router partial sums
  kErrTeamBarrier = 16u,  // batched expert kernel: waiting for the team's up-projections
  kErrBadLayer = 32u,     // batched router kernel: a chunk's layer index was outside [0, n_layers)
};

// First 256 bytes of every workspace.
struct alignas(256) WsHeader {
  uint32_t ticket;     // reserved
  uint32_t grid_bar;   // expert kernel: CTAs past the up-projection
  uint32_t err;        // error bits, cleared by blockffn_device_status
  uint32_t err_info;
  uint32_t router_bar; // expert kernel: CTAs whose router partial sums are written
  uint32_t exit_ctr;   // expert kernel: CTAs done; the last one sets the three counters back to 0
  uint32_t pad[58];
};
static_assert(sizeof(WsHeader) == 256, "header size");

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Decode up-projection output h: per expert, ceil(de/64) tiles of [2L rows][64 bf16] (hi rows, then
// lo rows) in the 128-byte-swizzled layout the down-projection loads.
size_t decode_h_bytes(int L, int E, int de);

// The tcgen05 decode path (decode_on_tc; namespace tcdec): its h image has tiles of 2 LC rows
// (LC = L rounded up to 16 or 32, at least 16), and its stream-K scratch holds the partial accumulators of blocks
// split between CTAs (two slots of 128 rows x LC fp32 per CTA) and one arrival counter per up- and
// down-projection block.
constexpr int kTcSmallL = 8;     // the mma.sync decode kernel takes chunks of at most this many tokens
constexpr int kTcMaxGrid = 160;  // CTAs of one tcgen05 decode launch
// Which decode kernel a shape takes: the tcgen05 one for chunks of more than kTcSmallL tokens, and for
// any chunk length once one expert's W1 and W2 hold 4 MiB or more (d de >= 2^20).  There its faster
// streaming outweighs its larger fixed cost (the split-block reductions): measured 11-14 % faster at
// d = 4096, de = 256 for L = 1..8, and 7 % slower at d = 2048, de = 256, L = 8.
inline bool decode_on_tc(int L, int d, int de) { return L > kTcSmallL || 1ll * d * de >= (1ll << 20); }
namespace tcdec {
inline int lc_of(int L) { return L <= 16 ? 16 : 32; }
inline size_t h_bytes(int L, int E, int de) { return size_t(E) * ((de + 63) / 64) * size_t(2 * lc_of(L)) * 128; }
inline size_t part_bytes(int L) { return size_t(kTcMaxGrid) * 2 * 128 * lc_of(L) * 4; }
inline size_t cnt_words(int d, int E, int de) { return size_t(E) * ((de + 127) / 128) + (d + 127) / 128; }
}  // namespace tcdec

// Prefill workspace regions (L > 32), after s: Wr as bf16 hi + lo pairs [2][d][E rounded up to 64], the
// router projection, per-token masks and RMS, per-expert counts and offsets, the pair lists (token, r)
// in expert-major order, and H = [pairs][2 de] bf16 (hi | lo).
struct PrefillLayout {
  size_t wsplit_off, spart_off, mask_off, rms_off, cnt_off, off_off, toff_off, npos_off, tok_off, rv_off, h_off,
      end;
};

inline PrefillLayout prefill_layout(size_t start, int L, int d, int E, int de) {
  PrefillLayout p;
  const size_t W = size_t(E + 31) / 32, P = size_t(L) * E, Ep = size_t(E + 63) / 64 * 64;
  p.wsplit_off = start;
  p.spart_off = p.wsplit_off + align256(2 * size_t(d) * Ep * 2);
  p.mask_off = p.spart_off + align256(size_t(4) * L * E * 4);  // up to 4 router parts (cls::kMaxRouterParts)
  p.rms_off = p.mask_off + align256(size_t(L) * W * 4);
  p.cnt_off = p.rms_off + align256(size_t(L) * 4);
  p.off_off = p.cnt_off + align256(size_t(E) * 4);
  p.toff_off = p.off_off + align256(size_t(E + 1) * 4);
  p.npos_off = p.toff_off + align256(size_t(E + 1) * 4);
  p.tok_off = p.npos_off + 256;
  p.rv_off = p.tok_off + align256(P * 4);
  p.h_off = p.rv_off + align256(P * 4);
  p.end = p.h_off + align256(P * size_t(2 * de) * 2);
  return p;
}

// Decode router split: d is cut into parts of R rows (a multiple of 8, at most 256); the expert
// kernel's CTAs write one fp32 partial projection [L,E] per part and add the parts in part order.
// Both numbers depend on d only, so the order of every sum does too.
inline int decode_router_rows(int d) {
  const int q0 = (d + 255) / 256;
  return (((d + q0 - 1) / q0) + 7) & ~7;
}
inline int decode_router_parts(int d) { return (d + decode_router_rows(d) - 1) / decode_router_rows(d); }

struct WsLayout {
  size_t s_off, h_off, part_off, cnt_off, total;  // part / cnt: tcgen05 decode path only
};

// Workspace: header | router projection (decode: per-part partials [parts][L,E]; prefill: s [L,E]) |
// decode h (L <= 32) or the prefill regions
inline WsLayout ws_layout(int L, int d, int E, int de) {
  WsLayout w;
  const size_t parts = L <= kDecodeMaxL ? size_t(decode_router_parts(d)) : 1;
  w.s_off = sizeof(WsHeader);
  w.h_off = w.s_off + align256(parts * size_t(L) * E * sizeof(float));
  w.part_off = w.cnt_off = 0;
  if (L <= kDecodeMaxL && !decode_on_tc(L, d, de)) {
    w.total = w.h_off + align256(decode_h_bytes(L, E, de));
  } else if (L <= kDecodeMaxL) {
    w.part_off = w.h_off + align256(tcdec::h_bytes(L, E, de));
    w.cnt_off = w.part_off + align256(tcdec::part_bytes(L));
    w.total = w.cnt_off + align256(tcdec::cnt_words(d, E, de) * 4);
  } else {
    w.total = prefill_layout(w.h_off, L, d, E, de).end;
  }
  return w;
}

// ------------------------------------------------------------------------------------ experts
struct DecodeParams {
  const __nv_bfloat16* x;     // [L,d]
  const float* Wr;            // [d,E]
  const float* br;            // [E] or null
  float* s_part;              // [rq][L,E] router partial projections (workspace)
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
  int inject_timeout;  // 1: the router barrier waits for one arrival more than the grid has (1 ms limit)
  int sum_norm;        // 1: r = g relu(s) / sum relu(s) (the ReMoE router) instead of the RMS
  int keep_l2;         // 1: expert weights are read with the L2 evict-last policy (BFFN_FLAG_KEEP_EXPERTS_IN_L2)
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
  int ustage_units; // its capacity in units of 8 rows; the epilogue runs once per full block
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
  // router: units of (part of rrows rows of d, block of 32 experts), unit u on CTA u mod G
  int rq;           // parts of d
  int rrows;        // rows per part (multiple of 8, <= 256)
  int rcb;          // blocks of 32 experts
  int pre_bytes;    // shared memory before the phase-B partials and the barriers: x, the ring, and room
                    // for the router's staging and the chunk's s [L,E]
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
// CTAs of the kernel the plan selected that fit on one SM at once with `smem` bytes of dynamic shared memory.
cudaError_t expert_decode_occupancy(const DecodeParams& p, size_t smem, int* ctas_per_sm);
cudaError_t expert_decode_launch(const DecodeParams& p, const TensorMaps& tm, const DecodeLaunch& plan,
                                 cudaStream_t st, bool pdl);

// ------------------------------------------------------------------------ decode on tcgen05 (decode_on_tc)
namespace tcdec {
struct Params {
  const __nv_bfloat16* x;     // [L,d]
  const float* Wr;            // [d,E]
  const float* br;            // [E] or null
  float* s_part;              // [rq][L,E] router partial projections (workspace)
  const float* g;             // [E]
  float* y;                   // [L,d]
  int32_t* active_idx;        // [E]
  int32_t* n_active;          // [1]
  uint32_t* tok_mask;         // [L, ceil(E/32)] or null
  int32_t* counts;            // [2] or null
  float* r_out;               // [L,E] or null
  uint8_t* h;                 // h_bytes(L, E, de)
  float* part;                // part_bytes(L): [CTA][2][128][LC] partial accumulators
  uint32_t* cntA;             // [E * nbpe] up-projection block arrivals (zeroed by every call)
  uint32_t* cntB;             // [nrb] down-projection block arrivals, right after cntA
  WsHeader* hdr;
  int L, d, E, de;
  int inject_timeout;  // 1: the router barrier waits for one arrival more than the grid has (1 ms limit)
  int sum_norm;        // 1: r = g relu(s) / sum relu(s) (the ReMoE router) instead of the RMS
  int keep_l2;         // 1: expert weights are read with the L2 evict-last policy (BFFN_FLAG_KEEP_EXPERTS_IN_L2)
  int nck;          // 64-column chunks of d (the last may be ragged: the tensor maps read zeros past d)
  int nbpe, HA;     // up-projection blocks per expert and their height (multiple of 8, <= 128)
  int nrb, HB;      // down-projection blocks of y rows and their height (multiple of 8, <= 128)
  int nJc;          // 64-column chunks of de
  int LB;           // rows of an x tile (L rounded up to 8)
  int NA;           // MMA N of the up-projection (LC)
  int NB;           // MMA N of the down-projection (2 LC)
  int HT;           // bytes of an h tile: 2 LC rows of 128 bytes
  int h_expert_bytes;  // bytes of one expert's h image: nJc tiles
  int S;            // ring slots
  int slot_bytes;   // bytes per slot (multiple of 1024)
  int tmem_cols;    // tensor-memory columns: two accumulators of each projection
  int rq, rrows, rcb;  // router split (decode_router.cuh)
  int pre_bytes;    // shared memory from the ring's start to the barriers: the ring, and room for the
                    // router's staging and the chunk's s [L,E]
  int tail_bytes;   // shared memory after that: barriers and per-CTA tables, at least the 16 KB that
                    // an M = 128 operand read starting in the ring's last slot may reach
};

// Tensor maps (128-byte swizzle, out-of-bounds elements read as zero).  W1 and W2 boxes are 64
// columns wide and 8 << k rows high (k = 0..4); a block of rows is loaded as a sum of such boxes.
struct Maps {
  CUtensorMap w1[5];     // [d, de, E]   box {64, 8 << k, 1}
  CUtensorMap w2[5];     // [de, d, E]   box {64, 8 << k, 1}
  CUtensorMap x;         // [d, L]       box {64, LB}
};

struct Launch {
  int grid;
  size_t smem;
};

bool plan(int L, int d, int E, int de, int grid, int max_smem, Params* p, Launch* out);
cudaError_t launch(const Params& p, const Maps& tm, const Launch& plan, cudaStream_t st, bool pdl);
// CTAs of the kernel for chunks of L tokens with `smem` bytes of dynamic shared memory that fit on one
// SM at once.
cudaError_t occupancy(int L, size_t smem, int* ctas_per_sm);
}  // namespace tcdec

// ------------------------------------------------------------------------ batched decode (decode_batch.cu)
// Many independent chunks of up to 8 tokens in two launches: a router kernel (one CTA per chunk: s,
// the RMSNorm statistics, masks, union and counts of every chunk) and a persistent expert kernel whose
// CTAs form `teams` teams of T; team k takes chunks k, k + teams, ... in order, and its CTAs split each
// chunk's rows.  Weights of several layers are stacked: W1 [n_layers E, de, d], W2 [n_layers E, d, de].
namespace batch {
constexpr int kMaxL = 8;          // tokens per chunk (the MMA's N)
constexpr int kHTile = 16 * 128;  // h tile of one 64-wide j chunk: 8 hi rows, then 8 lo rows, of 128 B
constexpr int kMaxRowsB = 256;    // y rows per CTA (16 m-tiles of 16, two per consumer warp)
constexpr int kMaxTeams = 15;
constexpr int kHImagesPerTeam = 4;  // h images per team (the expert kernel's schedule keeps four in use)

struct Params {
  const __nv_bfloat16* x;   // [C, L, d]
  const int32_t* layer;     // [C] weight set of each chunk, or null: chunk c uses c % n_layers
  const float* Wr;          // [n_layers, d, E]
  const float* g;           // [n_layers, E]
  const float* br;          // [n_layers, E] or null
  float* y;                 // [C, L, d]
  int32_t* active_idx;      // [C, E]
  int32_t* n_active;        // [C]
  int32_t* counts;          // [C, 2] or null
  uint32_t* tok_mask;       // [C, L, ceil(E/32)] or null
  float* r;                 // [C, L, E] router outputs (workspace)
  uint8_t* h;               // [teams][kHImagesPerTeam][E][nJc][kHTile] h images (workspace)
  uint32_t* chunk_bar;      // [C] CTAs whose up-projection of the chunk is published (workspace; zeroed by
                            // the router kernel)
  WsHeader* hdr;
  int C, L, d, E, de, n_layers;
  int sum_norm;             // 1: r = g relu(s) / sum relu(s) (the ReMoE router) instead of the RMS
  int teams, T;             // teams, CTAs per team
  int nKc, nJc;             // 64-wide chunks of d and of de
  int S, slot_bytes;        // ring slots and their size (multiple of 1024)
  int xbuf_bytes;           // x tile of a chunk: nKc x 8 rows x 128 B
  int KWB;                  // 64-wide j chunks per down-projection stage
  int nKf, nJf;             // full 64-wide chunks of d and de (the chunked views cover these)
  int hB[2];                // the two heights of the CTAs' y-row ranges (8 floor(d / 8 / T), + 8)
};

// Stages are one tensor box each: W1 through its chunked view, with a box of h rows x KS(h) chunks for
// every group height h = 8, 16, ..., 128; W2 likewise with a box of the CTA's y rows x KWB chunks.  A
// stage that holds the ragged last chunk of d or de takes per-chunk boxes of the plain views instead.
constexpr int kStageABytes = 32 * 1024;  // an up-projection stage holds at most this many bytes
__host__ __device__ inline int chunks_per_stage_a(int rows, int nKc) {
  const int r16 = (rows + 15) & ~15;
  const int ks = kStageABytes / (r16 * 128);
  return ks < 1 ? 1 : (ks > nKc ? nKc : ks);
}
struct Maps {
  CUtensorMap w1c[16];      // [64, de, d / 64, n_layers E]   box {64, 8 (k + 1), KS, 1}   (d >= 64 only)
  CUtensorMap w2c[2];       // [64, d, de / 64, n_layers E]   box {64, hB[k], KWB, 1}      (de >= 64 only)
  CUtensorMap w1[5];        // [d, de, n_layers E]   box {64, 8 << k, 1}
  CUtensorMap w2[5];        // [de, d, n_layers E]   box {64, 8 << k, 1}
  CUtensorMap x;            // [d, L, C]             box {64, 8, 1}
};

struct Launch {
  int grid;
  size_t smem;
};

// Workspace: header | r [C][L][E] | per-chunk counters | h images
struct Layout {
  size_t r_off, bar_off, h_off, total;
};
inline Layout layout(int C, int L, int E, int de, int teams) {
  Layout l;
  l.r_off = sizeof(WsHeader);
  l.bar_off = l.r_off + align256(size_t(C) * L * E * 4);
  l.h_off = l.bar_off + align256(size_t(C) * 4);
  l.total = l.h_off + size_t(teams) * kHImagesPerTeam * size_t(E) * ((de + 63) / 64) * kHTile;
  return l;
}

bool plan(int C, int L, int d, int E, int de, int teams, int num_sms, int max_smem, Params* p, Launch* out);
cudaError_t launch(const Params& p, const Maps& m, const Launch& plan, cudaStream_t st);
// The router kernel alone (it reads x, layer, Wr, g, br and writes r, active_idx, n_active, counts,
// tok_mask, chunk_bar and the header's error word).
cudaError_t launch_router(const Params& p, cudaStream_t st);
cudaError_t occupancy(size_t smem, int* ctas_per_sm);
}  // namespace batch

// Cross-chunk expert reuse (union_overlap.cu): overlap[c] = |U_a(c) ∩ U_b(c)| from two calls' active lists.
cudaError_t union_overlap_launch(const int32_t* idx_a, const int32_t* n_a, const int32_t* idx_b, const int32_t* n_b,
                                 int C, int E, int32_t* overlap, cudaStream_t st);

// ------------------------------------------------------------------------------------ prefill
struct PrefillParams {
  const __nv_bfloat16* x;   // [L,d]
  const float* Wr;          // [d,E]
  const float* br;          // [E] or null
  const float* g;           // [E]
  const __nv_bfloat16* W1;  // [E,de,d] (L2 prefetches; the GEMM reads it through its tensor map)
  const __nv_bfloat16* W2;  // [E,d,de]
  float* y;                 // [L,d] out (zeroed before the down-projection adds into it)
  int32_t* active_idx;
  int32_t* n_active;
  uint32_t* tok_mask;       // optional
  int32_t* counts;          // optional
  float* r_out;             // optional
  int L, d, E, de, W;       // W = ceil(E / 32)
  int sum_norm;             // 1: r = g relu(s) / sum relu(s) (the ReMoE router) instead of the RMS
  float* s;                 // [L,E]
  float* s_part;            // [ksplit][L,E] partial router projections x Wr over ranges of d (without b)
  int ksplit;               // their count
  __nv_bfloat16* wsplit;    // [2][d][Ep] Wr as bf16 hi + lo pairs, Ep = E rounded up to 64
  uint32_t* mask;           // [L,W]
  float* rms;               // [L]
  int32_t* cnt;             // [E] tokens per expert
  int32_t* off;             // [E+1] pair offset per expert
  int32_t* toff;            // [E+1] 128-row tile offset per expert (toff[E] = tiles)
  int32_t* n_pos;           // positive (t, e) entries of the call
  int32_t* tok;             // [L*E] pair -> token
  float* rv;                // [L*E] pair -> r_{t,e}
  __nv_bfloat16* H;         // [L*E][2 de] hi | lo
  WsHeader* hdr;
  int N1, S1;               // GEMM1: N (= de), pipeline stages
  int N2, S2;               // GEMM2: N tile of d, pipeline stages
};

struct PrefillMaps {
  CUtensorMap w1;   // W1 [E*de rows, d] box 64 x N1
  CUtensorMap h;    // H [L*E rows, 2 de] box 64 x 128
  CUtensorMap w2;   // W2 [E*d rows, de] box 64 x N2
};

struct PrefillLaunch {
  int grid;
  size_t smem1, smem2;
};

bool prefill_plan(int L, int d, int E, int de, int num_sms, int max_smem, PrefillParams* p, PrefillLaunch* out);
cudaError_t prefill_launch(const PrefillParams& p, const PrefillMaps& m, const PrefillLaunch& pl, int num_sms,
                           cudaStream_t st);

// ---------------------------------------------------------------- fp8 expert weights (fp8_decode.cu)
struct Fp8Params {
  const int32_t* layer;     // [C] or null
  const int32_t* active_idx;  // [C, E] (router output)
  const int32_t* n_active;  // [C]
  const float* r;           // [C, L, E] (router output)
  const uint8_t* W1q;       // [NE, de, d] e4m3 codes
  const uint8_t* W2q;       // [NE, d, de]
  const float* s1;          // [NE, de]
  const float* s2;          // [NE, de]
  const float* t2;          // [n_layers]
  __half* xh;               // [C, 8, d] x in f16, rows past L zero (workspace)
  int32_t* offs;            // [C + 1] up-projection items before each chunk (workspace)
  __half* h;                // [wave, E, 2, 8, de] h'' hi and lo planes (workspace)
  int4* desc;               // [wave * E * ceil(de / 64)] up-projection item descriptors (workspace)
  float* y;                 // [C, L, d]
  WsHeader* hdr;             // error word (a bounded wait that ran out)
  int C, L, d, E, de, n_layers, JB, wave;
};
namespace fp8 {
struct Maps {
  CUtensorMap w1;  // W1q as [NE de rows][d bytes], box 128 B x 64 rows, 128-byte swizzle
  CUtensorMap w2;  // W2q as [NE d rows][de bytes], the same box
};
constexpr size_t kHBufBytes = size_t(256) << 20;  // the h buffer: chunks per wave = this / (E 2 8 de 2)
struct Fp8Layout {
  size_t r_off, bar_off, offs_off, xh_off, h_off, desc_off, total;
  int wave;
};
Fp8Layout layout(int C, int L, int d, int E, int de);
size_t workspace_bytes(int C, int L, int d, int E, int de);
cudaError_t quantize(const __nv_bfloat16* W1, const __nv_bfloat16* W2, int n_layers, int E, int d, int de,
                     uint8_t* q1, uint8_t* q2, float* s1, float* s2, float* t2, cudaStream_t st);
cudaError_t forward(const Fp8Params& p, const Maps& m, const batch::Params& rp, int num_sms, cudaStream_t st);
}  // namespace fp8

// ---------------------------------------------------------------- layer backward (layer_backward.cu)
namespace bwd {
struct Layout {  // byte offsets into the workspace
  size_t wsplit, sparts, s, r, rho, dyhl, U, Q, rhhl, duhl, dr, ds, dgc, dshl, cnt, goff, tok, pexp, pidx, xp, total;
  int parts;
};
Layout layout(int T, int d, int E, int de, int num_sms);
cudaError_t launch(const __nv_bfloat16* x, int T, int d, const float* Wr, const float* br, const float* g,
                   const __nv_bfloat16* W1, const __nv_bfloat16* W2, int E, int de, const float* dy, float* dx,
                   float* dWr, float* db, float* dg, float* dW1, float* dW2, void* ws, int num_sms, cudaStream_t st);
}  // namespace bwd

// ---------------------------------------------------------------- CLS-aware losses (cls_losses.cu)
namespace cls {
constexpr int kTargetCtas = 296;               // dWr grid: two CTAs on each SM of a B200
constexpr int kTargetCtasTerms = 1184;         // chunk_terms grid: eight CTAs on each SM
constexpr int kMaxChunkTileBytes = 128 << 10;  // s tile of 4 chunks x 64 experts: L <= 128
struct Plan {
  int T, Ep, dtiles, tok_per_split, splits, b_rows;
  size_t wr_off, ds_off, part_off, loss_off, db_off, total;
};
Plan plan(int C, int L, int d, int E);
bool chunk_fits(int L);
cudaError_t launch(const void* x, int C, int L, int d, const float* Wr, const float* br, int E, float alpha,
                   float w_al, float w_cs, float* loss, float* dS, float* dWr, float* db, float* dx, void* ws,
                   int num_sms, cudaStream_t st);
// s = x [T, d] Wr [d, E] (no bias) on the warp tensor cores with Wr carried as bf16 hi + lo pairs
// (|error| <= 2^-18 sum_k |x_k Wr_k| from the pairs, plus fp32 accumulation), as `parts` partial
// products over consecutive ranges of d: s holds parts x [T, E] fp32, to be added in part order; wsplit
// holds 2 d (E rounded up to 64) bf16.  Two launches.  router_projection_parts picks the part count
// (1 .. kMaxRouterParts) that gives the GPU about two CTAs per SM.
constexpr int kMaxRouterParts = 4;
int router_projection_parts(int T, int d, int E, int num_sms);
cudaError_t router_projection(const __nv_bfloat16* x, int T, int d, const float* Wr, int E, __nv_bfloat16* wsplit,
                              float* s, int parts, int num_sms, cudaStream_t st);
}  // namespace cls

}  // namespace bffn
