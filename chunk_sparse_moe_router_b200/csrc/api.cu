// Host side of the C ABI declared in include/blockffn.h: argument checks, workspace handling and
// the kernel launches of one BlockFFN chunk-layer forward.
#include <cmath>
#include <cstdlib>
#include <mutex>

#include "blockffn.h"
#include "blockffn_internal.cuh"

namespace bffn {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int max_smem = 0;
  bool pdl = true;
};

struct DeviceWorkspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};

std::mutex g_mutex;
DeviceInfo g_info[kMaxDevices];
DeviceWorkspace g_ws[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

int cuda_fail(cudaError_t) {
  (void)cudaGetLastError();  // clear the sticky-free error state of this thread
  return BFFN_ECUDA;
}

int device_info(DeviceInfo* out, int* dev_out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err);
  if (dev < 0 || dev >= kMaxDevices) return BFFN_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& di = g_info[dev];
  if (!di.ready) {
    if ((err = cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(err);
    if ((err = cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
        cudaSuccess)
      return cuda_fail(err);
    di.ready = true;
  }
  *out = di;
  *dev_out = dev;
  return BFFN_OK;
}

// The library's per-device workspace, grown on demand (never during stream capture).
int internal_workspace(int dev, size_t need, cudaStream_t st, void** ws) {
  // BFFN_TEST_FAIL_ALLOC=1 makes every call that uses this workspace fail as its allocation would on a
  // device without free memory (BFFN_ENOMEM, nothing enqueued): a host-side stand-in that lets tests
  // reach that path without exhausting the GPU
  const char* fake = getenv("BFFN_TEST_FAIL_ALLOC");
  if (fake != nullptr && fake[0] == '1') return BFFN_ENOMEM;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceWorkspace& w = g_ws[dev];
  if (w.bytes < need) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t err = cudaStreamIsCapturing(st, &cap);
    if (err != cudaSuccess) return cuda_fail(err);
    if (cap != cudaStreamCaptureStatusNone) return BFFN_ENOMEM;
    if (w.ptr) {
      if ((err = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(err);
      cudaFree(w.ptr);
      w.ptr = nullptr;
      w.bytes = 0;
    }
    size_t bytes = need < (size_t(1) << 20) ? (size_t(1) << 20) : need;
    if (cudaMalloc(&w.ptr, bytes) != cudaSuccess) {
      (void)cudaGetLastError();
      w.ptr = nullptr;
      return BFFN_ENOMEM;
    }
    if ((err = cudaMemsetAsync(w.ptr, 0, bytes, st)) != cudaSuccess) return cuda_fail(err);
    w.bytes = bytes;
  }
  *ws = w.ptr;
  return BFFN_OK;
}

bool shapes_ok(int L, int d, int E, int de) {
  return L >= 1 && E >= 1 && E <= kMaxE && d >= 8 && d % 8 == 0 && de >= 8 && de % 8 == 0 &&
         (long long)L * d < (1ll << 31) && (long long)E * de * d < (1ll << 40);
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    (void)cudaGetLastError();
  });
  return fn;
}

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzle, out-of-bounds elements read as 0.
bool encode_tiled(CUtensorMap* tm, CUtensorMapDataType type, const void* base, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[5], gstride[4];
  cuuint32_t bdim[5], estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
  return fn(tm, type, cuuint32_t(rank), const_cast<void*>(base), gdim, gstride, bdim, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_bf16(CUtensorMap* tm, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                 const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[5], gstride[4];
  cuuint32_t bdim[5], estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base), gdim, gstride, bdim,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Decode shapes decode_on_tc selects: the tcgen05 decode kernel (expert_decode_tc.cu).
int forward_decode_tc(const void* x, int L, int d, const float* Wr, const float* g, const void* W1,
                      const void* W2, int E, int de, float* y, int32_t* active_idx, int32_t* n_active,
                      const float* br, uint32_t* tok_mask, int32_t* counts, float* r_out, void* ws,
                      const DeviceInfo& di, int share, bool inject, bool sum_norm, bool keep_l2,
                      cudaStream_t st) {
  const WsLayout lay = ws_layout(L, d, E, de);
  uint8_t* base = static_cast<uint8_t*>(ws);
  tcdec::Params dp;
  dp.inject_timeout = inject ? 1 : 0;
  dp.sum_norm = sum_norm ? 1 : 0;
  dp.keep_l2 = keep_l2 ? 1 : 0;
  dp.x = static_cast<const __nv_bfloat16*>(x);
  dp.Wr = Wr;
  dp.br = br;
  dp.s_part = reinterpret_cast<float*>(base + lay.s_off);
  dp.g = g;
  dp.y = y;
  dp.active_idx = active_idx;
  dp.n_active = n_active;
  dp.tok_mask = tok_mask;
  dp.counts = counts;
  dp.r_out = r_out;
  dp.h = base + lay.h_off;
  dp.part = reinterpret_cast<float*>(base + lay.part_off);
  dp.cntA = reinterpret_cast<uint32_t*>(base + lay.cnt_off);
  dp.cntB = dp.cntA + size_t(E) * ((de + 127) / 128);
  dp.hdr = reinterpret_cast<WsHeader*>(base);
  dp.L = L;
  dp.d = d;
  dp.E = E;
  dp.de = de;
  tcdec::Launch dl;
  const int grid = di.num_sms / share;  // one persistent CTA per SM of this call's share
  if (grid < 1 || !tcdec::plan(L, d, E, de, grid, di.max_smem, &dp, &dl)) return BFFN_EUNSUPPORTED;
  {
    // the kernel's grid barriers need every CTA resident at once
    int per_sm = 0;
    const cudaError_t oe = tcdec::occupancy(L, dl.smem, &per_sm);
    if (oe != cudaSuccess) return cuda_fail(oe);
    if (per_sm < 1) return BFFN_EUNSUPPORTED;
  }
  tcdec::Maps tm;
  {
    const uint64_t xrow = uint64_t(d) * 2, w1e = uint64_t(d) * de * 2;
    const uint64_t w2row = uint64_t(de) * 2, w2e = uint64_t(d) * de * 2;
    const uint64_t xd[2] = {uint64_t(d), uint64_t(L)}, xs[1] = {xrow};
    const uint32_t xb[2] = {64, uint32_t(dp.LB)};
    if (!encode_bf16(&tm.x, x, 2, xd, xs, xb)) return BFFN_ECUDA;
    const uint64_t w1d[3] = {uint64_t(d), uint64_t(de), uint64_t(E)}, w1s[2] = {xrow, w1e};
    const uint64_t w2d[3] = {uint64_t(de), uint64_t(d), uint64_t(E)}, w2s[2] = {w2row, w2e};
    for (int k = 0; k < 5; ++k) {
      const uint32_t b[3] = {64, uint32_t(8u << k), 1};
      if (!encode_bf16(&tm.w1[k], W1, 3, w1d, w1s, b)) return BFFN_ECUDA;
      if (!encode_bf16(&tm.w2[k], W2, 3, w2d, w2s, b)) return BFFN_ECUDA;
    }
  }
  const cudaError_t err = tcdec::launch(dp, tm, dl, st, di.pdl);
  if (err != cudaSuccess) return cuda_fail(err);
  return BFFN_OK;
}

int forward_decode(const void* x, int L, int d, const float* Wr, const float* g, const void* W1,
                   const void* W2, int E, int de, float* y, int32_t* active_idx, int32_t* n_active,
                   const float* br, uint32_t* tok_mask, int32_t* counts, float* r_out, void* ws,
                   const DeviceInfo& di, int share, bool inject, bool sum_norm, bool keep_l2, cudaStream_t st) {
  const WsLayout lay = ws_layout(L, d, E, de);
  uint8_t* base = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base);

  DecodeParams dp;
  dp.inject_timeout = inject ? 1 : 0;
  dp.sum_norm = sum_norm ? 1 : 0;
  dp.keep_l2 = keep_l2 ? 1 : 0;
  dp.x = static_cast<const __nv_bfloat16*>(x);
  dp.Wr = Wr;
  dp.br = br;
  dp.s_part = reinterpret_cast<float*>(base + lay.s_off);
  dp.g = g;
  dp.y = y;
  dp.active_idx = active_idx;
  dp.n_active = n_active;
  dp.tok_mask = tok_mask;
  dp.counts = counts;
  dp.r_out = r_out;
  dp.h = base + lay.h_off;
  dp.hdr = hdr;
  dp.L = L;
  dp.d = d;
  dp.E = E;
  dp.de = de;
  DecodeLaunch dl;
  const int grid = di.num_sms / share;  // one persistent CTA per SM of this call's share
  if (grid < 1 || !expert_decode_plan(L, d, E, de, grid, di.max_smem, &dp, &dl)) return BFFN_EUNSUPPORTED;
  {
    // the kernel's grid barriers need every CTA resident at once
    int per_sm = 0;
    const cudaError_t oe = expert_decode_occupancy(dp, dl.smem, &per_sm);
    if (oe != cudaSuccess) return cuda_fail(oe);
    if (per_sm < 1) return BFFN_EUNSUPPORTED;
  }

  TensorMaps tm;
  {
    const uint64_t xrow = uint64_t(d) * 2, w1e = uint64_t(d) * de * 2;
    const uint64_t w2row = uint64_t(de) * 2, w2e = uint64_t(d) * de * 2;
    const int KC = dp.nKf / dp.KP;
    // plain views: the ragged last chunk of d (and every stage when d < 64)
    const uint64_t x2d[2] = {uint64_t(d), uint64_t(L)}, x2s[1] = {xrow};
    const uint32_t x2b[2] = {64, uint32_t(dp.LB)};
    if (!encode_bf16(&tm.x_2d, x, 2, x2d, x2s, x2b)) return BFFN_ECUDA;
    const uint64_t w13d[3] = {uint64_t(d), uint64_t(de), uint64_t(E)}, w13s[2] = {xrow, w1e};
    for (int k = 0; k < 4; ++k) {
      const uint32_t b[3] = {64, uint32_t(1u << k), 1};
      if (!encode_bf16(&tm.w1_3d[k], W1, 3, w13d, w13s, b)) return BFFN_ECUDA;
    }
    // chunked views over the full chunks: a box is whole rows of one K pass
    if (KC > 0) {
      const uint64_t xcd[3] = {64, uint64_t(L), uint64_t(dp.nKf)}, xcs[2] = {xrow, 128};
      const uint32_t xcb[3] = {64, uint32_t(dp.LB), uint32_t(KC)};
      if (!encode_bf16(&tm.x_ch, x, 3, xcd, xcs, xcb)) return BFFN_ECUDA;
      const uint64_t w1cd[4] = {64, uint64_t(de), uint64_t(dp.nKf), uint64_t(E)}, w1cs[3] = {xrow, 128, w1e};
      for (int k = 0; k < 4; ++k) {
        const uint32_t b[4] = {64, uint32_t(1u << k), uint32_t(KC), 1};
        if (!encode_bf16(&tm.w1_ch[k], W1, 4, w1cd, w1cs, b)) return BFFN_ECUDA;
      }
    } else {
      tm.x_ch = tm.x_2d;
      for (int k = 0; k < 4; ++k) tm.w1_ch[k] = tm.w1_3d[k];
    }
    const uint64_t w23d[3] = {uint64_t(de), uint64_t(d), uint64_t(E)}, w23s[2] = {w2row, w2e};
    const uint32_t w2b3[3] = {64, uint32_t(dp.RBB), 1};
    if (!encode_bf16(&tm.w2_3d, W2, 3, w23d, w23s, w2b3)) return BFFN_ECUDA;
    if (dp.nJf > 0) {
      const uint64_t w2cd[4] = {64, uint64_t(d), uint64_t(dp.nJf), uint64_t(E)}, w2cs[3] = {w2row, 128, w2e};
      const uint32_t w2cb[4] = {64, uint32_t(dp.RBB), uint32_t(dp.KWB), 1};
      if (!encode_bf16(&tm.w2_ch, W2, 4, w2cd, w2cs, w2cb)) return BFFN_ECUDA;
    } else {
      tm.w2_ch = tm.w2_3d;
    }
  }

  const cudaError_t err = expert_decode_launch(dp, tm, dl, st, di.pdl);
  if (err != cudaSuccess) return cuda_fail(err);
  return BFFN_OK;
}

int forward_prefill(const void* x, int L, int d, const float* Wr, const float* g, const void* W1,
                    const void* W2, int E, int de, float* y, int32_t* active_idx, int32_t* n_active,
                    const float* br, uint32_t* tok_mask, int32_t* counts, float* r_out, void* ws,
                    const DeviceInfo& di, bool sum_norm, cudaStream_t st) {
  if (!aligned16(y)) return BFFN_EINVAL;  // the down-projection adds into y 16 bytes at a time
  const WsLayout lay = ws_layout(L, d, E, de);
  const PrefillLayout pl = prefill_layout(lay.h_off, L, d, E, de);
  uint8_t* base = static_cast<uint8_t*>(ws);
  PrefillParams p;
  p.sum_norm = sum_norm ? 1 : 0;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.Wr = Wr;
  p.br = br;
  p.g = g;
  p.W1 = static_cast<const __nv_bfloat16*>(W1);
  p.W2 = static_cast<const __nv_bfloat16*>(W2);
  p.y = y;
  p.active_idx = active_idx;
  p.n_active = n_active;
  p.tok_mask = tok_mask;
  p.counts = counts;
  p.r_out = r_out;
  p.L = L;
  p.d = d;
  p.E = E;
  p.de = de;
  p.s = reinterpret_cast<float*>(base + lay.s_off);
  p.s_part = reinterpret_cast<float*>(base + pl.spart_off);
  p.wsplit = reinterpret_cast<__nv_bfloat16*>(base + pl.wsplit_off);
  p.mask = reinterpret_cast<uint32_t*>(base + pl.mask_off);
  p.rms = reinterpret_cast<float*>(base + pl.rms_off);
  p.cnt = reinterpret_cast<int32_t*>(base + pl.cnt_off);
  p.off = reinterpret_cast<int32_t*>(base + pl.off_off);
  p.toff = reinterpret_cast<int32_t*>(base + pl.toff_off);
  p.n_pos = reinterpret_cast<int32_t*>(base + pl.npos_off);
  p.tok = reinterpret_cast<int32_t*>(base + pl.tok_off);
  p.rv = reinterpret_cast<float*>(base + pl.rv_off);
  p.H = reinterpret_cast<__nv_bfloat16*>(base + pl.h_off);
  p.hdr = reinterpret_cast<WsHeader*>(base);
  PrefillLaunch launch;
  if (!prefill_plan(L, d, E, de, di.num_sms, di.max_smem, &p, &launch)) return BFFN_EUNSUPPORTED;

  PrefillMaps m;
  {
    const uint64_t w1d[2] = {uint64_t(d), uint64_t(E) * de}, w1s[1] = {uint64_t(d) * 2};
    const uint32_t w1b[2] = {64, uint32_t(p.N1)};
    if (!encode_bf16(&m.w1, W1, 2, w1d, w1s, w1b)) return BFFN_ECUDA;
    const uint64_t hd[2] = {uint64_t(2 * de), uint64_t(L) * E}, hs[1] = {uint64_t(2 * de) * 2};
    const uint32_t hb[2] = {64, 128};
    if (!encode_bf16(&m.h, p.H, 2, hd, hs, hb)) return BFFN_ECUDA;
    const uint64_t w2d[2] = {uint64_t(de), uint64_t(E) * d}, w2s[1] = {uint64_t(de) * 2};
    const uint32_t w2b[2] = {64, uint32_t(p.N2)};
    if (!encode_bf16(&m.w2, W2, 2, w2d, w2s, w2b)) return BFFN_ECUDA;
  }
  const cudaError_t err = prefill_launch(p, m, launch, di.num_sms, st);
  if (err != cudaSuccess) return cuda_fail(err);
  return BFFN_OK;
}

int forward_batch(const void* x, int C, int L, int d, const int32_t* layer, int n_layers, const float* Wr,
                  const float* g, const float* br, const void* W1, const void* W2, int E, int de, float* y,
                  int32_t* active_idx, int32_t* n_active, int32_t* counts, uint32_t* tok_mask, int teams,
                  bool sum_norm, void* ws, const DeviceInfo& di, cudaStream_t st) {
  batch::Params p;
  batch::Launch launch;
  if (!batch::plan(C, L, d, E, de, teams, di.num_sms, di.max_smem, &p, &launch)) return BFFN_EUNSUPPORTED;
  {
    int per_sm = 0;  // the team barriers need every CTA of a team resident at once
    const cudaError_t oe = batch::occupancy(launch.smem, &per_sm);
    if (oe != cudaSuccess) return cuda_fail(oe);
    if (per_sm < 1) return BFFN_EUNSUPPORTED;
  }
  const batch::Layout lay = batch::layout(C, L, E, de, teams);
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.layer = layer;
  p.Wr = Wr;
  p.g = g;
  p.br = br;
  p.y = y;
  p.active_idx = active_idx;
  p.n_active = n_active;
  p.counts = counts;
  p.tok_mask = tok_mask;
  p.r = reinterpret_cast<float*>(base + lay.r_off);
  p.h = base + lay.h_off;
  p.chunk_bar = reinterpret_cast<uint32_t*>(base + lay.bar_off);
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.C = C;
  p.L = L;
  p.d = d;
  p.E = E;
  p.de = de;
  p.n_layers = n_layers;
  p.sum_norm = sum_norm ? 1 : 0;
  batch::Maps m;
  {
    const uint64_t NE = uint64_t(n_layers) * E;
    const uint64_t w1d[3] = {uint64_t(d), uint64_t(de), NE}, w1s[2] = {uint64_t(d) * 2, uint64_t(d) * de * 2};
    const uint64_t w2d[3] = {uint64_t(de), uint64_t(d), NE}, w2s[2] = {uint64_t(de) * 2, uint64_t(d) * de * 2};
    for (int k = 0; k < 5; ++k) {
      const uint32_t b[3] = {64, uint32_t(8u << k), 1};
      if (!encode_bf16(&m.w1[k], W1, 3, w1d, w1s, b)) return BFFN_ECUDA;
      if (!encode_bf16(&m.w2[k], W2, 3, w2d, w2s, b)) return BFFN_ECUDA;
    }
    // chunked views: one box is a whole stage (rows x consecutive 64-wide chunks)
    if (p.nKf > 0) {
      const uint64_t cd[4] = {64, uint64_t(de), uint64_t(p.nKf), NE};
      const uint64_t cs[3] = {uint64_t(d) * 2, 128, uint64_t(d) * de * 2};
      for (int k = 0; k < 16; ++k) {
        const int h = 8 * (k + 1);
        const uint32_t b[4] = {64, uint32_t(h), uint32_t(batch::chunks_per_stage_a(h, p.nKc)), 1};
        if (!encode_bf16(&m.w1c[k], W1, 4, cd, cs, b)) return BFFN_ECUDA;
      }
    }
    if (p.nJf > 0) {
      const uint64_t cd[4] = {64, uint64_t(d), uint64_t(p.nJf), NE};
      const uint64_t cs[3] = {uint64_t(de) * 2, 128, uint64_t(d) * de * 2};
      for (int k = 0; k < 2; ++k) {
        if (p.hB[k] < 8 || p.hB[k] > batch::kMaxRowsB) {
          m.w2c[k] = m.w2[0];  // a height no CTA has
          continue;
        }
        const uint32_t b[4] = {64, uint32_t(p.hB[k]), uint32_t(p.KWB), 1};
        if (!encode_bf16(&m.w2c[k], W2, 4, cd, cs, b)) return BFFN_ECUDA;
      }
    }
    const uint64_t xd[3] = {uint64_t(d), uint64_t(L), uint64_t(C)}, xs[2] = {uint64_t(d) * 2, uint64_t(L) * d * 2};
    const uint32_t xb[3] = {64, 8, 1};
    if (!encode_bf16(&m.x, x, 3, xd, xs, xb)) return BFFN_ECUDA;
  }
  const cudaError_t err = batch::launch(p, m, launch, st);
  if (err != cudaSuccess) return cuda_fail(err);
  return BFFN_OK;
}

bool batch_args_ok(int C, int L, int d, int n_layers, int E, int de) {
  return C >= 1 && n_layers >= 1 && shapes_ok(L, d, E, de) && (long long)n_layers * E < (1ll << 31) &&
         (long long)C * L * d < (1ll << 40) && (long long)n_layers * E * de * d < (1ll << 40);
}

int batch_teams(int flags, int C) {
  const int k = (flags >> 4) & 15;
  if (k != 0) return k;
  return C < 8 ? C : 8;
}

}  // namespace
}  // namespace bffn

using namespace bffn;

extern "C" {

int blockffn_abi_version(void) { return 100; }

const char* blockffn_status_string(int status) {
  switch (status) {
    case BFFN_OK: return "ok";
    case BFFN_EINVAL: return "invalid argument";
    case BFFN_ECUDA: return "CUDA runtime error";
    case BFFN_ENOMEM: return "workspace allocation failed or workspace too small";
    case BFFN_ETIMEOUT: return "a bounded device-side wait ran out";
    case BFFN_EUNSUPPORTED: return "shape not supported by this build";
    default: return "unknown status";
  }
}

size_t blockffn_workspace_size(int L, int d, int E, int de) {
  if (!shapes_ok(L, d, E, de)) return 0;
  return ws_layout(L, d, E, de).total;
}

int blockffn_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || !aligned256(workspace) || workspace_bytes < sizeof(WsHeader)) return BFFN_EINVAL;
  cudaError_t err = cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

int blockffn_chunk_forward_ex(const void* x, int L, int d, const float* Wr, const float* g,
                              const void* W1, const void* W2, int E, int de, float* y,
                              int32_t* active_idx, int32_t* n_active, const float* br,
                              uint32_t* tok_mask, int32_t* counts, float* r_out, int flags,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!shapes_ok(L, d, E, de)) return BFFN_EINVAL;
  // read by bulk / 16-byte copies: 16-byte alignment; everything else: 4-byte (natural) alignment
  const void* bulk[] = {x, Wr, W1, W2};
  for (const void* p : bulk)
    if (p == nullptr || !aligned16(p)) return BFFN_EINVAL;
  const void* scalar[] = {g, y, active_idx, n_active};
  for (const void* p : scalar)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  const void* optional[] = {br, tok_mask, counts, r_out};
  for (const void* p : optional)
    if (p != nullptr && !aligned4(p)) return BFFN_EINVAL;
  if (workspace != nullptr && !aligned256(workspace)) return BFFN_EINVAL;
  const int path = flags & 3;
  if (path == 3) return BFFN_EINVAL;
  const int share = ((flags >> 4) & 15) == 0 ? 1 : ((flags >> 4) & 15);
  if ((flags & ~(0xF3 | BFFN_FLAG_INJECT_ROUTER_TIMEOUT | BFFN_FLAG_ROUTER_SUM_NORM | BFFN_FLAG_KEEP_EXPERTS_IN_L2)) != 0)
    return BFFN_EINVAL;
  const bool inject = (flags & BFFN_FLAG_INJECT_ROUTER_TIMEOUT) != 0;
  const bool sum_norm = (flags & BFFN_FLAG_ROUTER_SUM_NORM) != 0;
  const bool keep_l2 = (flags & BFFN_FLAG_KEEP_EXPERTS_IN_L2) != 0;
  const bool decode = (path == BFFN_PATH_DECODE) || (path == BFFN_PATH_AUTO && L <= kDecodeMaxL);
  if (decode && L > kDecodeMaxL) return BFFN_EUNSUPPORTED;
  if (!decode && inject) return BFFN_EUNSUPPORTED;  // the injection exists on the decode path only
  if (!decode && L <= kDecodeMaxL) return BFFN_EUNSUPPORTED;  // the prefill path takes L > 32
  if (!decode && (d % 64 != 0 || de % 64 != 0 || de > 256)) return BFFN_EUNSUPPORTED;
  if (!decode && !aligned16(y)) return BFFN_EINVAL;  // the down-projection adds into y 16 bytes at a time

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceInfo di;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != BFFN_OK) return rc;
  const size_t need = ws_layout(L, d, E, de).total;
  void* ws = workspace;
  if (ws == nullptr) {
    rc = internal_workspace(dev, need, st, &ws);
    if (rc != BFFN_OK) return rc;
  } else if (workspace_bytes < need) {
    return BFFN_ENOMEM;
  }
  if (decode) {
    if (decode_on_tc(L, d, de))
      return forward_decode_tc(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, tok_mask, counts,
                               r_out, ws, di, share, inject, sum_norm, keep_l2, st);
    return forward_decode(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, tok_mask, counts,
                          r_out, ws, di, share, inject, sum_norm, keep_l2, st);
  }
  return forward_prefill(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, tok_mask, counts, r_out,
                         ws, di, sum_norm, st);
}

int blockffn_chunk_forward(const void* x, int L, int d, const float* Wr, const float* g,
                           const void* W1, const void* W2, int E, int de, float* y,
                           int32_t* active_idx, int32_t* n_active, void* stream) {
  return blockffn_chunk_forward_ex(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, nullptr,
                                   nullptr, nullptr, nullptr, BFFN_PATH_AUTO, nullptr, 0, stream);
}

size_t blockffn_batch_workspace_size(int C, int L, int d, int E, int de, int flags) {
  if (!batch_args_ok(C, L, d, 1, E, de) || (flags & ~(0xF0 | BFFN_FLAG_ROUTER_SUM_NORM)) != 0) return 0;
  return batch::layout(C, L, E, de, batch_teams(flags, C)).total;
}

int blockffn_chunk_forward_batch(const void* x, int C, int L, int d, const int32_t* layer, int n_layers,
                                 const float* Wr, const float* g, const float* br, const void* W1, const void* W2,
                                 int E, int de, float* y, int32_t* active_idx, int32_t* n_active, int32_t* counts,
                                 uint32_t* tok_mask, int flags, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!batch_args_ok(C, L, d, n_layers, E, de)) return BFFN_EINVAL;
  if ((flags & ~(0xF0 | BFFN_FLAG_ROUTER_SUM_NORM)) != 0) return BFFN_EINVAL;
  const void* bulk[] = {x, Wr, W1, W2};
  for (const void* p : bulk)
    if (p == nullptr || !aligned16(p)) return BFFN_EINVAL;
  const void* scalar[] = {g, y, active_idx, n_active};
  for (const void* p : scalar)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  const void* optional[] = {layer, br, counts, tok_mask};
  for (const void* p : optional)
    if (p != nullptr && !aligned4(p)) return BFFN_EINVAL;
  if (workspace != nullptr && !aligned256(workspace)) return BFFN_EINVAL;
  if (L > batch::kMaxL) return BFFN_EUNSUPPORTED;
  const int teams = batch_teams(flags, C);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceInfo di;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != BFFN_OK) return rc;
  const size_t need = batch::layout(C, L, E, de, teams).total;
  void* ws = workspace;
  if (ws == nullptr) {
    rc = internal_workspace(dev, need, st, &ws);
    if (rc != BFFN_OK) return rc;
  } else if (workspace_bytes < need) {
    return BFFN_ENOMEM;
  }
  return forward_batch(x, C, L, d, layer, n_layers, Wr, g, br, W1, W2, E, de, y, active_idx, n_active, counts,
                       tok_mask, teams, (flags & BFFN_FLAG_ROUTER_SUM_NORM) != 0, ws, di, st);
}

bool fp8_args_ok(int C, int L, int d, int n_layers, int E, int de) {
  return batch_args_ok(C, L, d, n_layers, E, de) && d % 16 == 0 && de % 16 == 0 && L <= batch::kMaxL &&
         1ll * C * 8 * d < (1ll << 40);
}

int blockffn_quantize_fp8(const void* W1, const void* W2, int n_layers, int E, int d, int de, uint8_t* W1q,
                          uint8_t* W2q, float* s1, float* s2, float* t2, void* stream) {
  if (n_layers < 1 || E < 1 || E > kMaxE || d < 16 || d % 16 != 0 || de < 16 || de % 16 != 0 ||
      1ll * n_layers * E * de * d >= (1ll << 40))
    return BFFN_EINVAL;
  const void* bulk[] = {W1, W2, W1q, W2q};
  for (const void* p : bulk)
    if (p == nullptr || !aligned16(p)) return BFFN_EINVAL;
  const void* scal[] = {s1, s2, t2};
  for (const void* p : scal)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  const cudaError_t err =
      fp8::quantize(static_cast<const __nv_bfloat16*>(W1), static_cast<const __nv_bfloat16*>(W2), n_layers, E, d, de,
                    W1q, W2q, s1, s2, t2, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

size_t blockffn_batch_fp8_workspace_size(int C, int L, int d, int E, int de) {
  if (!fp8_args_ok(C, L, d, 1, E, de)) return 0;
  return fp8::workspace_bytes(C, L, d, E, de);
}

int blockffn_chunk_forward_batch_fp8(const void* x, int C, int L, int d, const int32_t* layer, int n_layers,
                                     const float* Wr, const float* g, const float* br, const uint8_t* W1q,
                                     const float* s1, const uint8_t* W2q, const float* s2, const float* t2, int E,
                                     int de, float* y, int32_t* active_idx, int32_t* n_active, int32_t* counts,
                                     uint32_t* tok_mask, int flags, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!fp8_args_ok(C, L, d, n_layers, E, de)) return BFFN_EINVAL;
  if ((flags & ~BFFN_FLAG_ROUTER_SUM_NORM) != 0) return BFFN_EINVAL;
  const void* bulk[] = {x, W1q, W2q};
  for (const void* p : bulk)
    if (p == nullptr || !aligned16(p)) return BFFN_EINVAL;
  const void* scalar[] = {Wr, g, s1, s2, t2, y, active_idx, n_active};
  for (const void* p : scalar)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  const void* optional[] = {layer, br, counts, tok_mask};
  for (const void* p : optional)
    if (p != nullptr && !aligned4(p)) return BFFN_EINVAL;
  if (workspace != nullptr && !aligned256(workspace)) return BFFN_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceInfo di;
  int dev = 0;
  int rc = device_info(&di, &dev);
  if (rc != BFFN_OK) return rc;
  const fp8::Fp8Layout lay = fp8::layout(C, L, d, E, de);
  void* ws = workspace;
  if (ws == nullptr) {
    rc = internal_workspace(dev, lay.total, st, &ws);
    if (rc != BFFN_OK) return rc;
  } else if (workspace_bytes < lay.total) {
    return BFFN_ENOMEM;
  }
  uint8_t* base = static_cast<uint8_t*>(ws);
  batch::Params rp{};
  rp.x = static_cast<const __nv_bfloat16*>(x);
  rp.layer = layer;
  rp.Wr = Wr;
  rp.g = g;
  rp.br = br;
  rp.y = y;
  rp.active_idx = active_idx;
  rp.n_active = n_active;
  rp.counts = counts;
  rp.tok_mask = tok_mask;
  rp.r = reinterpret_cast<float*>(base + lay.r_off);
  rp.chunk_bar = reinterpret_cast<uint32_t*>(base + lay.bar_off);
  rp.hdr = reinterpret_cast<WsHeader*>(base);
  rp.C = C;
  rp.L = L;
  rp.d = d;
  rp.E = E;
  rp.de = de;
  rp.n_layers = n_layers;
  rp.sum_norm = (flags & BFFN_FLAG_ROUTER_SUM_NORM) != 0 ? 1 : 0;
  Fp8Params p{};
  p.layer = layer;
  p.active_idx = active_idx;
  p.n_active = n_active;
  p.r = rp.r;
  p.W1q = W1q;
  p.W2q = W2q;
  p.s1 = s1;
  p.s2 = s2;
  p.t2 = t2;
  p.xh = reinterpret_cast<__half*>(base + lay.xh_off);
  p.offs = reinterpret_cast<int32_t*>(base + lay.offs_off);
  p.h = reinterpret_cast<__half*>(base + lay.h_off);
  p.desc = reinterpret_cast<int4*>(base + lay.desc_off);
  p.y = y;
  p.C = C;
  p.L = L;
  p.d = d;
  p.E = E;
  p.de = de;
  p.n_layers = n_layers;
  p.JB = (de + 63) / 64;
  p.wave = lay.wave;
  p.hdr = rp.hdr;
  fp8::Maps maps;
  {  // the code matrices as 2D byte tensors, boxes of 128 bytes x 64 rows in the 128-byte swizzle
    const uint64_t NE = uint64_t(n_layers) * E;
    const uint64_t d1[2] = {uint64_t(d), NE * de}, s1b[1] = {uint64_t(d)};
    const uint64_t d2[2] = {uint64_t(de), NE * d}, s2b[1] = {uint64_t(de)};
    const uint32_t box[2] = {128, 64};
    if (!encode_tiled(&maps.w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, W1q, 2, d1, s1b, box)) return BFFN_ECUDA;
    if (!encode_tiled(&maps.w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, W2q, 2, d2, s2b, box)) return BFFN_ECUDA;
  }
  const cudaError_t err = fp8::forward(p, maps, rp, di.num_sms, st);
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

size_t blockffn_layer_backward_workspace_size(int T, int d, int E, int de) {
  if (T < 1 || T > 65535 * 128 || d < 8 || d % 8 != 0 || de < 8 || de % 8 != 0 || E < 1 || E > kMaxE ||
      1ll * T * E * de >= (1ll << 31) || 1ll * T * d >= (1ll << 31))
    return 0;
  DeviceInfo di;
  int dev = 0;
  const int sms = device_info(&di, &dev) == BFFN_OK ? di.num_sms : 148;
  return bwd::layout(T, d, E, de, sms).total;
}

int blockffn_layer_backward(const void* x, int T, int d, const float* Wr, const float* br, const float* g,
                            const void* W1, const void* W2, int E, int de, const float* dy, float* dx, float* dWr,
                            float* db, float* dg, float* dW1, float* dW2, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (T < 1 || T > 65535 * 128 || d < 8 || d % 8 != 0 || de < 8 || de % 8 != 0 || E < 1 || E > kMaxE ||
      1ll * T * E * de >= (1ll << 31) || 1ll * T * d >= (1ll << 31))
    return BFFN_EINVAL;
  const void* bulk[] = {x, W1, W2};
  for (const void* p : bulk)
    if (p == nullptr || !aligned16(p)) return BFFN_EINVAL;
  const void* req[] = {Wr, g, dy, dx, dWr, db, dg, dW1, dW2};
  for (const void* p : req)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  if (!aligned16(dy)) return BFFN_EINVAL;
  if (br != nullptr && !aligned4(br)) return BFFN_EINVAL;
  if (workspace == nullptr || !aligned256(workspace)) return BFFN_EINVAL;
  DeviceInfo di;
  int dev = 0;
  const int rc = device_info(&di, &dev);
  if (rc != BFFN_OK) return rc;
  if (workspace_bytes < bwd::layout(T, d, E, de, di.num_sms).total) return BFFN_ENOMEM;
  const cudaError_t err =
      bwd::launch(static_cast<const __nv_bfloat16*>(x), T, d, Wr, br, g, static_cast<const __nv_bfloat16*>(W1),
                  static_cast<const __nv_bfloat16*>(W2), E, de, dy, dx, dWr, db, dg, dW1, dW2, workspace, di.num_sms,
                  static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

int blockffn_union_overlap(const int32_t* active_idx_a, const int32_t* n_active_a, const int32_t* active_idx_b,
                           const int32_t* n_active_b, int C, int E, int32_t* overlap, void* stream) {
  if (C < 1 || E < 1 || E > kMaxE) return BFFN_EINVAL;
  const void* ptrs[] = {active_idx_a, n_active_a, active_idx_b, n_active_b, overlap};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned4(p)) return BFFN_EINVAL;
  const cudaError_t err =
      union_overlap_launch(active_idx_a, n_active_a, active_idx_b, n_active_b, C, E, overlap,
                           static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

size_t blockffn_cls_losses_workspace_size(int C, int L, int d, int E) {
  if (C < 1 || L < 1 || d < 8 || d % 8 != 0 || E < 1 || E > kMaxE || 1ll * C * L > (1ll << 30)) return 0;
  return cls::plan(C, L, d, E).total;
}

int blockffn_cls_losses(const void* x, int C, int L, int d, const float* Wr, const float* br, int E, float alpha,
                        float w_al, float w_cs, float* loss, float* dS, float* dWr, float* db, float* dx,
                        void* workspace, size_t workspace_bytes, void* stream) {
  const size_t need = blockffn_cls_losses_workspace_size(C, L, d, E);
  if (need == 0) return BFFN_EINVAL;
  if (!(alpha > 0.f) || !std::isfinite(alpha) || !std::isfinite(w_al) || !std::isfinite(w_cs)) return BFFN_EINVAL;
  if (x == nullptr || !aligned16(x) || Wr == nullptr || !aligned4(Wr) || loss == nullptr || !aligned4(loss) ||
      dS == nullptr || !aligned4(dS) || workspace == nullptr || !aligned256(workspace))
    return BFFN_EINVAL;
  if ((br != nullptr && !aligned4(br)) || (dWr != nullptr && !aligned4(dWr)) || (db != nullptr && !aligned4(db)) ||
      (dx != nullptr && !aligned16(dx)))
    return BFFN_EINVAL;
  if (!cls::chunk_fits(L)) return BFFN_EUNSUPPORTED;
  if (workspace_bytes < need) return BFFN_ENOMEM;
  DeviceInfo di;
  int dev = 0;
  const int rc = device_info(&di, &dev);
  if (rc != BFFN_OK) return rc;
  const cudaError_t err = cls::launch(x, C, L, d, Wr, br, E, alpha, w_al, w_cs, loss, dS, dWr, db, dx, workspace,
                                      di.num_sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? BFFN_OK : cuda_fail(err);
}

int blockffn_device_status(void* workspace, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaStreamSynchronize(st);
  if (err != cudaSuccess) return cuda_fail(err);
  void* ws = workspace;
  if (ws == nullptr) {
    int dev = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(err);
    if (dev < 0 || dev >= kMaxDevices) return BFFN_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    ws = g_ws[dev].ptr;
  }
  if (ws == nullptr) return BFFN_OK;
  WsHeader h;
  if ((err = cudaMemcpy(&h, ws, sizeof h, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(err);
  if (h.err == 0) return BFFN_OK;
  const uint32_t zero = 0;
  if ((err = cudaMemcpy(reinterpret_cast<uint8_t*>(ws) + offsetof(WsHeader, err), &zero, sizeof zero,
                        cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(err);
  // a wait that ran out outranks a bad layer index (both may be recorded)
  return (h.err & ~uint32_t(kErrBadLayer)) != 0 ? BFFN_ETIMEOUT : BFFN_EINVAL;
}

}  // extern "C"
