// Host side of the C ABI declared in include/blockffn.h: argument checks, workspace handling and
// the kernel launches of one BlockFFN chunk-layer forward.
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
  return L >= 1 && E >= 1 && E <= kMaxE && d >= 16 && d % 16 == 0 && de >= 16 && de % 16 == 0 &&
         (long long)L * d < (1ll << 31) && (long long)E * de * d < (1ll << 40);
}

int forward_decode(const void* x, int L, int d, const float* Wr, const float* g, const void* W1,
                   const void* W2, int E, int de, float* y, int32_t* active_idx, int32_t* n_active,
                   const float* br, uint32_t* tok_mask, int32_t* counts, float* r_out, void* ws,
                   const DeviceInfo& di, cudaStream_t st) {
  const WsLayout lay = ws_layout(L, d, E, de);
  uint8_t* base = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base);

  RouterParams rp;
  rp.x = static_cast<const __nv_bfloat16*>(x);
  rp.Wr = Wr;
  rp.br = br;
  rp.g = g;
  rp.L = L;
  rp.d = d;
  rp.E = E;
  rp.s_ws = reinterpret_cast<float*>(base + lay.s_off);
  rp.r_ws = reinterpret_cast<float*>(base + lay.r_off);
  rp.r_out = r_out;
  rp.tok_mask = tok_mask;
  rp.counts = counts;
  rp.active_idx = active_idx;
  rp.n_active = n_active;
  rp.hdr = hdr;
  RouterLaunch rl;
  if (!router_decode_plan(L, d, E, di.max_smem, &rl, &rp.Rq)) return BFFN_EUNSUPPORTED;
  rp.wreg_floats = rl.wreg_floats;

  DecodeParams dp;
  dp.x = rp.x;
  dp.W1 = static_cast<const __nv_bfloat16*>(W1);
  dp.W2 = static_cast<const __nv_bfloat16*>(W2);
  dp.y = y;
  dp.active_idx = active_idx;
  dp.n_active = n_active;
  dp.r = rp.r_ws;
  dp.h = reinterpret_cast<__nv_bfloat16*>(base + lay.h_off);
  dp.hdr = hdr;
  dp.L = L;
  dp.d = d;
  dp.E = E;
  dp.de = de;
  DecodeLaunch dl;
  if (!expert_decode_plan(L, d, de, di.num_sms, di.max_smem, &dp, &dl)) return BFFN_EUNSUPPORTED;

  cudaError_t err = router_decode_launch(rp, rl, st, di.pdl);
  if (err != cudaSuccess) return cuda_fail(err);
  err = expert_decode_launch(dp, dl, st, di.pdl);
  if (err != cudaSuccess) return cuda_fail(err);
  return BFFN_OK;
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
  const bool decode = (path == BFFN_PATH_DECODE) || (path == BFFN_PATH_AUTO && L <= kDecodeMaxL);
  if (!decode) return BFFN_EUNSUPPORTED;
  if (L > kDecodeMaxL) return BFFN_EUNSUPPORTED;

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
  return forward_decode(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, tok_mask, counts,
                        r_out, ws, di, st);
}

int blockffn_chunk_forward(const void* x, int L, int d, const float* Wr, const float* g,
                           const void* W1, const void* W2, int E, int de, float* y,
                           int32_t* active_idx, int32_t* n_active, void* stream) {
  return blockffn_chunk_forward_ex(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, nullptr,
                                   nullptr, nullptr, nullptr, BFFN_PATH_AUTO, nullptr, 0, stream);
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
  return BFFN_ETIMEOUT;
}

}  // extern "C"
