// blockffn_chunk_forward_noalloc: the chunk-layer forward for callers that cannot allocate device
// memory.  Its scratch is a fixed-size array compiled into this library instead of a cudaMalloc'd
// workspace; everything else is the regular decode path (blockffn_chunk_forward_ex with
// BFFN_PATH_DECODE).  blockffn_noalloc_device_status reads and clears that array's error word.
#include <mutex>

#include "blockffn.h"
#include "blockffn_internal.cuh"

namespace bffn {
namespace {

// Upper bound on the scratch one call may use (BFFN_NOALLOC_SCRATCH_BYTES, 8 MiB).  Every GPU that
// loads this library keeps this much device memory reserved until the process exits.
constexpr size_t kNoAllocScratchBytes = BFFN_NOALLOC_SCRATCH_BYTES;

// Zero-initialised when the module is loaded, as a fresh workspace must be.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory: the device address
// must come from cudaGetSymbolAddress, once per device, with that device current.  The address is kept
// for the life of the process; a device reset (which unloads this module's device copy) is not
// supported by this entry point.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return BFFN_ECUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return BFFN_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return BFFN_ECUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BFFN_OK;
}

}  // namespace
}  // namespace bffn

extern "C" {

int blockffn_chunk_forward_noalloc(const void* x, int L, int d, const float* Wr, const float* g,
                                   const void* W1, const void* W2, int E, int de, float* y,
                                   int32_t* active_idx, int32_t* n_active, const float* br,
                                   void* stream) {
  const size_t need = blockffn_workspace_size(L, d, E, de);
  if (need == 0) return BFFN_EINVAL;
  if (L > bffn::kDecodeMaxL) return BFFN_EUNSUPPORTED;  // the decode path only
  if (need > bffn::kNoAllocScratchBytes) return BFFN_ENOMEM;  // beyond the compiled-in maximum
  void* scratch = nullptr;
  const int rc = bffn::scratch_address(&scratch);
  if (rc != BFFN_OK) return rc;
  return blockffn_chunk_forward_ex(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, nullptr,
                                   nullptr, nullptr, BFFN_PATH_DECODE, scratch, bffn::kNoAllocScratchBytes,
                                   stream);
}

int blockffn_noalloc_device_status(void* stream) {
  void* scratch = nullptr;
  const int rc = bffn::scratch_address(&scratch);
  if (rc != BFFN_OK) return rc;
  // the array starts with the same header as every workspace: its error word is read and cleared
  return blockffn_device_status(scratch, stream);
}

}  // extern "C"
