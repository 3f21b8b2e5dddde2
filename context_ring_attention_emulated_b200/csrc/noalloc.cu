// noalloc.cu -- rattn_ring_bwd_noalloc: the ring backward with its scratch
// space in a fixed device array that is part of the library image, for
// callers that cannot allocate device memory themselves.
//
// The array is a file-scope __device__ object: every GPU that loads the
// library holds it (RATTN_NOALLOC_SCRATCH_BYTES) until the process exits.
// Host code cannot use the array's name as a device address, so its address
// is looked up once per device with cudaGetSymbolAddress, on the first call
// made while that device is current, and cached for the life of the process
// (the cache assumes the device's primary context is never reset).
#include <mutex>

#include "internal.h"

namespace rattn {
namespace {

constexpr size_t kScratchBytes = RATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_bwd_scratch on the current device (set up on first use).
rattn_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return RATTN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RATTN_OK;
}

}  // namespace
}  // namespace rattn

extern "C" rattn_status rattn_ring_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                               const void* dout, const float* lse, const int32_t* pos, int B, int H,
                                               int64_t Lp, int D, rattn_dtype dtype, int cp_size,
                                               rattn_layout layout, int causal, float scale, int64_t L_valid,
                                               void* dq, void* dk, void* dv, void* stream) {
  const size_t need = rattn_ring_bwd_workspace_size(B, H, Lp, D);
  if (need > rattn::kScratchBytes) return RATTN_ERR_UNSUPPORTED;  // larger than the built-in scratch array
  void* scratch = nullptr;
  if (need > 0) {
    const rattn_status st = rattn::scratch_address(&scratch);
    if (st != RATTN_OK) return st;
  }
  // Same validation and kernels as rattn_ring_bwd; the dQ accumulator part
  // of the scratch is zeroed on the device by the backward's first kernel.
  return rattn_ring_bwd(q, k, v, o, dout, lse, pos, B, H, Lp, D, dtype, cp_size, layout, causal, scale, L_valid, dq,
                        dk, dv, scratch, rattn::kScratchBytes, stream);
}
