// Library-owned step scratch for rc_step_noalloc.
//
// rc_step stages each call's rotated queries, log-sum-exps and token-score
// work buffers in the caller's memory block. rc_step_noalloc stages them here
// instead: a fixed-size array in the library's own device image, which the
// CUDA driver places on every GPU the library is loaded on and keeps until the
// process exits. No call allocates device memory.
//
// Host code must not use g_step_scratch's name as an address (it is the host
// shadow of the symbol, not device memory); it asks for the device address
// once per device with cudaGetSymbolAddress, with that device current.
#include <mutex>

#include "kernels.cuh"

namespace rc {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) uint8_t g_step_scratch[kStaticScratchBytes];

cudaError_t static_step_scratch(void** ptr, size_t* bytes) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_step_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  *bytes = kStaticScratchBytes;
  return cudaSuccess;
}

}  // namespace rc
