// device_cache.h -- launch set-up that depends only on the device, done once
// per device instead of on every call: the SM count, and each kernel's opt-in
// to more than 48 KB of dynamic shared memory.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace moe {

constexpr int kMaxDevices = 64;
constexpr int kMaxDynamicSmem = 232448;  // 227 KB: the most one CTA may use on sm_100a

// The current device's ordinal and SM count (looked up once per device).
cudaError_t current_device_sms(int* dev, int* sms);

// Opt `Kernel` in to kMaxDynamicSmem bytes of dynamic shared memory on the
// current device; the CUDA call runs once per (kernel, device).  The kernel is
// a template argument so that every kernel -- not every kernel signature --
// gets its own flags.
template <auto Kernel>
cudaError_t ensure_smem_optin() {
  static std::once_flag once[kMaxDevices];
  static cudaError_t result[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    result[dev] = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynamicSmem);
  });
  return result[dev];
}

}  // namespace moe
