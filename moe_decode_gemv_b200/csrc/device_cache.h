// device_cache.h -- launch set-up: what depends only on the device, done once
// per device instead of on every call (the SM count, each kernel's opt-in to
// more than 48 KB of dynamic shared memory), and the dependent launch that
// chains the kernels of a decode step.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <utility>

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

// Launch `kernel` with programmatic stream serialization: its CTAs may be
// scheduled while the previous kernel on the stream finishes (that kernel
// triggers it with griddepcontrol.launch_dependents), which hides the launch
// latency between back-to-back kernels of a decode step.  The kernel itself
// runs griddepcontrol.wait before it touches anything the previous kernel
// writes.  `coop` adds the cooperative attribute; if the driver refuses the
// pair, the launch is made again without serialization (same kernel, same
// work).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             bool coop, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (coop) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n++].val.cooperative = 1;
  }
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n++].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = n - 1;  // without serialization
    e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) (void)cudaGetLastError();  // leave no stale error for the next call to find
  }
  return e;
}

}  // namespace moe
