// device_cache.cu -- per-device SM counts, looked up once.
#include <atomic>

#include "device_cache.h"

namespace moe {

namespace {
std::atomic<int> g_sms[kMaxDevices];  // 0 until looked up
}

cudaError_t current_device_sms(int* dev, int* sms) {
  int d = 0;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) return e;
  if (d < 0 || d >= kMaxDevices) return cudaErrorInvalidDevice;
  int n = g_sms[d].load(std::memory_order_relaxed);
  if (n == 0) {
    if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d)) != cudaSuccess) return e;
    if (n <= 0) return cudaErrorInvalidDevice;
    g_sms[d].store(n, std::memory_order_relaxed);
  }
  *dev = d;
  *sms = n;
  return cudaSuccess;
}

}  // namespace moe
