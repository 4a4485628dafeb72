// selftest.cu -- a self-test of the bounded device waits.
//
// Every wait in this library's kernels (on an mbarrier phase, a grid barrier,
// a readiness counter) gives up after a time limit, records MOE_ERR_TIMEOUT
// in the workspace header and lets the kernel return, so that a wait that can
// never complete ends with a status the host reads instead of a hung GPU.
// This entry point runs that same wait on a flag nothing ever sets -- a word
// of the workspace header that no kernel writes -- with a short limit, so a
// test can watch the limit run out and the context stay usable afterwards.
#include <cuda_runtime.h>

#include "../../include/moe_gemv.h"
#include "common.cuh"

namespace moe {
namespace {

__global__ void wait_on_unset_flag_kernel(WsHeader* hdr, uint64_t limit_ns) {
  if (threadIdx.x != 0) return;
  const volatile uint32_t* flag = &hdr->pad[0];  // written by no kernel
  const bool ok = bounded_spin_for([&] { return *flag != 0u; }, limit_ns);
  if (!ok) report(hdr, MOE_ERR_TIMEOUT);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                               void* stream) {
  if (!workspace || workspace_bytes < sizeof(moe::WsHeader)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return MOE_ERR_MISALIGNED;
  if (limit_us < 1 || limit_us > 1000000) return MOE_ERR_INVALID_ARG;
  moe::wait_on_unset_flag_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<moe::WsHeader*>(workspace), (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
