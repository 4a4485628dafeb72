// lmhead_noalloc.cu -- lmhead_decode without a caller-provided workspace.
//
// Some callers cannot hand this library a workspace: a host that owns every
// device allocation and passes a plugin only its input and output buffers,
// or a latency-critical loop where a cudaMalloc (which may synchronise the
// device) is not allowed.  This entry point serves them.  Its scratch -- the
// 64-byte header with the last-CTA ticket, then one candidate list per CTA --
// lives in one file-scope device array of fixed size that every GPU loading
// the library holds until the process exits.  Nothing here allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe_gemv.h"
#include "common.cuh"
#include "device_cache.h"
#include "lmhead.h"

namespace {

constexpr size_t kScratchBytes = MOE_LMHEAD_NOALLOC_SCRATCH_BYTES;
constexpr size_t kHeaderBytes = sizeof(moe::WsHeader);

__device__ __align__(256) uint8_t g_lmhead_scratch[kScratchBytes];

// Device address of g_lmhead_scratch per device ordinal, looked up once.  In
// host code the array's name is only a host-side stand-in, never a device
// address, so it must not be passed to a kernel.
std::mutex g_mutex;
void* g_scratch_ptr[moe::kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= moe::kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lmhead_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status lmhead_decode_noalloc(const uint16_t* hidden_bf16, const moe_fp8_head* head, int32_t M,
                                            int32_t top_k, int32_t* topk_ids, float* topk_vals, float* logits,
                                            void* stream) {
  // the same argument checks as lmhead_decode, before any CUDA call
  if (!head) return MOE_ERR_INVALID_ARG;
  if (head->fmt != MOE_FMT_FP8_E4M3_TILED) return MOE_ERR_FORMAT_MISMATCH;
  if (!head->q || !head->row_scale || !hidden_bf16 || !topk_ids || !topk_vals) return MOE_ERR_INVALID_ARG;
  const int64_t V = head->vocab, H = head->hidden;
  if (M < 1 || M > 4 || top_k < 1 || top_k > 64 || top_k > V) return MOE_ERR_INVALID_ARG;
  if (V < 1 || V >= (int64_t(1) << 31) || H < 64 || H % 64 != 0 || (H / 64 + 7) / 8 > moe::lmhead_max_slices())
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(hidden_bf16) || !aligned16(head->q) || !aligned16(head->row_scale) || !aligned16(topk_ids) ||
      !aligned16(topk_vals) || (logits && !aligned16(logits)))
    return MOE_ERR_MISALIGNED;

  // one CTA per SM, as lmhead_decode launches; its candidate lists must fit
  int dev = 0, sms = 0;
  if (moe::current_device_sms(&dev, &sms) != cudaSuccess) return MOE_ERR_CUDA;
  const int grid = moe::lmhead_grid(sms, V);
  if (kHeaderBytes + moe::lmhead_cand_bytes(grid, M, top_k) > kScratchBytes) return MOE_ERR_WORKSPACE;
  int stages = 0;
  size_t smem = 0;
  if (!moe::lmhead_plan((int)H, 1, M, top_k, V, grid, &stages, &smem)) return MOE_ERR_UNSUPPORTED_SHAPE;

  void* scratch = nullptr;
  const moe_status st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the counters must start at zero: clear the header after its status word,
  // which keeps the first error until lmhead_noalloc_status reads it (the
  // lists need no clearing)
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + sizeof(int32_t), 0, kHeaderBytes - sizeof(int32_t), s) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  auto* hdr = static_cast<moe::WsHeader*>(scratch);
  void* cand = static_cast<uint8_t*>(scratch) + kHeaderBytes;
  const cudaError_t e = moe::launch_lmhead_fp8(hidden_bf16, head->q, head->row_scale, V, (int)H, M, top_k, logits,
                                               topk_ids, topk_vals, hdr, cand, grid, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status lmhead_noalloc_status(int32_t* status_out, void* stream) {
  if (!status_out) return MOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const moe_status st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  auto* hdr = static_cast<moe::WsHeader*>(scratch);
  int32_t status = 0;
  if (cudaMemcpy(&status, &hdr->status, sizeof(status), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (status != 0 && cudaMemset(&hdr->status, 0, sizeof(status)) != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = status;
  return MOE_OK;
}
