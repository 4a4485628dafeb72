// stack.h -- internal interface of the between-layer kernels (stack_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

cudaError_t launch_rmsnorm_bf16(const float* y, int M, int H, float eps, uint16_t* out, cudaStream_t st);
cudaError_t launch_embed_gather(const uint16_t* table, int64_t V, int H, const int32_t* ids, int ids_stride, int M,
                                uint16_t* out, cudaStream_t st);
cudaError_t launch_stream_read(const void* src, size_t bytes, uint32_t* sink, int sms, cudaStream_t st);

}  // namespace moe
