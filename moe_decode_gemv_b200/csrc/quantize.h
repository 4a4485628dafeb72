// quantize.h -- internal interface of the load-time quantisers (quantize_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

cudaError_t launch_mxfp4_quantize(const uint16_t* w, int64_t nblocks, uint8_t* data, uint8_t* scales,
                                  cudaStream_t st);
cudaError_t launch_fp8_rowquant(const uint16_t* w, int64_t V, int H, uint8_t* q, float* s, cudaStream_t st);

}  // namespace moe
