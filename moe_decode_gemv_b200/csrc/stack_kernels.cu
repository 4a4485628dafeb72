// stack_kernels.cu -- the two small steps between the weight streams of a
// decode step through a stack of MoE layers:
//  * RMSNorm of a layer's fp32 output into the next layer's bf16 input
//    (gain 1): out = bf16_RNE(y / sqrt(mean(y^2) + eps));
//  * the embedding row of each position's greedy token for the next step.
// Both move kilobytes; they exist so that a whole step (embedding, layers,
// norms, LM head) can run on the device and be captured in one CUDA graph.
#include <cuda_runtime.h>

#include "common.cuh"
#include "device_cache.h"
#include "stack.h"

namespace moe {
namespace {

// One CTA per row.
__global__ void rmsnorm_bf16_kernel(const float* __restrict__ y, int H, float eps, uint16_t* __restrict__ out) {
  pdl_wait();  // y comes from the previous kernel
  pdl_launch_dependents();
  const float* row = y + (size_t)blockIdx.x * H;
  float ss = 0.f;
  for (int j = threadIdx.x; j < H; j += blockDim.x) ss = fmaf(row[j], row[j], ss);
  ss = warp_sum(ss);
  __shared__ float part[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = ss;
  __syncthreads();
  if (warp == 0) {
    float v = lane < (int)(blockDim.x >> 5) ? part[lane] : 0.f;
    v = warp_sum(v);
    if (lane == 0) part[0] = sqrtf(__fdiv_rn(v, (float)H) + eps);
  }
  __syncthreads();
  const float rms = part[0];
  for (int j = threadIdx.x; j < H; j += blockDim.x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(__fdiv_rn(row[j], rms));
    out[(size_t)blockIdx.x * H + j] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

// One CTA per position; 16-byte copies.  An id outside [0, V) yields a zero
// row (no out-of-bounds read).
__global__ void embed_gather_kernel(const uint16_t* __restrict__ table, int64_t V, int H,
                                    const int32_t* __restrict__ ids, int ids_stride, uint16_t* __restrict__ out) {
  pdl_wait();  // ids come from the previous kernel
  pdl_launch_dependents();
  const int32_t id = ids[(size_t)blockIdx.x * ids_stride];
  const bool ok = id >= 0 && id < V;
  const uint4* src = reinterpret_cast<const uint4*>(table + (size_t)(ok ? id : 0) * H);
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)blockIdx.x * H);
  for (int j = threadIdx.x; j < H / 8; j += blockDim.x) dst[j] = ok ? src[j] : make_uint4(0, 0, 0, 0);
}

// Measurement aid: every thread streams 16-byte words with non-allocating
// loads (grid-stride) and folds them into one XOR, one atomic per warp.
__global__ void stream_read_kernel(const uint4* __restrict__ src, size_t n, uint32_t* __restrict__ sink) {
  uint32_t acc = 0;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {  // four independent loads in flight per thread
    const uint4 a = ld_stream_u4(src + i), b = ld_stream_u4(src + i + stride);
    const uint4 c = ld_stream_u4(src + i + 2 * stride), d = ld_stream_u4(src + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n; i += stride) {
    const uint4 v = ld_stream_u4(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace

cudaError_t launch_stream_read(const void* src, size_t bytes, uint32_t* sink, int sms, cudaStream_t st) {
  stream_read_kernel<<<4 * sms, 256, 0, st>>>(static_cast<const uint4*>(src), bytes / 16, sink);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bf16(const float* y, int M, int H, float eps, uint16_t* out, cudaStream_t st) {
  return launch_dependent(rmsnorm_bf16_kernel, dim3(M), dim3(256), 0, st, false, y, H, eps, out);
}

cudaError_t launch_embed_gather(const uint16_t* table, int64_t V, int H, const int32_t* ids, int ids_stride, int M,
                                uint16_t* out, cudaStream_t st) {
  return launch_dependent(embed_gather_kernel, dim3(M), dim3(128), 0, st, false, table, V, H, ids, ids_stride, out);
}

}  // namespace moe
