// quantize_kernels.cu -- load-time quantisers (not on the per-token path).
//
//  * MXFP4 (OCP Microscaling Formats v1.0): per 32-element block along K,
//    shared scale X = 2^(floor(log2(amax)) - 2) with the exponent clamped to
//    [-127, 127], elements V/X rounded to the nearest E2M1 value (ties to
//    even) and saturated at +-6.  A block holding Inf/NaN gets scale 0xFF.
//  * FP8 LM head: s_v = fp32(amax_v / 448) (1 for an all-zero row), then
//    q = E4M3 of fp32(w / s_v), rounded to nearest even and saturated at
//    +-448 -- the load-time FP8 conversion of the head that the pages
//    describe (ncijnetwork.com summary, "What are the 3 optimizations?",
//    item 2).  Both divisions are IEEE fp32 (__fdiv_rn).
//
// Rounding uses the sm_100a conversions cvt.rn.satfinite.{e2m1x2,e4m3x2}.f32.
#include <cuda_runtime.h>

#include "common.cuh"
#include "quantize.h"

namespace moe {
namespace {

// floor(log2(a)) for a finite a > 0, exact from the fp32 bits (subnormals included).
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)((b >> 23) & 0xffu);
  return e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
}

// One thread per 32-element block.
__global__ void mxfp4_quantize_kernel(const uint16_t* __restrict__ w, int64_t nblocks,
                                      uint8_t* __restrict__ data, uint8_t* __restrict__ scales) {
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + b * 32);
  uint32_t v[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 q = src[i];
    v[4 * i + 0] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
  }
  float amax = 0.f;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t bits = (v[i] >> (16 * h)) & 0xffffu;
      if ((bits & 0x7f80u) == 0x7f80u) finite = false;  // bf16 exponent all ones: Inf or NaN
      amax = fmaxf(amax, bf16_bits_to_f32(bits & 0x7fffu));
    }
  }
  uint4 out = make_uint4(0, 0, 0, 0);
  uint32_t sc;
  if (!finite) {
    sc = 0xffu;
  } else {
    int xexp = amax == 0.f ? -127 : floor_log2(amax) - 2;
    xexp = xexp < -127 ? -127 : (xexp > 127 ? 127 : xexp);
    sc = (uint32_t)(xexp + 127);
    // 2^-xexp is a normal fp32 (xexp <= 125 for any finite bf16 amax), so the
    // product below is V/X exactly unless it is far below the E2M1 grid.
    const float inv = __uint_as_float((uint32_t)(127 - xexp) << 23);
    uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float lo = bf16_bits_to_f32(v[i] & 0xffffu) * inv;
      const float hi = bf16_bits_to_f32(v[i] >> 16) * inv;
      o[i / 4] |= f32x2_to_e2m1x2(lo, hi) << (8 * (i % 4));
    }
    out = make_uint4(o[0], o[1], o[2], o[3]);
  }
  reinterpret_cast<uint4*>(data)[b] = out;
  scales[b] = (uint8_t)sc;
}

// One warp per row; H a multiple of 8.
__global__ void fp8_rowquant_kernel(const uint16_t* __restrict__ w, int64_t V, int H,
                                    uint8_t* __restrict__ q, float* __restrict__ s) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= V) return;
  const uint16_t* r = w + row * H;
  float amax = 0.f;
  for (int j = lane * 8; j < H; j += 256) {
    const uint4 p = *reinterpret_cast<const uint4*>(r + j);
    const uint32_t u[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, bf16_bits_to_f32(u[i] & 0x7fffu));
      amax = fmaxf(amax, bf16_bits_to_f32((u[i] >> 16) & 0x7fffu));
    }
  }
  amax = warp_max(amax);
  const float sv = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (lane == 0) s[row] = sv;
  for (int j = lane * 8; j < H; j += 256) {
    const uint4 p = *reinterpret_cast<const uint4*>(r + j);
    const uint32_t u[4] = {p.x, p.y, p.z, p.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __fdiv_rn(bf16_bits_to_f32(u[i] & 0xffffu), sv);
      const float hi = __fdiv_rn(bf16_bits_to_f32(u[i] >> 16), sv);
      o[i / 2] |= f32x2_to_e4m3x2(lo, hi) << (16 * (i % 2));
    }
    *reinterpret_cast<uint2*>(q + row * H + j) = make_uint2(o[0], o[1]);
  }
}

}  // namespace

cudaError_t launch_mxfp4_quantize(const uint16_t* w, int64_t nblocks, uint8_t* data, uint8_t* scales,
                                  cudaStream_t st) {
  if (nblocks == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t grid = (nblocks + threads - 1) / threads;
  mxfp4_quantize_kernel<<<(unsigned)grid, threads, 0, st>>>(w, nblocks, data, scales);
  return cudaGetLastError();
}

cudaError_t launch_fp8_rowquant(const uint16_t* w, int64_t V, int H, uint8_t* q, float* s, cudaStream_t st) {
  if (V == 0) return cudaSuccess;
  const int warps = 8;
  const int64_t grid = (V + warps - 1) / warps;
  fp8_rowquant_kernel<<<(unsigned)grid, warps * 32, 0, st>>>(w, V, H, q, s);
  return cudaGetLastError();
}

}  // namespace moe
