// pack_kernels.cu -- load-time re-layout of MXFP4 expert banks for moe_decode
// into the sliced layout of pack.h: one contiguous unit per work item, with
// the bytes in the order the kernel's MMAs read them (the tensor core's
// K-major gate/up operand and its scales, then the down fragments), plus the
// down scales per 32-column pair.  Load time only; the kernels gather bytes one
// at a time and favour plainness over speed.
#include <cuda_runtime.h>

#include "common.cuh"
#include "pack.h"

namespace moe {
namespace {

// One byte of two E2M1 codes (low nibble = element 2j, high = 2j+1) -> the
// packed bit placement of pack.h.
__device__ __forceinline__ uint32_t nibble_relayout(uint32_t b) {
  return ((b & 0x08u) << 4) | ((b & 0x07u) << 1) | ((b & 0x80u) >> 7) | (b & 0x70u);
}

// One thread per output byte of the units array.
__global__ void pack_units_kernel(const uint8_t* __restrict__ gate_d, const uint8_t* __restrict__ gate_s,
                                  const uint8_t* __restrict__ up_d, const uint8_t* __restrict__ up_s,
                                  const uint8_t* __restrict__ down_d, int64_t E, int H, int I,
                                  uint8_t* __restrict__ out) {
  const int nb = H / 32, n_sl = I / kSliceRows;
  const int ua = slice_a_bytes(H), ub = slice_b_bytes(H), unit = slice_unit_bytes(H), T = slice_ktiles(H);
  const int64_t total = E * n_sl * (int64_t)unit;
  const int64_t hb = H / 2, ib = I / 2;  // data bytes per gate/up row and per down row
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total; o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t item = o / unit;  // e * n_sl + j
    const int k = (int)(o - item * unit);
    const int64_t e = item / n_sl;
    const int j = (int)(item - e * n_sl);
    uint32_t v;
    if (k < ua) {
      // tile t, half c, operand row r = 32 s + R, byte bi of its 16
      const int t = k / 4096, c = (k % 4096) / 2048, r = (k % 2048) / 16, bi = k % 16;
      const int s = r / 32, R = r % 32;  // R: 0..15 gate rows, 16..31 up rows
      const int row = 16 * j + (R & 15);
      const int k0 = s * 64 * T + 64 * t + 32 * c + 2 * bi;  // the byte's first element
      const uint8_t* src = R < 16 ? gate_d : up_d;
      v = k0 < H ? src[(e * I + row) * hb + k0 / 2] : 0u;
    } else if (k < ua + ub) {
      const int kk = k - ua;
      const int t = kk / 256, R = (kk % 256) / 8, s = (kk % 8) / 2, c = kk % 2;
      const int b = 2 * T * s + 2 * t + c;
      const int row = 16 * j + (R & 15);
      const uint8_t* src = R < 16 ? gate_s : up_s;
      v = b < nb ? src[(e * I + row) * nb + b] : 0u;
    } else {
      // group G, lane l, row r of the four (32G + 8r + g), byte bw of its two
      const int kk = k - ua - ub;
      const int G = kk / 256, l = (kk % 256) / 8, r = (kk % 8) / 2, bw = kk % 2;
      const int g = l >> 2, t = l & 3;
      const int row = 32 * G + 8 * r + g;
      v = nibble_relayout(down_d[(e * H + row) * ib + 8 * j + 2 * t + bw]);
    }
    out[o] = (uint8_t)v;
  }
}

// One thread per output byte of the down-scale array [E][I/32][H].
__global__ void pack_dscales_kernel(const uint8_t* __restrict__ down_s, int64_t E, int H, int I,
                                    uint8_t* __restrict__ out) {
  const int np = I / 32;
  const int64_t total = E * np * (int64_t)H;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total; o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t ep = o / H;  // e * np + p
    const int k = (int)(o - ep * H);
    const int64_t e = ep / np;
    const int p = (int)(ep - e * np);
    const int G = k / 32, g = (k % 32) / 4, r = k % 4;
    const int row = 32 * G + 8 * r + g;
    out[o] = down_s[(e * H + row) * np + p];
  }
}

}  // namespace

size_t packed_units_bytes(int64_t E, int H, int I) { return (size_t)E * (I / kSliceRows) * slice_unit_bytes(H); }
size_t packed_dscales_bytes(int64_t E, int H, int I) { return (size_t)E * (I / 32) * H; }

cudaError_t launch_pack_experts(const uint8_t* gate_d, const uint8_t* gate_s, const uint8_t* up_d,
                                const uint8_t* up_s, const uint8_t* down_d, const uint8_t* down_s, int64_t E, int H,
                                int I, uint8_t* units, uint8_t* dscales, cudaStream_t st) {
  pack_units_kernel<<<8 * 148, 256, 0, st>>>(gate_d, gate_s, up_d, up_s, down_d, E, H, I, units);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pack_dscales_kernel<<<2 * 148, 256, 0, st>>>(down_s, E, H, I, dscales);
  return cudaGetLastError();
}

}  // namespace moe
