// pack.h -- the packed expert-bank layout shared by pack_kernels.cu (which
// writes it) and moe_fused.cu (which reads it).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Units of 16 bytes per data row -> the XOR mask applied to a unit's index
// within its row (row r stores unit c at position c ^ (r & mask)).
__host__ __device__ constexpr int swizzle_mask(int units_per_row) {
  return ((units_per_row & -units_per_row) < 8 ? (units_per_row & -units_per_row) : 8) - 1;
}
// One phase-1 item: 8 gate + 8 up rows of H/2 bytes, then their 16 scale rows of H/32 bytes.
__host__ __device__ constexpr int gateup_chunk_bytes(int H) { return 16 * (H / 2 + H / 32); }
// One phase-2 item: 32 down rows of I/2 bytes, then their 32 scale rows of I/32 bytes.
__host__ __device__ constexpr int down_tile_bytes(int I) { return 32 * (I / 2 + I / 32); }

size_t packed_gateup_bytes(int64_t E, int H, int I);
size_t packed_down_bytes(int64_t E, int H, int I);
cudaError_t launch_pack_experts(const uint8_t* gate_d, const uint8_t* gate_s, const uint8_t* up_d,
                                const uint8_t* up_s, const uint8_t* down_d, const uint8_t* down_s, int64_t E, int H,
                                int I, uint8_t* gateup, uint8_t* down, cudaStream_t st);

}  // namespace moe
