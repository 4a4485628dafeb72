// pack.h -- the sliced expert-bank layout shared by pack_kernels.cu (which
// writes it) and moe_layer.cu (which reads it).
//
// moe_decode splits every expert it runs into work items of kSliceRows rows
// of the intermediate dimension: item (e, j) computes gate and up rows
// 16j .. 16j+15 of expert e, h = silu(gate x) * (up x) for those rows, and
// applies down columns 16j .. 16j+15 to h.  Each item's weight bytes are one
// contiguous unit, already in the order of the kernel's MMA fragments:
//
//   A  gate/up data, (H/32) blocks x 512 bytes: for K block b and lane
//      l = 4g + t (g = l >> 2, t = l & 3), 16 bytes = the 4-byte words t of
//      block b of gate row 16j+g, up row 16j+g, gate row 16j+8+g and up row
//      16j+8+g (a word holds elements 32b + 8t .. 32b + 8t + 7);
//   B  gate/up scales, (H/32) x 32 bytes: for block b and g, 4 bytes = the
//      E8M0 scales of block b of those four rows, in the same order;
//   C  down data, (H/32) groups x 256 bytes: for 32-row group G and lane
//      l = 4g + t, 8 bytes = 2 bytes (columns 16j + 4t .. 16j + 4t + 3) of each
//      of down rows 32G + g, 32G + 8 + g, 32G + 16 + g, 32G + 24 + g.
//
// The down scales are per 32 columns, so two items share them: they sit in a
// second array, [E][I/32][H] bytes, where pair p's byte 32G + 4g + r is the
// scale of down row 32G + 8r + g, block p.  Within every data byte
// the two E2M1 codes are re-placed bit by bit (element 2j's sign|e1 e0 m at
// bits 7|3 2 1, element 2j+1's at 0|6 5 4) so that a mask gives the even
// elements of a word as E5M2 codes and two shifts the odd ones.  The layout
// moves bytes and bits only; no value changes.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kSliceRows = 16;  // intermediate rows per work item

// Bytes of one item's unit (parts A, B, C): 25 H.
__host__ __device__ constexpr int slice_unit_bytes(int H) { return (H / 32) * (512 + 32 + 256); }
__host__ __device__ constexpr int slice_a_bytes(int H) { return (H / 32) * 512; }
__host__ __device__ constexpr int slice_b_bytes(int H) { return (H / 32) * 32; }

size_t packed_units_bytes(int64_t E, int H, int I);
size_t packed_dscales_bytes(int64_t E, int H, int I);
cudaError_t launch_pack_experts(const uint8_t* gate_d, const uint8_t* gate_s, const uint8_t* up_d,
                                const uint8_t* up_s, const uint8_t* down_d, const uint8_t* down_s, int64_t E, int H,
                                int I, uint8_t* units, uint8_t* dscales, cudaStream_t st);

}  // namespace moe
