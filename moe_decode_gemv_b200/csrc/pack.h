// pack.h -- the sliced expert-bank layout shared by pack_kernels.cu (which
// writes it) and moe_layer.cu (which reads it).
//
// moe_decode splits every expert it runs into work items of kSliceRows rows
// of the intermediate dimension: item (e, j) computes gate and up rows
// 16j .. 16j+15 of expert e, h = silu(gate x) * (up x) for those rows, and
// applies down columns 16j .. 16j+15 to h.  Each item's weight bytes are one
// contiguous unit, already in the order its matrix instructions read them.
// The gate/up rows go to the tensor core as a 128-row operand: the item's 32
// rows (gate 16j .. 16j+15, then up 16j .. 16j+15) times four K segments of
// Ks = 64 T elements each, T = ceil(H / 256); row r = 32 s + R of the operand
// is row R over elements s Ks .. s Ks + Ks - 1.
//
//   A  gate/up data as the A operand of a block-scaled tensor-core MMA, in
//      the canonical K-major layout without swizzle: T K tiles of 4096 bytes,
//      each two halves of 2048 bytes; in half c of tile t, operand row r is
//      the 16 bytes at 16 r (8-row core matrices 128 bytes apart), holding
//      elements s Ks + 64t + 32c .. +31 of its gate/up row as packed E2M1
//      (element 2i in the low nibble of byte i).  Elements past H are zero.
//   B  gate/up scales, T x 256 bytes: for K tile t, row R, segment s and
//      half c, byte 256t + 8R + 2s + c = the E8M0 scale of block 2T s + 2t + c
//      of row R (0 past H).
//   C  down data, (H/32) groups x 256 bytes: for 32-row group G and lane
//      l = 4g + t, 8 bytes = 2 bytes (columns 16j + 4t .. 16j + 4t + 3) of each
//      of down rows 32G + g, 32G + 8 + g, 32G + 16 + g, 32G + 24 + g, with
//      the two E2M1 codes of each byte re-placed bit by bit (element 2j's
//      sign|e1 e0 m at bits 7|3 2 1, element 2j+1's at 0|6 5 4) so that a
//      mask gives the even elements of a word as E5M2 codes and two shifts
//      the odd ones.
//
// The down scales are per 32 columns, so two items share them: they sit in a
// second array, [E][I/32][H] bytes, where pair p's byte 32G + 4g + r is the
// scale of down row 32G + 8r + g, block p.  The layout moves bytes and bits
// only; no value changes.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kSliceRows = 16;  // intermediate rows per work item

// K tiles of 64 elements per K segment (four segments cover H).
__host__ __device__ constexpr int slice_ktiles(int H) { return (H + 255) / 256; }
// Bytes of one item's parts A, B, C and of the whole unit (25 H when H is a
// multiple of 256).
__host__ __device__ constexpr int slice_a_bytes(int H) { return slice_ktiles(H) * 4096; }
__host__ __device__ constexpr int slice_b_bytes(int H) { return slice_ktiles(H) * 256; }
__host__ __device__ constexpr int slice_c_bytes(int H) { return (H / 32) * 256; }
__host__ __device__ constexpr int slice_unit_bytes(int H) { return slice_a_bytes(H) + slice_b_bytes(H) + slice_c_bytes(H); }

size_t packed_units_bytes(int64_t E, int H, int I);
size_t packed_dscales_bytes(int64_t E, int H, int I);
cudaError_t launch_pack_experts(const uint8_t* gate_d, const uint8_t* gate_s, const uint8_t* up_d,
                                const uint8_t* up_s, const uint8_t* down_d, const uint8_t* down_s, int64_t E, int H,
                                int I, uint8_t* units, uint8_t* dscales, cudaStream_t st);

}  // namespace moe
