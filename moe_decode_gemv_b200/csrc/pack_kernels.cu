// pack_kernels.cu -- load-time re-layout of MXFP4 expert banks for moe_decode.
//
// moe_decode streams one unit of work at a time into shared memory: 8 gate +
// 8 up rows of one expert (a phase-1 item) or 32 rows of one expert's down
// matrix (a phase-2 item).  In the canonical layout such a unit is 18 or 33
// separate pieces (rows and scale rows), and a bulk copy costs a fixed time
// per copy, so a 384-byte down row streams at a fraction of the HBM rate.
// Packing makes every unit one contiguous, 16-byte-aligned run of bytes --
// one bulk copy -- already in the order the kernel reads it:
//   gate/up chunk q of expert e (bytes 16 * (H/2 + H/32)):
//     16 data rows of H/2 bytes: gate rows 8q..8q+7, then up rows 8q..8q+7;
//     then the 8 gate scale rows, then the 8 up scale rows (H/32 bytes each).
//   down tile t of expert e (bytes 32 * (I/2 + I/32)):
//     32 data rows of I/2 bytes (rows 32t..32t+31), then their 32 scale rows.
// Within a data row the 16-byte units (one 32-element MX block each) are
// permuted: unit c of row r is stored at position c ^ (r & mask), mask =
// min(8, largest power of two dividing the units per row) - 1.  The kernel's
// eight rows g = 0..7 that one instruction reads then fall on distinct
// shared-memory banks.  Within each data byte the two E2M1 codes are
// re-placed bit by bit (nibble_relayout): element 2j's sign|e1 e0 m go to
// bits 7|3 2 1 and element 2j+1's to bits 0|6 5 4.  Then a mask alone turns
// the four even elements of a word into E5M2 codes, and a shift pair the odd
// ones (see moe_fused.cu).  Packing moves bits only; no value changes.
#include <cuda_runtime.h>

#include "common.cuh"
#include "pack.h"

namespace moe {
namespace {

// Four data bytes: E2M1 pair (low nibble = element 2j, high = 2j+1) -> the
// packed bit placement described above.
__device__ __forceinline__ uint32_t nibble_relayout(uint32_t w) {
  return ((w & 0x08080808u) << 4) | ((w & 0x07070707u) << 1) | ((w & 0x80808080u) >> 7) | (w & 0x70707070u);
}
__device__ __forceinline__ uint4 nibble_relayout(uint4 v) {
  return make_uint4(nibble_relayout(v.x), nibble_relayout(v.y), nibble_relayout(v.z), nibble_relayout(v.w));
}

// One thread per 16-byte unit of the output.
__global__ void pack_gateup_kernel(const uint8_t* __restrict__ gate_d, const uint8_t* __restrict__ gate_s,
                                   const uint8_t* __restrict__ up_d, const uint8_t* __restrict__ up_s, int64_t E,
                                   int H, int I, uint8_t* __restrict__ out) {
  const int nb = H / 32;                      // 16-byte units per data row = MX blocks per row
  const int mask = swizzle_mask(nb);
  const int units = 16 * nb + nb;             // data units, then scale units (16 * nb bytes)
  const int n_chunks = I / 8;
  const int64_t total = E * n_chunks * units;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t chunk = u / units;          // e * n_chunks + q
    const int j = (int)(u - chunk * units);
    const int64_t e = chunk / n_chunks;
    const int q = (int)(chunk - e * n_chunks);
    uint4 v;
    if (j < 16 * nb) {
      const int r = j / nb, p = j - r * nb;
      const int c = p ^ (r & mask);           // stored at p, read from unit c of the source row
      const uint8_t* src = (r < 8 ? gate_d : up_d) + ((e * I + q * 8 + (r & 7)) * (int64_t)(H / 2)) + c * 16;
      v = nibble_relayout(*reinterpret_cast<const uint4*>(src));
    } else {
      const int b = (j - 16 * nb) * 16;       // byte offset in the 16 scale rows (8 gate, then 8 up)
      const uint8_t* src = (b < 8 * nb ? gate_s + b : up_s + (b - 8 * nb)) + (e * I + q * 8) * (int64_t)nb;
      v = *reinterpret_cast<const uint4*>(src);
    }
    *reinterpret_cast<uint4*>(out + u * 16) = v;
  }
}

__global__ void pack_down_kernel(const uint8_t* __restrict__ down_d, const uint8_t* __restrict__ down_s, int64_t E,
                                 int H, int I, uint8_t* __restrict__ out) {
  const int nb = I / 32;
  const int mask = swizzle_mask(nb);
  const int units = 32 * nb + 2 * nb;         // data units, then scale units (32 * nb bytes)
  const int n_tiles = H / 32;
  const int64_t total = E * n_tiles * units;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = u / units;           // e * n_tiles + t
    const int j = (int)(u - tile * units);
    const int64_t e = tile / n_tiles;
    const int t = (int)(tile - e * n_tiles);
    uint4 v;
    if (j < 32 * nb) {
      const int r = j / nb, p = j - r * nb;
      const int c = p ^ (r & mask);
      v = nibble_relayout(*reinterpret_cast<const uint4*>(down_d + ((e * H + t * 32 + r) * (int64_t)(I / 2)) + c * 16));
    } else {
      const int b = (j - 32 * nb) * 16;
      v = *reinterpret_cast<const uint4*>(down_s + (e * H + t * 32) * (int64_t)nb + b);
    }
    *reinterpret_cast<uint4*>(out + u * 16) = v;
  }
}

}  // namespace

size_t packed_gateup_bytes(int64_t E, int H, int I) { return (size_t)E * (I / 8) * gateup_chunk_bytes(H); }
size_t packed_down_bytes(int64_t E, int H, int I) { return (size_t)E * (H / 32) * down_tile_bytes(I); }

cudaError_t launch_pack_experts(const uint8_t* gate_d, const uint8_t* gate_s, const uint8_t* up_d,
                                const uint8_t* up_s, const uint8_t* down_d, const uint8_t* down_s, int64_t E, int H,
                                int I, uint8_t* gateup, uint8_t* down, cudaStream_t st) {
  pack_gateup_kernel<<<4 * 148, 256, 0, st>>>(gate_d, gate_s, up_d, up_s, E, H, I, gateup);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pack_down_kernel<<<4 * 148, 256, 0, st>>>(down_d, down_s, E, H, I, down);
  return cudaGetLastError();
}

}  // namespace moe
