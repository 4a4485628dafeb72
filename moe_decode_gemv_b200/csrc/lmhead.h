// lmhead.h -- internal interface of the LM-head kernels: the FP8 head
// (lmhead_fp8.cu) and the BF16 comparator head (lmhead_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

int lmhead_max_slices();
// Ring depth and shared memory of one launch (elem_bytes 1: the FP8 head, 2:
// the BF16 head); false if the shape does not fit in one CTA's shared memory
// (the CTA keeps its rows' logits there).
bool lmhead_plan(int H, int elem_bytes, int M, int top_k, int64_t V, int grid, int* stages, size_t* smem);
bool lmhead_fp8_plan(int H, int M, int top_k, int64_t V, int grid, int* stages, size_t* smem);
size_t lmhead_cand_bytes(int grid, int M, int top_k);
// CTAs of one head launch: one per SM, at most one per 16-row tile and at
// most kLmheadMaxGrid (every entry point launches this many).
constexpr int kLmheadMaxGrid = 1024;
inline int lmhead_grid(int sms, int64_t V) {
  const int64_t ntiles = (V + 15) / 16;
  int64_t g = sms < kLmheadMaxGrid ? sms : kLmheadMaxGrid;
  if (g > ntiles) g = ntiles;
  return (int)g;
}
// Bytes of the fragment-tiled FP8 head (whole 16-row tiles, zero rows past V).
size_t lmhead_tiled_bytes(int64_t V, int H);
cudaError_t launch_tile_fp8_head(const uint8_t* q, int64_t V, int H, uint8_t* out, cudaStream_t st);

// FP8 head over the tiled layout (qt: lmhead_tiled_bytes bytes).
cudaError_t launch_lmhead_fp8(const uint16_t* x, const uint8_t* qt, const float* s, int64_t V, int H, int M,
                              int top_k, float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand,
                              int grid, cudaStream_t st);
cudaError_t launch_lmhead_bf16(const uint16_t* x, const uint16_t* w, int64_t V, int H, int M, int top_k,
                               float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                               cudaStream_t st);

}  // namespace moe
