// abi.cu -- the extern "C" entry points declared in include/moe_gemv.h.
//
// Every entry point validates its arguments (shapes, alignment, format tags,
// workspace size) with plain integer checks before touching any CUDA API, so
// a bad call returns an error code and enqueues nothing.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>

#include "../../include/moe_gemv.h"
#include "common.cuh"
#include "device_cache.h"
#include "lmhead.h"
#include "moe.h"
#include "pack.h"
#include "quantize.h"
#include "stack.h"

namespace {



bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_mxfp4(const moe_mxfp4_tensor& t, int64_t count, int64_t rows, int64_t K) {
  if (t.fmt != MOE_FMT_MXFP4_E2M1_E8M0_32) return MOE_ERR_FORMAT_MISMATCH;
  if (!t.data || !t.scales) return MOE_ERR_INVALID_ARG;
  if (t.count != count || t.rows != rows || t.K != K) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(t.data) || !aligned16(t.scales)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status check_bank(const moe_expert_bank* b, int64_t count, int64_t H, int64_t I) {
  moe_status s;
  if ((s = check_mxfp4(b->gate, count, I, H)) != MOE_OK) return s;
  if ((s = check_mxfp4(b->up, count, I, H)) != MOE_OK) return s;
  return check_mxfp4(b->down, count, H, I);
}

bool pack_shape_ok(int64_t count, int64_t H, int64_t I) {
  return count >= 1 && count <= (int64_t(1) << 20) && H >= 32 && I >= 32 && H % 32 == 0 && I % 32 == 0 &&
         H <= 65536 && I <= 65536;
}

moe_status check_packed(const moe_packed_bank* b, int64_t count, int64_t H, int64_t I) {
  if (b->fmt != MOE_FMT_MXFP4_MOE_PACKED) return MOE_ERR_FORMAT_MISMATCH;
  if (!b->units || !b->dscales) return MOE_ERR_INVALID_ARG;
  if (b->count != count || b->hidden != H || b->inter != I) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(b->units) || !aligned16(b->dscales)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

bool head_shape_ok(int64_t vocab, int64_t hidden, int elem_bytes) {
  if (vocab < 1 || vocab >= (int64_t(1) << 31)) return false;
  if (hidden < 64 || (hidden * elem_bytes) % 64 != 0) return false;
  const int64_t slices = hidden * elem_bytes / 64;
  return (slices + 7) / 8 <= moe::lmhead_max_slices();
}

size_t head_ws_bytes(int32_t M, int32_t top_k) {
  return sizeof(moe::WsHeader) + moe::lmhead_cand_bytes(moe::kLmheadMaxGrid, M, top_k);
}

moe_status launch_head_common(const uint16_t* hidden, const void* w, const float* scale, bool fp8, int64_t V,
                              int64_t H, int32_t M, int32_t top_k, int32_t* ids, float* vals, float* logits,
                              void* ws, size_t ws_bytes, void* stream) {
  if (!hidden || !ids || !vals || !ws) return MOE_ERR_INVALID_ARG;
  if (M < 1 || M > 4 || top_k < 1 || top_k > 64 || top_k > V) return MOE_ERR_INVALID_ARG;
  if (!head_shape_ok(V, H, fp8 ? 1 : 2)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(hidden) || !aligned16(w) || (scale && !aligned16(scale)) || !aligned16(ids) ||
      !aligned16(vals) || (logits && !aligned16(logits)) || !aligned16(ws))
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < head_ws_bytes(M, top_k)) return MOE_ERR_WORKSPACE;

  int dev = 0, sms = 0;
  if (moe::current_device_sms(&dev, &sms) != cudaSuccess) return MOE_ERR_CUDA;
  const int grid = moe::lmhead_grid(sms, V);
  int stages = 0;
  size_t smem = 0;  // each CTA keeps its rows' logits in shared memory: a limit on vocab / SMs
  if (!moe::lmhead_plan((int)H, fp8 ? 1 : 2, M, top_k, V, grid, &stages, &smem)) return MOE_ERR_UNSUPPORTED_SHAPE;
  auto* hdr = static_cast<moe::WsHeader*>(ws);
  void* cand = static_cast<uint8_t*>(ws) + sizeof(moe::WsHeader);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      fp8 ? moe::launch_lmhead_fp8(hidden, static_cast<const uint8_t*>(w), scale, V, (int)H, M, top_k, logits, ids,
                                   vals, hdr, cand, grid, st)
          : moe::launch_lmhead_bf16(hidden, static_cast<const uint16_t*>(w), V, (int)H, M, top_k, logits, ids, vals,
                                    hdr, cand, grid, st);
  return cuda_status(e);
}

}  // namespace

extern "C" {

moe_status moe_quantize_mxfp4(const uint16_t* w_bf16, moe_mxfp4_tensor* out, void* stream) {
  if (!w_bf16 || !out || !out->data || !out->scales) return MOE_ERR_INVALID_ARG;
  if (out->count < 1 || out->rows < 1 || out->K < 32 || out->K % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(out->data) || !aligned16(out->scales)) return MOE_ERR_MISALIGNED;
  const int64_t nblocks = (int64_t)out->count * out->rows * (out->K / 32);
  cudaError_t e = moe::launch_mxfp4_quantize(w_bf16, nblocks, out->data, out->scales,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  out->fmt = MOE_FMT_MXFP4_E2M1_E8M0_32;
  return MOE_OK;
}

moe_status lmhead_quantize_fp8(const uint16_t* w_bf16, moe_fp8_head* out, void* stream) {
  if (!w_bf16 || !out || !out->q || !out->row_scale) return MOE_ERR_INVALID_ARG;
  if (!head_shape_ok(out->vocab, out->hidden, 1)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(out->q) || !aligned16(out->row_scale)) return MOE_ERR_MISALIGNED;
  cudaError_t e = moe::launch_fp8_rowquant(w_bf16, out->vocab, (int)out->hidden, out->q, out->row_scale,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  out->fmt = MOE_FMT_FP8_E4M3_ROWSCALE_F32;
  return MOE_OK;
}

size_t lmhead_tiled_bytes(int64_t vocab, int64_t hidden) {
  return head_shape_ok(vocab, hidden, 1) ? moe::lmhead_tiled_bytes(vocab, (int)hidden) : 0;
}

moe_status lmhead_tile_fp8(const moe_fp8_head* src, moe_fp8_head* dst, void* stream) {
  if (!src || !dst || !src->q || !dst->q || !dst->row_scale) return MOE_ERR_INVALID_ARG;
  if (src->fmt != MOE_FMT_FP8_E4M3_ROWSCALE_F32) return MOE_ERR_FORMAT_MISMATCH;
  if (dst->vocab != src->vocab || dst->hidden != src->hidden) return MOE_ERR_INVALID_ARG;
  if (!head_shape_ok(src->vocab, src->hidden, 1)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(src->q) || !aligned16(dst->q) || !aligned16(dst->row_scale)) return MOE_ERR_MISALIGNED;
  const cudaError_t e = moe::launch_tile_fp8_head(src->q, src->vocab, (int)src->hidden, dst->q,
                                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  dst->fmt = MOE_FMT_FP8_E4M3_TILED;
  return MOE_OK;
}

size_t moe_packed_units_bytes(int32_t count, int32_t hidden, int32_t inter) {
  return pack_shape_ok(count, hidden, inter) ? moe::packed_units_bytes(count, hidden, inter) : 0;
}

size_t moe_packed_dscales_bytes(int32_t count, int32_t hidden, int32_t inter) {
  return pack_shape_ok(count, hidden, inter) ? moe::packed_dscales_bytes(count, hidden, inter) : 0;
}

moe_status moe_pack_experts(const moe_expert_bank* src, moe_packed_bank* dst, void* stream) {
  if (!src || !dst || !dst->units || !dst->dscales) return MOE_ERR_INVALID_ARG;
  for (const moe_mxfp4_tensor* t : {&src->gate, &src->up, &src->down})
    if (t->fmt != MOE_FMT_MXFP4_E2M1_E8M0_32) return MOE_ERR_FORMAT_MISMATCH;
  const int64_t E = src->gate.count, H = src->gate.K, I = src->gate.rows;
  if (!pack_shape_ok(E, H, I) || dst->count != E || dst->hidden != H || dst->inter != I)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_status s;
  if ((s = check_bank(src, E, H, I)) != MOE_OK) return s;
  if (!aligned16(dst->units) || !aligned16(dst->dscales)) return MOE_ERR_MISALIGNED;
  cudaError_t e = moe::launch_pack_experts(src->gate.data, src->gate.scales, src->up.data, src->up.scales,
                                           src->down.data, src->down.scales, E, (int)H, (int)I, dst->units,
                                           dst->dscales, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  dst->fmt = MOE_FMT_MXFP4_MOE_PACKED;
  return MOE_OK;
}

size_t moe_workspace_bytes(int32_t M, int32_t top_k, int32_t num_experts, int32_t hidden, int32_t inter) {
  if (M < 1 || M > 4 || top_k < 1 || top_k > 8 || num_experts < 1 || num_experts > 1024) return 0;
  if (!moe::moe_layer_supported(hidden, inter)) return 0;
  return moe::moe_ws_bytes(num_experts, hidden);
}

moe_status moe_decode(const uint16_t* hidden_bf16, const float* router_w, const float* router_bias,
                      const moe_packed_bank* experts, const moe_packed_bank* shared, int32_t M, int32_t top_k,
                      float* out, int32_t* topk_ids, float* topk_w, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (!hidden_bf16 || !router_w || !experts || !shared || !out || !workspace) return MOE_ERR_INVALID_ARG;
  if (M < 1 || M > 4 || top_k < 1 || top_k > 8) return MOE_ERR_INVALID_ARG;
  // both tags first: a wrong-format bank is the error to report, whatever else is wrong
  if (experts->fmt != MOE_FMT_MXFP4_MOE_PACKED || shared->fmt != MOE_FMT_MXFP4_MOE_PACKED)
    return MOE_ERR_FORMAT_MISMATCH;
  const int64_t E = experts->count, H = experts->hidden, I = experts->inter;
  if (E < 1 || E > 1024 || top_k > E) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!moe::moe_layer_supported((int)H, (int)I)) return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_status s;
  if ((s = check_packed(experts, E, H, I)) != MOE_OK) return s;
  if ((s = check_packed(shared, 1, H, I)) != MOE_OK) return s;
  if (!aligned16(hidden_bf16) || !aligned16(router_w) || (router_bias && !aligned16(router_bias)) ||
      !aligned16(out) || (topk_ids && !aligned16(topk_ids)) || (topk_w && !aligned16(topk_w)) ||
      !aligned16(workspace))
    return MOE_ERR_MISALIGNED;
  if (workspace_bytes < moe_workspace_bytes(M, top_k, (int32_t)E, (int32_t)H, (int32_t)I)) return MOE_ERR_WORKSPACE;

  moe::MoeArgs a{};
  a.x = hidden_bf16;
  a.router_w = router_w;
  a.router_bias = router_bias;
  a.bank = moe::MoeBank{experts->units, experts->dscales};
  a.shared = moe::MoeBank{shared->units, shared->dscales};
  a.M = M; a.top_k = top_k; a.E = (int)E; a.H = (int)H; a.I = (int)I;
  a.out = out; a.ids_out = topk_ids; a.w_out = topk_w;
  a.ws = moe::MoeWs::carve(workspace, (int)E, (int)H);
  return cuda_status(moe::launch_moe_layer(a, static_cast<cudaStream_t>(stream)));
}

size_t lmhead_workspace_bytes(int32_t M, int32_t top_k, int64_t vocab, int64_t hidden) {
  if (M < 1 || M > 4 || top_k < 1 || top_k > 64 || top_k > vocab) return 0;
  if (!head_shape_ok(vocab, hidden, 1) && !head_shape_ok(vocab, hidden, 2)) return 0;
  return head_ws_bytes(M, top_k);
}

moe_status lmhead_decode(const uint16_t* hidden_bf16, const moe_fp8_head* head, int32_t M, int32_t top_k,
                         int32_t* topk_ids, float* topk_vals, float* logits, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (!head) return MOE_ERR_INVALID_ARG;
  if (head->fmt != MOE_FMT_FP8_E4M3_TILED) return MOE_ERR_FORMAT_MISMATCH;
  if (!head->q || !head->row_scale) return MOE_ERR_INVALID_ARG;
  return launch_head_common(hidden_bf16, head->q, head->row_scale, true, head->vocab, head->hidden, M, top_k,
                            topk_ids, topk_vals, logits, workspace, workspace_bytes, stream);
}

moe_status lmhead_decode_bf16(const uint16_t* hidden_bf16, const moe_bf16_head* head, int32_t M, int32_t top_k,
                              int32_t* topk_ids, float* topk_vals, float* logits, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!head) return MOE_ERR_INVALID_ARG;
  if (head->fmt != MOE_FMT_BF16) return MOE_ERR_FORMAT_MISMATCH;
  if (!head->w) return MOE_ERR_INVALID_ARG;
  return launch_head_common(hidden_bf16, head->w, nullptr, false, head->vocab, head->hidden, M, top_k, topk_ids,
                            topk_vals, logits, workspace, workspace_bytes, stream);
}

moe_status moe_rmsnorm_bf16(const float* y, int32_t M, int32_t H, float eps, uint16_t* out, void* stream) {
  if (!y || !out || M < 1 || H < 8 || H % 8 != 0 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  return cuda_status(moe::launch_rmsnorm_bf16(y, M, H, eps, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_embed_gather(const uint16_t* table, int64_t V, int64_t H, const int32_t* ids, int32_t ids_stride,
                            int32_t M, uint16_t* out, void* stream) {
  if (!table || !ids || !out || V < 1 || H < 8 || H % 8 != 0 || M < 1 || ids_stride < 1) return MOE_ERR_INVALID_ARG;
  if (!aligned16(table) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return MOE_ERR_MISALIGNED;
  return cuda_status(moe::launch_embed_gather(table, V, (int)H, ids, ids_stride, M, out,
                                              static_cast<cudaStream_t>(stream)));
}

moe_status moe_stream_read(const void* src, size_t bytes, uint32_t* sink, void* stream) {
  if (!src || !sink || bytes < 16 || bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(sink) & 3u)) return MOE_ERR_MISALIGNED;
  int dev = 0, sms = 0;
  if (moe::current_device_sms(&dev, &sms) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(moe::launch_stream_read(src, bytes, sink, sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_reset(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < sizeof(moe::WsHeader)) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_status(void* workspace, void* stream) {
  if (!workspace) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t status = 0;
  auto* hdr = static_cast<moe::WsHeader*>(workspace);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&status, &hdr->status, sizeof(status), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (status != 0) {
    if (cudaMemset(&hdr->status, 0, sizeof(status)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return static_cast<moe_status>(status);
}

moe_status moe_query_path(char* buf, size_t n) {
  if (!buf || n == 0) return MOE_ERR_INVALID_ARG;
  const char* desc =
      "sm_100a; moe: one persistent kernel, one CTA per SM (router fp32 GEMV with epoch-tagged logits, "
      "top-k softmax routing in every CTA, split-K over the intermediate: 16-row slices of MXFP4 "
      "E2M1/E8M0-32 gate/up + SiLU + down per work item, one bulk copy per item into a stage ring, "
      "gate/up as tcgen05.mma kind::mxf4 block-scaled on a 128-row operand of four K segments (TMEM "
      "accumulator, activations as 8 E2M1 base-4 digits), "
      "down as mma.sync f16 on E2M1 placed as E5M2, one grid barrier, fixed-order combine); "
      "lm-head: online-FP8 E4M3 per-row-scale GEMV over the fragment-tiled head (warp-specialised: bulk-copy "
      "ring, two mma.sync m16n8k32 e4m3 consumer groups, counter-scheduled tail tiles) fused top-k "
      "with temperature/top-p sampling; kernels chained by programmatic dependent launch; "
      "comparator: BF16 head GEMV";
  std::snprintf(buf, n, "%s", desc);
  return std::strlen(desc) < n ? MOE_OK : MOE_ERR_INVALID_ARG;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_FORMAT_MISMATCH: return "MOE_ERR_FORMAT_MISMATCH";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
  }
  return "MOE_ERR_UNKNOWN";
}

}  // extern "C"
