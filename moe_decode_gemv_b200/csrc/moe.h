// moe.h -- internal interface of the MoE-layer kernels (moe_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Raw pointers of one expert bank (stacked over experts), see moe_expert_bank.
struct MoeBank {
  const uint8_t* gate_d;
  const uint8_t* gate_s;
  const uint8_t* up_d;
  const uint8_t* up_s;
  const uint8_t* down_d;
  const uint8_t* down_s;
};

// Views into the caller's workspace.  Token-indexed arrays use a fixed stride
// of 4 tokens; slot arrays hold at most kMaxSlots = 4 * 8 + 1 entries.
struct MoeWs {
  static constexpr int kMaxSlots = 4 * 8 + 1;
  WsHeader* hdr;
  float* logits;        // [M][E]
  int32_t* nslots;      // number of live slots
  int32_t* slot_expert; // [kMaxSlots]: -1 for the shared expert
  uint32_t* slot_mask;  // [kMaxSlots]: bit m set if token m uses the slot
  float* slot_w;        // [kMaxSlots][4]: combine weight of the slot for token m
  float* h;             // [kMaxSlots][4][I]
  float* ypart;         // [kMaxSlots][4][H]
  uint32_t* slot_ready; // [kMaxSlots]: rows of h written (reset by the kernel's last CTA)
  uint32_t* hmax;       // [kMaxSlots][4]: max |h| as fp32 bits (reset likewise)
  uint32_t* tile_ticket;// [H/32]: slots finished per 32-row output tile (self-resetting)

  static size_t align(size_t v) { return (v + 255) & ~size_t(255); }
  static size_t bytes(int M, int top_k, int E, int H, int I) {
    (void)M; (void)top_k;
    size_t b = align(sizeof(WsHeader));
    b += align((size_t)4 * E * sizeof(float));
    b += align(64);
    b += align(kMaxSlots * sizeof(int32_t));
    b += align(kMaxSlots * sizeof(uint32_t));
    b += align((size_t)kMaxSlots * 4 * sizeof(float));
    b += align((size_t)kMaxSlots * 4 * I * sizeof(float));
    b += align((size_t)kMaxSlots * 4 * H * sizeof(float));
    b += align(kMaxSlots * sizeof(uint32_t));
    b += align((size_t)kMaxSlots * 4 * sizeof(uint32_t));
    b += align((size_t)(H / 32 + 1) * sizeof(uint32_t));
    return b;
  }
  static MoeWs carve(void* base, int E, int H, int I) {
    uint8_t* p = static_cast<uint8_t*>(base);
    MoeWs w;
    w.hdr = reinterpret_cast<WsHeader*>(p); p += align(sizeof(WsHeader));
    w.logits = reinterpret_cast<float*>(p); p += align((size_t)4 * E * sizeof(float));
    w.nslots = reinterpret_cast<int32_t*>(p); p += align(64);
    w.slot_expert = reinterpret_cast<int32_t*>(p); p += align(kMaxSlots * sizeof(int32_t));
    w.slot_mask = reinterpret_cast<uint32_t*>(p); p += align(kMaxSlots * sizeof(uint32_t));
    w.slot_w = reinterpret_cast<float*>(p); p += align((size_t)kMaxSlots * 4 * sizeof(float));
    w.h = reinterpret_cast<float*>(p); p += align((size_t)kMaxSlots * 4 * I * sizeof(float));
    w.ypart = reinterpret_cast<float*>(p); p += align((size_t)kMaxSlots * 4 * H * sizeof(float));
    w.slot_ready = reinterpret_cast<uint32_t*>(p); p += align(kMaxSlots * sizeof(uint32_t));
    w.hmax = reinterpret_cast<uint32_t*>(p); p += align((size_t)kMaxSlots * 4 * sizeof(uint32_t));
    w.tile_ticket = reinterpret_cast<uint32_t*>(p);
    return w;
  }
};

struct MoeArgs {
  const uint16_t* x;
  const float* router_w;
  const float* router_bias;
  MoeBank bank;
  MoeBank shared;
  int M, top_k, E, H, I;
  float* out;
  int32_t* ids_out;
  float* w_out;
  MoeWs ws;
};

inline size_t moe_ws_bytes(int M, int top_k, int E, int H, int I) { return MoeWs::bytes(M, top_k, E, H, I); }
size_t moe_fused_smem_bytes(int H, int I);
bool moe_fused_supported(int H, int I);
cudaError_t launch_moe_fused(const MoeArgs& a, cudaStream_t st);

}  // namespace moe
