// moe.h -- internal interface of the MoE-layer kernel (moe_fused.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Device arrays of one packed expert bank (see moe_packed_bank and pack.h).
struct MoeBank {
  const uint8_t* gateup;  // [E][I/8][gateup_chunk_bytes(H)]
  const uint8_t* down;    // [E][H/32][down_tile_bytes(I)]
};

// Views into the caller's workspace.  Token-indexed arrays use a fixed stride
// of 4 tokens; slot arrays hold at most kMaxSlots = 4 * 8 + 1 entries.  Every
// array is fully written before it is read in each call, and the header's
// barrier word returns to its starting value, so nothing needs resetting
// between calls.
struct MoeWs {
  static constexpr int kMaxSlots = 4 * 8 + 1;
  WsHeader* hdr;
  float* logits;        // [M][E]
  float* h;             // [kMaxSlots][4][I]: silu(gate) * up per slot and token
  uint8_t* hq;          // [kMaxSlots][4][I/32][3][32]: h per 32-element block as three E4M3 parts,
                        //   bytes in MMA B-fragment order (see moe_fused.cu)
  float* hf;            // [kMaxSlots][4][I/32]: 2^(6 - sigma) of each block (undoes its scale)
  float* ypart;         // [kMaxSlots][4][H]: down(h) per slot and token, before the weighted combine

  static size_t align(size_t v) { return (v + 255) & ~size_t(255); }
  static size_t bytes(int M, int top_k, int E, int H, int I) {
    (void)M; (void)top_k;
    size_t b = align(sizeof(WsHeader));
    b += align((size_t)4 * E * sizeof(float));
    b += align((size_t)kMaxSlots * 4 * I * sizeof(float));
    b += align((size_t)kMaxSlots * 4 * (I / 32) * 3 * 32);
    b += align((size_t)kMaxSlots * 4 * (I / 32) * sizeof(float));
    b += align((size_t)kMaxSlots * 4 * H * sizeof(float));
    return b;
  }
  static MoeWs carve(void* base, int E, int H, int I) {
    (void)H;
    uint8_t* p = static_cast<uint8_t*>(base);
    MoeWs w;
    w.hdr = reinterpret_cast<WsHeader*>(p); p += align(sizeof(WsHeader));
    w.logits = reinterpret_cast<float*>(p); p += align((size_t)4 * E * sizeof(float));
    w.h = reinterpret_cast<float*>(p); p += align((size_t)kMaxSlots * 4 * I * sizeof(float));
    w.hq = p; p += align((size_t)kMaxSlots * 4 * (I / 32) * 3 * 32);
    w.hf = reinterpret_cast<float*>(p); p += align((size_t)kMaxSlots * 4 * (I / 32) * sizeof(float));
    w.ypart = reinterpret_cast<float*>(p);
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
