// moe.h -- internal interface of the MoE-layer kernel (moe_layer.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Device arrays of one sliced expert bank (see pack.h).
struct MoeBank {
  const uint8_t* units;    // [E][I/16][slice_unit_bytes(H)]
  const uint8_t* dscales;  // [E][I/32][H]
};

// Views into the caller's workspace.  Token-indexed arrays use a fixed stride
// of 4 tokens.  The header's barrier word returns to its starting value after
// each call and its epoch counts calls, so nothing needs resetting between
// calls (the workspace is zeroed once before its first use).
struct MoeWs {
  static constexpr int kMaxGrid = 256;  // CTAs of one call at most (one per SM)
  WsHeader* hdr;
  uint64_t* logits;  // [4][E]: (epoch tag << 32) | fp32 bits of each router logit
  float* partials;   // [kMaxGrid][4][H]: each CTA's share of the layer output

  static size_t align(size_t v) { return (v + 255) & ~size_t(255); }
  static size_t bytes(int E, int H) {
    size_t b = align(sizeof(WsHeader));
    b += align((size_t)4 * E * sizeof(uint64_t));
    b += align((size_t)kMaxGrid * 4 * H * sizeof(float));
    return b;
  }
  static MoeWs carve(void* base, int E, int H) {
    (void)H;
    uint8_t* p = static_cast<uint8_t*>(base);
    MoeWs w;
    w.hdr = reinterpret_cast<WsHeader*>(p); p += align(sizeof(WsHeader));
    w.logits = reinterpret_cast<uint64_t*>(p); p += align((size_t)4 * E * sizeof(uint64_t));
    w.partials = reinterpret_cast<float*>(p);
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

inline size_t moe_ws_bytes(int E, int H) { return MoeWs::bytes(E, H); }
bool moe_layer_supported(int H, int I);
cudaError_t launch_moe_layer(const MoeArgs& a, cudaStream_t st);

}  // namespace moe
