// moe_kernels.cu -- the routed-expert MoE layer at M <= 4 tokens over MXFP4
// weights: router GEMV + top-k, gate/up GEMV with the SiLU gate fused, down
// GEMV per active expert, ordered weighted combine.
//
// The pages: each token goes to 8 of 512 routed experts plus a shared expert
// that always runs (saipien.org essay, "Why one user waits on weights"); the
// expert layer is narrow, intermediate 768 (same essay, "Kernels built for the
// shape you actually have"); verifying 4 positions wakes up to 32 routed
// experts (same essay, "Draft three tokens, verify four").  Only the selected
// experts' bytes are streamed, and each distinct expert once per call however
// many of the M tokens chose it.
//
// Work is expressed as "slots": slot 0 is the shared expert (every token,
// weight 1), slots 1.. are the distinct routed experts of the call in order of
// first appearance (token-major, rank order).  The router kernel's last CTA
// builds the slot table in the workspace; later kernels read it there, so no
// routing decision travels back to the host.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "moe.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

// ------------------------------- router ------------------------------------
// CTA = 8 warps = 4 experts x 2 halves of H.  Each lane keeps H/256 float4
// loads of its half-row in flight.  The last CTA to finish takes the top-k
// of every token, the renormalised softmax weights and the slot table.
template <int kM>
__global__ void __launch_bounds__(kThreads)
router_topk_kernel(const uint16_t* __restrict__ x, const float* __restrict__ Wr, const float* __restrict__ bias,
                   int E, int H, int top_k, MoeWs ws, int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
  __shared__ float part[8][kM];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 4 + (warp >> 1);
  const int half = warp & 1;
  float acc[kM];
#pragma unroll
  for (int m = 0; m < kM; ++m) acc[m] = 0.f;
  if (e < E) {
    const int hw = H / 2;
    const float* row = Wr + (size_t)e * H + half * hw;
    for (int j = lane * 4; j < hw; j += 128) {
      const float4 wv = ld_stream_f4(row + j);
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        const uint2 xv = *reinterpret_cast<const uint2*>(x + (size_t)m * H + half * hw + j);
        acc[m] += wv.x * bf16_bits_to_f32(xv.x & 0xffffu) + wv.y * bf16_bits_to_f32(xv.x >> 16) +
                  wv.z * bf16_bits_to_f32(xv.y & 0xffffu) + wv.w * bf16_bits_to_f32(xv.y >> 16);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kM; ++m) {
    const float v = warp_sum(acc[m]);
    if (lane == 0) part[warp][m] = v;
  }
  __syncthreads();
  if (threadIdx.x < 4 * kM) {
    const int ee = blockIdx.x * 4 + threadIdx.x / kM, m = threadIdx.x % kM;
    if (ee < E) {
      float l = part[2 * (threadIdx.x / kM)][m] + part[2 * (threadIdx.x / kM) + 1][m];
      if (bias) l += bias[ee];
      ws.logits[(size_t)m * E + ee] = l;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&ws.hdr->ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA: top-k per token (warp m), ties to the lower expert id ----
  __shared__ int32_t s_ids[kM][8];
  __shared__ float s_w[kM][8];
  if (warp < kM) {
    const int m = warp;
    uint32_t taken = 0u;  // bit i: expert lane + 32 i already selected (E <= 1024)
    float top[8];
    for (int r = 0; r < top_k; ++r) {
      float bv = -FLT_MAX;
      int32_t bi = INT32_MAX;
      for (int i = 0; lane + 32 * i < E; ++i) {
        if (taken >> i & 1u) continue;
        const float v = __ldcg(&ws.logits[(size_t)m * E + lane + 32 * i]);
        if (better(v, lane + 32 * i, bv, bi)) { bv = v; bi = lane + 32 * i; }
      }
      warp_best(bv, bi);
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      top[r] = bv;
      if (lane == 0) s_ids[m][r] = bi;
    }
    // renormalised softmax over the selected logits (top[0] is the largest)
    float z = 0.f;
    for (int r = 0; r < top_k; ++r) z += expf(top[r] - top[0]);
    if (lane == 0)
      for (int r = 0; r < top_k; ++r) s_w[m][r] = expf(top[r] - top[0]) / z;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // slot 0: shared expert; then distinct routed experts in first-appearance order
    int n = 1;
    ws.slot_expert[0] = -1;
    for (int m = 0; m < kM; ++m) ws.slot_w[0 * 4 + m] = 1.0f;
    ws.slot_mask[0] = (1u << kM) - 1u;
    for (int m = 0; m < kM; ++m) {
      for (int r = 0; r < top_k; ++r) {
        const int32_t ex = s_ids[m][r];
        int s = 1;
        while (s < n && ws.slot_expert[s] != ex) ++s;
        if (s == n) {
          ws.slot_expert[n] = ex;
          ws.slot_mask[n] = 0u;
          for (int mm = 0; mm < 4; ++mm) ws.slot_w[n * 4 + mm] = 0.f;
          ++n;
        }
        ws.slot_mask[s] |= 1u << m;
        ws.slot_w[s * 4 + m] = s_w[m][r];
        if (ids_out) ids_out[m * top_k + r] = ex;
        if (w_out) w_out[m * top_k + r] = s_w[m][r];
      }
    }
    *ws.nslots = n;
    __threadfence();
    ws.hdr->ticket = 0u;
  }
}

// Dot product of one MXFP4 block (16 code bytes, 32 elements) with 32 fp32
// activations in shared memory; the block scale is applied by the caller.
__device__ __forceinline__ float block_dot(const uint4 codes, const float* __restrict__ xs) {
  const uint32_t c[4] = {codes.x, codes.y, codes.z, codes.w};
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x0 = *reinterpret_cast<const float4*>(xs + 8 * i);
    const float4 x1 = *reinterpret_cast<const float4*>(xs + 8 * i + 4);
    const uint32_t h0 = e2m1x2_to_f16x2(c[i] & 0xffu), h1 = e2m1x2_to_f16x2((c[i] >> 8) & 0xffu);
    const uint32_t h2 = e2m1x2_to_f16x2((c[i] >> 16) & 0xffu), h3 = e2m1x2_to_f16x2(c[i] >> 24);
    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
    const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&h3));
    acc = fmaf(f0.x, x0.x, acc); acc = fmaf(f0.y, x0.y, acc);
    acc = fmaf(f1.x, x0.z, acc); acc = fmaf(f1.y, x0.w, acc);
    acc = fmaf(f2.x, x1.x, acc); acc = fmaf(f2.y, x1.y, acc);
    acc = fmaf(f3.x, x1.z, acc); acc = fmaf(f3.y, x1.w, acc);
  }
  return acc;
}

// ------------------------------ gate / up -----------------------------------
// grid (I/16, max slots).  Each warp owns 2 rows r of one slot's expert and
// computes gate and up for both; h = silu(g) * u for every token of the slot.
template <int kM>
__global__ void __launch_bounds__(kThreads)
gateup_kernel(const uint16_t* __restrict__ x, MoeBank bank, MoeBank shared, int H, int I, MoeWs ws) {
  extern __shared__ __align__(16) float xs[];  // [kM][H]
  const int slot = blockIdx.y;
  if (slot >= *ws.nslots) return;
  const int ex = ws.slot_expert[slot];
  const uint32_t mask = ws.slot_mask[slot];
  const MoeBank& b = ex < 0 ? shared : bank;
  const int64_t e = ex < 0 ? 0 : ex;
  for (int i = threadIdx.x; i < kM * H; i += blockDim.x) xs[i] = bf16_bits_to_f32(x[i]);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * 16 + warp * 2;
  const int nb = H / 32;
  const size_t mat_d = (size_t)I * H / 2, mat_s = (size_t)I * H / 32;
  const uint8_t* gd = b.gate_d + e * mat_d;
  const uint8_t* gs = b.gate_s + e * mat_s;
  const uint8_t* ud = b.up_d + e * mat_d;
  const uint8_t* us = b.up_s + e * mat_s;
  float acc[4][kM];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int m = 0; m < kM; ++m) acc[q][m] = 0.f;
  for (int blk = lane; blk < nb; blk += 32) {
    uint4 cd[4];
    float sc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + (q & 1);
      const uint8_t* d = (q < 2 ? gd : ud) + (size_t)r * (H / 2) + blk * 16;
      const uint8_t* s = (q < 2 ? gs : us) + (size_t)r * nb + blk;
      cd[q] = ld_stream_u4(d);
      sc[q] = e8m0_to_f32(*s);
    }
#pragma unroll
    for (int m = 0; m < kM; ++m) {
      if (!(mask >> m & 1u)) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q][m] = fmaf(block_dot(cd[q], xs + m * H + blk * 32), sc[q], acc[q][m]);
    }
  }
#pragma unroll
  for (int m = 0; m < kM; ++m) {
    if (!(mask >> m & 1u)) continue;
    float v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = warp_sum(acc[q][m]);
    if (lane == 0) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const float g = v[rr], u = v[2 + rr];
        ws.h[((size_t)slot * 4 + m) * I + r0 + rr] = g / (1.0f + expf(-g)) * u;
      }
    }
  }
}

// -------------------------------- down -------------------------------------
// grid (H/32, max slots).  Each warp owns 4 output rows of one slot; 8 lanes
// per row take every 8th block of the row.  Writes ypart[slot][m][row].
template <int kM>
__global__ void __launch_bounds__(kThreads)
down_kernel(MoeBank bank, MoeBank shared, int H, int I, MoeWs ws) {
  const int slot = blockIdx.y;
  if (slot >= *ws.nslots) return;
  const int ex = ws.slot_expert[slot];
  const uint32_t mask = ws.slot_mask[slot];
  const MoeBank& b = ex < 0 ? shared : bank;
  const int64_t e = ex < 0 ? 0 : ex;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 32 + warp * 4 + (lane >> 3);
  const int p = lane & 7;
  const int nb = I / 32;
  const uint8_t* dd = b.down_d + e * ((size_t)H * I / 2) + (size_t)row * (I / 2);
  const uint8_t* ds = b.down_s + e * ((size_t)H * I / 32) + (size_t)row * nb;
  float acc[kM];
#pragma unroll
  for (int m = 0; m < kM; ++m) acc[m] = 0.f;
  for (int blk = p; blk < nb; blk += 8) {
    const uint4 cd = ld_stream_u4(dd + blk * 16);
    const float sc = e8m0_to_f32(ds[blk]);
#pragma unroll
    for (int m = 0; m < kM; ++m) {
      if (!(mask >> m & 1u)) continue;
      acc[m] = fmaf(block_dot(cd, ws.h + ((size_t)slot * 4 + m) * I + blk * 32), sc, acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < kM; ++m) {
    float v = acc[m];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (p == 0 && (mask >> m & 1u)) ws.ypart[((size_t)slot * 4 + m) * H + row] = v;
  }
}

// ------------------------------- combine -----------------------------------
// out[m][i] = sum over slots, in slot order, of slot_w[s][m] * ypart[s][m][i].
template <int kM>
__global__ void combine_kernel(int H, MoeWs ws, float* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H) return;
  const int n = *ws.nslots;
#pragma unroll
  for (int m = 0; m < kM; ++m) {
    float y = 0.f;
    for (int s = 0; s < n; ++s)
      if (ws.slot_mask[s] >> m & 1u) y = fmaf(ws.slot_w[s * 4 + m], ws.ypart[((size_t)s * 4 + m) * H + i], y);
    out[(size_t)m * H + i] = y;
  }
}

template <int kM>
cudaError_t launch_t(const MoeArgs& a, cudaStream_t st) {
  const int max_slots = kM * a.top_k + 1;
  router_topk_kernel<kM><<<(a.E + 3) / 4, kThreads, 0, st>>>(a.x, a.router_w, a.router_bias, a.E, a.H, a.top_k,
                                                            a.ws, a.ids_out, a.w_out);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t xs_bytes = (size_t)kM * a.H * sizeof(float);
  if (xs_bytes > 48 * 1024) {
    err = cudaFuncSetAttribute(gateup_kernel<kM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)xs_bytes);
    if (err != cudaSuccess) return err;
  }
  gateup_kernel<kM><<<dim3(a.I / 16, max_slots), kThreads, xs_bytes, st>>>(a.x, a.bank, a.shared, a.H, a.I, a.ws);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  down_kernel<kM><<<dim3(a.H / 32, max_slots), kThreads, 0, st>>>(a.bank, a.shared, a.H, a.I, a.ws);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  combine_kernel<kM><<<(a.H + 255) / 256, 256, 0, st>>>(a.H, a.ws, a.out);
  return cudaGetLastError();
}

}  // namespace

size_t moe_ws_bytes(int M, int top_k, int E, int H, int I) {
  return MoeWs::bytes(M, top_k, E, H, I);
}

cudaError_t launch_moe(const MoeArgs& a, cudaStream_t st) {
  switch (a.M) {
    case 1: return launch_t<1>(a, st);
    case 2: return launch_t<2>(a, st);
    case 3: return launch_t<3>(a, st);
    case 4: return launch_t<4>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
