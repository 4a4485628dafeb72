// moe_layer.cu -- the whole MoE layer (router GEMV, top-k softmax routing,
// MXFP4 gate/up GEMV + SiLU gate, down GEMV, shared expert, weighted
// combine) as one cooperative persistent kernel, for M <= 4 tokens.
//
// The pages: each token goes to 8 of 512 routed experts plus a shared expert
// that always runs (saipien.org essay, "Why one user waits on weights"); the
// expert layer is narrow, intermediate 768 (same essay, "Kernels built for the
// shape you actually have"); verifying 4 positions wakes up to 32 routed
// experts (same essay, "Draft three tokens, verify four").  At batch 1 the
// layer is bound by weight reads, so the kernel keeps as many weight bytes in
// flight as it can and synchronises the grid once.
//
//  * One CTA per SM (cooperative launch: all CTAs resident), 16 warps.
//  * Work items split every expert along its intermediate dimension: item
//    (slot, j) computes gate and up rows 16j .. 16j+15, h = silu(gate) * up
//    for those rows, and applies the matching 16 columns of the down matrix
//    to h -- split-K over the intermediate, so that the narrow 768-wide layer
//    still gives 48 items per expert and h never leaves the CTA.  Each
//    item's bytes are one contiguous unit of the sliced bank (pack.h),
//    brought into a ring of shared-memory stages by bulk copies (no
//    multicast) that complete on an mbarrier per stage.  Item q goes to CTA
//    q mod G; the shared expert's items come first, so the CTAs that own them
//    start streaming and computing before routing is known.
//  * Router: the tokens are copied into shared memory at once; each CTA
//    scores its share of the router rows (fp32 weights, bf16 activations,
//    fp32 sums) and publishes each logit as one 64-bit word (epoch tag << 32
//    | value), so that readers need no barrier: every CTA polls the words
//    until all carry this call's tag, then takes the same top-k and builds
//    the same slot table (slot 0 = shared expert, then each distinct routed
//    expert once).  Top-k, one warp per token: the k-th best of the 32 lane
//    maxima bounds the k-th best logit from below, and the few logits not
//    worse than that bound are ranked by counting.
//  * Each lane owns a fixed set of output rows and accumulates its CTA's
//    weighted contributions in registers across items.  After the last item
//    the CTAs write these partial outputs, meet at one grid barrier, and sum
//    them in a fixed order (no float atomics: the result is the same on
//    every run).
//
// Arithmetic: mma.sync m16n8k32 E5M2 (weights) x E4M3 (activations) -> fp32.
// The packed nibbles become E5M2 codes of the E2M1 values times 2^-14 by one
// mask (even elements) or two shifts (odd ones).  Each 32-element block's MMA
// result is scaled by the weights' E8M0 scale and the activation block's own
// power of two before it joins an fp32 sum.
//  * x: per token and 32-element block, scaled so that the block's largest
//    magnitude lies in [2^7, 2^8), then carried by two E4M3 parts (exact for
//    bf16 values down to 2^-10 of the block's largest) in two columns of the
//    MMA: column n = part n & 1 of token n >> 1.
//  * h: per token and item (16 values), scaled by a power of two that puts
//    the largest magnitude in [2^14, 2^15) and carried by two f16 parts (about
//    22 significant bits) into mma.sync m16n8k16 f16 x f16 -> fp32, whose K of
//    16 is exactly the item's slice.  The weights' E5M2 bytes are the top
//    bytes of f16 values (one byte permute each pair); column n of B = part
//    n & 1 of token n >> 1, so one MMA covers 16 output rows of all tokens.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "moe.h"
#include "pack.h"

namespace moe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxBlocksPerWarp = 8;  // H <= 8 * 16 * 32 = 4096
constexpr int kMaxStages = 4;
constexpr int kMaxSlots = 4 * 8 + 1;
constexpr int kRouterChunk = 8;        // float4 router loads in flight per lane
constexpr int kMaxE = 1024;
constexpr uint32_t kFull = 0xffffffffu;

struct Geo {
  int H, I, nb, n_sl, n_pairs, a_bytes, b_bytes, unit_bytes, stage_bytes;
  __host__ __device__ Geo(int H_, int I_) : H(H_), I(I_) {
    nb = H / 32;
    n_sl = I / kSliceRows;
    n_pairs = I / 32;
    a_bytes = slice_a_bytes(H);
    b_bytes = slice_b_bytes(H);
    unit_bytes = slice_unit_bytes(H);
    stage_bytes = (unit_bytes + H + 127) / 128 * 128;  // the unit, then its pair's down scales
  }
};

constexpr int kCandCap = 256;  // routing candidates per token: at most top_k lanes' E/32 logits

struct Ctl {
  uint64_t full[kMaxStages];                 // one phase per item copied into the stage
  uint64_t xbar;                             // the tokens' copy into shared memory
  float router_part[kWarps][4];
  int32_t sigma_x[4][kMaxBlocksPerWarp * kWarps];
  uint16_t cand[4][kCandCap];                // routing: candidate experts of each token
  int32_t ids[4][8];
  float topv[4][8];
  float wts[4][8];
  int32_t slot_expert[kMaxSlots];
  uint32_t slot_mask[kMaxSlots];
  float slot_w[kMaxSlots][4];
  alignas(16) uint16_t hp[4][2][4][4];       // h of one item as f16: [token][part][t][elements 4t, 4t+2, 4t+1, 4t+3]
  float hfw[4];
  int nslots;
  int poison;
};
constexpr int kCtlBytes = (int)((sizeof(Ctl) + 127) / 128 * 128);
// The scratch area holds, one after the other: the tokens (bf16, while the
// router and the activation fragments read them), the M x E router logits
// (while routing), each item's gate/up partial sums (after).
__host__ __device__ constexpr int scratch_bytes(int H) {
  const int xb = 4 * H * 2, lb = 4 * kMaxE * 4, rb = kWarps * 32 * 16;
  const int m = xb > lb ? (xb > rb ? xb : rb) : (lb > rb ? lb : rb);
  return (m + 127) / 128 * 128;
}

struct LayerArgs {
  const uint16_t* x;
  const float* router_w;
  const float* router_bias;
  MoeBank bank, shared;
  int M, top_k, E, H, I, stages;
  float* out;
  int32_t* ids_out;
  float* w_out;
  MoeWs ws;
};

// ---- memory helpers ----
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_router(const float* p, uint64_t policy) {
  float4 r;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "l"(p), "l"(policy));
  return r;
}

// ---- power-of-two scaling of activation blocks ----
// sigma such that amax * 2^sigma lies in [2^7, 2^8) (the top of E4M3's normal
// range, max 448), clamped to [-113, 140] so that 2^(14 - sigma) is a normal
// fp32 number; 140 covers every bf16 value (the smallest is 2^-133).  0 for
// amax = 0 (or NaN).
__device__ __forceinline__ int pow2_sigma(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int e = (int)((b >> 23) & 0xffu);
  const int fl = e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
  const int s = 7 - fl;
  return s > 140 ? 140 : (s < -113 ? -113 : s);
}
// 2^e for e in [-126, 127], exactly.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }
// v * 2^s for s in [-113, 140], exactly (two steps above 2^126).
__device__ __forceinline__ float scale_pow2(float v, int s) {
  return s > 126 ? v * exp2i(126) * exp2i(s - 126) : v * exp2i(s);
}

// ---- routing: the best 8 of up to 1,024 logits across warps ----
// (value, expert) pairs under `better`: larger value first, lower id on ties.
struct VI {
  float v;
  int32_t i;
};
// A padding entry ranks below every real entry (real logits are clamped to
// >= -FLT_MAX, real ids are < 1024); entries further down a sorted list get
// larger padding ids, so padded lists stay sorted.
__device__ __forceinline__ VI pad_entry(int pos) { return VI{-FLT_MAX, 0x7fffff00 + pos}; }

// Grid barrier on one word (all CTAs are resident: cooperative launch).  The
// first CTA adds 2^31 - (G - 1), the others 1, so the top bit flips exactly
// when all G have arrived and the low bits return to where they were: the
// same word serves every call.  Arrival publishes the caller's earlier writes
// (fence first); the wait is bounded.
__device__ __forceinline__ uint32_t grid_arrive(uint32_t* word, int c, int G) {
  __threadfence();
  return atomicAdd(word, c == 0 ? 0x80000000u - (uint32_t)(G - 1) : 1u);
}
__device__ __forceinline__ bool grid_wait(uint32_t* word, uint32_t old) {
  return bounded_spin([&] { return ((ld_acquire(word) ^ old) & 0x80000000u) != 0u; });
}

template <int kB>
__global__ void __launch_bounds__(kThreads, 1) moe_layer_kernel(LayerArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  Ctl& C = *reinterpret_cast<Ctl*>(smem);
  uint8_t* scratch = smem + kCtlBytes;
  const Geo geo(a.H, a.I);
  uint8_t* stages = scratch + scratch_bytes(a.H);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int G = gridDim.x, c = blockIdx.x;
  const int M = a.M, H = a.H, E = a.E, NS = a.stages;
  const int nb = geo.nb, n_sl = geo.n_sl;
  const MoeWs ws = a.ws;
  WsHeader* hdr = ws.hdr;
  const uint64_t policy = l2_evict_first_policy();
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(scratch);  // the tokens, [M][H] bf16

  // The shared expert's items of this CTA are known before routing; item j
  // (q = c + G j) sits in stage j % NS.
  const int n_pre = c < n_sl ? (n_sl - c + G - 1) / G : 0;
  auto issue = [&](int j) {  // one thread: the item's unit and its pair's down scales, two bulk copies
    const int s = j % NS;
    const int q = c + G * j;
    const int slot = q / n_sl, sl = q - slot * n_sl;
    const MoeBank& bk = slot == 0 ? a.shared : a.bank;
    const size_t e = slot == 0 ? 0 : (size_t)C.slot_expert[slot];
    uint8_t* dst = stages + (size_t)s * geo.stage_bytes;
    mbar_arrive_expect_tx(&C.full[s], (uint32_t)(geo.unit_bytes + H));
    bulk_g2s(dst, bk.units + (e * n_sl + sl) * (size_t)geo.unit_bytes, (uint32_t)geo.unit_bytes, &C.full[s], policy);
    bulk_g2s(dst + geo.unit_bytes, bk.dscales + (e * geo.n_pairs + (sl >> 1)) * (size_t)H, (uint32_t)H, &C.full[s],
             policy);
  };
  int issued = 0, consumed = 0;  // kept by thread 0, the only issuer
  auto top_up = [&](int limit) {
    if (threadIdx.x == 0)
      while (issued < limit && issued < consumed + NS) issue(issued++);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&C.full[s], 1);
    mbar_init(&C.xbar, 1);
    fence_mbar_init();
    C.poison = 0;
    top_up(n_pre);  // the shared expert's items: weights, which no kernel writes
  }

  // ---- router loads of this CTA's rows: the first chunk goes out now ----
  const int e_begin = (int)((int64_t)E * c / G), e_end = (int)((int64_t)E * (c + 1) / G);
  const int R = e_end - e_begin;
  const int RR = R < kWarps ? R : kWarps;    // rows per round
  const int wpr = RR > 0 ? kWarps / RR : 1;  // warps per row
  const int F = H / 4;                       // float4 per router row
  auto router_slot = [&](int base, int& row, int& f0, int& f1) {  // this warp's share of a round
    const int lr = warp / wpr, part = warp - lr * wpr;
    row = (lr < RR && base + lr < R) ? base + lr : -1;
    f0 = part * F / wpr;
    f1 = (part + 1) * F / wpr;
  };
  float4 wv[kRouterChunk];
  auto router_load = [&](int row, int f, int f1) {
#pragma unroll
    for (int i = 0; i < kRouterChunk; ++i) wv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < 0) return;
#pragma unroll
    for (int i = 0; i < kRouterChunk; ++i) {
      const int ff = f + 32 * i;
      if (ff < f1) wv[i] = ld_router(a.router_w + (size_t)(e_begin + row) * H + 4 * ff, policy);
    }
  };
  int r_row, r_f0, r_f1;
  router_slot(0, r_row, r_f0, r_f1);
  if (R > 0) router_load(r_row, r_f0 + lane, r_f1);
  __syncthreads();  // the barriers are initialised
  // Everything below may read what the previous kernel on the stream wrote
  // (the tokens, the workspace): wait for it.  The weight copies and loads
  // above are already on their way.
  pdl_wait();
  pdl_launch_dependents();  // the next kernel may launch; its CTAs start as this one's exit
  // This call's tag: the epoch advances once per call, after every CTA has read it.
  const uint32_t tag = ld_relaxed_u32(&hdr->epoch) + 1u;
  if (threadIdx.x == 0) {
    const uint32_t xbytes = (uint32_t)(M * H * 2);
    mbar_arrive_expect_tx(&C.xbar, xbytes);
    bulk_g2s(scratch, a.x, xbytes, &C.xbar, l2_evict_last_policy());
  }

  auto poisoned = [&]() -> bool { return *(volatile int*)&C.poison != 0; };
  auto fail = [&]() {  // the first wait of this CTA that ran out
    if (!poisoned()) {
      report(hdr, MOE_ERR_TIMEOUT);
      atomicExch(&C.poison, 1);
    }
  };
  if (!mbar_wait(&C.xbar, 0)) fail();

  // ---- router GEMV: finish the first chunk, then any further chunks/rounds ----
  float racc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int base = 0; base < R; base += RR) {
    router_slot(base, r_row, r_f0, r_f1);
    for (int f = r_f0 + lane; f < r_f1; f += 32 * kRouterChunk) {
      if (!(base == 0 && f == r_f0 + lane)) router_load(r_row, f, r_f1);
      if (r_row >= 0) {
#pragma unroll
        for (int i = 0; i < kRouterChunk; ++i) {
          const int ff = f + 32 * i;
          if (ff < r_f1) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              if (m < M) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xs + m * H + 4 * ff);
                racc[m] += wv[i].x * bf16_bits_to_f32(xv.x & 0xffffu) + wv[i].y * bf16_bits_to_f32(xv.x >> 16) +
                           wv[i].z * bf16_bits_to_f32(xv.y & 0xffffu) + wv[i].w * bf16_bits_to_f32(xv.y >> 16);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float v = warp_sum(racc[m]);
      if (lane == 0) C.router_part[warp][m] = v;
      racc[m] = 0.f;
    }
    __syncthreads();
    if (threadIdx.x < RR * 4) {
      const int lr = threadIdx.x >> 2, m = threadIdx.x & 3;
      const int e = e_begin + base + lr;
      if (m < M && base + lr < R) {
        float l = 0.f;
        for (int p = 0; p < wpr; ++p) l += C.router_part[lr * wpr + p][m];
        if (a.router_bias) l += a.router_bias[e];
        st_relaxed_u64(&ws.logits[(size_t)m * E + e], ((uint64_t)tag << 32) | __float_as_uint(l));
      }
    }
    __syncthreads();
  }

  // ---- x: per (token, block) power-of-two scale, then this lane's B fragments ----
  for (int t = threadIdx.x; t < M * nb; t += kThreads) {
    const int m = t / nb, b = t - m * nb;
    const uint4* p = reinterpret_cast<const uint4*>(xs + m * H + 32 * b);
    float am = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = p[q];
      am = fmaxf(am, fmaxf(fmaxf(bf16_bits_to_f32(v.x & 0x7fffu), bf16_bits_to_f32((v.x >> 16) & 0x7fffu)),
                           fmaxf(bf16_bits_to_f32(v.y & 0x7fffu), bf16_bits_to_f32((v.y >> 16) & 0x7fffu))));
      am = fmaxf(am, fmaxf(fmaxf(bf16_bits_to_f32(v.z & 0x7fffu), bf16_bits_to_f32((v.z >> 16) & 0x7fffu)),
                           fmaxf(bf16_bits_to_f32(v.w & 0x7fffu), bf16_bits_to_f32((v.w >> 16) & 0x7fffu))));
    }
    C.sigma_x[m][b] = pow2_sigma(am);
  }
  __syncthreads();
  // Lane (g, t) of warp w, block b = w + 16 jb: column g of B = part g & 1 of
  // token g >> 1; its even elements 32b + 8t + 2i fill b0, the odd ones b1
  // (the order of the weight nibbles).  fx undoes the scale of token t's block
  // and the E5M2 weights' 2^-14 on the D side (columns 2t, 2t+1 = token t).
  uint32_t bx[kB][2];
  float fx[kB];
  {
    const int mB = g >> 1, part = g & 1;
#pragma unroll
    for (int jb = 0; jb < kB; ++jb) {
      const int b = warp + kWarps * jb;
      uint32_t b0 = 0u, b1 = 0u;
      if (b < nb && mB < M) {
        const int sg = C.sigma_x[mB][b];
        const uint4 q = *reinterpret_cast<const uint4*>(xs + mB * H + 32 * b + 8 * tq);
        auto xsc = [&](uint32_t bits) { return scale_pow2(bf16_bits_to_f32(bits), sg); };
        uint32_t pe[2], po[2];
        split_e4m3x4<2>(xsc(q.x & 0xffffu), xsc(q.y & 0xffffu), xsc(q.z & 0xffffu), xsc(q.w & 0xffffu), pe);
        split_e4m3x4<2>(xsc(q.x >> 16), xsc(q.y >> 16), xsc(q.z >> 16), xsc(q.w >> 16), po);
        b0 = part ? pe[1] : pe[0];
        b1 = part ? po[1] : po[0];
      }
      bx[jb][0] = b0;
      bx[jb][1] = b1;
      fx[jb] = (b < nb && tq < M) ? exp2i(14 - C.sigma_x[tq][b]) : 0.f;
    }
  }
  __syncthreads();  // the tokens' shared memory is free from here on

  // ---- one work item: gate/up over H, SiLU gate, down over its 16 columns ----
  float yacc[kB][4];
#pragma unroll
  for (int jg = 0; jg < kB; ++jg) yacc[jg][0] = yacc[jg][1] = yacc[jg][2] = yacc[jg][3] = 0.f;
  auto compute = [&](int j) {
    const int s = j % NS;
    const int slot = (c + G * j) / n_sl;
    if (!poisoned() && !mbar_wait(&C.full[s], (uint32_t)((j / NS) & 1))) fail();
    const uint8_t* st = stages + (size_t)s * geo.stage_bytes;
    const uint32_t all = (1u << M) - 1u;
    const uint32_t mask = slot == 0 ? all : C.slot_mask[slot];
    // gate/up: this warp's K blocks, two 16-row tiles (gate rows g, up rows g
    // of the slice's first and second half)
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jb = 0; jb < kB; ++jb) {
      const int b = warp + kWarps * jb;
      if (b < nb) {
        const uint4 q = *reinterpret_cast<const uint4*>(st + (b * 32 + lane) * 16);
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(st + geo.a_bytes + (b * 8 + g) * 4);
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
        mma_e5m2_e4m3(d0, packed_even_to_e5m2x4(q.x), packed_even_to_e5m2x4(q.y), packed_odd_to_e5m2x4(q.x),
                      packed_odd_to_e5m2x4(q.y), bx[jb][0], bx[jb][1]);
        mma_e5m2_e4m3(d1, packed_even_to_e5m2x4(q.z), packed_even_to_e5m2x4(q.w), packed_odd_to_e5m2x4(q.z),
                      packed_odd_to_e5m2x4(q.w), bx[jb][0], bx[jb][1]);
        const float f = fx[jb];
        acc[0] = fmaf(d0[0] + d0[1], e8m0_to_f32_fast(sc & 0xffu) * f, acc[0]);          // gate row g, token t
        acc[1] = fmaf(d0[2] + d0[3], e8m0_to_f32_fast((sc >> 8) & 0xffu) * f, acc[1]);   // up row g
        acc[2] = fmaf(d1[0] + d1[1], e8m0_to_f32_fast((sc >> 16) & 0xffu) * f, acc[2]);  // gate row 8 + g
        acc[3] = fmaf(d1[2] + d1[3], e8m0_to_f32_fast(sc >> 24) * f, acc[3]);            // up row 8 + g
      }
    }
    float4* red = reinterpret_cast<float4*>(scratch);
    red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    // h for the slice's 16 rows and each token, in fp32; then its f16 parts
    if (threadIdx.x < 64) {
      const int m = threadIdx.x >> 4, r = threadIdx.x & 15;
      const float2* rp = reinterpret_cast<const float2*>(red + (r & 7) * 4 + m) + (r >> 3);
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float2 p = rp[w * 64];
        gs += p.x;
        us += p.y;
      }
      const bool live = m < M && ((mask >> m) & 1u);
      const float h = live ? gs / (1.0f + expf(-gs)) * us : 0.f;
      float am = fabsf(h);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(kFull, am, o));
      // sigma such that the largest |h| of the slice lies in [2^14, 2^15)
      const int sig = min(pow2_sigma(am) + 7, 140);
      const float v = scale_pow2(h, sig);
      const __half hi = __float2half_rn(v);
      const __half lo = __float2half_rn(v - __half2float(hi));
      const int pos = ((r & 1) << 1) | ((r >> 1) & 1);  // element r = 4t + i sits at [t][0, 2, 1, 3 -> 0..3]
      C.hp[m][0][r >> 2][pos] = __half_as_ushort(hi);
      C.hp[m][1][r >> 2][pos] = __half_as_ushort(lo);
      if (r == 0) C.hfw[m] = live ? (slot == 0 ? 1.0f : C.slot_w[slot][m]) * exp2i(14 - sig) : 0.f;
    }
    __syncthreads();
    // down: this warp's 32-row output groups, two MMAs (16 rows each) per group
    // for all tokens; lane (g, t) ends with rows 32G + 8r + g of token t
    const uint2 bh = (g >> 1) < M ? *reinterpret_cast<const uint2*>(&C.hp[g >> 1][g & 1][tq][0]) : make_uint2(0u, 0u);
    const float hw = tq < M ? C.hfw[tq] : 0.f;
    const uint8_t* cdat = st + geo.a_bytes + geo.b_bytes;
    const uint8_t* cscl = st + geo.unit_bytes;
#pragma unroll
    for (int jg = 0; jg < kB; ++jg) {
      const int Gi = warp + kWarps * jg;
      if (Gi < nb) {
        const uint2 aw = *reinterpret_cast<const uint2*>(cdat + (Gi * 32 + lane) * 8);
        const uint32_t sd4 = *reinterpret_cast<const uint32_t*>(cscl + Gi * 32 + 4 * g);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // rows 32G + 16hf + (g, g + 8)
          const uint32_t w = hf ? aw.y : aw.x;
          const uint32_t ev = packed_even_to_e5m2x4(w), od = packed_odd_to_e5m2x4(w);
          // bytes 0, 1: row g, columns 4t / 4t+2 (even) and 4t+1 / 4t+3 (odd);
          // bytes 2, 3: row g + 8.  Each E5M2 byte is the top byte of an f16.
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          mma_f16(d, __byte_perm(ev, 0u, 0x1404u), __byte_perm(ev, 0u, 0x3424u), __byte_perm(od, 0u, 0x1404u),
                  __byte_perm(od, 0u, 0x3424u), bh.x, bh.y);
          const float s0 = e8m0_to_f32_fast((sd4 >> (16 * hf)) & 0xffu) * hw;
          const float s1 = e8m0_to_f32_fast((sd4 >> (16 * hf + 8)) & 0xffu) * hw;
          yacc[jg][2 * hf] = fmaf(d[0] + d[1], s0, yacc[jg][2 * hf]);
          yacc[jg][2 * hf + 1] = fmaf(d[2] + d[3], s1, yacc[jg][2 * hf + 1]);
        }
      }
    }
    __syncthreads();  // the stage, the partial sums and h are free for the next item
  };

  // ---- routing: every CTA takes the same top-k of each token ----
  auto route = [&]() {
    float* lg = reinterpret_cast<float*>(scratch);  // [M][E]
    {
      // this thread's words (at most 8: M * E <= 4096), all read at once;
      // only stale ones are read again
      constexpr int kPer = 4 * kMaxE / kThreads;
      uint64_t v[kPer];
      uint32_t stale = 0u;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kThreads;
        if (i < M * E) {
          v[u] = ld_relaxed_u64(&ws.logits[i]);
          if ((uint32_t)(v[u] >> 32) != tag) stale |= 1u << u;
        }
      }
      const uint64_t start = global_ns();
      while (stale && !poisoned()) {
        if (global_ns() - start > kWaitLimitNs) {
          fail();
          break;
        }
        __nanosleep(32);
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          if (stale >> u & 1u) {
            v[u] = ld_relaxed_u64(&ws.logits[threadIdx.x + u * kThreads]);
            if ((uint32_t)(v[u] >> 32) == tag) stale &= ~(1u << u);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kThreads;
        if (i < M * E) {
          const float x = __uint_as_float((uint32_t)v[u]);
          lg[i] = x > -FLT_MAX ? x : -FLT_MAX;  // NaN and -inf rank as -FLT_MAX
        }
      }
    }
    __syncthreads();
    // One warp per token: lane l holds experts l, l + 32, ...  The k-th best
    // of the 32 lane maxima bounds the k-th best logit from below (those are k
    // real logits), so only logits not worse than it are candidates; they are
    // ranked by counting (ids are distinct, so ranks are).
    if (warp < M) {
      const int m = warp;
      const float* lm = lg + m * E;
      VI b = pad_entry(0);
#pragma unroll 8
      for (int e = lane; e < E; e += 32)
        if (better(lm[e], e, b.v, b.i)) b = VI{lm[e], e};
      int rank = 0;
#pragma unroll
      for (int o = 0; o < 32; ++o) {
        const float ov = __shfl_sync(kFull, b.v, o);
        const int32_t oi = __shfl_sync(kFull, b.i, o);
        rank += better(ov, oi, b.v, b.i);
      }
      const uint32_t hit = __ballot_sync(kFull, rank == a.top_k - 1 && b.i < E);
      VI bound = pad_entry(0);  // none: fewer than k lanes hold an expert, every expert is a candidate
      if (hit) {
        bound.v = __shfl_sync(kFull, b.v, __ffs(hit) - 1);
        bound.i = __shfl_sync(kFull, b.i, __ffs(hit) - 1);
      }
      int nc = 0;
#pragma unroll 4
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const bool keep = e < E && !better(bound.v, bound.i, lm[e], e);
        const uint32_t bal = __ballot_sync(kFull, keep);
        const int pos = nc + __popc(bal & ((1u << lane) - 1u));
        if (keep && pos < kCandCap) C.cand[m][pos] = (uint16_t)e;  // never more: k lanes' experts at most
        nc += __popc(bal);
      }
      __syncwarp();
      nc = min(nc, kCandCap);
      for (int q = lane; q < nc; q += 32) {
        const int e = C.cand[m][q];
        const float v = lm[e];
        int r = 0;
#pragma unroll 8
        for (int o = 0; o < nc; ++o) {
          const int f = C.cand[m][o];
          r += better(lm[f], f, v, e);
        }
        if (r < a.top_k) {
          C.ids[m][r] = e;
          C.topv[m][r] = v;
        }
      }
      __syncwarp();
      // softmax over the selected k, renormalised
      const float v0 = C.topv[m][0];
      const float ex = lane < a.top_k ? expf(C.topv[m][lane] - v0) : 0.f;
      float z = ex;
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
      if (lane < a.top_k) C.wts[m][lane] = ex / z;
    }
    __syncthreads();
    if (warp == 0) {
      // Slot table: slot 0 is the shared expert, then one slot per distinct
      // routed expert in order of first appearance over (token, rank).
      // Lane l holds choice l = m * top_k + r (M * top_k <= 32).
      const int k = a.top_k, n_in = M * k;
      const bool act = lane < n_in;
      const int mm = act ? lane / k : 0, r = act ? lane - mm * k : 0;
      int32_t ex = act ? C.ids[mm][r] : -1 - lane;  // idle lanes get ids of their own
      if (act && (ex < 0 || ex >= E)) {  // cannot happen (every rank below k is filled); never index out of range
        report(hdr, MOE_ERR_DEVICE_CHECK);
        ex = 0;
      }
      const uint32_t same = __match_any_sync(kFull, ex);
      const int leader = __ffs(same) - 1;
      const uint32_t leaders = __ballot_sync(kFull, act && leader == lane);
      const int slot = 1 + __popc(leaders & ((1u << leader) - 1u));
      if (act && leader == lane) {
        C.slot_expert[slot] = ex;
        C.slot_mask[slot] = 0u;
        for (int t = 0; t < 4; ++t) C.slot_w[slot][t] = 0.f;
      }
      if (lane == 0) {
        C.slot_expert[0] = -1;
        C.slot_mask[0] = (1u << M) - 1u;
        for (int t = 0; t < 4; ++t) C.slot_w[0][t] = 1.0f;
      }
      __syncwarp();
      if (act) {
        atomicOr(&C.slot_mask[slot], 1u << mm);
        C.slot_w[slot][mm] = C.wts[mm][r];  // a token picks an expert at most once
      }
      __syncwarp();
      if (lane == 0) C.nslots = 1 + __popc(leaders);
    }
    __syncthreads();
    if (c == 0) {
      for (int i = threadIdx.x; i < M * a.top_k; i += kThreads) {
        if (a.ids_out) a.ids_out[i] = C.ids[i / a.top_k][i % a.top_k];
        if (a.w_out) a.w_out[i] = C.wts[i / a.top_k][i % a.top_k];
      }
    }
  };

  // ---- the items: the shared expert's first, routing when they are done ----
  int n_my = n_pre;
  for (int j = 0;; ++j) {
    if (j == n_pre) {
      route();
      const int n_items = C.nslots * n_sl;
      n_my = c < n_items ? (n_items - c + G - 1) / G : 0;
      top_up(n_my);
    }
    if (j >= n_my) break;
    compute(j);
    consumed = j + 1;
    top_up(n_my);
  }

  // After a wait ran out, copies may still be in flight: let them land
  // (bounded) before this CTA can exit.
  if (threadIdx.x == 0 && poisoned())
    for (int j = issued > NS ? issued - NS : 0; j < issued; ++j) mbar_wait(&C.full[j % NS], (uint32_t)((j / NS) & 1));

  // ---- this CTA's partial outputs; one grid barrier; the fixed-order sum ----
  const int n_items = C.nslots * n_sl;
  const int P = n_items < G ? n_items : G;  // CTAs that hold items
  if (c < P) {
#pragma unroll
    for (int jg = 0; jg < kB; ++jg) {
      const int Gi = warp + kWarps * jg;
      if (Gi < nb) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
          if (tq < M) __stcg(&ws.partials[((size_t)c * 4 + tq) * H + 32 * Gi + 8 * r + g], yacc[jg][r]);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t old = grid_arrive(&hdr->barrier, c, G);
    if (!poisoned() && !grid_wait(&hdr->barrier, old)) fail();
    if (c == 0) hdr->epoch = tag;  // every CTA of this call has read the epoch
  }
  __syncthreads();
  {
    const int n4 = M * H / 4;
    const int o0 = (int)((int64_t)n4 * c / G), o1 = (int)((int64_t)n4 * (c + 1) / G);
    for (int o = o0 + warp; o < o1; o += kWarps) {  // one warp per 4 outputs
      const int m = (4 * o) / H, row = 4 * o - m * H;
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int p0 = 0; p0 < P; p0 += 32 * 8) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int p = p0 + lane + 32 * i;
          v[i] = p < P ? __ldcg(reinterpret_cast<const float4*>(&ws.partials[((size_t)p * 4 + m) * H + row]))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s.x += v[i].x;
          s.y += v[i].y;
          s.z += v[i].z;
          s.w += v[i].w;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        s.x += __shfl_xor_sync(kFull, s.x, off);
        s.y += __shfl_xor_sync(kFull, s.y, off);
        s.z += __shfl_xor_sync(kFull, s.z, off);
        s.w += __shfl_xor_sync(kFull, s.w, off);
      }
      if (lane == 0) *reinterpret_cast<float4*>(&a.out[(size_t)m * H + row]) = s;
    }
  }
}

int moe_stages(int H) {
  const Geo geo(H, 32);
  const int avail = kMaxDynamicSmem - kCtlBytes - scratch_bytes(H);
  int n = avail / geo.stage_bytes;
  return n > kMaxStages ? kMaxStages : n;
}

template <int kB>
cudaError_t launch_layer_t(const LayerArgs& a, cudaStream_t st) {
  cudaError_t e = ensure_smem_optin<moe_layer_kernel<kB>>();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = current_device_sms(&dev, &sms)) != cudaSuccess) return e;
  const Geo geo(a.H, a.I);
  const int grid = sms < MoeWs::kMaxGrid ? sms : MoeWs::kMaxGrid;  // one CTA per SM, all resident
  const size_t smem = (size_t)kCtlBytes + scratch_bytes(a.H) + (size_t)a.stages * geo.stage_bytes;
  e = launch_dependent(moe_layer_kernel<kB>, dim3(grid), dim3(kThreads), smem, st, true, a);
  return e;
}

}  // namespace

bool moe_layer_supported(int H, int I) {
  return H >= 32 && H % 32 == 0 && H <= kMaxBlocksPerWarp * kWarps * 32 && I >= 32 && I % 32 == 0 &&
         I <= 65536 && moe_stages(H) >= 1;
}

cudaError_t launch_moe_layer(const MoeArgs& m, cudaStream_t st) {
  LayerArgs a{m.x, m.router_w, m.router_bias, m.bank, m.shared, m.M, m.top_k, m.E, m.H, m.I,
              moe_stages(m.H), m.out, m.ids_out, m.w_out, m.ws};
  const int need = (m.H / 32 + kWarps - 1) / kWarps;  // K blocks (= output groups) per warp
  if (need <= 1) return launch_layer_t<1>(a, st);
  if (need <= 2) return launch_layer_t<2>(a, st);
  if (need <= 3) return launch_layer_t<3>(a, st);
  if (need <= 4) return launch_layer_t<4>(a, st);
  if (need <= 5) return launch_layer_t<5>(a, st);
  if (need <= 6) return launch_layer_t<6>(a, st);
  return launch_layer_t<kMaxBlocksPerWarp>(a, st);
}

}  // namespace moe
