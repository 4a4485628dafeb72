// moe_layer.cu -- the whole MoE layer (router GEMV, top-k softmax routing,
// MXFP4 gate/up GEMV + SiLU gate, down GEMV, shared expert, weighted
// combine) as one persistent kernel, for M <= 4 tokens.
//
// The pages: each token goes to 8 of 512 routed experts plus a shared expert
// that always runs (saipien.org essay, "Why one user waits on weights"); the
// expert layer is narrow, intermediate 768 (same essay, "Kernels built for the
// shape you actually have"); verifying 4 positions wakes up to 32 routed
// experts (same essay, "Draft three tokens, verify four").  At batch 1 the
// layer is bound by weight reads, so the kernel keeps as many weight bytes in
// flight as it can and synchronises the grid once.
//
//  * One CTA per SM (all CTAs resident; see launch_layer_t), 16 warps.
//  * Work items split every expert along its intermediate dimension: item
//    (slot, j) computes gate and up rows 16j .. 16j+15, h = silu(gate) * up
//    for those rows, and applies the matching 16 columns of the down matrix
//    to h -- split-K over the intermediate, so that the narrow 768-wide layer
//    still gives 48 items per expert and h never leaves the CTA.  Each
//    item's bytes are one contiguous unit of the sliced bank (pack.h),
//    brought into a ring of shared-memory stages by bulk copies (no
//    multicast) that complete on an mbarrier per stage.  Item q goes to CTA
//    q mod G; the shared expert's items come first, so the CTAs that own them
//    stream those bytes while routing runs.
//  * Router: the tokens are copied into shared memory at once; each CTA
//    scores its share of the router rows (fp32 weights, bf16 activations,
//    fp32 sums) and publishes each logit as one 64-bit word (epoch tag << 32
//    | value), so that readers need no barrier.  Then warps 0..7 poll the
//    words until all carry this call's tag, take the same top-k as every
//    other CTA and build the same slot table (slot 0 = shared expert, then
//    each distinct routed expert once), while warps 8..15 turn the tokens
//    into the gate/up MMA's operand.  Top-k, one warp per token: the k-th
//    best of the 32 lane maxima bounds the k-th best logit from below, and
//    the few logits not worse than that bound are ranked by counting; at
//    M = 1 the routed items are issued as soon as they are ranked.
//  * Each lane owns a fixed set of output rows and accumulates its CTA's
//    weighted contributions in registers across items.  After the last item
//    the CTAs write these partial outputs, meet at one grid barrier, and sum
//    them in a fixed order (no float atomics: the result is the same on
//    every run).
//
// Arithmetic.
//  * gate/up on the fifth-generation tensor cores: one block-scaled FP4 MMA
//    (tcgen05.mma kind::mxf4, E8M0 scale per 32 elements, fp32 accumulator in
//    TMEM) per 64-element K tile, issued by one thread.  A = the item's 32
//    gate/up rows as stored (E2M1, with the bank's own E8M0 scales), cut
//    into four K segments stacked as 128 operand rows, so that every row the
//    tensor core reads is a weight row; B = the tokens, each as eight E2M1
//    base-4 digits per 32-element block and K segment; only the diagonal
//    (segment s of A with segment s of B) of the product is read.  The
//    digits carry a bf16 value exactly when it is within 2^-8 of its block's
//    largest, and to within 2^-16 of the largest below.  The tensor core
//    applies both scales, so no instruction decodes a weight.  An MMA takes
//    about 75 cycles: an item's ten (H = 2,560) take about a quarter of the
//    time its 64 KB take to arrive at one SM's share of HBM bandwidth.
//  * h: per token and item (16 values), scaled by a power of two that puts
//    the largest magnitude in [2^14, 2^15) and carried by two f16 parts (about
//    22 significant bits) into mma.sync m16n8k16 f16 x f16 -> fp32, whose K of
//    16 is exactly the item's slice.  The down weights' E5M2 bytes (E2M1
//    codes placed by the bank's bit layout) are the top bytes of f16 values;
//    column n of B = part n & 1 of token n >> 1, so one MMA covers 16 output
//    rows of all tokens.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "moe.h"
#include "pack.h"
#include "tcgen05.cuh"

namespace moe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxBlocksPerWarp = 8;  // down: 32-row groups per warp, H <= 8 * 16 * 32 = 4096
constexpr int kMaxH = 3840;           // a multiple of 256: the K segments' padded blocks stay within kMaxBlocks
constexpr int kMaxBlocks = kMaxH / 32;
constexpr int kParts = 8;             // E2M1 digits per activation value
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemD = 0;        // the gate/up accumulator: 128 lanes x up to 128 columns
constexpr uint32_t kTmemSfa = 128;    // the item's weight scales: 4 columns per K tile
constexpr int16_t kZeroBlock = -32768;
constexpr int kMaxStages = 4;
constexpr int kMaxSlots = 4 * 8 + 1;
constexpr int kRouterChunk = 8;        // float4 router loads in flight per lane
constexpr int kRouteWarps = 8;         // warps 0..7 route while warps 8..15 build the activation digits
constexpr int kGroupThreads = 32 * kRouteWarps;
constexpr int kMaxE = 1024;
constexpr uint32_t kFull = 0xffffffffu;

// Token columns of the gate/up MMA's B operand per K segment: 8 digits of
// each of mp tokens, mp = M rounded up to 1, 2 or 4 (N = 32 mp).
__host__ __device__ constexpr int padded_tokens(int M) { return M <= 1 ? 1 : (M == 2 ? 2 : 4); }

struct Geo {
  int H, I, nb, n_sl, n_pairs, kt, a_bytes, b_bytes, unit_bytes, stage_bytes, xparts_bytes;
  __host__ __device__ Geo(int H_, int I_, int M) : H(H_), I(I_) {
    nb = H / 32;
    n_sl = I / kSliceRows;
    n_pairs = I / 32;
    kt = slice_ktiles(H);
    a_bytes = slice_a_bytes(H);
    b_bytes = slice_b_bytes(H);
    unit_bytes = slice_unit_bytes(H);
    stage_bytes = (unit_bytes + H + 127) / 128 * 128;  // the unit, then its pair's down scales
    xparts_bytes = kt * 1024 * padded_tokens(M);       // the activation digits: 32 mp rows x 64 T elements, E2M1
  }
};

constexpr int kCandCap = 256;  // routing candidates per token: at most top_k lanes' E/32 logits

struct Ctl {
  uint64_t full[kMaxStages];                 // one phase per item copied into the stage
  uint64_t xbar;                             // the tokens' copy into shared memory
  uint64_t mma_bar;                          // one phase per item's gate/up MMAs
  uint32_t tmem;                             // TMEM base address
  float router_part[kWarps][4];
  int16_t ex[4][kMaxBlocks + 1];             // per token and block: floor(log2) of the largest magnitude, or kZeroBlock
  int16_t tshift[kMaxBlocks + 1];            // per block: powers of two moved from the weights' scales to the digits'
  float gu[4][4][32];                        // gate/up of one item: [K segment][token][row R]
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
  int shifted;  // some block's t is not 0
};
constexpr int kCtlBytes = (int)((sizeof(Ctl) + 127) / 128 * 128);
// The scratch area holds, side by side, the tokens (bf16; the router and the
// activation digits read them), the digits' scale table (T x 512 B) and the
// M x E router logits (routing runs beside the digits): sized for this call,
// so that a small M leaves room for another stage.
__host__ __device__ constexpr int scratch_tokens_bytes(int H, int M) { return (M * H * 2 + 127) / 128 * 128; }
__host__ __device__ constexpr int scratch_table_bytes(int H) { return slice_ktiles(H) * 512; }
__host__ __device__ constexpr int scratch_bytes(int H, int M, int E) {
  return scratch_tokens_bytes(H, M) + scratch_table_bytes(H) + (M * E * 4 + 127) / 128 * 128;
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

// Barrier among `n` threads (whole warps) of the CTA, id 1..15.
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

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

// ---- power-of-two scaling of h ----
// sigma such that amax * 2^sigma lies in [2^7, 2^8), clamped to [-113, 140]
// so that 2^(14 - sigma) is a normal fp32 number; 140 covers every bf16
// value (the smallest is 2^-133).  0 for amax = 0 (or NaN).  h's slice uses
// sigma + 7, which puts its largest magnitude in [2^14, 2^15).
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
// floor(log2(a)) of a positive finite float (subnormals included).
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)((b >> 23) & 0xffu);
  return e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
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

// Grid barrier on one word (all CTAs are resident; see launch_layer_t).  The
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
  const Geo geo(a.H, a.I, a.M);
  uint8_t* xparts = scratch + scratch_bytes(a.H, a.M, a.E);   // the gate/up B operand: [K tile][half][32 mp rows][16 B]
  uint8_t* stages = xparts + geo.xparts_bytes;
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
    mbar_init(&C.mma_bar, 1);
    fence_mbar_init();
    C.poison = 0;
    C.shifted = 0;
  }
  if (warp == 0) tmem_alloc(&C.tmem, kTmemCols);  // one CTA per SM: all of the SM's TMEM

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
  tc_fence_before_sync();
  __syncthreads();  // the barriers are initialised, TMEM is allocated
  tc_fence_after_sync();
  // The shared expert's items (weights, which no kernel writes) go out after
  // the router rows: those are on the path to routing, these are needed
  // only after it.
  top_up(n_pre);
  const uint32_t tm = C.tmem;
  const int T = geo.kt;
  const uint32_t tm_sfb = kTmemSfa + 4u * (uint32_t)T;  // the activation digits' scales: 4 columns per K tile
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

  // ---- routing (warps 0..7): every CTA takes the same top-k of each token ----
  auto route = [&]() {
    float* lg = reinterpret_cast<float*>(scratch + scratch_tokens_bytes(H, M) + scratch_table_bytes(H));  // [M][E]
    {
      // this thread's words (at most 16: M * E <= 4096), eight loads at a
      // time; only stale ones are read again
      for (int i0 = threadIdx.x; i0 < M * E; i0 += 8 * kGroupThreads) {
        uint64_t v[8];
        uint32_t stale = 0u;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kGroupThreads;
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
          for (int u = 0; u < 8; ++u) {
            if (stale >> u & 1u) {
              v[u] = ld_relaxed_u64(&ws.logits[i0 + u * kGroupThreads]);
              if ((uint32_t)(v[u] >> 32) == tag) stale &= ~(1u << u);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kGroupThreads;
          if (i < M * E) {
            const float x = __uint_as_float((uint32_t)v[u]);
            lg[i] = x > -FLT_MAX ? x : -FLT_MAX;  // NaN and -inf rank as -FLT_MAX
          }
        }
      }
    }
    named_sync(2, kGroupThreads);
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
      // compaction, eight ballots at a time (independent loads and votes,
      // then the running count)
      int nc = 0;
      for (int e0 = 0; e0 < E; e0 += 256) {
        uint32_t bal[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + 32 * u + lane;
          bal[u] = __ballot_sync(kFull, e < E && !better(bound.v, bound.i, lm[e], e));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int pos = nc + __popc(bal[u] & ((1u << lane) - 1u));
          if (((bal[u] >> lane) & 1u) && pos < kCandCap)  // never more: k lanes' experts at most
            C.cand[m][pos] = (uint16_t)(e0 + 32 * u + lane);
          nc += __popc(bal[u]);
        }
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
      if (M == 1) {
        // one token: its k experts are the routed slots in rank order, so the
        // CTA's routed items can go out now, before the softmax and the table
        if (lane < a.top_k) C.slot_expert[1 + lane] = C.ids[0][lane];
        if (lane == 0) C.nslots = 1 + a.top_k;
        __syncwarp();
        if (threadIdx.x == 0) {
          const int n_items = C.nslots * n_sl;
          top_up(c < n_items ? (n_items - c + G - 1) / G : 0);
        }
      }
      // softmax over the selected k, renormalised
      const float v0 = C.topv[m][0];
      const float ex = lane < a.top_k ? expf(C.topv[m][lane] - v0) : 0.f;
      float z = ex;
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
      if (lane < a.top_k) C.wts[m][lane] = ex / z;
    }
    named_sync(2, kGroupThreads);
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
    named_sync(2, kGroupThreads);
    if (c == 0) {
      for (int i = threadIdx.x; i < M * a.top_k; i += kGroupThreads) {
        if (a.ids_out) a.ids_out[i] = C.ids[i / a.top_k][i % a.top_k];
        if (a.w_out) a.w_out[i] = C.wts[i / a.top_k][i % a.top_k];
      }
    }
  };

  const int mp = padded_tokens(M);
  const int lmp = mp == 1 ? 0 : (mp == 2 ? 1 : 2);
  if (warp < kRouteWarps) {
    route();
  } else {
    const int xt = threadIdx.x - kGroupThreads;  // warps 8..15
    // ---- x: eight E2M1 digits per token and 32-element block ----
    // The gate/up MMA's B operand has N = 32 mp rows: row n = 8 mp s + 8 m + p
    // holds digit p of token m over K segment s (elements 64 T s ..), K-major
    // like the weights.  For a block whose largest magnitude lies in [2^E,
    // 2^(E+1)), each value v is rounded to N = round(|v| 2^(15 - E)), an
    // integer below 2^16 (exact when v is within 2^-8 of the block's largest,
    // else off by at most 2^(E-16)), and written in base 4: digit p = bits
    // 14 - 2p, 15 - 2p of N, stored as the E2M1 code of d / 2 (codes 0..3 are
    // 0, 0.5, 1, 1.5) with v's sign, scale 2^(E - 2p).  The tensor core
    // applies the scales, so the eight digit columns of a token sum to N
    // 2^(E-15) x the weights.  The digits' E8M0 scales go to TMEM.
    // 1. E per (token, block)
    for (int u = xt; u < M * nb; u += kGroupThreads) {
      const int m = u / nb, b = u - m * nb;
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
      C.ex[m][b] = am > 0.f ? (int16_t)floor_log2(am) : kZeroBlock;
    }
    named_sync(3, kGroupThreads);
    // 2. per block, t: the product of a weight scale 2^(c - 127) and a digit
    // scale 2^(E - 2p) is taken as 2^(c - t - 127) x 2^(E - 2p + t), with t
    // chosen so that every token's digit codes E - 2p + t + 127 lie in [0,
    // 254] (0 unless the block is below about 2^-113 or above 2^127).
    for (int b = xt; b < 8 * T; b += kGroupThreads) {
      int lo = -100000, hi = 100000;
      for (int m = 0; m < M; ++m) {
        const int eb = b < nb ? C.ex[m][b] : kZeroBlock;
        if (eb != kZeroBlock) {
          lo = max(lo, -127 - (eb - 2 * (kParts - 1)));
          hi = min(hi, 127 - eb);
        }
      }
      int t = 0;
      if (t < lo) t = lo;
      if (t > hi) t = hi;  // the leading digits win if no shift fits all
      C.tshift[b] = (int16_t)t;
      if (t != 0) C.shifted = 1;
    }
    // 3. the digits: one thread per (token, block, 8 elements, 4 digits),
    // four 4-byte words; zero for padding
    for (int u = xt; u < mp * 64 * T; u += kGroupThreads) {
      const int ph = u & 1, u8 = u >> 1;
      const int m = u8 / (32 * T), rest = u8 - m * (32 * T), b = rest >> 2, q = rest & 3;
      const int sg = b / (2 * T), lb = b - sg * (2 * T), t = lb >> 1, hf = lb & 1;
      uint8_t* dst = xparts + (size_t)t * (1024 * mp) + hf * (512 * mp) + (sg * mp + m) * 128 + 64 * ph + 4 * q;
      const int eb = (m < M && b < nb) ? C.ex[m][b] : kZeroBlock;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (eb != kZeroBlock) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xs + m * H + 32 * b + 8 * q);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t pr[4] = {0u, 0u, 0u, 0u}, sgn = 0u;  // pr[i] = N_i | N_(i+4) << 16
        // 2^(15 - E) as one or two exact factors (15 - E <= 148), found once
        // per unit: a range test per element costs a branch per element
        const int kk = 15 - eb;
        const float f1 = kk > 126 ? exp2i(126) : 1.0f, f2 = exp2i(kk > 126 ? kk - 126 : kk);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t bits = (xw[i >> 1] >> (16 * (i & 1))) & 0xffffu;
          const uint32_t n = __float2uint_rn(bf16_bits_to_f32(bits & 0x7fffu) * f1 * f2);
          pr[i & 3] |= n << (16 * (i >> 2));
          sgn |= (bits >> 15) << (4 * i + 3);
        }
        const int sh0 = 14 - 8 * ph;  // digit 4 ph: bits sh0, sh0 + 1
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          uint32_t v = sgn;
#pragma unroll
          for (int i = 0; i < 4; ++i) v |= ((pr[i] >> (sh0 - 2 * p)) & 0x00030003u) << (4 * i);
          w[p] = v;
        }
      }
#pragma unroll
      for (int p = 0; p < 4; ++p) *reinterpret_cast<uint32_t*>(dst + 16 * p) = w[p];
    }
    fence_proxy_async_smem();  // the tensor core reads these through the async proxy
    named_sync(3, kGroupThreads);  // every block's t is written
    // 4. the digits' scales: K tile t, operand row n = 32 q + lane in column q
    // of the tile's group, in every lane quarter; bytes 0, 1 = the two halves;
    // 127 where the digit is zero.  These warps fill a table [T][4][32] in the
    // scratch area, then warps 8..11 copy it into lane quarters 0..3.
    uint32_t* sfbt = reinterpret_cast<uint32_t*>(scratch + scratch_tokens_bytes(H, M));
    for (int e = xt; e < 128 * T; e += kGroupThreads) {
      const int t = e >> 7, q = (e >> 5) & 3, n = e & 127;
      const int sg = n >> (3 + lmp), m = (n >> 3) & (mp - 1), p = n & 7;
      uint32_t w = 0u;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int b = 2 * T * sg + 2 * t + hf;
        const int eb = (q < mp && m < M && b < nb) ? C.ex[m][b] : kZeroBlock;
        int code = 127;
        if (eb != kZeroBlock) code = min(max(eb - 2 * p + C.tshift[b] + 127, 0), 254);
        w |= (uint32_t)code << (8 * hf);
      }
      sfbt[e] = w;
    }
    named_sync(3, kGroupThreads);
    if (warp < kRouteWarps + 4) {
      for (int t0 = 0; t0 < T; t0 += 8) {
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = t0 + (i >> 2) < T ? sfbt[(t0 * 4 + i) * 32 + lane] : 0u;
        const uint32_t ta = tm + ((uint32_t)(32 * (warp & 3)) << 16) + tm_sfb + 4u * t0;
        if (T - t0 >= 8) {
          tmem_st_x32(ta, v);
        } else {
#pragma unroll
          for (int tt = 0; tt < 7; ++tt)
            if (tt < T - t0) tmem_st_x4(ta + 4u * tt, v[4 * tt], v[4 * tt + 1], v[4 * tt + 2], v[4 * tt + 3]);
        }
      }
      tmem_wait_st();
    }

  }
  tc_fence_before_sync();
  __syncthreads();  // routed, and the digits are built; the tokens' shared memory is free from here on
  tc_fence_after_sync();
  const bool shifted = C.shifted != 0;

  // ---- one work item: gate/up over H, SiLU gate, down over its 16 columns ----
  float yacc[kB][4];
#pragma unroll
  for (int jg = 0; jg < kB; ++jg) yacc[jg][0] = yacc[jg][1] = yacc[jg][2] = yacc[jg][3] = 0.f;
  int n_done = 0;  // items computed: the phase of the MMA barrier
  auto compute = [&](int j) {
    const int s = j % NS;
    const int slot = (c + G * j) / n_sl;
    if (!poisoned() && !mbar_wait(&C.full[s], (uint32_t)((j / NS) & 1))) fail();
    const uint8_t* st = stages + (size_t)s * geo.stage_bytes;
    const uint32_t all = (1u << M) - 1u;
    const uint32_t mask = slot == 0 ? all : C.slot_mask[slot];
    // gate/up on the tensor core.  The item's weight scales go to TMEM
    // (warps 0..3, each its lane quarter; operand row 32 s + R in lane R,
    // column s of the K tile's group), shifted by the blocks' t; then one
    // thread issues one block-scaled MMA per K tile: D[32 s + R][n] = gate/up
    // row R over K segment s times B row n, summed over the segment's tiles.
    // Only the 8 mp columns of segment s are wanted from lanes 32 s ..
    {
      // warp w writes lane quarter w % 4 for K tiles w / 4, w / 4 + 4, ...;
      // both tiles' values are loaded before either store (a TMEM store
      // between shared-memory loads costs hundreds of cycles)
      const uint2* sb = reinterpret_cast<const uint2*>(st + geo.a_bytes);  // [T][32 rows][4 segments][2 halves]
      const uint32_t tq = tm + ((uint32_t)(32 * (warp & 3)) << 16) + kTmemSfa;
      for (int t0 = warp >> 2; t0 < T; t0 += 8) {
        const bool two = t0 + 4 < T;
        const uint2 c0 = sb[t0 * 32 + lane];
        const uint2 c1 = two ? sb[(t0 + 4) * 32 + lane] : make_uint2(0u, 0u);
        uint32_t v[8] = {c0.x & 0xffffu, c0.x >> 16, c0.y & 0xffffu, c0.y >> 16,
                         c1.x & 0xffffu, c1.x >> 16, c1.y & 0xffffu, c1.y >> 16};
        if (shifted) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int t = t0 + 4 * (i >> 2), sg = i & 3;
            uint32_t w = 0u;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int cc = (int)((v[i] >> (8 * hf)) & 0xffu);
              const int cs = (cc == 255 || t >= T) ? cc : min(max(cc - C.tshift[2 * T * sg + 2 * t + hf], 0), 254);
              w |= (uint32_t)cs << (8 * hf);
            }
            v[i] = w;
          }
        }
        tmem_st_x4(tq + 4u * t0, v[0], v[1], v[2], v[3]);
        if (two) tmem_st_x4(tq + 4u * (t0 + 4), v[4], v[5], v[6], v[7]);
      }
      tmem_wait_st();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after_sync();
      const uint32_t bt = 1024u * (uint32_t)mp, idesc = mxf4_idesc(32u * (uint32_t)mp);
      // tile t's descriptors are tile 0's plus t times the tile size in
      // 16-byte units (the start-address field; no carry: shared memory is
      // below 256 KB)
      uint64_t ad = umma_desc_kmajor(smem_addr(st), 2048u, 128u);
      uint64_t bd = umma_desc_kmajor(smem_addr(xparts), bt >> 1, 128u);
      uint32_t sfa = tm + kTmemSfa, sfb = tm + tm_sfb;
      mma_mxf4(tm + kTmemD, ad, bd, idesc, sfa, sfb, false);
      for (int t = 1; t < T; ++t) {
        ad += 4096u >> 4;
        bd += bt >> 4;
        sfa += 4u;
        sfb += 4u;
        mma_mxf4(tm + kTmemD, ad, bd, idesc, sfa, sfb, true);
      }
      mma_commit(&C.mma_bar);
    }
    // h from the accumulator: warp s < 4 adds the digit columns of segment s
    // for each token (lane R = gate/up row R); warp m < M then sums the four
    // segments of token m, h = silu(gate) * up, the slice's power of two and
    // its two f16 parts
    if (warp < 4) {
      if (!poisoned() && !mbar_wait(&C.mma_bar, (uint32_t)(n_done & 1))) fail();
      tc_fence_after_sync();
      uint32_t d[32];
      const uint32_t ta = tm + ((uint32_t)(32 * warp) << 16) + kTmemD + 8u * (uint32_t)(mp * warp);
      if (mp == 1) tmem_ld_x8(ta, d);
      else if (mp == 2) tmem_ld_x16(ta, d);
      else tmem_ld_x32(ta, d);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        if (m < mp) {
          float gv = 0.f;
#pragma unroll
          for (int p = 0; p < kParts; ++p) gv += __uint_as_float(d[8 * m + p]);
          C.gu[warp][m][lane] = gv;
        }
      }
      tc_fence_before_sync();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // warps 0..3: the segments' sums are in shared memory
      if (warp < M) {
        const int m = warp, r = lane & 15;
        const float gv = (C.gu[0][m][lane] + C.gu[1][m][lane]) + (C.gu[2][m][lane] + C.gu[3][m][lane]);
        const float uv = __shfl_down_sync(kFull, gv, 16);
        const bool live = lane < 16 && ((mask >> m) & 1u);
        // silu with the fast exponential and division (relative error near 2^-21; a very negative
        // gate gives 0 where silu is below 2^-125 in magnitude)
        const float h = live ? __fdividef(gv, 1.0f + __expf(-gv)) * uv : 0.f;
        float am = fabsf(h);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(kFull, am, o));
        // sigma such that the largest |h| of the slice lies in [2^14, 2^15)
        const int sig = min(pow2_sigma(am) + 7, 140);
        const float v = scale_pow2(h, sig);
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        const int pos = ((r & 1) << 1) | ((r >> 1) & 1);  // element r = 4t + i sits at [t][0, 2, 1, 3 -> 0..3]
        if (lane < 16) {
          C.hp[m][0][r >> 2][pos] = __half_as_ushort(hi);
          C.hp[m][1][r >> 2][pos] = __half_as_ushort(lo);
        }
        if (lane == 0) C.hfw[m] = live ? (slot == 0 ? 1.0f : C.slot_w[slot][m]) * exp2i(14 - sig) : 0.f;
      }
    }
    ++n_done;
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

  // ---- the items: the shared expert's first (its copies went out at the start) ----
  const int n_all = C.nslots * n_sl;
  const int n_my = c < n_all ? (n_all - c + G - 1) / G : 0;
  top_up(n_my);
  for (int j = 0; j < n_my; ++j) {
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
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, kTmemCols);
}

int moe_stages(int H, int M, int E) {
  const Geo geo(H, 32, M);
  const int avail = kMaxDynamicSmem - kCtlBytes - scratch_bytes(H, M, E) - geo.xparts_bytes;
  int n = avail / geo.stage_bytes;
  return n > kMaxStages ? kMaxStages : n;
}

template <int kB>
cudaError_t launch_layer_t(const LayerArgs& a, cudaStream_t st) {
  cudaError_t e = ensure_smem_optin<moe_layer_kernel<kB>>();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = current_device_sms(&dev, &sms)) != cudaSuccess) return e;
  const Geo geo(a.H, a.I, a.M);
  const int grid = sms < MoeWs::kMaxGrid ? sms : MoeWs::kMaxGrid;  // one CTA per SM, all resident
  const size_t smem =
      (size_t)kCtlBytes + scratch_bytes(a.H, a.M, a.E) + geo.xparts_bytes + (size_t)a.stages * geo.stage_bytes;
  // A regular launch, not a cooperative one: a cooperative launch waits for the
  // whole previous kernel to finish (about 5 us after the LM head's last CTA),
  // while this one's CTAs take SMs as the previous kernel's CTAs leave.  All
  // G CTAs (one per SM, the shared memory allows no second) still become
  // resident: nothing launched after this kernel starts before every CTA
  // has run griddepcontrol.launch_dependents, and kernels before it finish
  // on their own.  Should another process hold SMs, the grid barrier's wait
  // is bounded and the call reports MOE_ERR_TIMEOUT instead of hanging.
  e = launch_dependent(moe_layer_kernel<kB>, dim3(grid), dim3(kThreads), smem, st, false, a);
  return e;
}

}  // namespace

bool moe_layer_supported(int H, int I) {
  return H >= 32 && H % 32 == 0 && H <= kMaxH && I >= 32 && I % 32 == 0 &&
         I <= 65536 && moe_stages(H, 4, kMaxE) >= 1;
}

cudaError_t launch_moe_layer(const MoeArgs& m, cudaStream_t st) {
  LayerArgs a{m.x, m.router_w, m.router_bias, m.bank, m.shared, m.M, m.top_k, m.E, m.H, m.I,
              moe_stages(m.H, m.M, m.E), m.out, m.ids_out, m.w_out, m.ws};
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
