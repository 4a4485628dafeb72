// moe_fused.cu -- the whole MoE layer (router GEMV, top-k softmax routing,
// MXFP4 gate/up GEMV + SiLU gate, down GEMV, shared expert, weighted
// combine) as one persistent kernel, for M <= 4 tokens.
//
// The pages: each token goes to 8 of 512 routed experts plus a shared expert
// that always runs (saipien.org essay, "Why one user waits on weights"); the
// expert layer is narrow, intermediate 768 (same essay, "Kernels built for the
// shape you actually have"); verifying 4 positions wakes up to 32 routed
// experts (same essay, "Draft three tokens, verify four").  At batch 1 the
// layer is bound by weight reads, so the kernel is organised around keeping
// HBM busy from the first microsecond:
//
//  * One CTA per SM (cooperative launch: all CTAs are resident, which the
//    grid barrier and the readiness counters below rely on).  A producer warp
//    streams every weight tile the CTA will need into a ring of shared-memory
//    stages with bulk copies (cp.async.bulk, no multicast); eight consumer
//    warps compute.
//  * Phase 0: each CTA scores its share of the router rows (fp32 weights,
//    bf16 activations, fp32 sums) and arrives at a split grid barrier.  The
//    shared expert needs no routing, so its tiles are loaded and computed
//    while the barrier completes.
//  * Phase 1: every CTA takes the same top-k from the logits and builds the
//    same slot table (slot 0 = shared expert, then the distinct routed
//    experts in first-appearance order), so each distinct expert is streamed
//    once however many tokens chose it.  Items of 8 gate rows + 8 up rows of
//    one slot form one 16-row MMA tile; h = silu(g) * u is written in fp32 and
//    a per-slot counter is bumped.
//  * Phase 2: items of 32 output rows of one slot's down matrix wait on that
//    slot's counter (bounded), then multiply by h.  The last CTA to finish a
//    32-row tile sums the slot partials in slot order: no float atomics, the
//    result is reproducible run to run.
//
// Arithmetic: mma.sync m16n8k16 f16 x f16 -> fp32.  E2M1 codes widen to f16
// exactly (cvt.rn.f16x2.e2m1x2).  bf16 activations become f16 exactly after a
// per-token power-of-two scale.  h (fp32) enters the down GEMV as an f16
// hi/lo pair, which carries 22 of fp32's 24 significand bits.  Each MMA
// spans one 32-element block (two k16 steps), so its fp32 result is scaled
// by that block's E8M0 scale before it joins the running fp32 sum.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "moe.h"

namespace moe {
namespace {

constexpr int kCons = 8;                   // consumer warps
constexpr int kProd = kCons;               // producer warp index
constexpr int kGuRows = 8;                 // gate rows (and up rows) per phase-1 item
constexpr int kDnRows = 32;                // output rows per phase-2 item
constexpr int kStages = 6;
constexpr int kMaxGuBlocksPerWarp = 16;    // H <= 16 * 8 * 32 = 4096
constexpr int kMaxDnBlocksPerWarp = 4;     // I <= 4 * 8 * 32 = 1024
// The x fragments of the gate/up GEMV live in registers for the whole kernel:
// the kernel is instantiated for these blocks-per-warp buckets and the
// launcher picks the smallest that fits.  The down GEMV's fragments are
// rebuilt per item and sized for the largest case.
constexpr int kGuBuckets[] = {1, 2, 4, 8, 10, 16};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Fire-and-forget atomics with release semantics: writes ordered before them
// (in this thread, or in lanes synchronised with it by __syncwarp) become
// visible to a reader that acquires the counter.
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_max(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// One round trip that both publishes this thread's (and its warp's) earlier
// writes and makes other CTAs' published writes visible.
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// f32 pair -> f16x2 (lo in the low half)
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ int pow2_sigma(float amax) {
  // sigma such that amax * 2^sigma lies in [2^14, 2^15)
  if (!(amax > 0.f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int e = (int)((b >> 23) & 0xffu);
  const int fl = e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
  int s = 14 - fl;
  return s > 126 ? 126 : (s < -126 ? -126 : s);
}

__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

struct FusedArgs {
  const uint16_t* x;
  const float* router_w;
  const float* router_bias;
  MoeBank bank, shared;
  int M, top_k, E, H, I;
  float* out;
  int32_t* ids_out;
  float* w_out;
  MoeWs ws;
};

// Shared-memory layout of one ring stage.  Phase-1 item: 16 data rows
// (8 gate, then 8 up) at a padded stride, then the 8 gate and 8 up scale rows.
// Phase-2 item: 32 down data rows at a padded stride, then their 32 scale rows.
// Strides are 16 * odd bytes, so the 8 rows a quarter of a warp reads from
// land on distinct banks.
struct Geometry {
  int H, I, nbH, nbI;   // blocks of 32 along H and along I
  int gu_stride;        // H/2 + 16
  int dn_stride;        // I/2 + 16
  int gu_bytes, dn_bytes, stage_bytes;
  int n_chunks;         // I / 8 phase-1 items per slot
  int n_tiles;          // H / 32 phase-2 items per slot
  __host__ __device__ Geometry(int H_, int I_) : H(H_), I(I_) {
    nbH = H / 32;
    nbI = I / 32;
    gu_stride = H / 2 + 16;
    dn_stride = I / 2 + 16;
    gu_bytes = 16 * gu_stride + 16 * nbH;
    dn_bytes = kDnRows * dn_stride + kDnRows * nbI;
    stage_bytes = ((gu_bytes > dn_bytes ? gu_bytes : dn_bytes) + 127) / 128 * 128;
    n_chunks = I / kGuRows;
    n_tiles = H / kDnRows;
  }
};

// Shared memory outside the ring.
constexpr int kRed = 4;                    // partial-sum buffers between consumers and the epilogue warp
constexpr int kEpi = kCons + 1;            // first epilogue warp
constexpr int kNumEpi = 2;                 // epilogue warps; item i goes to epilogue warp i % kNumEpi
constexpr int kThreadsAll = (kCons + 1 + kNumEpi) * 32;
constexpr int kRouterF4 = 16;              // float4 loads per lane per half router row: H <= 4096

struct SmemCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t red_full[kRed];
  uint64_t red_empty[kRed];
  uint64_t routed;                         // slot table ready (producer and epilogue wait on it)
  alignas(16) float red[kRed][kCons][32][8];  // per-item partials (float4 access)
  float logit_part[kCons][4];              // router: half-row partial sums
  int32_t ids[4][8];
  float wts[4][8];
  int32_t slot_expert[MoeWs::kMaxSlots];
  uint32_t slot_mask[MoeWs::kMaxSlots];
  float slot_w[MoeWs::kMaxSlots][4];
  int sigma_x[4];
  int nslots;
  int poison;
  int last;
};

__device__ __forceinline__ void consumer_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kCons * 32) : "memory");
}

// The work of one CTA, enumerated identically by the producer, the consumers
// and the epilogue warp: phase-1 items are global items c, c+G, ... of
// S * n_chunks (the first n_chunks belong to the shared expert, slot 0), then
// phase-2 items c, c+G, ... of S * n_tiles.
struct ItemIter {
  int c, G, n_chunks, n_tiles;
  __device__ int n_shared() const { return c < n_chunks ? (n_chunks - c + G - 1) / G : 0; }
  __device__ int n_phase1(int S) const { return c < S * n_chunks ? (S * n_chunks - c + G - 1) / G : 0; }
  __device__ int n_phase2(int S) const { return c < S * n_tiles ? (S * n_tiles - c + G - 1) / G : 0; }
};

template <int kGuB>
__global__ void __launch_bounds__(kThreadsAll, 1) moe_fused_kernel(FusedArgs a) {
  constexpr int kDnB = kMaxDnBlocksPerWarp;
  extern __shared__ __align__(128) uint8_t smem[];
  SmemCtl& C = *reinterpret_cast<SmemCtl*>(smem);
  uint8_t* ring = smem + ((sizeof(SmemCtl) + 127) / 128) * 128;
  const Geometry geo(a.H, a.I);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int M = a.M, H = a.H, I = a.I, E = a.E;
  const MoeWs ws = a.ws;
  const ItemIter items{c, G, geo.n_chunks, geo.n_tiles};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], kCons);
    }
    for (int r = 0; r < kRed; ++r) {
      mbar_init(&C.red_full[r], kCons);
      mbar_init(&C.red_empty[r], 1);
    }
    mbar_init(&C.routed, 1);
    fence_mbar_init();
    C.poison = 0;
  }
  if (warp < M) {
    float amax = 0.f;
    for (int j = lane; j < H; j += 32) amax = fmaxf(amax, fabsf(bf16_bits_to_f32(a.x[(size_t)warp * H + j])));
    amax = warp_max(amax);
    if (lane == 0) C.sigma_x[warp] = pow2_sigma(amax);
  }
  __syncthreads();

  auto bounded_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    bool ok = !*(volatile int*)&C.poison;
    if (ok && lane == 0) ok = mbar_wait(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0 && !*(volatile int*)&C.poison) {
      report(ws.hdr, MOE_ERR_TIMEOUT);
      atomicExch(&C.poison, 1);
    }
    return ok;
  };

  if (warp == kProd) {
    // ============================== producer ==============================
    const uint64_t policy = l2_evict_first_policy();
    int it = 0, issued = 0;
    auto issue = [&](int s_slot, bool phase1, int row0) {
      const int st = it % kStages;
      const uint32_t ph = (uint32_t)((it / kStages) & 1);
      bool ok = true;
      if (it >= kStages) ok = bounded_wait(&C.empty[st], ph ^ 1u);
      if (ok && !*(volatile int*)&C.poison) {
        uint8_t* dst = ring + (size_t)st * geo.stage_bytes;
        const int ex = s_slot == 0 ? -1 : C.slot_expert[s_slot];
        const MoeBank& b = ex < 0 ? a.shared : a.bank;
        const size_t e = ex < 0 ? 0 : (size_t)ex;
        if (phase1) {
          const size_t mat_d = (size_t)I * H / 2, mat_s = (size_t)I * geo.nbH;
          const uint32_t rowb = (uint32_t)(H / 2), scb = (uint32_t)(kGuRows * geo.nbH);
          if (lane == 0) mbar_arrive_expect_tx(&C.full[st], 16u * rowb + 2u * scb);
          __syncwarp();
          if (lane < 16) {
            const uint8_t* src = (lane < 8 ? b.gate_d : b.up_d) + e * mat_d + (size_t)(row0 + (lane & 7)) * rowb;
            bulk_g2s(dst + lane * geo.gu_stride, src, rowb, &C.full[st], policy);
          } else if (lane < 18) {
            const uint8_t* src = (lane == 16 ? b.gate_s : b.up_s) + e * mat_s + (size_t)row0 * geo.nbH;
            bulk_g2s(dst + 16 * geo.gu_stride + (lane - 16) * scb, src, scb, &C.full[st], policy);
          }
        } else {
          const size_t mat_d = (size_t)H * I / 2, mat_s = (size_t)H * geo.nbI;
          const uint32_t rowb = (uint32_t)(I / 2), scb = (uint32_t)(kDnRows * geo.nbI);
          if (lane == 0) mbar_arrive_expect_tx(&C.full[st], kDnRows * rowb + scb);
          __syncwarp();
          bulk_g2s(dst + lane * geo.dn_stride, b.down_d + e * mat_d + (size_t)(row0 + lane) * rowb, rowb,
                   &C.full[st], policy);
          if (lane == 0)
            bulk_g2s(dst + kDnRows * geo.dn_stride, b.down_s + e * mat_s + (size_t)row0 * geo.nbI, scb,
                     &C.full[st], policy);
        }
        issued = it + 1;
      }
      ++it;
    };
    // the shared expert's items come first: they are known before routing
    const int ns = items.n_shared();
    int n1 = ns, n2 = 0;
    for (int j = 0;; ++j) {
      if (j == ns) {
        const int S = bounded_wait(&C.routed, 0) ? *(volatile int*)&C.nslots : 0;
        n1 = items.n_phase1(S);
        n2 = items.n_phase2(S);
      }
      if (j >= n1) break;
      const int q = c + j * G;
      issue(q / geo.n_chunks, true, (q % geo.n_chunks) * kGuRows);
    }
    for (int j = 0; j < n2; ++j) {
      const int q = c + j * G;
      issue(q / geo.n_tiles, false, (q % geo.n_tiles) * kDnRows);
    }
    // every issued copy must land before this CTA may exit
    if (lane == 0) {
      const int first = issued > kStages ? issued - kStages : 0;
      for (int k2 = first; k2 < issued; ++k2) mbar_wait(&C.full[k2 % kStages], (uint32_t)((k2 / kStages) & 1));
    }
  } else if (warp >= kEpi) {
    // ============================== epilogue ==============================
    // Owns everything that leaves the CTA: h and its max, the readiness
    // counters, the partial outputs, the tile tickets and the combine.  Items
    // alternate between the epilogue warps so that one item's memory round
    // trips overlap the next item's.
    const int ew = warp - kEpi;
    const int g = lane >> 2, tq = lane & 3;
    int idx = 0;  // item index, counted by every epilogue warp
    auto take = [&]() -> bool {
      return bounded_wait(&C.red_full[idx % kRed], (uint32_t)((idx / kRed) & 1));
    };
    auto give = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.red_empty[idx % kRed]);
    };
    auto gateup_out = [&](int slot, int row0) {
      const bool ok = take();
      const float* rb = &C.red[idx % kRed][0][0][0];
      float gs[2] = {0.f, 0.f}, us[2] = {0.f, 0.f};
#pragma unroll
      for (int w2 = 0; w2 < kCons; ++w2) {
        const float4 p = *reinterpret_cast<const float4*>(rb + (w2 * 32 + lane) * 8);
        gs[0] += p.x; gs[1] += p.y; us[0] += p.z; us[1] += p.w;
      }
      give();
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int m = 2 * tq + q;
        float hv = 0.f;
        if (ok && tq < 2 && m < M && (mask >> m & 1u)) {
          const float inv = exp2i(-C.sigma_x[m]);
          const float gg = gs[q] * inv, uu = us[q] * inv;
          hv = gg / (1.0f + expf(-gg)) * uu;
          ws.h[((size_t)slot * 4 + m) * I + row0 + g] = hv;
        }
        float mx = fabsf(hv);  // max |h| over the 8 rows (lanes with equal tq)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (g == 0 && tq < 2 && m < M && mx > 0.f) red_max(&ws.hmax[slot * 4 + m], __float_as_uint(mx));
      }
      __syncwarp();
      if (lane == 0) red_release_add(&ws.slot_ready[slot], (uint32_t)kGuRows);
    };
    auto down_out = [&](int slot, int row0, int S) {
      const bool ok = take();
      const float* rb = &C.red[idx % kRed][0][0][0];
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w2 = 0; w2 < kCons; ++w2) {
        const float4 p0 = *reinterpret_cast<const float4*>(rb + (w2 * 32 + lane) * 8);
        const float4 p1 = *reinterpret_cast<const float4*>(rb + (w2 * 32 + lane) * 8 + 4);
        s8[0] += p0.x; s8[1] += p0.y; s8[2] += p0.z; s8[3] += p0.w;
        s8[4] += p1.x; s8[5] += p1.y; s8[6] += p1.z; s8[7] += p1.w;
      }
      give();
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int m = 2 * tq + q;
        if (ok && tq < 2 && m < M && (mask >> m & 1u)) {
          const float inv = exp2i(-pow2_sigma(__uint_as_float(__ldcg(&ws.hmax[slot * 4 + m]))));
          float* yp = ws.ypart + ((size_t)slot * 4 + m) * H + row0;
          yp[g] = s8[q] * inv;            // row g of the first 16
          yp[g + 8] = s8[2 + q] * inv;    // row g + 8
          yp[16 + g] = s8[4 + q] * inv;   // second 16 rows
          yp[24 + g] = s8[6 + q] * inv;
        }
      }
      __syncwarp();
      // the last CTA to finish this 32-row tile combines the slots in order
      const int tile = row0 / kDnRows;
      uint32_t tk = 0;
      if (lane == 0) tk = atom_acq_rel_add(&ws.tile_ticket[tile], 1u);
      tk = __shfl_sync(0xffffffffu, tk, 0);
      __syncwarp();
      if (tk == (uint32_t)(S - 1)) {
        const int row = row0 + lane;
        for (int m = 0; m < M; ++m) {
          float y = 0.f;
          for (int s2 = 0; s2 < S; ++s2) {
            const uint32_t mk = s2 == 0 ? 0xfu : C.slot_mask[s2];
            if (mk >> m & 1u) y = fmaf(C.slot_w[s2][m], __ldcg(&ws.ypart[((size_t)s2 * 4 + m) * H + row]), y);
          }
          a.out[(size_t)m * H + row] = y;
        }
        if (lane == 0) ws.tile_ticket[tile] = 0u;
      }
    };
    const int ns = items.n_shared();
    int S = 0, n1 = ns, n2 = 0;
    for (int j = 0;; ++j, ++idx) {
      if (j == ns) {
        S = bounded_wait(&C.routed, 0) ? *(volatile int*)&C.nslots : 0;
        n1 = items.n_phase1(S);
        n2 = items.n_phase2(S);
      }
      if (j >= n1) break;
      if (idx % kNumEpi != ew) continue;
      const int q = c + j * G;
      gateup_out(q / geo.n_chunks, (q % geo.n_chunks) * kGuRows);
    }
    for (int j = 0; j < n2; ++j, ++idx) {
      if (idx % kNumEpi != ew) continue;
      const int q = c + j * G;
      down_out(q / geo.n_tiles, (q % geo.n_tiles) * kDnRows, S);
    }
  } else {
    // ============================== consumers =============================
    const int g = lane >> 2, tq = lane & 3;
    const int cw = warp;  // consumer warp index 0..7

    // ---- phase 0: router rows of this CTA (2 warps per expert row) ----
    const int e_begin = (int)((int64_t)E * c / G), e_end = (int)((int64_t)E * (c + 1) / G);
    for (int base = e_begin; base < e_end; base += kCons / 2) {
      const int e = base + (cw >> 1), half = cw & 1;
      const int hw = H / 2;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (e < e_end) {
        const float* row = a.router_w + (size_t)e * H + half * hw;
        float4 wv[kRouterF4];
#pragma unroll
        for (int i = 0; i < kRouterF4; ++i) {  // every load of the half row in flight at once
          const int jj = lane * 4 + i * 128;
          wv[i] = jj < hw ? ld_stream_f4(row + jj) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kRouterF4; ++i) {
          const int jj = lane * 4 + i * 128;
          if (jj < hw) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              if (m < M) {
                const uint2 xv = *reinterpret_cast<const uint2*>(a.x + (size_t)m * H + half * hw + jj);
                acc[m] += wv[i].x * bf16_bits_to_f32(xv.x & 0xffffu) + wv[i].y * bf16_bits_to_f32(xv.x >> 16) +
                          wv[i].z * bf16_bits_to_f32(xv.y & 0xffffu) + wv[i].w * bf16_bits_to_f32(xv.y >> 16);
              }
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float v = warp_sum(acc[m]);
        if (lane == 0) C.logit_part[cw][m] = v;
      }
      consumer_bar_sync();
      if (threadIdx.x < (kCons / 2) * 4) {
        const int ee = base + threadIdx.x / 4, m = threadIdx.x % 4;
        if (ee < e_end && m < M) {
          float l = C.logit_part[2 * (threadIdx.x / 4)][m] + C.logit_part[2 * (threadIdx.x / 4) + 1][m];
          if (a.router_bias) l += a.router_bias[ee];
          ws.logits[(size_t)m * E + ee] = l;
        }
      }
      consumer_bar_sync();
    }
    // split grid barrier: arrive now, wait after the shared expert's items
    uint32_t bar_old = 0;
    if (threadIdx.x == 0) {
      __threadfence();
      const uint32_t inc = c == 0 ? 0x80000000u - (uint32_t)(G - 1) : 1u;
      bar_old = atomicAdd(&ws.hdr->barrier, inc);
    }

    // x as f16 B fragments for this warp's K blocks of the gate/up GEMV
    const int nbw_gu = (geo.nbH + kCons - 1) / kCons;
    const int b0_gu = cw * nbw_gu;
    uint32_t bx[kGuB][2][2];
    {
      const bool live = g < M;
      const float scl = live ? exp2i(C.sigma_x[g]) : 0.f;
#pragma unroll
      for (int bi = 0; bi < kGuB; ++bi) {
        const int blk = b0_gu + bi;
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            uint32_t v = 0u;
            if (live && bi < nbw_gu && blk < geo.nbH) {
              const int k0 = blk * 32 + tq * 8 + mm * 4 + p * 2;
              const uint32_t pair = *reinterpret_cast<const uint32_t*>(a.x + (size_t)g * H + k0);
              v = pack_h2(bf16_bits_to_f32(pair & 0xffffu) * scl, bf16_bits_to_f32(pair >> 16) * scl);
            }
            bx[bi][mm][p] = v;
          }
        }
      }
    }

    int it = 0;     // ring position
    int nitem = 0;  // items handed to the epilogue warp
    auto hand_off = [&](const float (&v)[8]) {
      const int r = nitem % kRed;
      if (nitem >= kRed) bounded_wait(&C.red_empty[r], (uint32_t)(((nitem / kRed) & 1) ^ 1));
      float* rb = &C.red[r][0][0][0];
      *reinterpret_cast<float4*>(rb + (cw * 32 + lane) * 8) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(rb + (cw * 32 + lane) * 8 + 4) = make_float4(v[4], v[5], v[6], v[7]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.red_full[r]);
      ++nitem;
    };

    // ---- phase-1 item: partial gate/up sums for 8 rows of one slot ----
    auto gateup_item = [&]() {
      const int st = it % kStages;
      const bool ok = bounded_wait(&C.full[st], (uint32_t)((it / kStages) & 1));
      const uint8_t* base = ring + (size_t)st * geo.stage_bytes;
      const uint8_t* gsc = base + 16 * geo.gu_stride;
      const uint8_t* usc = gsc + kGuRows * geo.nbH;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
#pragma unroll
        for (int bi = 0; bi < kGuB; ++bi) {
          const int blk = b0_gu + bi;
          if (bi < nbw_gu && blk < geo.nbH) {
            const uint32_t ga = lds32(base + g * geo.gu_stride + blk * 16 + tq * 4);
            const uint32_t ua = lds32(base + (8 + g) * geo.gu_stride + blk * 16 + tq * 4);
            const float sg = e8m0_to_f32(gsc[g * geo.nbH + blk]);
            const float su = e8m0_to_f32(usc[g * geo.nbH + blk]);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma16816(d, e2m1x2_to_f16x2(ga & 0xffu), e2m1x2_to_f16x2(ua & 0xffu), e2m1x2_to_f16x2((ga >> 8) & 0xffu),
                     e2m1x2_to_f16x2((ua >> 8) & 0xffu), bx[bi][0][0], bx[bi][0][1]);
            mma16816(d, e2m1x2_to_f16x2((ga >> 16) & 0xffu), e2m1x2_to_f16x2((ua >> 16) & 0xffu),
                     e2m1x2_to_f16x2(ga >> 24), e2m1x2_to_f16x2(ua >> 24), bx[bi][1][0], bx[bi][1][1]);
            acc[0] = fmaf(d[0], sg, acc[0]);
            acc[1] = fmaf(d[1], sg, acc[1]);
            acc[2] = fmaf(d[2], su, acc[2]);
            acc[3] = fmaf(d[3], su, acc[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[st]);
      ++it;
      hand_off(acc);
    };

    // ---- phase-2 item: partial sums of 32 output rows of one slot's down matrix ----
    const int nbw_dn = (geo.nbI + kCons - 1) / kCons;
    const int b0_dn = cw * nbw_dn;
    auto down_item = [&](int slot) {
      // wait until every row of h for this slot is written (bounded)
      bool ok = !*(volatile int*)&C.poison;
      if (ok && lane == 0) ok = bounded_spin([&] { return ld_acquire(&ws.slot_ready[slot]) >= (uint32_t)I; });
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();  // orders lane 0's acquire before the other lanes' reads of h
      if (!ok && lane == 0 && !*(volatile int*)&C.poison) {
        report(ws.hdr, MOE_ERR_TIMEOUT);
        atomicExch(&C.poison, 1);
      }
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
      // B fragments: h of token g as an f16 hi/lo pair, scaled by 2^sigma
      uint32_t bh[kDnB][2][2], bl[kDnB][2][2];
      {
        const bool live = ok && g < M && (mask >> g & 1u);
        const float hm = live ? __uint_as_float(__ldcg(&ws.hmax[slot * 4 + g])) : 0.f;
        const float scl = live ? exp2i(pow2_sigma(hm)) : 0.f;
        float v[kDnB][8];
#pragma unroll
        for (int bi = 0; bi < kDnB; ++bi) {  // all loads first
          const int blk = b0_dn + bi;
          if (live && bi < nbw_dn && blk < geo.nbI) {
            const float* hp = ws.h + ((size_t)slot * 4 + g) * I + blk * 32 + tq * 8;
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(hp));
            const float4 v1 = __ldcg(reinterpret_cast<const float4*>(hp + 4));
            v[bi][0] = v0.x; v[bi][1] = v0.y; v[bi][2] = v0.z; v[bi][3] = v0.w;
            v[bi][4] = v1.x; v[bi][5] = v1.y; v[bi][6] = v1.z; v[bi][7] = v1.w;
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[bi][q] = 0.f;
          }
        }
#pragma unroll
        for (int bi = 0; bi < kDnB; ++bi) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float x0 = v[bi][2 * q] * scl, x1 = v[bi][2 * q + 1] * scl;
            const __half2 hi = __floats2half2_rn(x0, x1);
            const float2 hf = __half22float2(hi);
            bh[bi][q >> 1][q & 1] = *reinterpret_cast<const uint32_t*>(&hi);
            bl[bi][q >> 1][q & 1] = pack_h2(x0 - hf.x, x1 - hf.y);
          }
        }
      }
      const int st = it % kStages;
      ok = bounded_wait(&C.full[st], (uint32_t)((it / kStages) & 1)) && ok;
      const uint8_t* base = ring + (size_t)st * geo.stage_bytes;
      const uint8_t* dsc = base + kDnRows * geo.dn_stride;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
          for (int bi = 0; bi < kDnB; ++bi) {
            const int blk = b0_dn + bi;
            if (bi < nbw_dn && blk < geo.nbI) {
              const int r_lo = 16 * tt + g, r_hi = r_lo + 8;
              const uint32_t wa = lds32(base + r_lo * geo.dn_stride + blk * 16 + tq * 4);
              const uint32_t wb = lds32(base + r_hi * geo.dn_stride + blk * 16 + tq * 4);
              const float sa = e8m0_to_f32(dsc[r_lo * geo.nbI + blk]);
              const float sb = e8m0_to_f32(dsc[r_hi * geo.nbI + blk]);
              const uint32_t a00 = e2m1x2_to_f16x2(wa & 0xffu), a01 = e2m1x2_to_f16x2(wb & 0xffu);
              const uint32_t a02 = e2m1x2_to_f16x2((wa >> 8) & 0xffu), a03 = e2m1x2_to_f16x2((wb >> 8) & 0xffu);
              const uint32_t a10 = e2m1x2_to_f16x2((wa >> 16) & 0xffu), a11 = e2m1x2_to_f16x2((wb >> 16) & 0xffu);
              const uint32_t a12 = e2m1x2_to_f16x2(wa >> 24), a13 = e2m1x2_to_f16x2(wb >> 24);
              float d[4] = {0.f, 0.f, 0.f, 0.f};
              mma16816(d, a00, a01, a02, a03, bh[bi][0][0], bh[bi][0][1]);
              mma16816(d, a00, a01, a02, a03, bl[bi][0][0], bl[bi][0][1]);
              mma16816(d, a10, a11, a12, a13, bh[bi][1][0], bh[bi][1][1]);
              mma16816(d, a10, a11, a12, a13, bl[bi][1][0], bl[bi][1][1]);
              acc[4 * tt + 0] = fmaf(d[0], sa, acc[4 * tt + 0]);
              acc[4 * tt + 1] = fmaf(d[1], sa, acc[4 * tt + 1]);
              acc[4 * tt + 2] = fmaf(d[2], sb, acc[4 * tt + 2]);
              acc[4 * tt + 3] = fmaf(d[3], sb, acc[4 * tt + 3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[st]);
      ++it;
      hand_off(acc);
    };

    // ---- phase 1: the shared expert's items (no routing needed), then,
    //      once every CTA's logits are in, routing and the routed items ----
    const int ns = items.n_shared();
    int S = 0, n1 = ns, n2 = 0;
    for (int j = 0;; ++j) {
      if (j == ns) {
        // ---- wait for every CTA's logits (bounded), then route ----
        if (threadIdx.x == 0 && !*(volatile int*)&C.poison) {
          const bool ok = bounded_spin([&] { return ((ld_acquire(&ws.hdr->barrier) ^ bar_old) & 0x80000000u) != 0u; });
          if (!ok) {
            report(ws.hdr, MOE_ERR_TIMEOUT);
            atomicExch(&C.poison, 1);
          }
        }
        consumer_bar_sync();
        if (cw < M) {
          const int m = cw;
          float lv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            lv[i] = (lane + 32 * i < E) ? __ldcg(&ws.logits[(size_t)m * E + lane + 32 * i]) : -FLT_MAX;
          uint32_t taken = 0u;
          float top[8];
          for (int r = 0; r < a.top_k; ++r) {
            float bv = -FLT_MAX;
            int32_t bi = INT32_MAX;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int e2 = lane + 32 * i;
              if (e2 < E && !(taken >> i & 1u) && better(lv[i], e2, bv, bi)) { bv = lv[i]; bi = e2; }
            }
            warp_best(bv, bi);
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            top[r] = bv;
            if (lane == 0) C.ids[m][r] = bi;
          }
          float z = 0.f;
          for (int r = 0; r < a.top_k; ++r) z += expf(top[r] - top[0]);
          if (lane == 0)
            for (int r = 0; r < a.top_k; ++r) C.wts[m][r] = expf(top[r] - top[0]) / z;
        }
        consumer_bar_sync();
        if (threadIdx.x == 0) {
          int n = 1;
          C.slot_expert[0] = -1;
          C.slot_mask[0] = 0xfu;
          for (int m = 0; m < 4; ++m) C.slot_w[0][m] = 1.0f;
          for (int m = 0; m < M; ++m) {
            for (int r = 0; r < a.top_k; ++r) {
              const int32_t ex = C.ids[m][r];
              int sl = 1;
              while (sl < n && C.slot_expert[sl] != ex) ++sl;
              if (sl == n) {
                C.slot_expert[n] = ex;
                C.slot_mask[n] = 0u;
                for (int mm = 0; mm < 4; ++mm) C.slot_w[n][mm] = 0.f;
                ++n;
              }
              C.slot_mask[sl] |= 1u << m;
              C.slot_w[sl][m] = C.wts[m][r];
            }
          }
          C.nslots = n;
          __threadfence_block();
          mbar_arrive(&C.routed);  // the producer and the epilogue warp may go on
        }
        consumer_bar_sync();
        S = C.nslots;
        if (c == 0) {
          for (int i = threadIdx.x; i < M * a.top_k; i += kCons * 32) {
            if (a.ids_out) a.ids_out[i] = C.ids[i / a.top_k][i % a.top_k];
            if (a.w_out) a.w_out[i] = C.wts[i / a.top_k][i % a.top_k];
          }
        }

        n1 = items.n_phase1(S);
        n2 = items.n_phase2(S);
      }
      if (j >= n1) break;
      gateup_item();
    }
    for (int j = 0; j < n2; ++j) down_item((c + j * G) / geo.n_tiles);
  }

  // ---- the last CTA to finish resets the per-call counters ----
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    C.last = atomicAdd(&ws.hdr->ticket, 1u) == (uint32_t)(G - 1);
  }
  __syncthreads();
  if (C.last) {
    __threadfence();
    for (int i = threadIdx.x; i < MoeWs::kMaxSlots; i += blockDim.x) ws.slot_ready[i] = 0u;
    for (int i = threadIdx.x; i < MoeWs::kMaxSlots * 4; i += blockDim.x) ws.hmax[i] = 0u;
    __syncthreads();
    if (threadIdx.x == 0) ws.hdr->ticket = 0u;
  }
}

}  // namespace

size_t moe_fused_smem_bytes(int H, int I) {
  const Geometry geo(H, I);
  return ((sizeof(SmemCtl) + 127) / 128) * 128 + (size_t)kStages * geo.stage_bytes;
}

bool moe_fused_supported(int H, int I) {
  return H % 64 == 0 && I % 64 == 0 && H / 32 <= kMaxGuBlocksPerWarp * kCons &&
         I / 32 <= kMaxDnBlocksPerWarp * kCons && moe_fused_smem_bytes(H, I) <= 232448;
}

template <int kGuB>
static cudaError_t launch_fused_t(const FusedArgs& a, size_t smem, cudaStream_t st) {
  auto kern = moe_fused_kernel<kGuB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreadsAll, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(sms);  // one CTA per SM; all resident (cooperative launch)
  cfg.blockDim = dim3(kThreadsAll);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_moe_fused(const MoeArgs& m, cudaStream_t st) {
  FusedArgs a{m.x, m.router_w, m.router_bias, m.bank, m.shared, m.M, m.top_k, m.E, m.H, m.I,
              m.out, m.ids_out, m.w_out, m.ws};
  const size_t smem = moe_fused_smem_bytes(m.H, m.I);
  const int need_gu = (m.H / 32 + kCons - 1) / kCons;
  int gub = 0;
  for (int b : kGuBuckets) if (!gub && b >= need_gu) gub = b;
  switch (gub) {
    case 1: return launch_fused_t<1>(a, smem, st);
    case 2: return launch_fused_t<2>(a, smem, st);
    case 4: return launch_fused_t<4>(a, smem, st);
    case 8: return launch_fused_t<8>(a, smem, st);
    case 10: return launch_fused_t<10>(a, smem, st);
    case 16: return launch_fused_t<16>(a, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
