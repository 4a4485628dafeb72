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
//    grid barriers below rely on).  A producer warp streams every weight unit
//    the CTA will need into a ring of shared-memory stages, one bulk copy
//    (cp.async.bulk, no multicast) per unit of the packed bank; eight
//    consumer warps compute; two epilogue warps finish each item and own
//    everything that leaves the CTA.
//  * Phase 0: each CTA scores its share of the router rows (fp32 weights,
//    bf16 activations, fp32 sums) and arrives at a split grid barrier.  The
//    shared expert needs no routing, so its tiles are loaded and computed
//    while the barrier completes.
//  * Phase 1: every CTA takes the same top-k from the logits and builds the
//    same slot table (slot 0 = shared expert, then the distinct routed
//    experts in first-appearance order), so each distinct expert is streamed
//    once however many tokens chose it.  Items of 8 gate rows + 8 up rows of
//    one slot form one 16-row MMA tile; h = silu(g) * u is written in fp32.
//  * A grid barrier publishes h.  No fence or atomic sits on the per-item
//    path: the producer streams the down tiles meanwhile.
//  * Split pass: one warp per (slot, token, 32-element block) of h scales the
//    block by a power of two and writes it as three E4M3 parts in MMA
//    fragment order -- once, instead of once per down item that reads it.
//    Another grid barrier publishes the parts.
//  * Phase 2: items of 32 output rows of one slot's down matrix multiply by h
//    and write per-slot partial outputs.  After one more grid barrier each
//    CTA sums, for the 32-row tiles it owns, the slot partials in slot order:
//    no float atomics, the result is reproducible run to run.
//
// Arithmetic: mma.sync m16n8k32 E5M2 (weights) x E4M3 (activations) -> fp32,
// one MMA per 32-element MX block and 16 weight rows, so that its fp32
// result is scaled by that block's E8M0 scale before it joins the running
// fp32 sum.  The weights need no conversion instruction: the packed bank
// places each E2M1 code's bits so that a mask (even elements) or two shifts
// (odd ones) give the E5M2 code of its value times 2^-14.  Activations are
// scaled by a per-token power of two that puts their largest magnitude in
// [2^7, 2^8); bf16 x is then carried by two E4M3 parts (exactly for scaled
// magnitudes of 2^-2 and up, within 2^-17 of the largest below), which ride in
// two columns of the same MMA.  h is scaled per 32-element block and token
// (largest magnitude into [2^7, 2^8)) and carried by three E4M3 parts (12
// significant bits) in three columns; one MMA covers two tokens.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "moe.h"
#include "pack.h"

namespace moe {
namespace {

constexpr int kCons = 16;                  // consumer warps
constexpr int kProd = kCons;               // producer warp index
constexpr int kGuRows = 8;                 // gate rows (and up rows) per phase-1 item
constexpr int kDnRows = 32;                // output rows per phase-2 item
constexpr int kStages = 6;
constexpr int kMaxGuBlocksPerWarp = 8;     // H <= 8 * 16 * 32 = 4096
constexpr int kMaxDnBlocksPerWarp = 2;     // I <= 2 * 16 * 32 = 1024
// The x fragments of the gate/up GEMV live in registers for the whole kernel:
// the kernel is instantiated for blocks-per-warp buckets (GuBuckets, at the
// launcher) and a launch picks the smallest that fits.  The down GEMV's
// fragments are rebuilt per item and sized for the largest case.
constexpr int kHParts = 3;  // E4M3 parts carrying h into the down GEMV

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int pow2_sigma(float amax) {
  // sigma such that amax * 2^sigma lies in [2^7, 2^8): the largest value sits
  // at the top of E4M3's normal range (max 448)
  if (!(amax > 0.f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int e = (int)((b >> 23) & 0xffu);
  const int fl = e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
  int s = 7 - fl;
  return s > 126 ? 126 : (s < -126 ? -126 : s);
}

__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// v rounded to 4 significant bits (E4M3's precision), to nearest even, as an
// fp32 value: integer operations only.  For |v| in E4M3's normal range
// [2^-6, 448] the result is exactly an E4M3 value.
__device__ __forceinline__ float round_sig4(float v) {
  uint32_t b = __float_as_uint(v);
  b += 0x7ffffu + ((b >> 20) & 1u);
  return __uint_as_float(b & 0xfff00000u);
}

// ---- routing: top-8 of up to 1,024 logits in one warp ----
// (value, expert) pairs under `better`: larger value first, lower id on ties.
struct VI {
  float v;
  int32_t i;
};

// Leave the better of the two in a.
__device__ __forceinline__ void cas(VI& a, VI& b) {
  const bool sw = better(b.v, b.i, a.v, a.i);
  const VI t = a;
  a = sw ? b : a;
  b = sw ? t : b;
}

// Sorting network for 8 entries, best first (19 comparators, depth 6).
__device__ __forceinline__ void sort8(VI (&a)[8]) {
  cas(a[0], a[2]); cas(a[1], a[3]); cas(a[4], a[6]); cas(a[5], a[7]);
  cas(a[0], a[4]); cas(a[1], a[5]); cas(a[2], a[6]); cas(a[3], a[7]);
  cas(a[0], a[1]); cas(a[2], a[3]); cas(a[4], a[5]); cas(a[6], a[7]);
  cas(a[2], a[4]); cas(a[3], a[5]);
  cas(a[1], a[4]); cas(a[3], a[6]);
  cas(a[1], a[2]); cas(a[3], a[4]); cas(a[5], a[6]);
}

// R (sorted) <- the best 8 of R and S (both sorted), sorted.  The pairwise
// better of R[j] and S[7 - j] is exactly that set, in bitonic order; a
// bitonic sorter of 8 (12 comparators) orders it.
__device__ __forceinline__ void merge8(VI (&R)[8], const VI (&S)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const VI o = S[7 - j];
    if (better(o.v, o.i, R[j].v, R[j].i)) R[j] = o;
  }
  cas(R[0], R[4]); cas(R[1], R[5]); cas(R[2], R[6]); cas(R[3], R[7]);
  cas(R[0], R[2]); cas(R[1], R[3]); cas(R[4], R[6]); cas(R[5], R[7]);
  cas(R[0], R[1]); cas(R[2], R[3]); cas(R[4], R[5]); cas(R[6], R[7]);
}

// The best 8 of logits[0..E) (E <= 1024, in shared memory), sorted, in every
// lane of the warp.
// Logits that are NaN or -inf count as -FLT_MAX, so that every real expert
// ranks above the padding entries (-FLT_MAX, INT32_MAX): with E >= 8 the
// result holds only experts in [0, E).  Each lane sorts its logits 8 at a time
// (read chunk by chunk, to keep few registers live) into its running best 8;
// a butterfly of merges then gives every lane the warp's best 8.
__device__ __forceinline__ void warp_top8(const float* logits, int E, int lane, VI (&R)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) R[j] = VI{-FLT_MAX, INT32_MAX};
#pragma unroll 1
  for (int ch = 0; ch * 256 < E; ++ch) {  // this lane's values lane + 32 i, i in [8 ch, 8 ch + 8)
    VI S[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * (8 * ch + j);
      const float v = e < E ? logits[e] : -FLT_MAX;
      S[j] = e < E ? VI{v > -FLT_MAX ? v : -FLT_MAX, e} : VI{-FLT_MAX, INT32_MAX};
    }
    sort8(S);
    merge8(R, S);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {  // butterfly: both partners end with the same list
    VI P[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      P[j].v = __shfl_xor_sync(0xffffffffu, R[j].v, o);
      P[j].i = __shfl_xor_sync(0xffffffffu, R[j].i, o);
    }
    merge8(R, P);
  }
}

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

// Shared-memory layout of one ring stage: one packed unit, exactly as it sits
// in HBM (see pack.h), brought by one bulk copy.  Phase-1 item: 16 data rows
// (8 gate, then 8 up) of H/2 bytes, then the 8 gate and 8 up scale rows.
// Phase-2 item: 32 down data rows of I/2 bytes, then their 32 scale rows.
// Within a data row the 16-byte units are XOR-permuted by the row index, so
// the 8 rows a quarter of a warp reads from land on distinct banks.
struct Geometry {
  int H, I, nbH, nbI;   // blocks of 32 along H and along I (= 16-byte units per data row)
  int mH, mI;           // unit swizzle masks of the gate/up and the down rows
  int gu_bytes, dn_bytes, stage_bytes;
  int n_chunks;         // I / 8 phase-1 items per slot
  int n_tiles;          // H / 32 phase-2 items per slot
  __host__ __device__ Geometry(int H_, int I_) : H(H_), I(I_) {
    nbH = H / 32;
    nbI = I / 32;
    mH = swizzle_mask(nbH);
    mI = swizzle_mask(nbI);
    gu_bytes = gateup_chunk_bytes(H);
    dn_bytes = down_tile_bytes(I);
    stage_bytes = ((gu_bytes > dn_bytes ? gu_bytes : dn_bytes) + 127) / 128 * 128;
    n_chunks = I / kGuRows;
    n_tiles = H / kDnRows;
  }
};

// Shared memory outside the ring.
constexpr int kRed = 4;                    // partial-sum buffers between consumers and the epilogue warps
constexpr int kEpi = kCons + 1;            // first epilogue warp
constexpr int kNumEpi = 2;                 // epilogue warps; item i goes to epilogue warp i % kNumEpi
constexpr int kThreadsAll = (kCons + 1 + kNumEpi) * 32;
constexpr int kRouterSplit = 4;           // consumer warps per router row
constexpr int kRouterF4 = 8;               // float4 loads per lane per quarter router row: H <= 4096

struct SmemCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t red_full[kRed];
  uint64_t red_empty[kRed];
  uint64_t routed;                         // slot table ready (producer and epilogue warps wait on it)
  uint64_t h_ready;                        // every CTA's h written (consumers wait on it)
  uint64_t parts_ready;                    // this CTA passed the split-pass barrier (epilogue waits on it)
  uint64_t partials_ready;                 // every CTA's partial outputs written (consumers wait on it)
  alignas(16) float red[kRed][kCons][32][8];  // per-item partials (float4 access)
  float logit_part[kCons][4];              // router: quarter-row partial sums
  int32_t ids[4][8];
  float wts[4][8];
  float topv[4][8];
  int32_t slot_expert[MoeWs::kMaxSlots];
  uint32_t slot_mask[MoeWs::kMaxSlots];
  float slot_w[MoeWs::kMaxSlots][4];
  int sigma_x[4];
  int nslots;
  int poison;
};

static_assert(sizeof(SmemCtl::red) >= 4 * 1024 * sizeof(float), "routing stages M x E <= 4 x 1024 logits in red");

__device__ __forceinline__ void consumer_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kCons * 32) : "memory");
}
__device__ __forceinline__ void epilogue_bar_sync() {
  asm volatile("bar.sync 2, %0;" ::"r"(kNumEpi * 32) : "memory");
}

// Grid barrier on one word (all CTAs are resident: cooperative launch).  The
// first CTA adds 2^31 - (G - 1), the others 1, so the top bit flips exactly
// when all G have arrived and the low bits return to where they were: the
// same word serves every barrier of every call.  A CTA may arrive at barrier
// n + 1 only after it has seen barrier n complete -- otherwise its early
// arrival would count toward barrier n -- which the warps that arrive for a
// CTA (consumers: router, split pass; epilogue: h, partial outputs) ensure
// with the CTA-local mbarriers h_ready and parts_ready.  Arrival publishes
// the caller's earlier writes (fence first); the wait is bounded.
__device__ __forceinline__ uint32_t grid_arrive(uint32_t* word, int c, int G) {
  __threadfence();
  return atomicAdd(word, c == 0 ? 0x80000000u - (uint32_t)(G - 1) : 1u);
}
__device__ __forceinline__ bool grid_wait(uint32_t* word, uint32_t old) {
  return bounded_spin([&] { return ((ld_acquire(word) ^ old) & 0x80000000u) != 0u; });
}

// The work of one CTA, enumerated identically by the producer, the consumers
// and the epilogue warps: phase-1 items are global items c, c+G, ... of
// S * n_chunks (the first n_chunks belong to the shared expert, slot 0, so
// that most CTAs have one to load before routing), then phase-2 items are
// the contiguous range [S n_tiles c / G, S n_tiles (c + 1) / G) of
// S * n_tiles: consecutive down tiles of the same slot, which share their
// B fragments (h of that slot).
struct ItemIter {
  int c, G, n_chunks, n_tiles;
  __device__ int n_shared() const { return c < n_chunks ? (n_chunks - c + G - 1) / G : 0; }
  __device__ int n_phase1(int S) const { return c < S * n_chunks ? (S * n_chunks - c + G - 1) / G : 0; }
  __device__ int p2_begin(int S) const { return (int)((int64_t)S * n_tiles * c / G); }
  __device__ int n_phase2(int S) const { return (int)((int64_t)S * n_tiles * (c + 1) / G) - p2_begin(S); }
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
  uint32_t* bar_word = &ws.hdr->barrier;

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
    mbar_init(&C.h_ready, 1);
    mbar_init(&C.parts_ready, 1);
    mbar_init(&C.partials_ready, 1);
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

  auto poisoned = [&]() -> bool { return *(volatile int*)&C.poison != 0; };
  auto fail = [&]() {  // the first wait of this CTA that ran out
    if (!poisoned()) {
      report(ws.hdr, MOE_ERR_TIMEOUT);
      atomicExch(&C.poison, 1);
    }
  };
  // bounded wait on an mbarrier phase: lane 0 polls, the warp agrees
  auto bounded_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    bool ok = !poisoned();
    if (ok && lane == 0) ok = mbar_wait(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0) fail();
    return ok;
  };

  if (warp == kProd) {
    // ============================== producer ==============================
    // Streams every weight tile of this CTA's items, phase 1 then phase 2:
    // no tile depends on h, so the down tiles arrive while phase 1 finishes.
    const uint64_t policy = l2_evict_first_policy();
    int it = 0, issued = 0;
    auto issue = [&](int s_slot, bool phase1, int row0) {
      const int st = it % kStages;
      const uint32_t ph = (uint32_t)((it / kStages) & 1);
      bool ok = true;
      if (it >= kStages) ok = bounded_wait(&C.empty[st], ph ^ 1u);
      if (ok && !poisoned()) {
        uint8_t* dst = ring + (size_t)st * geo.stage_bytes;
        const int ex = s_slot == 0 ? -1 : C.slot_expert[s_slot];
        const MoeBank& b = ex < 0 ? a.shared : a.bank;
        const size_t e = ex < 0 ? 0 : (size_t)ex;
        // one packed unit = one bulk copy
        const uint8_t* src = phase1 ? b.gateup + (e * geo.n_chunks + row0 / kGuRows) * (size_t)geo.gu_bytes
                                    : b.down + (e * geo.n_tiles + row0 / kDnRows) * (size_t)geo.dn_bytes;
        const uint32_t bytes = (uint32_t)(phase1 ? geo.gu_bytes : geo.dn_bytes);
        if (lane == 0) {
          mbar_arrive_expect_tx(&C.full[st], bytes);
          bulk_g2s(dst, src, bytes, &C.full[st], policy);
        }
        __syncwarp();
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
    const int q2 = n2 > 0 ? items.p2_begin(*(volatile int*)&C.nslots) : 0;
    for (int j = 0; j < n2; ++j) {
      const int q = q2 + j;
      issue(q / geo.n_tiles, false, (q % geo.n_tiles) * kDnRows);
    }
    // every issued copy must land before this CTA may exit
    if (lane == 0) {
      const int first = issued > kStages ? issued - kStages : 0;
      for (int k2 = first; k2 < issued; ++k2) mbar_wait(&C.full[k2 % kStages], (uint32_t)((k2 / kStages) & 1));
    }
  } else if (warp >= kEpi) {
    // ============================== epilogue ==============================
    // Owns everything that leaves the CTA: h, the partial outputs, the two
    // grid barriers that publish them, and the final combine.  Items
    // alternate between the epilogue warps so that one item's memory traffic
    // overlaps the next item's.  No fence or atomic sits on the per-item path.
    const int ew = warp - kEpi;
    const int g = lane >> 2, tq = lane & 3;
    int idx = 0;  // item index, counted by every epilogue warp
    auto take = [&]() -> bool { return bounded_wait(&C.red_full[idx % kRed], (uint32_t)((idx / kRed) & 1)); };
    auto give = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.red_empty[idx % kRed]);
    };
    auto gateup_out = [&](int slot, int row0) {
      const bool ok = take();
      const float* rb = &C.red[idx % kRed][0][0][0];
      float gs = 0.f, us = 0.f;  // gate row g and up row g of token tq: the two parts summed
#pragma unroll
      for (int w2 = 0; w2 < kCons; ++w2) {
        const float4 p = *reinterpret_cast<const float4*>(rb + (w2 * 32 + lane) * 8);
        gs += p.x + p.y;
        us += p.z + p.w;
      }
      give();
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
      const int m = tq;
      if (ok && m < M && (mask >> m & 1u)) {
        const float inv = exp2i(6 - C.sigma_x[m]) * 256.0f;  // undo 2^sigma and the E5M2 weights' 2^-14
        const float gg = gs * inv, uu = us * inv;
        ws.h[((size_t)slot * 4 + m) * I + row0 + g] = gg / (1.0f + expf(-gg)) * uu;
      }
    };
    auto down_out = [&](int slot, int row0) {
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
      // lanes tq and tq ^ 1 hold the parts of the same token: after the sum,
      // the even lanes hold s8[4 tt + 2 half + r] = row 16tt + 8half + g of
      // token 2r + (tq >> 1)
#pragma unroll
      for (int q = 0; q < 8; ++q) s8[q] += __shfl_xor_sync(0xffffffffu, s8[q], 1);
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
      if (ok && (tq & 1) == 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int m = 2 * r + (tq >> 1);
          if (m < M && (mask >> m & 1u)) {
            float* yp = ws.ypart + ((size_t)slot * 4 + m) * H + row0;
            yp[g] = s8[r];
            yp[8 + g] = s8[2 + r];
            yp[16 + g] = s8[4 + r];
            yp[24 + g] = s8[6 + r];
          }
        }
      }
    };
    // grid barrier of the epilogue warps: both finish their writes, one thread
    // publishes and waits, both go on
    auto epilogue_grid_barrier = [&]() {
      epilogue_bar_sync();
      if (ew == 0 && lane == 0) {
        const uint32_t old = grid_arrive(bar_word, c, G);
        if (!poisoned() && !grid_wait(bar_word, old)) fail();
      }
      epilogue_bar_sync();
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
    // h of every CTA is written: release the consumers into phase 2
    epilogue_grid_barrier();
    if (ew == 0 && lane == 0) mbar_arrive(&C.h_ready);
    // This CTA's next arrival on the grid-barrier word must follow its
    // consumers' arrival at the split-pass barrier, even when it has no
    // phase-2 items: arrivals on the word stay in barrier order.
    bounded_wait(&C.parts_ready, 0);
    const int q2 = items.p2_begin(S);
    for (int j = 0; j < n2; ++j, ++idx) {
      if (idx % kNumEpi != ew) continue;
      const int q = q2 + j;
      down_out(q / geo.n_tiles, (q % geo.n_tiles) * kDnRows);
    }
    // every slot's partial outputs are written: the consumers combine them
    epilogue_grid_barrier();
    if (ew == 0 && lane == 0) mbar_arrive(&C.partials_ready);
  } else {
    // ============================== consumers =============================
    const int g = lane >> 2, tq = lane & 3;
    const int cw = warp;  // consumer warp index 0..kCons-1

    // ---- phase 0: router rows of this CTA (4 warps per expert row) ----
    const int e_begin = (int)((int64_t)E * c / G), e_end = (int)((int64_t)E * (c + 1) / G);
    constexpr int kRowsPerRound = kCons / kRouterSplit;
    for (int base = e_begin; base < e_end; base += kRowsPerRound) {
      const int e = base + cw / kRouterSplit, part = cw % kRouterSplit;
      const int hw = H / kRouterSplit;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (e < e_end) {
        const float* row = a.router_w + (size_t)e * H + part * hw;
        float4 wv[kRouterF4];
#pragma unroll
        for (int i = 0; i < kRouterF4; ++i) {  // every load of the quarter row in flight at once
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
                const uint2 xv = *reinterpret_cast<const uint2*>(a.x + (size_t)m * H + part * hw + jj);
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
      if (threadIdx.x < kRowsPerRound * 4) {
        const int rr = threadIdx.x / 4, m = threadIdx.x % 4, ee = base + rr;
        if (ee < e_end && m < M) {
          float l = 0.f;
#pragma unroll
          for (int q = 0; q < kRouterSplit; ++q) l += C.logit_part[rr * kRouterSplit + q][m];
          if (a.router_bias) l += a.router_bias[ee];
          ws.logits[(size_t)m * E + ee] = l;
        }
      }
      consumer_bar_sync();
    }
    // split grid barrier: arrive now, wait after the shared expert's items
    uint32_t bar_old = 0;
    if (threadIdx.x == 0) bar_old = grid_arrive(bar_word, c, G);

    // x as E4M3 B fragments for this warp's K blocks of the gate/up GEMV.
    // Column n of B is part n & 1 of token n >> 1: each token, scaled by
    // 2^sigma, is carried by two E4M3 parts (hi, lo; exact for scaled
    // magnitudes of 2^-2 and up, within 2^-17 of the largest below), and the two
    // parts ride in two columns of ONE MMA (their sum is taken after it).
    // Within a 32-element block, lane (g, tq) covers elements 8tq..8tq+7 of
    // column g: the even ones fill k-slots 4tq..4tq+3 (b0), the odd ones
    // 16+4tq.. (b1), matching the even/odd split of the weight nibbles.
    uint32_t bx[kGuB][2];  // [block][b0, b1]; this warp's blocks are cw, cw + kCons, ...
    {
      const int m = g >> 1, part = g & 1;
      const bool live = m < M;
      const float scl = live ? exp2i(C.sigma_x[m]) : 0.f;
#pragma unroll
      for (int bi = 0; bi < kGuB; ++bi) {
        const int blk = cw + kCons * bi;
        uint32_t pe[2] = {0u, 0u}, po[2] = {0u, 0u};
        if (live && blk < geo.nbH) {
          const uint4 q = *reinterpret_cast<const uint4*>(a.x + (size_t)m * H + blk * 32 + tq * 8);
          const float v0 = bf16_bits_to_f32(q.x & 0xffffu) * scl, v1 = bf16_bits_to_f32(q.x >> 16) * scl;
          const float v2 = bf16_bits_to_f32(q.y & 0xffffu) * scl, v3 = bf16_bits_to_f32(q.y >> 16) * scl;
          const float v4 = bf16_bits_to_f32(q.z & 0xffffu) * scl, v5 = bf16_bits_to_f32(q.z >> 16) * scl;
          const float v6 = bf16_bits_to_f32(q.w & 0xffffu) * scl, v7 = bf16_bits_to_f32(q.w >> 16) * scl;
          split_e4m3x4<2>(v0, v2, v4, v6, pe);
          split_e4m3x4<2>(v1, v3, v5, v7, po);
        }
        bx[bi][0] = part ? pe[1] : pe[0];
        bx[bi][1] = part ? po[1] : po[0];
      }
    }
    // Shared-memory offsets of this lane's words.  Block blk = cw + kCons*bi of
    // row r sits at unit blk ^ (r & mask) = kCons*bi + (cw ^ (r & mask)) (the
    // mask is below 8 and cw below kCons), so every block is a constant stride
    // from the lane's base; rows g and 8+g share the permutation.
    const int gu_rowb = H / 2;
    const int gu_lane = g * gu_rowb + ((cw ^ (g & geo.mH)) * 16) + tq * 4;  // gate row g; up row 8+g adds 8 rows
    const int gu_scl = 16 * gu_rowb + g * geo.nbH + cw;                    // gate scale; up scale adds 8 rows
    int it = 0;     // ring position
    int nitem = 0;  // items handed to the epilogue warps
    auto hand_off = [&](const float (&v)[8], bool two) {
      const int r = nitem % kRed;
      if (nitem >= kRed) bounded_wait(&C.red_empty[r], (uint32_t)(((nitem / kRed) & 1) ^ 1));
      float* rb = &C.red[r][0][0][0];
      *reinterpret_cast<float4*>(rb + (cw * 32 + lane) * 8) = make_float4(v[0], v[1], v[2], v[3]);
      if (two) *reinterpret_cast<float4*>(rb + (cw * 32 + lane) * 8 + 4) = make_float4(v[4], v[5], v[6], v[7]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.red_full[r]);
      ++nitem;
    };

    // ---- phase-1 item: partial gate/up sums for 8 rows of one slot ----
    // All shared loads first, then one MMA per block (E5M2 weights from the
    // packed nibbles, x's two parts in two columns), then the block scales.
    auto gateup_item = [&]() {
      const int st = it % kStages;
      const bool ok = bounded_wait(&C.full[st], (uint32_t)((it / kStages) & 1));
      const uint8_t* base = ring + (size_t)st * geo.stage_bytes;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        uint32_t gw[kGuB], uw[kGuB];
#pragma unroll
        for (int bi = 0; bi < kGuB; ++bi) {
          const bool in = cw + kCons * bi < geo.nbH;
          gw[bi] = in ? lds32(base + gu_lane + 256 * bi) : 0u;
          uw[bi] = in ? lds32(base + gu_lane + 8 * gu_rowb + 256 * bi) : 0u;
        }
        float d[kGuB][4];
#pragma unroll
        for (int bi = 0; bi < kGuB; ++bi) {
          // A: gate row g (a0, a2) and up row g (a1, a3), 32 elements = one MX block
          d[bi][0] = d[bi][1] = d[bi][2] = d[bi][3] = 0.f;
          if (cw + kCons * bi < geo.nbH)
            mma_e5m2_e4m3(d[bi], packed_even_to_e5m2x4(gw[bi]), packed_even_to_e5m2x4(uw[bi]),
                          packed_odd_to_e5m2x4(gw[bi]), packed_odd_to_e5m2x4(uw[bi]), bx[bi][0], bx[bi][1]);
        }
#pragma unroll
        for (int bi = 0; bi < kGuB; ++bi) {
          if (cw + kCons * bi < geo.nbH) {
            const float sg = e8m0_to_f32_fast(base[gu_scl + kCons * bi]);
            const float su = e8m0_to_f32_fast(base[gu_scl + 8 * geo.nbH + kCons * bi]);
            acc[0] = fmaf(d[bi][0], sg, acc[0]);  // gate row g, token tq: hi part
            acc[1] = fmaf(d[bi][1], sg, acc[1]);  //                       lo part
            acc[2] = fmaf(d[bi][2], su, acc[2]);  // up row g, token tq
            acc[3] = fmaf(d[bi][3], su, acc[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[st]);
      ++it;
      hand_off(acc, false);
    };

    // ---- phase-2 item: partial sums of 32 output rows of one slot's down matrix ----
    const int dn_rowb = I / 2;
    const int dn_lane = g * dn_rowb + ((cw ^ (g & geo.mI)) * 16) + tq * 4;  // rows 16tt + g (+ 8) share it
    const int dn_scl = kDnRows * dn_rowb + g * geo.nbI + cw;
    // The B fragments of a down item: h of one slot for this warp's blocks,
    // already split into three E4M3 parts by the split pass.  MMA group r
    // covers tokens 2r and 2r+1: column n holds part n & 3 of token
    // 2r + (n >> 2) (part 3 is zero), so lane (g, tq) loads one part of one
    // token (uint2 = its even and odd 4-byte groups) and its results are the
    // parts of token 2r + (tq >> 1), whose block factor (undoing the block's
    // scale and the E5M2 weights' 2^-14) it holds in f.  Issued one item
    // ahead, so the L2 round trip overlaps the previous item.
    struct HFrag {
      uint2 q[kDnB][2];
      float f[kDnB][2];
    };
    auto load_h = [&](int slot, HFrag& hf) {
      const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
      const bool ok = !poisoned();
#pragma unroll
      for (int bi = 0; bi < kDnB; ++bi) {
        const int blk = cw + kCons * bi;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int mb = 2 * r + (g >> 2), p = g & 3, mo = 2 * r + (tq >> 1);
          const bool lb = ok && blk < geo.nbI && p < kHParts && mb < M && (mask >> mb & 1u);
          const bool lf = ok && blk < geo.nbI && mo < M && (mask >> mo & 1u);
          const size_t ub = ((size_t)slot * 4 + mb) * geo.nbI + blk, uo = ((size_t)slot * 4 + mo) * geo.nbI + blk;
          hf.q[bi][r] = lb ? __ldcg(reinterpret_cast<const uint2*>(ws.hq + (ub * kHParts + p) * 32 + tq * 8))
                           : make_uint2(0u, 0u);
          hf.f[bi][r] = lf ? __ldcg(ws.hf + uo) : 0.f;
        }
      }
    };
    auto down_item = [&](const HFrag& hf) {
      const int st = it % kStages;
      const bool ok = bounded_wait(&C.full[st], (uint32_t)((it / kStages) & 1));
      const uint8_t* base = ring + (size_t)st * geo.stage_bytes;
      // acc[4 tt + 2 half + r]: rows 16tt + 8half + g, token group r, the
      // lane's columns summed (parts of token 2r + (tq >> 1))
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        uint32_t wa[2][kDnB], wb[2][kDnB];  // rows 16tt + g and 16tt + 8 + g
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
          for (int bi = 0; bi < kDnB; ++bi) {
            const bool in = cw + kCons * bi < geo.nbI;
            const int off = dn_lane + 16 * tt * dn_rowb + 256 * bi;
            wa[tt][bi] = in ? lds32(base + off) : 0u;
            wb[tt][bi] = in ? lds32(base + off + 8 * dn_rowb) : 0u;
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (r == 1 && M <= 2) break;
          float d[2][kDnB][4];
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
            for (int bi = 0; bi < kDnB; ++bi) {
              d[tt][bi][0] = d[tt][bi][1] = d[tt][bi][2] = d[tt][bi][3] = 0.f;
              if (cw + kCons * bi < geo.nbI)
                mma_e5m2_e4m3(d[tt][bi], packed_even_to_e5m2x4(wa[tt][bi]), packed_even_to_e5m2x4(wb[tt][bi]),
                              packed_odd_to_e5m2x4(wa[tt][bi]), packed_odd_to_e5m2x4(wb[tt][bi]), hf.q[bi][r].x,
                              hf.q[bi][r].y);
            }
          }
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
            for (int bi = 0; bi < kDnB; ++bi) {
              if (cw + kCons * bi < geo.nbI) {
                const float ta = e8m0_to_f32_fast(base[dn_scl + 16 * tt * geo.nbI + kCons * bi]) * hf.f[bi][r];
                const float tb = e8m0_to_f32_fast(base[dn_scl + (16 * tt + 8) * geo.nbI + kCons * bi]) * hf.f[bi][r];
                acc[4 * tt + r] = fmaf(d[tt][bi][1], ta, fmaf(d[tt][bi][0], ta, acc[4 * tt + r]));
                acc[4 * tt + 2 + r] = fmaf(d[tt][bi][3], tb, fmaf(d[tt][bi][2], tb, acc[4 * tt + 2 + r]));
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[st]);
      ++it;
      hand_off(acc, true);
    };

    // ---- phase 1: once every CTA's logits are in, routing; then the shared
    //      expert's items (prefetched by the producer while the barrier
    //      completed) and the routed items.  Routing comes first so that the
    //      routed items' copies start as early as possible. ----
    int n1 = 1, n2 = 0;
    for (int j = 0;; ++j) {
      if (j == 0) {
        // ---- wait for every CTA's logits (bounded), then route ----
        if (threadIdx.x == 0 && !poisoned() && !grid_wait(bar_word, bar_old)) fail();
        consumer_bar_sync();
        // all M x E logits into shared memory with one round of loads (the
        // reduce buffers are idle until the first item is handed off)
        float* lg = &C.red[0][0][0][0];
        for (int i = threadIdx.x; i < M * E; i += kCons * 32) lg[i] = __ldcg(ws.logits + i);
        consumer_bar_sync();
        if (cw < M) {  // warp m routes token m
          const int m = cw;
          VI R[8];
          warp_top8(lg + (size_t)m * E, E, lane, R);
          if (lane == 0) {
#pragma unroll
            for (int r = 0; r < 8; ++r)
              if (r < a.top_k) { C.ids[m][r] = R[r].i; C.topv[m][r] = R[r].v; }
            float z = 0.f;
            for (int r = 0; r < a.top_k; ++r) z += expf(C.topv[m][r] - C.topv[m][0]);
            for (int r = 0; r < a.top_k; ++r) C.wts[m][r] = expf(C.topv[m][r] - C.topv[m][0]) / z;
          }
        }
        consumer_bar_sync();
        if (cw == 0) {
          // Slot table: slot 0 is the shared expert, then one slot per distinct
          // routed expert in order of first appearance over (token, rank).
          // Lane l holds choice l = m * top_k + r (M * top_k <= 32).
          const int k = a.top_k, n_in = M * k;
          const bool act = lane < n_in;
          const int m = act ? lane / k : 0, r = act ? lane - (lane / k) * k : 0;
          int32_t ex = act ? C.ids[m][r] : -1 - lane;  // idle lanes get ids of their own
          if (act && (ex < 0 || ex >= E)) {  // cannot happen (see warp_top8); never index out of range
            report(ws.hdr, MOE_ERR_DEVICE_CHECK);
            ex = 0;
          }
          const uint32_t same = __match_any_sync(0xffffffffu, ex);
          const int leader = __ffs(same) - 1;
          const uint32_t leaders = __ballot_sync(0xffffffffu, act && leader == lane);
          const int slot = 1 + __popc(leaders & ((1u << leader) - 1u));
          if (act && leader == lane) {
            C.slot_expert[slot] = ex;
            C.slot_mask[slot] = 0u;
            for (int mm = 0; mm < 4; ++mm) C.slot_w[slot][mm] = 0.f;
          }
          if (lane == 0) {
            C.slot_expert[0] = -1;
            C.slot_mask[0] = 0xfu;
            for (int mm = 0; mm < 4; ++mm) C.slot_w[0][mm] = 1.0f;
          }
          __syncwarp();
          if (act) {
            atomicOr(&C.slot_mask[slot], 1u << m);
            C.slot_w[slot][m] = C.wts[m][r];  // a token picks an expert at most once
          }
          __syncwarp();
          if (lane == 0) {
            C.nslots = 1 + __popc(leaders);
            __threadfence_block();
            mbar_arrive(&C.routed);  // the producer and the epilogue warps may go on
          }
        }
        consumer_bar_sync();
        const int S = C.nslots;
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
    // phase 2 reads every CTA's h: wait until the epilogue warps have seen the
    // grid barrier that follows phase 1
    bounded_wait(&C.h_ready, 0);
    // ---- split pass: h -> per-block scale and three E4M3 parts, once per
    //      (slot, token, 32-element block) across the grid (one warp per
    //      block: lane l holds element l), instead of once per down item ----
    {
      const int S = C.nslots;
      const int units = S * M * geo.nbI;
      for (int u = c * kCons + cw; u < units; u += G * kCons) {
        const int blk = u % geo.nbI, sm = u / geo.nbI, m = sm % M, slot = sm / M;
        const uint32_t mask = slot == 0 ? 0xfu : C.slot_mask[slot];
        const size_t unit = ((size_t)slot * 4 + m) * geo.nbI + blk;
        if (!(mask >> m & 1u)) continue;  // this token does not use the slot: its h is never read
        const float v = __ldcg(ws.h + ((size_t)slot * 4 + m) * I + blk * 32 + lane);
        const int sig = pow2_sigma(warp_max(fabsf(v)));
        float r = v * exp2i(sig);
        // element l goes to the lane tq = l / 8 of the B fragment: even ones
        // to its first 4-byte group (b0), odd ones to its second (b1)
        const int j = lane & 7;
        uint8_t* dst = ws.hq + unit * kHParts * 32 + (lane >> 3) * 8 + (j & 1) * 4 + (j >> 1);
#pragma unroll
        for (int part = 0; part < kHParts; ++part) {
          const float q = round_sig4(r);
          dst[part * 32] = (uint8_t)f32x2_to_e4m3x2(q, 0.f);
          r -= q;
        }
        if (lane == 0) ws.hf[unit] = exp2i(6 - sig) * 256.0f;  // 2^-sig and the E5M2 weights' 2^-14
      }
      // every CTA's parts are written before any down item reads them
      consumer_bar_sync();
      if (threadIdx.x == 0) {
        const uint32_t old = grid_arrive(bar_word, c, G);
        if (!poisoned() && !grid_wait(bar_word, old)) fail();
        mbar_arrive(&C.parts_ready);  // the epilogue warps may arrive at the next barrier
      }
      consumer_bar_sync();
    }
    // B fragments are loaded once per slot (the CTA's items are consecutive
    // tiles), one item ahead of the first item that needs them
    const int q2 = items.p2_begin(C.nslots);
    HFrag nxt;
    int nslot = n2 > 0 ? q2 / geo.n_tiles : -1;
    if (n2 > 0) load_h(nslot, nxt);
    for (int j = 0; j < n2; ++j) {
      const HFrag cur = nxt;
      if (j + 1 < n2) {
        const int s1 = (q2 + j + 1) / geo.n_tiles;
        if (s1 != nslot) load_h(s1, nxt);
        nslot = s1;
      }
      down_item(cur);
    }
    // ---- combine: out = sum over slots, in slot order, of w * partial.  One
    //      warp per (32-row tile, token) across the grid, lane = row, every
    //      slot's load in flight at once: no float atomics, the same result
    //      on every run ----
    if (bounded_wait(&C.partials_ready, 0)) {
      const int S = C.nslots;
      for (int u = c + G * cw; u < geo.n_tiles * M; u += G * kCons) {
        const int tile = u % geo.n_tiles, m = u / geo.n_tiles;
        const int row = tile * kDnRows + lane;
        float p[MoeWs::kMaxSlots];
#pragma unroll
        for (int s2 = 0; s2 < MoeWs::kMaxSlots; ++s2) {
          const uint32_t mk = s2 == 0 ? 0xfu : C.slot_mask[s2 < S ? s2 : 0];
          p[s2] = (s2 < S && (mk >> m & 1u)) ? __ldcg(&ws.ypart[((size_t)s2 * 4 + m) * H + row]) : 0.f;
        }
        float y = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < MoeWs::kMaxSlots; ++s2)
          if (s2 < S) y = fmaf(C.slot_w[s2][m], p[s2], y);
        a.out[(size_t)m * H + row] = y;
      }
    }
  }
}

}  // namespace

size_t moe_fused_smem_bytes(int H, int I) {
  const Geometry geo(H, I);
  return ((sizeof(SmemCtl) + 127) / 128) * 128 + (size_t)kStages * geo.stage_bytes;
}

bool moe_fused_supported(int H, int I) {
  return H % 64 == 0 && I % 64 == 0 && H / 32 <= kMaxGuBlocksPerWarp * kCons &&
         I / 32 <= kMaxDnBlocksPerWarp * kCons && moe_fused_smem_bytes(H, I) <= (size_t)kMaxDynamicSmem;
}

template <int kGuB>
static cudaError_t launch_fused_t(const FusedArgs& a, size_t smem, cudaStream_t st) {
  auto kern = moe_fused_kernel<kGuB>;
  cudaError_t e = ensure_smem_optin<moe_fused_kernel<kGuB>>();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = current_device_sms(&dev, &sms)) != cudaSuccess) return e;
  // one CTA per SM; the cooperative launch fails (it does not wait) if they
  // cannot all be resident at once
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
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) (void)cudaGetLastError();  // leave no stale error for the next call to find
  return e;
}

// The instantiations of the gate/up blocks-per-warp buckets, smallest first;
// a launch takes the first bucket that covers ceil((H / 32) / kCons).
template <int... kBuckets>
struct GuDispatch {
  static cudaError_t run(int, const FusedArgs&, size_t, cudaStream_t) { return cudaErrorInvalidValue; }
};
template <int kB, int... kRest>
struct GuDispatch<kB, kRest...> {
  static cudaError_t run(int need, const FusedArgs& a, size_t smem, cudaStream_t st) {
    return need <= kB ? launch_fused_t<kB>(a, smem, st) : GuDispatch<kRest...>::run(need, a, smem, st);
  }
};
using GuBuckets = GuDispatch<1, 2, 4, 5, kMaxGuBlocksPerWarp>;

cudaError_t launch_moe_fused(const MoeArgs& m, cudaStream_t st) {
  FusedArgs a{m.x, m.router_w, m.router_bias, m.bank, m.shared, m.M, m.top_k, m.E, m.H, m.I,
              m.out, m.ids_out, m.w_out, m.ws};
  const size_t smem = moe_fused_smem_bytes(m.H, m.I);
  const int need_gu = (m.H / 32 + kCons - 1) / kCons;
  return GuBuckets::run(need_gu, a, smem, st);
}

}  // namespace moe
