// lmhead_fp8.cu -- the online-FP8 LM head: one pass over the tiled E4M3 head
// for all M tokens, fused with the per-row scale, an optional logits write
// and a top-k reduction.
//
// The pages: every generated token reads the whole 157,184 x 2,560 head, and
// quantising only this layer to FP8 at load time halves those reads
// (ncijnetwork.com summary, "What are the 3 optimizations?", item 2;
// generativeaipub.com blog, "2. Compressing the Output Head").
//
// Design (sm_100a, one GPU), warp-specialised with no CTA-wide barrier in the
// stream:
//  * One CTA per SM over 16-row tiles of the fragment-tiled head
//    (lmhead_tile_fp8): half of the tiles in one contiguous range per CTA,
//    the rest handed out by a global counter so that SMs that stream at
//    different rates finish together.  A producer warp streams the tiles into
//    a ring of shared-memory stages, one bulk copy (no multicast) per tile
//    plus one for its 16 row scales, completing on an mbarrier per stage; the
//    ring keeps four tiles (~160 KB) in flight per SM, two when a call's other
//    shared-memory needs leave no room for four (always an even count: see
//    lmhead_fp8_plan).
//  * Two groups of ten consumer warps take alternate tiles, so that each
//    group has two tiles' time for one: warp w of a group takes 64-byte
//    slices w, w + 10, ... of its tiles, loads its A fragments from the stage
//    (one 512-byte run per warp and half tile) and runs mma.sync m16n8k32
//    E4M3 x E4M3 -> fp32; the B fragments (the tokens) live in registers for
//    the whole kernel.  The tensor-core instruction retires 4,096
//    multiply-adds per issue with no per-weight decode; the contraction is
//    not reshaped.
//  * Activations: per token and 64-element slice, scaled by a power of two
//    that puts the slice's largest magnitude in [2^7, 2^8) and split into two
//    E4M3 parts hi + lo (exact for bf16 values down to 2^-10 of the slice's
//    largest, within 2^-17 of it below), which ride in two columns of the
//    MMA: column n = part n & 1 of token n >> 1.  Each slice's result is
//    scaled back before it joins the row's fp32 sum.
//  * Each group hands a tile's partial sums to its epilogue warp through
//    mbarrier-guarded buffers; the epilogue sums them, applies the row scale,
//    writes the logits if asked, keeps the values in shared memory and keeps
//    64 running maxima per token.
//  * Top-k (k <= 64) after the stream, all tokens at once: the k-th largest
//    running maximum bounds the k-th best value from below, and the few
//    values not below it are ranked by counting.  Each CTA writes its sorted
//    list; the last CTA to finish bulk-copies all lists into shared memory
//    and merges them: the k-th best list head L bounds the answer, only
//    lists whose head is not worse than L hold survivors (a prefix of each,
//    at most k * k in all), and the survivors are ranked by counting (ties
//    go to the lower token id everywhere).
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "lmhead.h"

namespace moe {
namespace {

constexpr int kRows = 16;             // rows per tile
constexpr int kGrp = 10;              // consumer warps per group; a group splits K of one tile
constexpr int kCons = 2 * kGrp;       // two groups take alternate tiles
constexpr int kProdWarp = kCons;      // the producer warp
constexpr int kEpi0 = kCons + 1;      // epilogue warp e serves group e
constexpr int kNumEpi = 2;
constexpr int kWarpsF = kCons + 1 + kNumEpi;
constexpr int kThreadsF = kWarpsF * 32;
constexpr int kMaxSlicesF = 8;        // 64-byte slices per consumer warp: H <= 8 * 10 * 64 = 5120
constexpr int kMaxStagesF = 5;
constexpr int kRedF = 4;              // partial-sum buffers; group q uses buffers q and q + 2
constexpr int kGroupsF = 64;          // running maxima per token for the top-k bound (k <= 64)
constexpr int kMaxHF = kMaxSlicesF * kGrp * 64;
static_assert(kRedF == 2 * kNumEpi, "two partial-sum buffers per group");

struct HeadCand {
  float v;
  int32_t id;
};

struct HeadCtl {
  uint64_t full[kMaxStagesF];
  uint64_t empty[kMaxStagesF];
  uint64_t red_full[kRedF];
  uint64_t red_empty[kRedF];
  uint64_t xbar;                    // the tokens
  uint64_t lbar;                    // the merge's lists
  int32_t stile[kMaxStagesF];       // tile in each stage; -1: no more tiles
  int32_t rtile[kRedF];             // tile in each partial-sum buffer; -1: no more tiles
  float rsc[kRedF][kRows];          // row scales of the tile in each partial-sum buffer
  int sigma[4][kMaxHF / 64];        // per token and 64-element slice
  float gmax[4][kGroupsF];          // running maxima (admissible values only; -FLT_MAX if none)
  float vstar[4];                   // per token: the k-th largest running maximum
  int vkey[4];                      // merge: per token, the k-th largest head value (ordered-int key)
  HeadCand bound[4];                // merge: per token, the k-th best list head
  int cnt[4];                       // per token: candidates or survivors
  int end[kNumEpi];                 // the slot at which each epilogue warp stopped
  int last;
  int poison;
};
constexpr int kHeadCtlBytes = (int)((sizeof(HeadCtl) + 127) / 128 * 128);

__host__ __device__ constexpr int tile_stage_bytes(int H) { return (kRows * H + 64 + 127) / 128 * 128; }

// Shared-memory plan and tile schedule.  CTA c first takes tiles
// c * ps .. c * ps + ps - 1 (half of the head, in order), then tiles from a
// counter until the head is done or it holds `cap` tiles; the counter
// evens out the finishing times of SMs that stream at different rates.
struct HeadGeo {
  int64_t ntiles;
  int64_t dyn0;       // first tile handed out by the counter
  int ps;             // tiles per CTA taken in order
  int cap;            // most tiles one CTA takes
  int stage_bytes, stages;
  int red_bytes;      // partial sums: [kRedF][kGrp][M][16] fp32
  int cval_off;       // this CTA's values: [M][cap * 16] fp32
  int tile_off;       // the tile in each slot: [cap] int32
  int work_bytes;     // the tokens first ([M][H] bf16), then the three arrays above
  int tok_stride;     // candidate entries per token in global memory (G * k, even)
  int tpp;            // tokens per merge pass (lists, survivors and head values of a token)
  size_t ring_bytes;  // the stages; after the stream, the top-k candidates and the merge's lists
  size_t smem;
};

__host__ __device__ inline HeadGeo head_geo(int64_t V, int H, int M, int grid, int stages, int top_k) {
  HeadGeo g;
  g.ntiles = (V + kRows - 1) / kRows;
  g.ps = (int)(g.ntiles / 2 / grid);
  g.dyn0 = (int64_t)grid * g.ps;
  const int64_t dyn = g.ntiles - g.dyn0;
  g.cap = g.ps + 2 * (int)((dyn + grid - 1) / grid) + 8;
  g.stage_bytes = tile_stage_bytes(H);
  g.stages = stages;
  g.red_bytes = kRedF * kGrp * M * kRows * 4;
  g.cval_off = g.red_bytes;
  g.tile_off = g.cval_off + M * g.cap * kRows * 4;
  const int rc = g.tile_off + g.cap * 4, xb = M * H * 2;
  g.work_bytes = ((xb > rc ? xb : rc) + 127) / 128 * 128;
  g.tok_stride = (grid * top_k + 1) & ~1;
  const size_t cands = (size_t)M * g.cap * kRows * sizeof(HeadCand);
  // a merge pass holds, per token: the lists, k * k survivors, and the
  // heads' values, ids and two counts
  const size_t per_tok = (size_t)g.tok_stride * sizeof(HeadCand) + (size_t)top_k * top_k * sizeof(HeadCand) +
                         (size_t)((grid + 3) & ~3) * 16;
  const size_t ring = (size_t)stages * g.stage_bytes;
  size_t need = cands > per_tok ? cands : per_tok;
  need = ring > need ? ring : need;
  need = (need + 127) / 128 * 128;
  const size_t fixed = (size_t)kHeadCtlBytes + g.work_bytes;
  const size_t all_tok = ((size_t)M * per_tok + 127) / 128 * 128;
  if (need < all_tok && fixed + all_tok <= (size_t)kMaxDynamicSmem) need = all_tok;  // one merge pass
  g.ring_bytes = need;
  g.tpp = (int)(g.ring_bytes / per_tok);
  if (g.tpp > M) g.tpp = M;
  g.smem = (size_t)kHeadCtlBytes + g.work_bytes + g.ring_bytes;
  return g;
}

__device__ __forceinline__ int pow2_sigma_e4m3(float amax) {
  // sigma such that amax * 2^sigma lies in [2^7, 2^8), clamped so that 2^sigma
  // and 2^-sigma are normal fp32 numbers; 0 for amax = 0 or NaN
  if (!(amax > 0.f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int e = (int)((b >> 23) & 0xffu);
  const int fl = e ? e - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
  const int s = 7 - fl;
  return s > 126 ? 126 : (s < -126 ? -126 : s);
}
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// A float's bits as an int that orders like the float (finite values and
// +-inf; NaN never reaches these).
__device__ __forceinline__ int float_order_key(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}

// The number of entries of list[0..n) better than e.
__device__ __forceinline__ int count_better(const HeadCand* list, int n, const HeadCand& e) {
  int r = 0;
#pragma unroll 8
  for (int o = 0; o < n; ++o) r += better(list[o].v, list[o].id, e.v, e.id);
  return r;
}

template <int kS>
__global__ void __launch_bounds__(kThreadsF, 1)
lmhead_fp8_kernel(const uint16_t* __restrict__ x,       // [M][H] bf16
                  const uint8_t* __restrict__ qt,       // tiled E4M3 head
                  const float* __restrict__ row_scale,  // [V]
                  int64_t V, int H, int M, int top_k, int stages,
                  float* __restrict__ logits,           // [M][V] or nullptr
                  int32_t* __restrict__ out_ids,        // [M][top_k]
                  float* __restrict__ out_vals,         // [M][top_k]
                  WsHeader* __restrict__ hdr,
                  HeadCand* __restrict__ cand)          // [M][tok_stride]: CTA c's list at c * top_k
{
  extern __shared__ __align__(128) uint8_t smem[];
  HeadCtl& C = *reinterpret_cast<HeadCtl*>(smem);
  const HeadGeo geo = head_geo(V, H, M, gridDim.x, stages, top_k);
  uint8_t* work = smem + kHeadCtlBytes;
  uint8_t* ring = work + geo.work_bytes;
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(work);   // [M][H], until the fragments are built
  float* red = reinterpret_cast<float*>(work);                     // then the partial sums,
  float* cvals = reinterpret_cast<float*>(work + geo.cval_off);    // this CTA's values
  int32_t* slot_tile = reinterpret_cast<int32_t*>(work + geo.tile_off);
  const int cap16 = geo.cap * kRows;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int nsl = H / 64;
  const int k = top_k;
  const uint32_t tile_bytes = (uint32_t)(kRows * H);

  if (t == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], kGrp);
    }
    for (int r = 0; r < kRedF; ++r) {
      mbar_init(&C.red_full[r], kGrp);
      mbar_init(&C.red_empty[r], 1);
    }
    mbar_init(&C.xbar, 1);
    mbar_init(&C.lbar, 1);
    fence_mbar_init();
    C.poison = 0;
  }
  __syncthreads();
  pdl_launch_dependents();  // the next kernel may launch; its CTAs start as this one's exit
  if (t == 0) {
    // The tokens (and, after them, everything this kernel writes) may come
    // from the previous kernel on the stream: wait for it here, while the
    // producer already streams weights.  The other threads see its results
    // through the tokens' barrier; the producer waits on its own before it
    // takes tiles from the workspace's counter.
    pdl_wait();
    const uint32_t xbytes = (uint32_t)(M * H * 2);
    mbar_arrive_expect_tx(&C.xbar, xbytes);
    bulk_g2s(work, x, xbytes, &C.xbar, l2_evict_last_policy());
  }
  auto poisoned = [&]() -> bool { return *(volatile int*)&C.poison != 0; };
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {  // bounded; every lane polls
    if (poisoned()) return false;
    if (mbar_wait(bar, parity)) return true;
    report(hdr, MOE_ERR_TIMEOUT);
    atomicExch(&C.poison, 1);
    return false;
  };

  uint32_t bfrag[kS][2][2];
  float fx[kS];  // undoes the scale of token t's slice (columns 2t, 2t + 1)
  if (warp == kProdWarp) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      int uses[kMaxStagesF] = {0, 0, 0, 0, 0};    // phases started per stage (tiles and end markers)
      uint32_t next = 0;                          // a counter value fetched one tile ahead
      bool have_next = false;
      int ends = 0;                               // end markers sent (one per group)
      for (int it = 0; ends < 2; ++it) {
        const int s = it % stages;
        if (it >= stages && !wait(&C.empty[s], (uint32_t)((it / stages - 1) & 1))) break;
        int64_t tile = -1;
        if (ends == 0 && it < geo.cap) {
          if (it < geo.ps) {
            tile = (int64_t)blockIdx.x * geo.ps + it;
          } else {
            if (it == geo.ps) pdl_wait();  // the counter belongs to the workspace: after the previous kernel
            if (!have_next) next = atomicAdd(&hdr->tiles, 1u);
            have_next = false;
            tile = geo.dyn0 + next;
            if (tile >= geo.ntiles) tile = -1;
          }
        }
        if (tile >= 0 && it + 1 >= geo.ps && it + 1 < geo.cap) {  // every fetched value is used next
          if (it + 1 == geo.ps) pdl_wait();
          next = atomicAdd(&hdr->tiles, 1u);
          have_next = true;
        }
        C.stile[s] = (int32_t)tile;
        ++uses[s];
        if (tile < 0) {
          ++ends;
          mbar_arrive(&C.full[s]);  // the end marker: no bytes
          continue;
        }
        const bool full_tile = (tile + 1) * kRows <= V;  // a ragged last tile's scales are read from global
        uint8_t* dst = ring + (size_t)s * geo.stage_bytes;
        mbar_arrive_expect_tx(&C.full[s], tile_bytes + (full_tile ? 64u : 0u));
        bulk_g2s(dst, qt + (size_t)tile * tile_bytes, tile_bytes, &C.full[s], pol);
        if (full_tile) bulk_g2s(dst + tile_bytes, row_scale + tile * kRows, 64u, &C.full[s], pol);
      }
      if (poisoned()) {  // let the copies in flight land before the CTA exits
        for (int s = 0; s < stages; ++s)
          if (uses[s] > 0) mbar_wait(&C.full[s], (uint32_t)((uses[s] - 1) & 1));
      }
    }
  } else {
    wait(&C.xbar, 0);
    // ---- per (token, slice) scale (consumers) ----
    for (int u = t; u < M * nsl; u += kCons * 32) {
      if (warp >= kCons) break;
      const int m = u / nsl, sl = u - m * nsl;
      const uint4* p = reinterpret_cast<const uint4*>(xs + m * H + 64 * sl);
      float am = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 v = p[q];
        am = fmaxf(am, fmaxf(fmaxf(bf16_bits_to_f32(v.x & 0x7fffu), bf16_bits_to_f32((v.x >> 16) & 0x7fffu)),
                             fmaxf(bf16_bits_to_f32(v.y & 0x7fffu), bf16_bits_to_f32((v.y >> 16) & 0x7fffu))));
        am = fmaxf(am, fmaxf(fmaxf(bf16_bits_to_f32(v.z & 0x7fffu), bf16_bits_to_f32((v.z >> 16) & 0x7fffu)),
                             fmaxf(bf16_bits_to_f32(v.w & 0x7fffu), bf16_bits_to_f32((v.w >> 16) & 0x7fffu))));
      }
      C.sigma[m][sl] = pow2_sigma_e4m3(am);
    }
    asm volatile("bar.sync 1, %0;" ::"r"((kWarpsF - 1) * 32) : "memory");  // every warp but the producer
    // Warp wq of a group, slice sl = wq + 10 si, MMA j, register r, lane
    // (g, t): elements 64 sl + 16 t + 8 j + 4 r .. +3 of column g = part
    // g & 1 of token g >> 1.
    const int grp = warp / kGrp, wq = warp - grp * kGrp;
    if (warp < kCons) {
      const int m = g >> 1, part = g & 1;
#pragma unroll
      for (int si = 0; si < kS; ++si) {
        const int sl = wq + kGrp * si;
        const bool in = sl < nsl && m < M;
        const float scl = in ? pow2f(C.sigma[m][sl]) : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t hw = 0u, lw = 0u;
          if (in) {
            const uint2 p = *reinterpret_cast<const uint2*>(xs + m * H + 64 * sl + 16 * tq + 4 * q);
            uint32_t pp[2];
            split_e4m3x4<2>(bf16_bits_to_f32(p.x & 0xffffu) * scl, bf16_bits_to_f32(p.x >> 16) * scl,
                            bf16_bits_to_f32(p.y & 0xffffu) * scl, bf16_bits_to_f32(p.y >> 16) * scl, pp);
            hw = pp[0];
            lw = pp[1];
          }
          bfrag[si][q >> 1][q & 1] = part ? lw : hw;
        }
        fx[si] = (sl < nsl && tq < M) ? pow2f(-C.sigma[tq][sl]) : 0.f;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"((kWarpsF - 1) * 32) : "memory");  // the tokens' memory becomes red + cvals

    if (warp < kCons) {
      // ------------------------------ consumers -----------------------------
      for (int it = grp;; it += 2) {
        const int s = it % stages, r = it % kRedF;
        if (!wait(&C.full[s], (uint32_t)((it / stages) & 1))) break;
        const int32_t tile = C.stile[s];
        if (tile < 0) {  // pass the end marker to this group's epilogue warp
          if (it >= kRedF && !wait(&C.red_empty[r], (uint32_t)(((it / kRedF) & 1) ^ 1))) break;
          if (wq == 0 && lane == 0) C.rtile[r] = -1;
          __syncwarp();
          if (lane == 0) mbar_arrive(&C.red_full[r]);
          break;
        }
        const uint8_t* st = ring + (size_t)s * geo.stage_bytes;
        float rs = 0.f;  // the group's first warp carries the tile's row scales to the epilogue
        const int64_t row = (int64_t)tile * kRows + lane;
        if (wq == 0 && lane < kRows && row < V)
          rs = ((int64_t)tile + 1) * kRows <= V ? *reinterpret_cast<const float*>(st + tile_bytes + 4 * lane)
                                                 : __ldg(row_scale + row);
        float ag = 0.f, ag8 = 0.f;  // rows g and g + 8, token t
#pragma unroll
        for (int si = 0; si < kS; ++si) {
          const int sl = wq + kGrp * si;
          if (sl < nsl) {
            const uint4 a = *reinterpret_cast<const uint4*>(st + sl * 1024 + lane * 16);        // row g
            const uint4 b = *reinterpret_cast<const uint4*>(st + sl * 1024 + 512 + lane * 16);  // row g + 8
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_e4m3(d, a.x, b.x, a.y, b.y, bfrag[si][0][0], bfrag[si][0][1]);
            mma_e4m3(d, a.z, b.z, a.w, b.w, bfrag[si][1][0], bfrag[si][1][1]);
            ag = fmaf(d[0] + d[1], fx[si], ag);
            ag8 = fmaf(d[2] + d[3], fx[si], ag8);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[s]);  // this warp is done with the stage
        if (it >= kRedF && !wait(&C.red_empty[r], (uint32_t)(((it / kRedF) & 1) ^ 1))) break;
        float* rb = red + ((size_t)r * kGrp + wq) * M * kRows;
        if (tq < M) {
          rb[tq * kRows + g] = ag;
          rb[tq * kRows + g + 8] = ag8;
        }
        if (wq == 0) {
          if (lane < kRows) C.rsc[r][lane] = rs;
          if (lane == 0) C.rtile[r] = tile;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.red_full[r]);
      }
    } else {
      // ------------------------------ epilogue ------------------------------
      // Lane l owns values idx = l and l + 32 (token idx / 16, row idx % 16)
      // and keeps their running maxima per slot pair phase: group
      // 32 e + 16 phase + row of each token.
      const int e = warp - kEpi0;
      float gm[2][2] = {{-FLT_MAX, -FLT_MAX}, {-FLT_MAX, -FLT_MAX}};
      int it = e;
      for (;; it += 2) {
        const int r = it % kRedF;
        if (!wait(&C.red_full[r], (uint32_t)((it / kRedF) & 1))) break;
        const int32_t tile = C.rtile[r];
        if (tile < 0) break;
        const float* rb = red + (size_t)r * kGrp * M * kRows;
        const int ph = (it >> 1) & 1;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = lane + 32 * u;
          if (idx < M * kRows) {
            const int m = idx >> 4, rr = idx & 15;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kGrp; ++w) v += rb[(w * M + m) * kRows + rr];
            v *= C.rsc[r][rr];
            const int64_t row = (int64_t)tile * kRows + rr;
            const bool in = row < V;
            if (in && logits) logits[(size_t)m * V + row] = v;
            const float cv = in ? v : -INFINITY;
            cvals[m * cap16 + it * kRows + rr] = cv;
            if (cv >= -FLT_MAX) gm[u][ph] = fmaxf(gm[u][ph], cv);
          }
        }
        if (lane == 0) slot_tile[it] = tile;
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.red_empty[r]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int idx = lane + 32 * u;
        if (idx < M * kRows) {
          C.gmax[idx >> 4][32 * e + (idx & 15)] = gm[u][0];
          C.gmax[idx >> 4][32 * e + 16 + (idx & 15)] = gm[u][1];
        }
      }
      if (lane == 0) C.end[e] = it;
    }
  }
  __syncthreads();  // every tile consumed: the ring is free

  // ---- this CTA's top-k per token, all tokens at once ----
  // 1. v*: the k-th largest of the token's 64 running maxima.  Each maximum
  // is one of the CTA's admissible values (or -FLT_MAX for an empty group),
  // so at least k values are >= v* and v* bounds the k-th best from below.
  if (warp < M) {
    const float a = C.gmax[warp][lane], b = C.gmax[warp][lane + 32];
    int ca = 0, cb = 0;
#pragma unroll 16
    for (int o = 0; o < kGroupsF; ++o) {
      const float q = C.gmax[warp][o];
      ca += q > a;
      cb += q > b;
    }
    float c = ca < k ? a : INFINITY;  // values with fewer than k larger ones: v* is their minimum
    if (cb < k) c = fminf(c, b);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c = fminf(c, __shfl_xor_sync(0xffffffffu, c, o));
    if (lane == 0) {
      C.vstar[warp] = c;
      C.cnt[warp] = 0;
    }
  }
  const int ntl = min(min(C.end[0], C.end[1]), geo.cap);  // slots 0 .. ntl - 1 hold tiles
  __syncthreads();
  // 2. candidates: every admissible value >= v* (a few per token; each
  // thread claims its slots with its own shared atomic)
  const int nv = ntl * kRows;
  HeadCand* cl = reinterpret_cast<HeadCand*>(ring);  // [M][cap16]
  for (int i = t; i < nv; i += kThreadsF) {
    const int32_t id = slot_tile[i >> 4] * kRows + (i & 15);
    for (int m = 0; m < M; ++m) {
      const float v = cvals[m * cap16 + i];
      if (v >= C.vstar[m]) {
        const int pos = atomicAdd(&C.cnt[m], 1);
        if (pos < cap16) cl[m * cap16 + pos] = HeadCand{v, id};
      }
    }
  }
  __syncthreads();
  // 3. rank them by counting; the best k become this CTA's list
  bool wrote = false;
  {
    const int per = kThreadsF / M, m = t / per, q0 = t - m * per;
    if (m < M) {
      const int n = min(C.cnt[m], cap16);
      const HeadCand* clm = cl + m * cap16;
      HeadCand* dst = cand + (size_t)m * geo.tok_stride + (size_t)blockIdx.x * k;
      for (int q = q0; q < n; q += per) {
        const HeadCand e = clm[q];
        const int r = count_better(clm, n, e);
        if (r < k) {
          dst[r] = e;
          wrote = true;
        }
      }
      for (int r = n + q0; r < k; r += per) {
        dst[r] = HeadCand{-FLT_MAX, INT32_MAX};
        wrote = true;
      }
    }
  }

  // ---- the last CTA merges every CTA's lists ----
  if (wrote) __threadfence();  // this CTA's list entries, before it counts itself done
  __syncthreads();
  if (t == 0) C.last = atomicAdd(&hdr->ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!C.last) return;
  if (t == 0) {
    hdr->ticket = 0u;  // every CTA has counted itself and taken its last tile
    hdr->tiles = 0u;
    __threadfence();
  }
  if (poisoned()) return;
  const int G = gridDim.x;
  HeadCand* lists = reinterpret_cast<HeadCand*>(ring);           // [tpp][tok_stride]
  HeadCand* surv = lists + (size_t)geo.tpp * geo.tok_stride;     // [tpp][k * k]
  float* hv = reinterpret_cast<float*>(surv + (size_t)geo.tpp * k * k);  // [tpp][G] head values
  int32_t* hid = reinterpret_cast<int32_t*>(hv + geo.tpp * G);            // [tpp][G] head ids
  int32_t* hcnt = hid + geo.tpp * G;                                      // [tpp][G] larger head values
  int32_t* heq = hcnt + geo.tpp * G;                                      // [tpp][G] equal head values
  const uint32_t tok_bytes = (uint32_t)geo.tok_stride * (uint32_t)sizeof(HeadCand);
  for (int m0 = 0, pass = 0; m0 < M; m0 += geo.tpp, ++pass) {
    const int mt = min(geo.tpp, M - m0);
    if (t == 0) {
      fence_proxy_async();  // the other CTAs' lists, acquired above, before the bulk reads
      mbar_arrive_expect_tx(&C.lbar, (uint32_t)mt * tok_bytes);
      for (int j = 0; j < mt; ++j)
        bulk_g2s(lists + (size_t)j * geo.tok_stride, cand + (size_t)(m0 + j) * geo.tok_stride, tok_bytes, &C.lbar,
                 l2_evict_first_policy());
    }
    if (t < mt) {
      C.vkey[t] = INT32_MAX;
      C.bound[t] = HeadCand{-FLT_MAX, INT32_MAX};
      C.cnt[t] = 0;
    }
    if (!mbar_wait(&C.lbar, (uint32_t)(pass & 1))) {  // bounded; the copies are known to be in bounds
      report(hdr, MOE_ERR_TIMEOUT);
      return;
    }
    const int nh = mt * G;
    for (int h = t; h < nh; h += kThreadsF) {
      const int j = h / G;
      const HeadCand e = lists[(size_t)j * geo.tok_stride + (size_t)(h - j * G) * k];
      hv[h] = e.v;
      hid[h] = e.id;
    }
    __syncthreads();
    // 1. per token, v* = the k-th largest head value.  p = 4, 2 or 1
    // threads count the heads with a larger value than one head.
    const int lp = nh * 4 <= kThreadsF ? 2 : (nh * 2 <= kThreadsF ? 1 : 0);
    const int p = 1 << lp;
    for (int u0 = 0; u0 < (nh << lp); u0 += kThreadsF) {  // the same trip count in every thread
      const int u = u0 + t, h = u >> lp, part = u & (p - 1);
      int cnt = 0, eq = 0;
      if (h < nh) {
        const int j = h / G;
        const float* hj = hv + j * G;
        const float a = hv[h];
#pragma unroll 8
        for (int o = part; o < G; o += p) {
          const float q = hj[o];
          cnt += q > a;
          eq += q == a;
        }
      }
      for (int d = 1; d < p; d <<= 1) {
        cnt += __shfl_xor_sync(0xffffffffu, cnt, d);
        eq += __shfl_xor_sync(0xffffffffu, eq, d);
      }
      if (h < nh && part == 0) {
        hcnt[h] = cnt;
        heq[h] = eq;
        if (cnt < k) atomicMin(&C.vkey[h / G], float_order_key(hv[h]));
      }
    }
    __syncthreads();
    // 2. L = the k-th best head: among the heads whose value is v*, the one
    // whose rank by id completes k (none when fewer than k heads are
    // admissible).  Usually one head has value v*.
    for (int h = t; h < nh; h += kThreadsF) {
      const int j = h / G;
      const float a = hv[h];
      if (float_order_key(a) == C.vkey[j] && hid[h] != INT32_MAX) {
        const float* hj = hv + j * G;
        const int32_t* ij = hid + j * G;
        int r = hcnt[h];
        if (heq[h] > 1)  // ties on the value: rank by id among them
          for (int o = 0; o < G; ++o) r += (hj[o] == a) & (ij[o] < hid[h]);
        if (r == k - 1) C.bound[j] = HeadCand{a, hid[h]};
      }
    }
    __syncthreads();
    // 3. survivors: the entries not worse than L in lists whose head is not
    // worse than L -- at most k lists, a prefix of each: at most k * k
    for (int u0 = 0; u0 < (nh << lp); u0 += kThreadsF) {
      const int u = u0 + t, h = u >> lp, part = u & (p - 1);
      if (h < nh) {
        const int j = h / G, c = h - j * G;
        const HeadCand L = C.bound[j];
        const HeadCand* lst = lists + (size_t)j * geo.tok_stride + (size_t)c * k;
        for (int o = part; o < k; o += p) {
          const HeadCand e = lst[o];
          if (e.id == INT32_MAX || better(L.v, L.id, e.v, e.id)) break;  // the list is sorted
          const int pos = atomicAdd(&C.cnt[j], 1);
          if (pos < k * k) surv[(size_t)j * k * k + pos] = e;
        }
      }
    }
    __syncthreads();
    // 4. rank the survivors by counting; pad when fewer than k values are
    // admissible
    {
      const int per = kThreadsF / mt, j = t / per, q0 = t - j * per;
      if (j < mt) {
        const int m = m0 + j;
        const int n = min(C.cnt[j], k * k);
        const HeadCand* sj = surv + (size_t)j * k * k;
        for (int q = q0; q < n; q += per) {
          const HeadCand e = sj[q];
          const int r = count_better(sj, n, e);
          if (r < k) {
            out_ids[m * k + r] = e.id;
            out_vals[m * k + r] = e.v;
          }
        }
        for (int r = n + q0; r < k; r += per) {
          out_ids[m * k + r] = INT32_MAX;
          out_vals[m * k + r] = -FLT_MAX;
        }
      }
    }
    __syncthreads();  // before the next pass reuses the lists
  }
}

__global__ void tile_fp8_head_kernel(const uint8_t* __restrict__ q, int64_t V, int H, uint8_t* __restrict__ out) {
  const int64_t ntiles = (V + kRows - 1) / kRows;
  const int64_t units = ntiles * H;  // 16-byte units: 16 * H bytes per tile
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < units; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = u / H;
    const int j = (int)(u - t * H);
    const int s = j >> 6, h = (j >> 5) & 1, l = j & 31;
    const int64_t row = t * kRows + (l >> 2) + 8 * h;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < V) v = *reinterpret_cast<const uint4*>(q + row * H + 64 * s + 16 * (l & 3));
    *reinterpret_cast<uint4*>(out + u * 16) = v;
  }
}

template <int kS>
cudaError_t launch_fp8_t(const uint16_t* x, const uint8_t* qt, const float* s, int64_t V, int H, int M, int top_k,
                         float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid, int stages,
                         size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem_optin<lmhead_fp8_kernel<kS>>();
  if (e != cudaSuccess) return e;
  return launch_dependent(lmhead_fp8_kernel<kS>, dim3(grid), dim3(kThreadsF), smem, st, false, x, qt, s, V, H, M,
                          top_k, stages, logits, ids, vals, hdr, reinterpret_cast<HeadCand*>(cand));
}

}  // namespace

bool lmhead_fp8_plan(int H, int M, int top_k, int64_t V, int grid, int* stages, size_t* smem) {
  if (grid < 1 || grid > kLmheadMaxGrid) return false;
  if (H < 64 || H % 64 != 0 || H > kMaxHF || M < 1 || M > 4 || top_k < 1 || top_k > 64) return false;
  // An even number of stages: the two consumer groups take alternate
  // iterations and iteration i uses stage i % stages, so each stage then
  // belongs to one group, and a group never waits on a stage's barrier two
  // phases ahead of it.  With an odd count a stage alternates between the
  // groups, and a group running ahead could take the other group's earlier
  // phase of the barrier for its own (the parities match) and read the
  // other group's tile.
  for (int st = kMaxStagesF & ~1; st >= 2; st -= 2) {
    const HeadGeo g = head_geo(V, H, M, grid, st, top_k);
    if (g.smem <= (size_t)kMaxDynamicSmem) {
      *stages = st;
      *smem = g.smem;
      return true;
    }
  }
  return false;
}

size_t lmhead_tiled_bytes(int64_t V, int H) { return (size_t)((V + kRows - 1) / kRows) * kRows * H; }

cudaError_t launch_tile_fp8_head(const uint8_t* q, int64_t V, int H, uint8_t* out, cudaStream_t st) {
  tile_fp8_head_kernel<<<4 * 148, 256, 0, st>>>(q, V, H, out);
  return cudaGetLastError();
}

size_t lmhead_cand_bytes(int grid, int M, int top_k) {
  return (size_t)M * (size_t)(((int64_t)grid * top_k + 1) & ~int64_t(1)) * sizeof(HeadCand);
}

cudaError_t launch_lmhead_fp8(const uint16_t* x, const uint8_t* qt, const float* s, int64_t V, int H, int M,
                              int top_k, float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand,
                              int grid, cudaStream_t st) {
  int stages = 0;
  size_t smem = 0;
  if (!lmhead_fp8_plan(H, M, top_k, V, grid, &stages, &smem)) return cudaErrorInvalidConfiguration;
  const int need = (H / 64 + kGrp - 1) / kGrp;  // slices per consumer warp
  switch (need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : need <= 8 ? 8 : 0) {
    case 1: return launch_fp8_t<1>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 2: return launch_fp8_t<2>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 4: return launch_fp8_t<4>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 8: return launch_fp8_t<8>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
