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
//  * One CTA per SM, persistent over a contiguous range of 16-row tiles of
//    the fragment-tiled head (lmhead_tile_fp8).  A producer warp streams the
//    tiles into a ring of shared-memory stages, one bulk copy (no multicast)
//    per tile plus one for its 16 row scales, completing on an mbarrier per
//    stage; the ring keeps four or five tiles (~160-200 KB) in flight per SM.
//  * Twenty consumer warps split K: warp w takes 64-byte slices w, w + 20, ...
//    of every tile, loads its A fragments from the stage (the tiled layout
//    puts them in one 512-byte run per warp and half tile), releases the stage
//    and runs mma.sync m16n8k32 E4M3 x E4M3 -> fp32; the B fragments (the
//    tokens) live in registers for the whole kernel.  The tensor-core
//    instruction is used because it retires 4,096 multiply-adds per issue with
//    no per-weight decode; the contraction is not reshaped.
//  * Activations: per token and 64-element slice, scaled by a power of two
//    that puts the slice's largest magnitude in [2^7, 2^8) and split into two
//    E4M3 parts hi + lo (exact for bf16 values down to 2^-10 of the slice's
//    largest, within 2^-17 of it below), which ride in two columns of the
//    MMA: column n = part n & 1 of token n >> 1.  Each slice's result is
//    scaled back before it joins the row's fp32 sum.
//  * The consumers hand each tile's partial sums to one of two epilogue warps
//    (alternate tiles) through mbarrier-guarded buffers; the epilogue sums
//    them, applies the row scale, writes the logits if asked and keeps them in
//    shared memory.
//  * Top-k (k <= 64) after the stream, with all threads: the k-th best of 64
//    group maxima bounds the k-th best value from below, and the few values
//    not worse than the bound are ranked by counting.  Each CTA writes its
//    sorted list; the last CTA to finish merges the lists: the k-th best list
//    head bounds the answer, only lists whose head is not worse hold
//    survivors, and the survivors are ranked by counting (ties go to the lower
//    token id everywhere).
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "lmhead.h"

namespace moe {
namespace {

constexpr int kRows = 16;           // rows per tile
constexpr int kCons = 20;           // consumer warps splitting K
constexpr int kProdWarp = kCons;    // the producer warp
constexpr int kEpi0 = kCons + 1;    // the first epilogue warp
constexpr int kNumEpi = 2;          // epilogue warps, alternate tiles
constexpr int kWarpsF = kCons + 1 + kNumEpi;
constexpr int kThreadsF = kWarpsF * 32;
constexpr int kMaxSlicesF = 4;      // 64-byte slices per consumer warp: H <= 4 * 20 * 64 = 5120
constexpr int kMaxStagesF = 5;
constexpr int kRedF = 4;            // partial-sum buffers (a multiple of kNumEpi)
constexpr int kGroupsF = 64;        // group maxima for the top-k bound (k <= 64)
constexpr int kGroupThreads = (kThreadsF / kGroupsF) * kGroupsF;
constexpr int kMaxHF = kMaxSlicesF * kCons * 64;
static_assert(kRedF % kNumEpi == 0, "each reduce buffer belongs to one epilogue warp");

struct HeadCand {
  float v;
  int32_t id;
};

struct HeadCtl {
  uint64_t full[kMaxStagesF];
  uint64_t empty[kMaxStagesF];
  uint64_t red_full[kRedF];
  uint64_t red_empty[kRedF];
  uint64_t xbar;
  int sigma[4][kMaxHF / 64];        // per token and 64-element slice
  float rsc[kRedF][kRows];          // row scales of the tile in each reduce buffer
  float gmax_v[kGroupsF];
  int32_t gmax_i[kGroupsF];
  HeadCand bound;
  int n0, n1;                       // compaction counters
  int last;
  int poison;
};
constexpr int kHeadCtlBytes = (int)((sizeof(HeadCtl) + 127) / 128 * 128);

__host__ __device__ constexpr int tile_stage_bytes(int H) { return (kRows * H + 64 + 127) / 128 * 128; }

struct HeadGeo {
  int64_t ntiles;
  int n_cap;          // rows of the largest CTA range
  int stage_bytes, stages;
  int red_bytes;      // partial sums: [kRedF][kCons][M][16] fp32
  int work_bytes;     // the tokens (first), then the partial sums + this CTA's logits [M][n_cap]
  size_t ring_bytes;  // the stages; after the stream, the top-k scratch and the merge's lists
  size_t smem;
};

__host__ __device__ inline HeadGeo head_geo(int64_t V, int H, int M, int grid, int stages, int top_k) {
  HeadGeo g;
  g.ntiles = (V + kRows - 1) / kRows;
  g.n_cap = (int)((g.ntiles + grid - 1) / grid) * kRows;
  g.stage_bytes = tile_stage_bytes(H);
  g.stages = stages;
  g.red_bytes = kRedF * kCons * M * kRows * 4;
  const int xb = M * H * 2, rc = g.red_bytes + M * g.n_cap * 4;
  g.work_bytes = ((xb > rc ? xb : rc) + 127) / 128 * 128;
  const size_t topk_scratch = (size_t)kThreadsF * 8 + (size_t)g.n_cap * 8;
  const size_t merge = (size_t)grid * top_k * 8 + (size_t)grid * 4 + (size_t)top_k * top_k * 8;
  const size_t post = topk_scratch > merge ? topk_scratch : merge;
  const size_t ring = (size_t)stages * g.stage_bytes;
  g.ring_bytes = ((ring > post ? ring : post) + 127) / 128 * 128;
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

// Append `e` to `list` (counter *cnt) when `keep`, one shared atomic per
// warp.  Every lane of the warp calls this.
__device__ __forceinline__ void warp_append(bool keep, const HeadCand& e, HeadCand* list, int* cnt, int cap) {
  const uint32_t bal = __ballot_sync(0xffffffffu, keep);
  const int lane = threadIdx.x & 31;
  int base = 0;
  if (lane == 0 && bal) base = atomicAdd(cnt, __popc(bal));
  base = __shfl_sync(0xffffffffu, base, 0);
  const int pos = base + __popc(bal & ((1u << lane) - 1u));
  if (keep && pos < cap) list[pos] = e;
}

// Rank each entry of list[0..n) by counting the entries better than it and
// write rank r < k to out[r]; ranks are distinct because ids are.
__device__ __forceinline__ void rank_into(const HeadCand* list, int n, int k, HeadCand* out_c, int32_t* out_ids,
                                          float* out_vals) {
  for (int q = threadIdx.x; q < n; q += blockDim.x) {
    const HeadCand e = list[q];
    int r = 0;
#pragma unroll 8
    for (int o = 0; o < n; ++o) r += better(list[o].v, list[o].id, e.v, e.id);
    if (r < k) {
      if (out_c) out_c[r] = e;
      if (out_ids) {
        out_ids[r] = e.id;
        out_vals[r] = e.v;
      }
    }
  }
}

// The best k of the n shared-memory values vals[0..n) (entry i has id
// id0 + i), sorted, into out[0..k) -- padded with (-FLT_MAX, INT32_MAX) when
// fewer than k values are admissible (NaN and -inf are not).  The 64 groups
// (i mod 64) give maxima whose k-th best bounds the k-th best value from
// below (those maxima are k admissible values), so only values not worse than
// the bound are candidates.  Every thread of the CTA calls this.
__device__ void cta_topk(const float* vals, int n, int64_t id0, int k, HeadCand* tmp, HeadCand* cl, HeadCtl& C,
                         HeadCand* out) {
  const int t = threadIdx.x;
  if (t == 0) {
    C.bound = HeadCand{-FLT_MAX, INT32_MAX};
    C.n0 = 0;
  }
  // 1. group j = values i = j (mod 64); threads t < kGroupThreads: group t % 64
  if (t < kGroupThreads) {
    HeadCand best{-FLT_MAX, INT32_MAX};
    for (int i = t % kGroupsF + kGroupsF * (t / kGroupsF); i < n; i += kGroupThreads) {
      const float v = vals[i];
      const int32_t id = (int32_t)(id0 + i);
      if (v >= -FLT_MAX && better(v, id, best.v, best.id)) best = HeadCand{v, id};
    }
    tmp[t] = best;
  }
  __syncthreads();
  if (t < kGroupsF) {
    HeadCand b = tmp[t];
#pragma unroll 4
    for (int u = t + kGroupsF; u < kGroupThreads; u += kGroupsF)
      if (better(tmp[u].v, tmp[u].id, b.v, b.id)) b = tmp[u];
    C.gmax_v[t] = b.v;
    C.gmax_i[t] = b.id;
  }
  __syncthreads();
  // 2. the bound: the k-th best group maximum, if it is admissible
  if (t < kGroupsF) {
    const float mv = C.gmax_v[t];
    const int32_t mi = C.gmax_i[t];
    int rank = 0;
#pragma unroll 16
    for (int o = 0; o < kGroupsF; ++o) rank += better(C.gmax_v[o], C.gmax_i[o], mv, mi);
    if (rank == k - 1 && mi != INT32_MAX) C.bound = HeadCand{mv, mi};
  }
  __syncthreads();
  // 3. candidates (no bound: every admissible value)
  const HeadCand L = C.bound;
  for (int i0 = 0; i0 < n; i0 += kThreadsF) {
    const int i = i0 + t;
    HeadCand e{-FLT_MAX, INT32_MAX};
    bool keep = false;
    if (i < n) {
      e = HeadCand{vals[i], (int32_t)(id0 + i)};
      keep = e.v >= -FLT_MAX && !better(L.v, L.id, e.v, e.id);
    }
    warp_append(keep, e, cl, &C.n0, n);
  }
  __syncthreads();
  // 4. rank them
  const int nc = C.n0;
  rank_into(cl, nc, k, out, nullptr, nullptr);
  for (int r = nc + t; r < k; r += kThreadsF) out[r] = HeadCand{-FLT_MAX, INT32_MAX};
  __syncthreads();
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
                  HeadCand* __restrict__ cand)          // [gridDim][M][top_k]
{
  extern __shared__ __align__(128) uint8_t smem[];
  HeadCtl& C = *reinterpret_cast<HeadCtl*>(smem);
  const HeadGeo geo = head_geo(V, H, M, gridDim.x, stages, top_k);
  uint8_t* work = smem + kHeadCtlBytes;
  uint8_t* ring = work + geo.work_bytes;
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(work);  // [M][H], until the fragments are built
  float* red = reinterpret_cast<float*>(work);                    // [kRedF][kCons][M][16], after
  float* cvals = reinterpret_cast<float*>(work + geo.red_bytes);  // [M][n_cap]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int nsl = H / 64;
  const int64_t t_begin = geo.ntiles * blockIdx.x / gridDim.x;
  const int64_t t_end = geo.ntiles * (blockIdx.x + 1) / gridDim.x;
  const int ntl = (int)(t_end - t_begin);
  const uint32_t tile_bytes = (uint32_t)(kRows * H);

  auto issue = [&](int it) {  // the producer: tile t_begin + it into stage it % stages
    const int s = it % stages;
    const int64_t t = t_begin + it;
    const bool full_tile = (t + 1) * kRows <= V;  // a ragged last tile's scales are read from global
    uint8_t* dst = ring + (size_t)s * geo.stage_bytes;
    const uint64_t pol = l2_evict_first_policy();
    mbar_arrive_expect_tx(&C.full[s], tile_bytes + (full_tile ? 64u : 0u));
    bulk_g2s(dst, qt + (size_t)t * tile_bytes, tile_bytes, &C.full[s], pol);
    if (full_tile) bulk_g2s(dst + tile_bytes, row_scale + t * kRows, 64u, &C.full[s], pol);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], kCons);
    }
    for (int r = 0; r < kRedF; ++r) {
      mbar_init(&C.red_full[r], kCons);
      mbar_init(&C.red_empty[r], 1);
    }
    mbar_init(&C.xbar, 1);
    fence_mbar_init();
    C.poison = 0;
    const uint32_t xbytes = (uint32_t)(M * H * 2);
    mbar_arrive_expect_tx(&C.xbar, xbytes);
    bulk_g2s(work, x, xbytes, &C.xbar, l2_evict_last_policy());
  }
  __syncthreads();
  auto poisoned = [&]() -> bool { return *(volatile int*)&C.poison != 0; };
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {  // bounded; every lane polls
    if (poisoned()) return false;
    if (mbar_wait(bar, parity)) return true;
    report(hdr, MOE_ERR_TIMEOUT);
    atomicExch(&C.poison, 1);
    return false;
  };

  uint32_t bfrag[kS][2][2];
  float fx[kS];  // undoes the scale of token t's slice (columns 2t, 2t+1)
  if (warp == kProdWarp) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      for (int it = 0; it < ntl; ++it) {
        if (it >= stages && !wait(&C.empty[it % stages], (uint32_t)((it / stages - 1) & 1))) break;
        issue(it);
      }
    }
  } else {
    wait(&C.xbar, 0);
    // ---- per (token, slice) scale (consumers and epilogue warps) ----
    for (int u = threadIdx.x; u < M * nsl; u += kCons * 32) {
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
    // Lane (g, t), slice sl = warp + 20 si, MMA j, register r: elements
    // 64 sl + 16 t + 8 j + 4 r .. +3 of column g = part g & 1 of token g >> 1.
    if (warp < kCons) {
      const int m = g >> 1, part = g & 1;
#pragma unroll
      for (int si = 0; si < kS; ++si) {
        const int sl = warp + kCons * si;
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
      for (int it = 0; it < ntl; ++it) {
        const int s = it % stages;
        wait(&C.full[s], (uint32_t)((it / stages) & 1));
        const uint8_t* st = ring + (size_t)s * geo.stage_bytes;
        uint4 a[kS], b[kS];
#pragma unroll
        for (int si = 0; si < kS; ++si) {
          const int sl = warp + kCons * si;
          if (sl < nsl) {
            a[si] = *reinterpret_cast<const uint4*>(st + sl * 1024 + lane * 16);        // row g
            b[si] = *reinterpret_cast<const uint4*>(st + sl * 1024 + 512 + lane * 16);  // row g + 8
          }
        }
        float rs = 0.f;  // warp 0 carries the tile's row scales to the epilogue
        const int64_t row = (t_begin + it) * kRows + lane;
        if (warp == 0 && lane < kRows && row < V)
          rs = (t_begin + it + 1) * kRows <= V ? *reinterpret_cast<const float*>(st + tile_bytes + 4 * lane)
                                                : __ldg(row_scale + row);
        float ag = 0.f, ag8 = 0.f;  // rows g and g + 8, token t
#pragma unroll
        for (int si = 0; si < kS; ++si) {
          const int sl = warp + kCons * si;
          if (sl < nsl) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_e4m3(d, a[si].x, b[si].x, a[si].y, b[si].y, bfrag[si][0][0], bfrag[si][0][1]);
            mma_e4m3(d, a[si].z, b[si].z, a[si].w, b[si].w, bfrag[si][1][0], bfrag[si][1][1]);
            ag = fmaf(d[0] + d[1], fx[si], ag);
            ag8 = fmaf(d[2] + d[3], fx[si], ag8);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[s]);  // this warp is done with the stage
        const int r = it % kRedF;
        if (it >= kRedF) wait(&C.red_empty[r], (uint32_t)(((it / kRedF) & 1) ^ 1));
        float* rb = red + ((size_t)r * kCons + warp) * M * kRows;
        if (tq < M) {
          rb[tq * kRows + g] = ag;
          rb[tq * kRows + g + 8] = ag8;
        }
        if (warp == 0 && lane < kRows) C.rsc[r][lane] = rs;
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.red_full[r]);
      }
    } else {
      // ------------------------------ epilogue ------------------------------
      const int e = warp - kEpi0;
      for (int it = e; it < ntl; it += kNumEpi) {
        const int r = it % kRedF;
        wait(&C.red_full[r], (uint32_t)((it / kRedF) & 1));
        const float* rb = red + (size_t)r * kCons * M * kRows;
        for (int idx = lane; idx < M * kRows; idx += 32) {
          const int m = idx / kRows, rr = idx - m * kRows;
          const int64_t row = (t_begin + it) * kRows + rr;
          float v = 0.f;
#pragma unroll 4
          for (int w = 0; w < kCons; ++w) v += rb[(w * M + m) * kRows + rr];
          v *= C.rsc[r][rr];
          if (row < V) {
            if (logits) logits[(size_t)m * V + row] = v;
            cvals[m * geo.n_cap + it * kRows + rr] = v;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.red_empty[r]);
      }
    }
  }
  __syncthreads();  // every tile consumed: the ring is free

  // ---- this CTA's top-k per token ----
  const int n_local = (int)((t_end * kRows < V ? t_end * kRows : V) - t_begin * kRows);
  HeadCand* tmp = reinterpret_cast<HeadCand*>(ring);  // [kThreadsF]
  HeadCand* cl = tmp + kThreadsF;                     // [n_cap]
  for (int m = 0; m < M; ++m)
    cta_topk(cvals + m * geo.n_cap, n_local, t_begin * kRows, top_k, tmp, cl, C,
             cand + ((size_t)blockIdx.x * M + m) * top_k);

  // ---- the last CTA merges every CTA's lists ----
  __threadfence();  // this CTA's lists, before it counts itself done
  __syncthreads();
  if (threadIdx.x == 0) C.last = atomicAdd(&hdr->ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!C.last) return;
  __threadfence();
  const int G = gridDim.x, k = top_k;
  // Every token's lists at once when they fit in the ring, else one token at
  // a time; the loads of a pass are all issued before any is stored.
  const size_t per_tok = (size_t)G * k * sizeof(HeadCand);
  const size_t fixed = (size_t)k * k * sizeof(HeadCand) + (size_t)G * sizeof(int);
  const int tpp = (per_tok * M + fixed <= geo.ring_bytes) ? M : 1;  // tokens per pass
  HeadCand* lists = reinterpret_cast<HeadCand*>(ring);                  // [tpp][G][k]
  HeadCand* surv = lists + (size_t)tpp * G * k;                         // [k * k]
  int* qual = reinterpret_cast<int*>(surv + (size_t)k * k);             // [G]
  for (int m0 = 0; m0 < M; m0 += tpp) {
    const int n = tpp * G * k;  // entry i: token m0 + i / (G k), list (i / k) % G, rank i % k
    for (int i0 = 0; i0 < n; i0 += 8 * kThreadsF) {
      HeadCand e[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kThreadsF + threadIdx.x;
        if (i < n) {
          const int mm = m0 + i / (G * k), c2 = (i / k) % G, j = i % k;
          const HeadCand* src = cand + ((size_t)c2 * M + mm) * k + j;
          e[u] = HeadCand{__ldcg(&src->v), __ldcg(&src->id)};
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kThreadsF + threadIdx.x;
        if (i < n) lists[i] = e[u];
      }
    }
    __syncthreads();
    for (int m = m0; m < m0 + tpp; ++m) {
      const HeadCand* lm = lists + (size_t)(m - m0) * G * k;
      if (threadIdx.x == 0) {
        C.bound = HeadCand{-FLT_MAX, INT32_MAX};
        C.n0 = C.n1 = 0;
      }
      __syncthreads();
      // 1. L = the k-th best list head (none: fewer than k admissible heads)
      for (int c2 = threadIdx.x; c2 < G; c2 += kThreadsF) {
        const HeadCand h = lm[(size_t)c2 * k];
        int rank = 0;
#pragma unroll 8
        for (int o = 0; o < G; ++o) rank += better(lm[(size_t)o * k].v, lm[(size_t)o * k].id, h.v, h.id);
        if (rank == k - 1 && h.id != INT32_MAX) C.bound = h;
      }
      __syncthreads();
      const HeadCand L = C.bound;
      // 2. lists whose head is not worse than L (at most k of them)
      for (int c0 = 0; c0 < G; c0 += kThreadsF) {
        const int c2 = c0 + threadIdx.x;
        bool keep = false;
        if (c2 < G) {
          const HeadCand h = lm[(size_t)c2 * k];
          keep = h.id != INT32_MAX && !better(L.v, L.id, h.v, h.id);
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&C.n1, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (keep) qual[base + __popc(bal & ((1u << lane) - 1u))] = c2;
      }
      __syncthreads();
      // 3. their entries not worse than L (at most k * k survivors)
      const int nq = C.n1;
      for (int i0 = 0; i0 < nq * k; i0 += kThreadsF) {
        const int i = i0 + threadIdx.x;
        HeadCand e{-FLT_MAX, INT32_MAX};
        bool keep = false;
        if (i < nq * k) {
          e = lm[(size_t)qual[i / k] * k + (i % k)];
          keep = e.id != INT32_MAX && !better(L.v, L.id, e.v, e.id);
        }
        warp_append(keep, e, surv, &C.n0, k * k);
      }
      __syncthreads();
      // 4. rank the survivors
      const int ns = min(C.n0, k * k);
      rank_into(surv, ns, k, nullptr, out_ids + m * k, out_vals + m * k);
      for (int r = ns + threadIdx.x; r < k; r += kThreadsF) {  // fewer admissible values than k
        out_ids[m * k + r] = INT32_MAX;
        out_vals[m * k + r] = -FLT_MAX;
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) hdr->ticket = 0u;
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
  lmhead_fp8_kernel<kS><<<grid, kThreadsF, smem, st>>>(x, qt, s, V, H, M, top_k, stages, logits, ids, vals, hdr,
                                                      reinterpret_cast<HeadCand*>(cand));
  return cudaGetLastError();
}

}  // namespace

bool lmhead_fp8_plan(int H, int M, int top_k, int64_t V, int grid, int* stages, size_t* smem) {
  if (H < 64 || H % 64 != 0 || H > kMaxHF || M < 1 || M > 4 || top_k < 1 || top_k > 64) return false;
  for (int st = kMaxStagesF; st >= 2; --st) {
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

size_t lmhead_cand_bytes(int grid, int M, int top_k) { return (size_t)grid * M * top_k * sizeof(HeadCand); }

cudaError_t launch_lmhead_fp8(const uint16_t* x, const uint8_t* qt, const float* s, int64_t V, int H, int M,
                              int top_k, float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand,
                              int grid, cudaStream_t st) {
  int stages = 0;
  size_t smem = 0;
  if (!lmhead_fp8_plan(H, M, top_k, V, grid, &stages, &smem)) return cudaErrorInvalidConfiguration;
  const int need = (H / 64 + kWarpsF - 1) / kWarpsF;
  switch (need) {
    case 1: return launch_fp8_t<1>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 2: return launch_fp8_t<2>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 3: return launch_fp8_t<3>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    case 4: return launch_fp8_t<4>(x, qt, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, stages, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
