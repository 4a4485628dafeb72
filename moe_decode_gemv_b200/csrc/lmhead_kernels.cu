// lmhead_kernels.cu -- the BF16 comparator head: the same GEMV + top-k as the
// FP8 head (lmhead_fp8.cu), without a row scale, over the unquantised BF16
// [V][H] head, which the FP8 head halves in bytes.  One pass over the head
// for all M tokens, fused with an optional logits write and a top-k.
//
// The pages: quantising only the vocabulary projection to FP8 at load time
// halves the bytes each token reads (ncijnetwork.com summary, "What are the 3
// optimizations?", item 2; generativeaipub.com blog, "2. Compressing the
// Output Head"); this kernel is the BF16 side of that comparison.
//
// Design (sm_100a, one GPU):
//  * One CTA per SM, persistent over a contiguous range of 16-row tiles.
//  * A producer warp streams tiles HBM -> shared memory with bulk copies
//    (cp.async.bulk, no multicast) into a ring of stages guarded by
//    mbarriers; rows are copied one by one into a padded stride so that the
//    consumers' 16-byte shared loads are free of bank conflicts.
//  * Eight consumer warps split K, each computing 16 rows x 8 token columns
//    with mma.sync m16n8k16 (bf16 x bf16 -> fp32); the B fragments hold the
//    tokens and stay in registers for the whole kernel.
//  * Two epilogue warps, on alternate tiles, sum the consumers' partials,
//    write logits when asked and keep each value in shared memory; after the stream one warp per
//    token takes the CTA's top-k, and the last CTA to finish merges all
//    CTAs' lists (ties to the lower id).
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "device_cache.h"
#include "lmhead.h"

namespace moe {
namespace {

constexpr int kTileRows = 16;
constexpr int kConsumerWarps = 8;
constexpr int kEpilogueWarps = 2;  // alternate tiles
constexpr int kThreads = (kConsumerWarps + 1 + kEpilogueWarps) * 32;  // consumers + producer + epilogue
constexpr int kMaxSlicesPerWarp = 10;  // row bytes <= 10 * 8 * 64 = 5120: H <= 5120 (fp8), 2560 (bf16)
constexpr size_t kMaxSmem = kMaxDynamicSmem;

template <typename W>
struct HeadTraits;

// FP8 E4M3 weights: a 64-byte K slice is 64 elements = 2 MMAs of k32, each
// run twice (hi and lo parts of the activations): 4 MMAs per slice.
template <>
struct HeadTraits<uint8_t> {
  static constexpr int kElemBytes = 1;
  static constexpr int kMmasPerSlice = 4;
};
// BF16 weights: a 64-byte K slice is 32 elements; 2 MMAs of k16 each.
template <>
struct HeadTraits<uint16_t> {
  static constexpr int kElemBytes = 2;
  static constexpr int kMmasPerSlice = 2;
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__host__ __device__ constexpr int padded_stride(int row_bytes) {
  // Rows are a multiple of 64 bytes.  A stride of 64 (mod 128) bytes puts rows
  // g and g+1 on opposite halves of the 32 banks, so each quarter-warp of a
  // 16-byte shared load is conflict-free.
  return (row_bytes % 128 == 0) ? row_bytes + 64 : row_bytes;
}

// One ring stage: 16 rows at the padded stride, then the 16 rows' fp32 scales
// (64 B), rounded up to 128 B.  (Measured: one contiguous 40 KB copy per tile
// into unpadded rows streams no faster than 16 row copies, and its shared
// loads take two wavefronts instead of one.)
__host__ __device__ constexpr int stage_bytes(int row_bytes) {
  return (kTileRows * padded_stride(row_bytes) + 64 + 127) / 128 * 128;
}

struct Cand {
  float v;
  int32_t id;
};

constexpr uint32_t kFull = 0xffffffffu;

// A sorted top-k list (k <= 64) held in one warp's registers: rank r < 32 sits
// in lane r of row 0, rank 32 + r in lane r of row 1.  Ranks >= k are unused.
// Empty entries are (-FLT_MAX, INT32_MAX), below every admissible candidate.
// (tv, ti), replicated in every lane, is the entry at rank k - 1: a candidate
// enters only if it is better than that one.
struct WarpList {
  float v0, v1;
  int32_t i0, i1;
  float tv;
  int32_t ti;
};

__device__ __forceinline__ void list_init(WarpList& L) {
  L.v0 = L.v1 = L.tv = -FLT_MAX;
  L.i0 = L.i1 = L.ti = INT32_MAX;
}

// Insert (cv, ci), known to be better than the threshold (warp-uniform call).
// Its rank p is the number of kept entries better than it; entries at ranks
// >= p move down one place and the one at rank k - 1 drops out.
__device__ __forceinline__ void list_insert(WarpList& L, float cv, int32_t ci, int k, int lane) {
  const uint32_t m0 = k >= 32 ? kFull : ((1u << k) - 1u);
  int p = __popc(__ballot_sync(kFull, better(L.v0, L.i0, cv, ci)) & m0);
  if (k > 32) {
    const uint32_t m1 = k >= 64 ? kFull : ((1u << (k - 32)) - 1u);
    p += __popc(__ballot_sync(kFull, better(L.v1, L.i1, cv, ci)) & m1);
    float u = __shfl_up_sync(kFull, L.v1, 1);
    int32_t j = __shfl_up_sync(kFull, L.i1, 1);
    const float carry_v = __shfl_sync(kFull, L.v0, 31);  // rank 31 moves to rank 32
    const int32_t carry_i = __shfl_sync(kFull, L.i0, 31);
    if (lane == 0) { u = carry_v; j = carry_i; }
    if (32 + lane > p) { L.v1 = u; L.i1 = j; }
    else if (32 + lane == p) { L.v1 = cv; L.i1 = ci; }
  }
  const float u = __shfl_up_sync(kFull, L.v0, 1);
  const int32_t j = __shfl_up_sync(kFull, L.i0, 1);
  if (lane > p) { L.v0 = u; L.i0 = j; }
  else if (lane == p) { L.v0 = cv; L.i0 = ci; }
  const int t = k - 1;
  L.tv = __shfl_sync(kFull, t < 32 ? L.v0 : L.v1, t & 31);
  L.ti = __shfl_sync(kFull, t < 32 ? L.i0 : L.i1, t & 31);
}

// Offer one candidate per lane (ignored where !valid).  Candidates that beat
// the threshold are inserted one at a time, lowest lane first, re-testing the
// rest against the raised threshold after each insertion.
__device__ __forceinline__ void list_offer(WarpList& L, float v, int32_t id, bool valid, int k, int lane) {
  uint32_t bal = __ballot_sync(kFull, valid && better(v, id, L.tv, L.ti));
  while (bal) {
    const int src = __ffs(bal) - 1;
    const float cv = __shfl_sync(kFull, v, src);
    const int32_t ci = __shfl_sync(kFull, id, src);
    list_insert(L, cv, ci, k, lane);
    bal &= (bal - 1u) & __ballot_sync(kFull, valid && better(v, id, L.tv, L.ti));
  }
}

constexpr int kCandCap = 256;  // candidates a warp ranks by counting (more: the list path)

// The best k (<= 64) of vals[0..n) under `better`, entry i carrying the id
// row0 + i, by one warp; writes the sorted list (padded with empty entries
// when fewer than k are admissible) to out[0..k).  NaN and -inf values are
// not admissible.  The values fall into 64 groups (i mod 64); the k-th best
// of the group maxima, L, is a lower bound on the k-th best value (those are
// k real entries), so only values not worse than L can be selected -- a few
// dozen -- and they are ranked by counting.  `scratch` holds kCandCap entries.
__device__ void warp_topk_rows(const float* vals, int n, int64_t row0, int k, int lane, Cand* scratch, Cand* out) {
  // 1. group maxima: value i is in group i mod 64 (lane i mod 32, row (i / 32) mod 2)
  float m0 = -FLT_MAX, m1 = -FLT_MAX;
  int32_t j0 = INT32_MAX, j1 = INT32_MAX;
  for (int b = 0; b < n; b += 256) {  // 8 loads in flight per step
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = b + 32 * u + lane;
      v[u] = i < n ? vals[i] : -FLT_MAX;
    }
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
      const int i0 = b + 32 * u + lane, i1 = i0 + 32;
      const int32_t id0 = (int32_t)(row0 + i0), id1 = (int32_t)(row0 + i1);
      if (i0 < n && better(v[u], id0, m0, j0)) { m0 = v[u]; j0 = id0; }
      if (i1 < n && better(v[u + 1], id1, m1, j1)) { m1 = v[u + 1]; j1 = id1; }
    }
  }
  // 2. L = the k-th best group maximum
  int r0 = 0, r1 = 0;
#pragma unroll 8
  for (int j = 0; j < 32; ++j) {
    const float a = __shfl_sync(kFull, m0, j), b = __shfl_sync(kFull, m1, j);
    const int32_t ai = __shfl_sync(kFull, j0, j), bi = __shfl_sync(kFull, j1, j);
    r0 += better(a, ai, m0, j0) + better(b, bi, m0, j0);
    r1 += better(a, ai, m1, j1) + better(b, bi, m1, j1);
  }
  // real maxima have distinct ids, so at most one has rank k - 1; none when
  // fewer than k groups hold an admissible value (then there is no bound)
  const uint32_t s0 = __ballot_sync(kFull, r0 == k - 1 && j0 != INT32_MAX);
  const uint32_t s1 = __ballot_sync(kFull, r1 == k - 1 && j1 != INT32_MAX);
  float Lv = -FLT_MAX;
  int32_t Li = INT32_MAX;
  if (s0) {
    Lv = __shfl_sync(kFull, m0, __ffs(s0) - 1);
    Li = __shfl_sync(kFull, j0, __ffs(s0) - 1);
  } else if (s1) {
    Lv = __shfl_sync(kFull, m1, __ffs(s1) - 1);
    Li = __shfl_sync(kFull, j1, __ffs(s1) - 1);
  }
  // 3. candidates: admissible values not worse than L, gathered in one pass
  //    (a ballot per 32 values gives each its slot)
  int nc = 0;
  for (int b = 0; b < n; b += 256) {  // 8 loads in flight per step
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = b + 32 * u + lane;
      v[u] = i < n ? vals[i] : -FLT_MAX;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = b + 32 * u + lane;
      const int32_t id = (int32_t)(row0 + i);
      const bool keep = i < n && v[u] >= -FLT_MAX && !better(Lv, Li, v[u], id);
      const uint32_t bal = __ballot_sync(kFull, keep);
      const int pos = nc + __popc(bal & ((1u << lane) - 1u));
      if (keep && pos < kCandCap) scratch[pos] = Cand{v[u], id};
      nc += __popc(bal);
    }
  }
  __syncwarp();
  if (nc <= kCandCap) {
    // 4. rank by counting; ranks are distinct because ids are
    for (int q = lane; q < nc; q += 32) {
      const Cand e = scratch[q];
      int r = 0;
#pragma unroll 8
      for (int o = 0; o < nc; ++o) {
        const Cand f = scratch[o];
        r += better(f.v, f.id, e.v, e.id);
      }
      if (r < k) out[r] = e;
    }
    for (int j = nc + lane; j < k; j += 32) out[j] = Cand{-FLT_MAX, INT32_MAX};
  } else {  // heavy ties: a sorted register list over every value
    WarpList L;
    list_init(L);
    for (int b = 0; b < n; b += 32) {
      const bool valid = b + lane < n;
      list_offer(L, valid ? vals[b + lane] : -FLT_MAX, (int32_t)(row0 + b + lane), valid, k, lane);
    }
    if (lane < k) out[lane] = Cand{L.v0, L.i0};
    if (32 + lane < k) out[32 + lane] = Cand{L.v1, L.i1};
  }
  __syncwarp();
}

// The end of every head kernel, run by the whole CTA once its rows' values
// (cvals [M][n_cap], rows t_begin * 16 ...) are in shared memory: this CTA's
// top-k per token (one warp per token, warp_scratch holds M * kCandCap
// entries), then the last CTA to finish merges every CTA's lists.
__device__ void head_tail(const float* cvals, int n_cap, Cand* warp_scratch, int64_t t_begin, int64_t t_end,
                          int64_t V, int M, int top_k, int warp, int lane, WsHeader* hdr, Cand* cand, uint8_t* smem,
                          int* s_last, int32_t* out_ids, float* out_vals) {
  // ------------------- this CTA's top-k, one warp per token -------------------
  __syncthreads();
  if (warp < M) {
    const int64_t row0 = t_begin * kTileRows;
    const int n_local = (int)((t_end * kTileRows < V ? t_end * kTileRows : V) - row0);
    warp_topk_rows(cvals + (size_t)warp * n_cap, n_local, row0, top_k, lane,
                   warp_scratch + warp * kCandCap, cand + ((size_t)blockIdx.x * M + warp) * top_k);
    __threadfence();  // this list, before the CTA counts itself done (only the lists are read by the merge)
  }

  // ------------------------- all lists written? ----------------------------
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t tk = atomicAdd(&hdr->ticket, 1u);
    *s_last = (tk == gridDim.x - 1);
  }
  __syncthreads();
  const bool last = *s_last;
  __syncthreads();  // every thread holds the flag before the merge reuses shared memory
  if (!last) return;
  __threadfence();

  // ------------------------ last CTA: merge the lists ------------------------
  // Per token, over G sorted lists of k entries (G = gridDim.x):
  //  1. L = the k-th best of the lists' first entries.  Those are k real
  //     candidates, so the global k-th best is not worse than L, and only
  //     entries not worse than L can be in the top k.
  //  2. Only a list whose first entry is not worse than L can hold such an
  //     entry: exactly k lists (all G when G < k), so at most k * k survivors.
  //  3. Each survivor's rank is the number of survivors better than it; ranks
  //     are distinct because ids are.  Ranks below k are the output.
  // Every step is spread over the whole CTA; all of shared memory is free by now.
  const int G = (int)gridDim.x;
  Cand* heads = reinterpret_cast<Cand*>(smem);                       // [G]
  int* qual = reinterpret_cast<int*>(heads + G);                     // [G]
  Cand* surv = reinterpret_cast<Cand*>(qual + ((G + 1) & ~1));       // [k * k]
  int* s_cnt = reinterpret_cast<int*>(surv + (size_t)top_k * top_k); // [2]: lists, survivors
  Cand* s_bound = reinterpret_cast<Cand*>(s_cnt + 2);
  for (int m = 0; m < M; ++m) {
    for (int c = threadIdx.x; c < G; c += blockDim.x) {
      const Cand* src = cand + ((size_t)c * M + m) * top_k;
      heads[c] = Cand{__ldcg(&src->v), __ldcg(&src->id)};
    }
    if (threadIdx.x == 0) {
      s_cnt[0] = s_cnt[1] = 0;
      *s_bound = Cand{-FLT_MAX, INT32_MAX};  // no bound when G < k
    }
    __syncthreads();
    for (int c = threadIdx.x; c < G; c += blockDim.x) {
      const Cand h = heads[c];
      int rank = 0;
#pragma unroll 8
      for (int o = 0; o < G; ++o) {
        const Cand e = heads[o];
        rank += better(e.v, e.id, h.v, h.id);
      }
      if (rank == top_k - 1) *s_bound = h;
    }
    __syncthreads();
    const Cand L = *s_bound;
    for (int c = threadIdx.x; c < G; c += blockDim.x)
      if (!better(L.v, L.id, heads[c].v, heads[c].id)) qual[atomicAdd(&s_cnt[0], 1)] = c;
    __syncthreads();
    const int nq = s_cnt[0];
    for (int i = threadIdx.x; i < nq * top_k; i += blockDim.x) {
      const int c = qual[i / top_k], j = i - (i / top_k) * top_k;
      const Cand* src = cand + ((size_t)c * M + m) * top_k + j;
      const Cand e{__ldcg(&src->v), __ldcg(&src->id)};
      if (e.id != INT32_MAX && !better(L.v, L.id, e.v, e.id)) {
        const int pos = atomicAdd(&s_cnt[1], 1);
        if (pos < top_k * top_k) surv[pos] = e;  // never false: at most k lists hold survivors
      }
    }
    __syncthreads();
    const int ns = min(s_cnt[1], top_k * top_k);
    for (int i = threadIdx.x; i < ns; i += blockDim.x) {
      const Cand e = surv[i];
      int rank = 0;
#pragma unroll 8
      for (int o = 0; o < ns; ++o) {
        const Cand f = surv[o];
        rank += better(f.v, f.id, e.v, e.id);
      }
      if (rank < top_k) {
        out_ids[m * top_k + rank] = e.id;
        out_vals[m * top_k + rank] = e.v;
      }
    }
    // fewer admissible candidates than k (only when logits are NaN or -inf): pad
    for (int j = ns + threadIdx.x; j < top_k; j += blockDim.x) {
      out_ids[m * top_k + j] = INT32_MAX;
      out_vals[m * top_k + j] = -FLT_MAX;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) hdr->ticket = 0u;
}

// Warp roles: warp 0..7 consumers (K split), warp 8 producer (bulk copies),
// warp 9 epilogue (cross-warp sum, row scale, logits, top-k).  Consumers hand
// each tile's partial sums to the epilogue warp through kRed buffers guarded
// by mbarriers, so no CTA-wide barrier sits in the streaming loop.
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kRed = 4;

template <typename W, int kSlices>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_topk_kernel(const uint16_t* __restrict__ x,       // [M][H] bf16
                   const W* __restrict__ w,              // [V][H]
                   const float* __restrict__ row_scale,  // [V] or nullptr (bf16 head)
                   int64_t V, int H, int M, int top_k, int stages,
                   float* __restrict__ logits,           // [M][V] or nullptr
                   int32_t* __restrict__ out_ids,        // [M][top_k]
                   float* __restrict__ out_vals,         // [M][top_k]
                   WsHeader* __restrict__ hdr,
                   Cand* __restrict__ cand)              // [gridDim][M][top_k]
{
  using T = HeadTraits<W>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int row_bytes = H * T::kElemBytes;
  const int stride = padded_stride(row_bytes);
  const int tile_bytes = stage_bytes(row_bytes);  // 16 rows at `stride`, then their 16 fp32 row scales
  const int scale_off = kTileRows * stride;

  const int64_t ntiles = (V + kTileRows - 1) / kTileRows;
  const int n_cap = (int)((ntiles + gridDim.x - 1) / gridDim.x) * kTileRows;  // rows of the largest CTA range

  // shared-memory carve-up: [ring][reduce buffers][row scales][logits of this CTA's rows][barriers][scalars]
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(ring + (size_t)stages * tile_bytes);  // [kRed][8][16][4]
  float* rsc = red + kRed * kConsumerWarps * kTileRows * 4;                    // [kRed][16] row scales
  float* cvals = rsc + kRed * kTileRows;                                       // [M][n_cap]
  uint64_t* full = reinterpret_cast<uint64_t*>(cvals + (size_t)M * ((n_cap + 1) & ~1));
  uint64_t* empty = full + stages;
  uint64_t* red_full = empty + stages;
  uint64_t* red_empty = red_full + kRed;
  int* s_sigma = reinterpret_cast<int*>(red_empty + kRed);  // [4]
  int* s_poison = s_sigma + 4;  // set once any bounded wait ran out
  int* s_last = s_sigma + 5;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t_begin = ntiles * blockIdx.x / gridDim.x;
  const int64_t t_end = ntiles * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int r = 0; r < kRed; ++r) {
      mbar_init(&red_full[r], kConsumerWarps);
      mbar_init(&red_empty[r], 1);
    }
    fence_mbar_init();
    *s_poison = 0;
  }
  // per-token power-of-two scale for the f16 activations (fp8 head only)
  if (warp < M) {
    float amax = 0.f;
#pragma unroll 8
    for (int j = lane; j < H; j += 32) amax = fmaxf(amax, fabsf(bf16_bits_to_f32(x[(size_t)warp * H + j])));
    amax = warp_max(amax);
    if (lane == 0) {
      int sigma = 0;
      if (sizeof(W) == 1 && amax > 0.f) {
        int e = (int)((__float_as_uint(amax) >> 23) & 0xff);
        int fl = e ? e - 127 : (31 - __clz(__float_as_uint(amax) & 0x7fffff)) - 149;
        sigma = 7 - fl;  // max |x * 2^sigma| in [2^7, 2^8): inside E4M3's normal range
        sigma = sigma > 126 ? 126 : (sigma < -126 ? -126 : sigma);
      }
      s_sigma[warp] = sigma;
    }
  }
  __syncthreads();

  // bounded wait shared by all roles: lane 0 polls, the warp agrees on the result
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    bool ok = !*(volatile int*)s_poison;
    if (ok && lane == 0) ok = mbar_wait(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0 && !*(volatile int*)s_poison) {
      report(hdr, MOE_ERR_TIMEOUT);
      atomicExch(s_poison, 1);
    }
    return ok;
  };

  if (warp == kProducerWarp) {
    // ------------------------------ producer ------------------------------
    const uint64_t policy = l2_evict_first_policy();
    int64_t it = 0, issued = 0;
    for (int64_t t = t_begin; t < t_end; ++t, ++it) {
      const int s = (int)(it % stages);
      const uint32_t ph = (uint32_t)((it / stages) & 1);
      if (it >= stages && !wait_all(&empty[s], ph ^ 1u)) continue;  // after a timeout: issue nothing more
      if (*(volatile int*)s_poison) continue;
      const int64_t r0 = t * kTileRows;
      const int nrows = (int)(V - r0 < kTileRows ? V - r0 : kTileRows);
      // the row scales travel with the tile: 16 B per 4 rows (a ragged last
      // tile's 1..3 leftover scales are read from global by the epilogue)
      const uint32_t sbytes = row_scale ? (uint32_t)(nrows & ~3) * 4u : 0u;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * row_bytes) + sbytes);
      __syncwarp();
      uint8_t* stage = ring + (size_t)s * tile_bytes;
      if (lane < nrows)
        bulk_g2s(stage + (size_t)lane * stride, reinterpret_cast<const uint8_t*>(w) + (size_t)(r0 + lane) * row_bytes,
                 (uint32_t)row_bytes, &full[s], policy);
      if (lane == 16 && sbytes) bulk_g2s(stage + scale_off, row_scale + r0, sbytes, &full[s], policy);
      issued = it + 1;
    }
    // every issued copy must land before this CTA may exit
    if (lane == 0) {
      const int64_t first = issued > stages ? issued - stages : 0;
      for (int64_t j = first; j < issued; ++j) mbar_wait(&full[j % stages], (uint32_t)((j / stages) & 1));
    }
  } else if (warp < kConsumerWarps) {
    // ------------------------------ consumers -----------------------------
    const int g = lane >> 2, tq = lane & 3;
    // B fragments: token n = g, this warp's K slices, resident for the whole kernel.
    // FP8 head: the token, scaled by 2^sigma, is split into two E4M3 parts,
    // x' = hi + lo, exact for every element of scaled magnitude 2^-2 or more
    // (the rest within 2^-17 of the token's largest).  Each part takes its own
    // MMA; the weights enter the MMA as raw E4M3 bytes.
    uint32_t bfrag[kSlices][T::kMmasPerSlice][2];
    {
      const bool live = g < M;
      const float scl = live ? __uint_as_float((uint32_t)(127 + s_sigma[g]) << 23) : 0.f;
#pragma unroll
      for (int si = 0; si < kSlices; ++si) {
        const int slice = warp + si * kConsumerWarps;
        const bool in = live && slice * 64 < row_bytes;
        if constexpr (sizeof(W) == 1) {
          const int e0 = slice * 64 + tq * 16;
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // four groups of 4 elements: mma (q / 2), register (q % 2)
            uint32_t hw = 0u, lw = 0u;
            if (in) {
              const uint2 p = *reinterpret_cast<const uint2*>(x + (size_t)g * H + e0 + 4 * q);
              const float v0 = bf16_bits_to_f32(p.x & 0xffffu) * scl, v1 = bf16_bits_to_f32(p.x >> 16) * scl;
              const float v2 = bf16_bits_to_f32(p.y & 0xffffu) * scl, v3 = bf16_bits_to_f32(p.y >> 16) * scl;
              const uint32_t h01 = f32x2_to_e4m3x2(v0, v1), h23 = f32x2_to_e4m3x2(v2, v3);
              const uint32_t f01 = e4m3x2_to_f16x2(h01), f23 = e4m3x2_to_f16x2(h23);
              const float2 r01 = __half22float2(*reinterpret_cast<const __half2*>(&f01));
              const float2 r23 = __half22float2(*reinterpret_cast<const __half2*>(&f23));
              hw = h01 | (h23 << 16);
              lw = f32x2_to_e4m3x2(v0 - r01.x, v1 - r01.y) | (f32x2_to_e4m3x2(v2 - r23.x, v3 - r23.y) << 16);
            }
            bfrag[si][2 * (q / 2)][q % 2] = hw;      // j = 0 (mma 0, hi), 2 (mma 1, hi)
            bfrag[si][2 * (q / 2) + 1][q % 2] = lw;  // j = 1 (mma 0, lo), 3 (mma 1, lo)
          }
        } else {
          const int e0 = slice * 32 + tq * 8;
#pragma unroll
          for (int j = 0; j < T::kMmasPerSlice; ++j) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
              const int k0 = e0 + 4 * j + 2 * p;
              bfrag[si][j][p] = in ? *reinterpret_cast<const uint32_t*>(x + (size_t)g * H + k0) : 0u;
            }
          }
        }
      }
    }

    int64_t it = 0;
    for (int64_t t = t_begin; t < t_end; ++t, ++it) {
      const int s = (int)(it % stages);
      const bool ok = wait_all(&full[s], (uint32_t)((it / stages) & 1));
      // one accumulator per MMA index: four independent chains instead of one
      float acc[T::kMmasPerSlice][4];
#pragma unroll
      for (int j = 0; j < T::kMmasPerSlice; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      if (ok) {
        const uint8_t* tile = ring + (size_t)s * tile_bytes;
        uint4 ra[kSlices], rb[kSlices];
#pragma unroll
        for (int si = 0; si < kSlices; ++si) {  // all shared loads of the tile first
          const int slice = warp + si * kConsumerWarps;
          if (slice * 64 < row_bytes) {
            ra[si] = *reinterpret_cast<const uint4*>(tile + (size_t)g * stride + slice * 64 + tq * 16);
            rb[si] = *reinterpret_cast<const uint4*>(tile + (size_t)(g + 8) * stride + slice * 64 + tq * 16);
          }
        }
#pragma unroll
        for (int si = 0; si < kSlices; ++si) {
          const int slice = warp + si * kConsumerWarps;
          if (slice * 64 < row_bytes) {
            const uint32_t wa[4] = {ra[si].x, ra[si].y, ra[si].z, ra[si].w};
            const uint32_t wb[4] = {rb[si].x, rb[si].y, rb[si].z, rb[si].w};
            if constexpr (sizeof(W) == 1) {
              // rows g and g+8, 16 bytes each: words 0,1 feed MMA 0 and words 2,3 MMA 1
              mma_e4m3(acc[0], wa[0], wb[0], wa[1], wb[1], bfrag[si][0][0], bfrag[si][0][1]);
              mma_e4m3(acc[1], wa[0], wb[0], wa[1], wb[1], bfrag[si][1][0], bfrag[si][1][1]);
              mma_e4m3(acc[2], wa[2], wb[2], wa[3], wb[3], bfrag[si][2][0], bfrag[si][2][1]);
              mma_e4m3(acc[3], wa[2], wb[2], wa[3], wb[3], bfrag[si][3][0], bfrag[si][3][1]);
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t a[4] = {wa[2 * j], wb[2 * j], wa[2 * j + 1], wb[2 * j + 1]};
                mma_bf16(acc[j], a, bfrag[si][j][0], bfrag[si][j][1]);
              }
            }
          }
        }
      }
      float d[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        d[q] = acc[0][q];
#pragma unroll
        for (int j = 1; j < T::kMmasPerSlice; ++j) d[q] += acc[j][q];
      }
      // warp 0 also passes the tile's row scales on (the stage is recycled next)
      float sc = 1.0f;
      if (warp == 0 && lane < kTileRows && row_scale && ok)
        sc = *reinterpret_cast<const float*>(ring + (size_t)s * tile_bytes + scale_off + lane * 4);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // hand the partial sums to the epilogue warp of this tile
      const int r = (int)(it % kRed);
      if (it >= kRed) wait_all(&red_empty[r], (uint32_t)(((it / kRed) & 1) ^ 1));
      float* rb = red + (size_t)r * kConsumerWarps * kTileRows * 4;
      if (warp == 0 && lane < kTileRows) rsc[r * kTileRows + lane] = sc;
      if (tq < 2) {  // tokens 2tq, 2tq+1 (M <= 4)
        rb[(warp * kTileRows + g) * 4 + 2 * tq] = d[0];
        rb[(warp * kTileRows + g) * 4 + 2 * tq + 1] = d[1];
        rb[(warp * kTileRows + g + 8) * 4 + 2 * tq] = d[2];
        rb[(warp * kTileRows + g + 8) * 4 + 2 * tq + 1] = d[3];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_full[r]);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    // Two epilogue warps take alternate tiles: sum the 8 partials, apply the
    // row scale and 2^-sigma_m, write logits when asked, and keep each value
    // in shared memory for this CTA's top-k, taken after the stream.
    const int ew = warp - kConsumerWarps - 1;  // 0 or 1
    float inv[4];  // 2^-sigma_m
#pragma unroll
    for (int m = 0; m < 4; ++m) inv[m] = __uint_as_float((uint32_t)(127 - (m < M ? s_sigma[m] : 0)) << 23);
    int64_t it = ew;
    for (int64_t t = t_begin + ew; t < t_end; t += kEpilogueWarps, it += kEpilogueWarps) {
      const int r = (int)(it % kRed);
      const int64_t row = t * kTileRows + lane;
      const int nrows = (int)(V - t * kTileRows < kTileRows ? V - t * kTileRows : kTileRows);
      const bool valid = lane < nrows;
      const bool ok = wait_all(&red_full[r], (uint32_t)((it / kRed) & 1));
      const float* rb = red + (size_t)r * kConsumerWarps * kTileRows * 4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      float rs = 1.0f;
      if (valid && ok) {
#pragma unroll
        for (int ww = 0; ww < kConsumerWarps; ++ww) {
          const float4 p = *reinterpret_cast<const float4*>(rb + (ww * kTileRows + lane) * 4);
          acc[0] += p.x; acc[1] += p.y; acc[2] += p.z; acc[3] += p.w;
        }
        if (row_scale) rs = lane < (nrows & ~3) ? rsc[r * kTileRows + lane] : __ldg(row_scale + row);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[r]);
      if (valid) {
        const int local = (int)((t - t_begin) * kTileRows) + lane;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          if (m < M) {
            const float v = acc[m] * rs * inv[m];
            if (logits) logits[(size_t)m * V + row] = v;
            cvals[(size_t)m * n_cap + local] = v;
          }
        }
      }
    }
  }

  // every value is in shared memory and every copy has landed: the ring is free
  head_tail(cvals, n_cap, reinterpret_cast<Cand*>(ring), t_begin, t_end, V, M, top_k, warp, lane, hdr, cand, smem,
            s_last, out_ids, out_vals);
}


}  // namespace

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------

static size_t merge_smem_bytes(int grid, int top_k) {
  return (size_t)grid * sizeof(Cand) + (size_t)((grid + 1) & ~1) * sizeof(int) +
         (size_t)top_k * top_k * sizeof(Cand) + 2 * sizeof(int) + sizeof(Cand);
}

static size_t stream_smem_bytes(int H, int elem_bytes, int stages, int M, int64_t V, int grid) {
  const int64_t ntiles = (V + kTileRows - 1) / kTileRows;
  const int64_t n_cap = (ntiles + grid - 1) / grid * kTileRows;
  size_t bytes = (size_t)stages * stage_bytes(H * elem_bytes);
  bytes += kRed * kConsumerWarps * kTileRows * 4 * sizeof(float);  // reduce buffers
  bytes += kRed * kTileRows * sizeof(float);                        // row scales
  bytes += (size_t)M * ((n_cap + 1) & ~1) * sizeof(float);          // this CTA's logits
  bytes += (2 * stages + 2 * 4) * sizeof(uint64_t) + 8 * sizeof(int);
  return bytes;
}

// elem_bytes 1: the FP8 head kernel (lmhead_fp8.cu); 2: the BF16 ring kernel.
bool lmhead_plan(int H, int elem_bytes, int M, int top_k, int64_t V, int grid, int* stages, size_t* smem) {
  if (elem_bytes == 1) return lmhead_fp8_plan(H, M, top_k, V, grid, stages, smem);
  const size_t merge = merge_smem_bytes(grid, top_k);  // the final merge reuses the whole dynamic buffer
  for (int st = 4; st >= 2; --st) {
    size_t b = stream_smem_bytes(H, elem_bytes, st, M, V, grid);
    if (merge > b) b = merge;
    if (b <= kMaxSmem) {
      *stages = st;
      *smem = b;
      return true;
    }
  }
  return false;
}

template <typename W, int kSlices>
static cudaError_t launch_head_t(const uint16_t* x, const W* w, const float* s, int64_t V, int H, int M, int top_k,
                                 float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                                 cudaStream_t st) {
  int stages = 0;
  size_t smem = 0;
  if (!lmhead_plan(H, (int)sizeof(W), M, top_k, V, grid, &stages, &smem)) return cudaErrorInvalidConfiguration;
  auto kern = lmhead_topk_kernel<W, kSlices>;
  cudaError_t e = ensure_smem_optin<lmhead_topk_kernel<W, kSlices>>();
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(x, w, s, V, H, M, top_k, stages, logits, ids, vals, hdr,
                                     reinterpret_cast<Cand*>(cand));
  return cudaGetLastError();
}

template <typename W>
static cudaError_t launch_head(const uint16_t* x, const W* w, const float* s, int64_t V, int H, int M, int top_k,
                               float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                               cudaStream_t st) {
  const int slices = (H * (int)sizeof(W) / 64 + kConsumerWarps - 1) / kConsumerWarps;
  switch (slices) {
#define MOE_CASE(S) \
  case S: return launch_head_t<W, S>(x, w, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, st);
    MOE_CASE(1) MOE_CASE(2) MOE_CASE(3) MOE_CASE(4) MOE_CASE(5) MOE_CASE(6) MOE_CASE(7) MOE_CASE(8)
    MOE_CASE(9) MOE_CASE(10)
#undef MOE_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_lmhead_bf16(const uint16_t* x, const uint16_t* w, int64_t V, int H, int M, int top_k,
                               float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                               cudaStream_t st) {
  return launch_head<uint16_t>(x, w, nullptr, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, st);
}

int lmhead_max_slices() { return kMaxSlicesPerWarp; }

}  // namespace moe
