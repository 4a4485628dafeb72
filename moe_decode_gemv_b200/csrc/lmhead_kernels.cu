// lmhead_kernels.cu -- the online-FP8 LM head (and its BF16 comparator):
// one pass over the [V][H] head for all M tokens, fused with the per-row
// scale, an optional logits write and a top-k reduction.
//
// The pages: every generated token reads the whole 157,184 x 2,560 head, and
// quantising only this layer to FP8 at load time halves those reads
// (ncijnetwork.com summary, "What are the 3 optimizations?", item 2;
// generativeaipub.com blog, "2. Compressing the Output Head").
//
// Design (sm_100a, one GPU):
//  * One CTA per SM, persistent over a contiguous range of 16-row tiles.
//  * A producer warp streams tiles HBM -> shared memory with bulk copies
//    (cp.async.bulk, no multicast) into a ring of kStages buffers guarded by
//    mbarriers; rows are copied one by one into a padded stride so that the
//    consumers' 16-byte shared loads are free of bank conflicts.
//  * Eight consumer warps split K.  Each computes 16 rows x 8 token columns
//    with mma.sync m16n8k32 (E4M3 x E4M3 -> fp32): the weight bytes from
//    shared memory ARE the A fragments -- no conversion instruction per
//    weight -- and the B fragments hold the token activations, resident in
//    registers for the whole kernel.  This is a GEMV: the tensor-core
//    instruction is used because it retires 4,096 multiply-adds per issue and
//    needs no per-weight decode, which keeps the instruction count per weight
//    byte far below what the HBM stream allows, at M = 1 and M = 4 alike.
//  * Activations: each bf16 token is scaled by 2^sigma_m (max |x| into
//    [2^7, 2^8)) and split into two E4M3 parts hi + lo, which represent the
//    bf16 value exactly (8 significand bits = 4 + 4) for every element above
//    E4M3's subnormal range; the two parts take two MMAs.  The logit is
//    acc * s_v * 2^-sigma_m.
//  * Epilogue per tile: the consumers' partial sums meet in shared memory;
//    one warp per token applies the row scale, writes logits when asked and
//    merges the 16 candidates into the CTA's running top-k list (sorted, ties
//    to the lower id).  The last CTA to finish merges all CTAs' lists.
#include <cuda_runtime.h>

#include <cfloat>

#include "common.cuh"
#include "lmhead.h"

namespace moe {
namespace {

constexpr int kTileRows = 16;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 2) * 32;  // consumers + producer + epilogue
constexpr int kMaxSlicesPerWarp = 10;  // row bytes <= 10 * 8 * 64 = 5120: H <= 5120 (fp8), 2560 (bf16)
constexpr size_t kMaxSmem = 232448;    // 227 KB of dynamic shared memory per CTA

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

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
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

struct Cand {
  float v;
  int32_t id;
};

constexpr int kCandBuf = 128;     // per-token candidate buffer of the epilogue warp
constexpr int kSurvivors = 2048;  // entries kept by the final merge's lower bound

// Warp-cooperative: move the best min(k, n) of buf[0..n) to buf[0..) in order
// (value descending, ties to the lower id), padding with empty candidates up
// to k.  Returns min(k, n).  Selection by repeated warp argmax: O(n k / 32).
__device__ int select_top(Cand* buf, int n, int k, int lane) {
  constexpr int kPer = kCandBuf / 32;
  Cand c[kPer];
  bool taken[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = lane + 32 * i;
    c[i] = j < n ? buf[j] : Cand{-FLT_MAX, INT32_MAX};
    taken[i] = j >= n;
  }
  __syncwarp();
  const int keep = n < k ? n : k;
  for (int r = 0; r < k; ++r) {
    float bv = -FLT_MAX;
    int32_t bi = INT32_MAX;
    int bslot = -1;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (!taken[i] && (bslot < 0 || better(c[i].v, c[i].id, bv, bi))) { bv = c[i].v; bi = c[i].id; bslot = i; }
    float wv = bv;
    int32_t wi = bi;
    warp_best(wv, wi);
    // the owner of the winner marks it taken (ids are unique among real candidates)
    if (r < keep && bslot >= 0 && bi == wi && bv == wv) taken[bslot] = true;
    if (lane == 0) buf[r] = r < keep ? Cand{wv, wi} : Cand{-FLT_MAX, INT32_MAX};
  }
  __syncwarp();
  return keep;
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
  const int tile_bytes = kTileRows * stride;

  // shared-memory carve-up: [ring][reduce buffers][top-k lists][barriers][scalars]
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(ring + (size_t)stages * tile_bytes);       // [kRed][8][16][4]
  Cand* lists = reinterpret_cast<Cand*>(red + kRed * kConsumerWarps * kTileRows * 4);  // [M][top_k]
  Cand* cbuf = lists + 4 * 64;                                                       // [M][kCandBuf]
  uint64_t* full = reinterpret_cast<uint64_t*>(cbuf + 4 * kCandBuf);
  uint64_t* empty = full + stages;
  uint64_t* red_full = empty + stages;
  uint64_t* red_empty = red_full + kRed;
  int* s_sigma = reinterpret_cast<int*>(red_empty + kRed);  // [4]
  int* s_poison = s_sigma + 4;  // set once any bounded wait ran out
  int* s_last = s_sigma + 5;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (V + kTileRows - 1) / kTileRows;
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
  for (int i = threadIdx.x; i < M * top_k; i += blockDim.x) lists[i] = Cand{-FLT_MAX, INT32_MAX};
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
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * row_bytes));
      __syncwarp();
      if (lane < nrows)
        bulk_g2s(ring + (size_t)s * tile_bytes + (size_t)lane * stride,
                 reinterpret_cast<const uint8_t*>(w) + (size_t)(r0 + lane) * row_bytes, (uint32_t)row_bytes,
                 &full[s], policy);
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
    // x' = hi + lo, exact for every element whose magnitude is above E4M3's
    // subnormal range (more than 2^-14 of the token's largest).  Each part
    // takes its own MMA; the weights enter the MMA as raw E4M3 bytes.
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // hand the partial sums to the epilogue warp
      const int r = (int)(it % kRed);
      if (it >= kRed) wait_all(&red_empty[r], (uint32_t)(((it / kRed) & 1) ^ 1));
      float* rb = red + (size_t)r * kConsumerWarps * kTileRows * 4;
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
    int cnt[4] = {0, 0, 0, 0};
    Cand thr[4] = {{-FLT_MAX, INT32_MAX}, {-FLT_MAX, INT32_MAX}, {-FLT_MAX, INT32_MAX}, {-FLT_MAX, INT32_MAX}};
    // Per token: a buffer of candidates better than the current threshold (the
    // k-th best kept so far).  Appends are one ballot; when the buffer could
    // overflow, a selection pass keeps the best k and raises the threshold.
    int64_t it = 0;
    for (int64_t t = t_begin; t < t_end; ++t, ++it) {
      const int r = (int)(it % kRed);
      const int64_t row = t * kTileRows + lane;
      const bool valid = lane < kTileRows && row < V;
      const float rs = (valid && row_scale) ? __ldg(row_scale + row) : 1.0f;
      const bool ok = wait_all(&red_full[r], (uint32_t)((it / kRed) & 1));
      const float* rb = red + (size_t)r * kConsumerWarps * kTileRows * 4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid && ok) {
#pragma unroll
        for (int ww = 0; ww < kConsumerWarps; ++ww) {
          const float4 p = *reinterpret_cast<const float4*>(rb + (ww * kTileRows + lane) * 4);
          acc[0] += p.x; acc[1] += p.y; acc[2] += p.z; acc[3] += p.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[r]);
      for (int m = 0; m < M; ++m) {
        float v = -FLT_MAX;
        if (valid) {
          v = acc[m] * rs * __uint_as_float((uint32_t)(127 - s_sigma[m]) << 23);
          if (logits) logits[(size_t)m * V + row] = v;
        }
        Cand* buf = cbuf + m * kCandBuf;
        if (cnt[m] + kTileRows > kCandBuf) {
          cnt[m] = select_top(buf, cnt[m], top_k, lane);
          if (cnt[m] >= top_k) thr[m] = buf[top_k - 1];
        }
        const bool pass = valid && better(v, (int32_t)row, thr[m].v, thr[m].id);
        const uint32_t bal = __ballot_sync(0xffffffffu, pass);
        if (pass) buf[cnt[m] + __popc(bal & ((1u << lane) - 1u))] = Cand{v, (int32_t)row};
        cnt[m] += __popc(bal);
        __syncwarp();
      }
    }
    for (int m = 0; m < M; ++m) {
      Cand* buf = cbuf + m * kCandBuf;
      select_top(buf, cnt[m], top_k, lane);
      for (int i = lane; i < top_k; i += 32) lists[m * top_k + i] = buf[i];
    }
    __syncwarp();
  }

  // ------------------------- CTA lists -> global ---------------------------
  __syncthreads();
  Cand* my = cand + (size_t)blockIdx.x * M * top_k;
  for (int i = threadIdx.x; i < M * top_k; i += blockDim.x) my[i] = lists[i];
  __threadfence();
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
  // Per token: stage every CTA's sorted list in shared memory.  The k best of
  // the lists' first entries are k real candidates, so the k-th best of them,
  // L, is a lower bound on the global k-th best: only entries not worse than
  // L can be in the top k.  Keep those (typically a few dozen) and select the
  // top k of them with one warp.
  Cand* stage = reinterpret_cast<Cand*>(smem);                 // [G * top_k]  (the ring is free now)
  Cand* surv = stage + (size_t)gridDim.x * top_k;              // [kSurvivors]
  Cand* wbuf = surv + kSurvivors;                              // [kCandBuf] selection buffer of warp 0
  int* s_cnt = reinterpret_cast<int*>(wbuf + kCandBuf);
  Cand* s_bound = reinterpret_cast<Cand*>(s_cnt + 4);
  const int nl = (int)gridDim.x * top_k;
  // warp 0's chunked selection: the best top_k of src[0..n) into wbuf[0..top_k)
  auto select_from = [&](const Cand* src, int n, int stride) {
    int cnt = 0, pos = 0;
    do {
      const int take = min(kCandBuf - cnt, n - pos);
      for (int i = lane; i < take; i += 32) wbuf[cnt + i] = src[(size_t)(pos + i) * stride];
      __syncwarp();
      pos += take;
      cnt = select_top(wbuf, cnt + take, top_k, lane);
    } while (pos < n);
  };
  for (int m = 0; m < M; ++m) {
    for (int i = threadIdx.x; i < nl; i += blockDim.x) {
      const int cc = i / top_k, j = i - cc * top_k;
      const Cand* src = cand + ((size_t)cc * M + m) * top_k + j;
      stage[i] = Cand{__ldcg(&src->v), __ldcg(&src->id)};
    }
    if (threadIdx.x == 0) *s_cnt = 0;
    __syncthreads();
    if (warp == 0) {
      select_from(stage, (int)gridDim.x, top_k);  // the lists' first entries
      if (lane == 0) *s_bound = wbuf[top_k - 1];  // an empty slot (worst) when fewer than top_k lists
    }
    __syncthreads();
    const Cand L = *s_bound;
    for (int i = threadIdx.x; i < nl; i += blockDim.x) {
      const Cand e = stage[i];
      if (!better(L.v, L.id, e.v, e.id)) {  // e is L or better
        const int pos = atomicAdd(s_cnt, 1);
        if (pos < kSurvivors) surv[pos] = e;
      }
    }
    __syncthreads();
    if (warp == 0) {
      const int n = *s_cnt;
      // more survivors than the buffer holds (heavy ties): select from all staged entries instead
      if (n <= kSurvivors) select_from(surv, n, 1);
      else select_from(stage, nl, 1);
      for (int i = lane; i < top_k; i += 32) {
        out_ids[m * top_k + i] = wbuf[i].id;
        out_vals[m * top_k + i] = wbuf[i].v;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) hdr->ticket = 0u;
}

}  // namespace

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------

size_t lmhead_smem_bytes(int H, int elem_bytes, int stages);

int lmhead_stages(int H, int elem_bytes) {
  int stages = 4;
  while (stages > 2 && lmhead_smem_bytes(H, elem_bytes, stages) > kMaxSmem) --stages;
  return stages;
}

size_t lmhead_merge_smem_bytes(int grid, int top_k) {
  return ((size_t)grid * top_k + kSurvivors + kCandBuf) * sizeof(Cand) + 4 * sizeof(int) + sizeof(Cand);
}

size_t lmhead_smem_bytes(int H, int elem_bytes, int stages) {
  const int stride = padded_stride(H * elem_bytes);
  size_t bytes = (size_t)stages * kTileRows * stride;
  bytes += 4 * kConsumerWarps * kTileRows * 4 * sizeof(float);  // kRed reduce buffers
  bytes += 4 * 64 * sizeof(Cand) + 4 * kCandBuf * sizeof(Cand);
  bytes += (2 * stages + 2 * 4) * sizeof(uint64_t) + 8 * sizeof(int);
  return bytes;
}

size_t lmhead_cand_bytes(int grid, int M, int top_k) { return (size_t)grid * M * top_k * sizeof(Cand); }

template <typename W, int kSlices>
static cudaError_t launch_head_t(const uint16_t* x, const W* w, const float* s, int64_t V, int H, int M, int top_k,
                                 float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                                 cudaStream_t st) {
  const int stages = lmhead_stages(H, (int)sizeof(W));
  size_t smem = lmhead_smem_bytes(H, (int)sizeof(W), stages);
  const size_t merge = lmhead_merge_smem_bytes(grid, top_k);
  if (merge > smem) smem = merge;  // the final merge reuses the whole dynamic buffer
  if (smem > kMaxSmem) return cudaErrorInvalidConfiguration;
  auto kern = lmhead_topk_kernel<W, kSlices>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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

cudaError_t launch_lmhead_fp8(const uint16_t* x, const uint8_t* q, const float* s, int64_t V, int H, int M,
                              int top_k, float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand,
                              int grid, cudaStream_t st) {
  return launch_head<uint8_t>(x, q, s, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, st);
}

cudaError_t launch_lmhead_bf16(const uint16_t* x, const uint16_t* w, int64_t V, int H, int M, int top_k,
                               float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                               cudaStream_t st) {
  return launch_head<uint16_t>(x, w, nullptr, V, H, M, top_k, logits, ids, vals, hdr, cand, grid, st);
}

int lmhead_max_slices() { return kMaxSlicesPerWarp; }

}  // namespace moe
