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
//    with mma.sync m16n8k16 (f16 x f16 -> fp32): the A fragments are built in
//    registers straight from the E4M3 bytes (one cvt per pair; every E4M3
//    value is an f16 value, so this is exact) and the B fragments hold the
//    token activations, resident in registers for the whole kernel.  This is
//    a GEMV: the tensor-core instruction is used because it retires 2,048
//    multiply-adds per issue, which keeps the instruction count per weight
//    byte far below what the HBM stream allows at M = 4.
//  * bf16 activations become f16 exactly after a per-token power-of-two
//    scale 2^sigma_m that puts max|x_m| in [2^14, 2^15); the logit is
//    acc * s_v * 2^-sigma_m.  Only elements more than 2^28 below the token's
//    largest fall into the f16 subnormal range.
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
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxSlicesPerWarp = 10;  // row bytes <= 10 * 8 * 64 = 5120: H <= 5120 (fp8), 2560 (bf16)
constexpr size_t kMaxSmem = 232448;    // 227 KB of dynamic shared memory per CTA

template <typename W>
struct HeadTraits;

// FP8 E4M3 weights: a 64-byte K slice is 64 elements; 4 MMAs of k16 each.
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

  // shared-memory carve-up: [ring][reduce 2x][top-k lists][barriers]
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(ring + (size_t)stages * tile_bytes);      // [2][W][16][4]
  Cand* lists = reinterpret_cast<Cand*>(red + 2 * kConsumerWarps * kTileRows * 4);  // [M][top_k]
  uint64_t* full = reinterpret_cast<uint64_t*>(lists + 4 * 64);
  uint64_t* empty = full + stages;
  int* s_sigma = reinterpret_cast<int*>(empty + stages);  // [4]
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
        sigma = 14 - fl;
        sigma = sigma > 126 ? 126 : (sigma < -126 ? -126 : sigma);
      }
      s_sigma[warp] = sigma;
    }
  }
  for (int i = threadIdx.x; i < M * top_k; i += blockDim.x) lists[i] = Cand{-FLT_MAX, INT32_MAX};
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------ producer ------------------------------
    const uint64_t policy = l2_evict_first_policy();
    int64_t it = 0, issued = 0;
    for (int64_t t = t_begin; t < t_end; ++t, ++it) {
      const int s = (int)(it % stages);
      const uint32_t ph = (uint32_t)((it / stages) & 1);
      bool ok = !*(volatile int*)s_poison;
      if (ok && it >= stages && lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        // after a timeout nothing more is issued; the consumers run on without waiting
        if (lane == 0 && !*(volatile int*)s_poison) { report(hdr, MOE_ERR_TIMEOUT); atomicExch(s_poison, 1); }
        continue;
      }
      const int64_t r0 = t * kTileRows;
      const int nrows = (int)(V - r0 < kTileRows ? V - r0 : kTileRows);
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(nrows * row_bytes));
      __syncwarp();
      if (lane < nrows)
        bulk_g2s(ring + (size_t)s * tile_bytes + (size_t)lane * stride,
                 reinterpret_cast<const uint8_t*>(w) + (size_t)(r0 + lane) * row_bytes, (uint32_t)row_bytes, &full[s], policy);
      issued = it + 1;
    }
    // drain: every issued copy must land before this CTA may exit
    if (lane == 0) {
      const int64_t first = issued > stages ? issued - stages : 0;
      for (int64_t j = first; j < issued; ++j) mbar_wait(&full[j % stages], (uint32_t)((j / stages) & 1));
    }
  } else {
    // ------------------------------ consumers -----------------------------
    const int g = lane >> 2, tq = lane & 3;
    // B fragments: token n = g, this warp's K slices
    uint32_t bfrag[kSlices][T::kMmasPerSlice][2];
    {
      const bool live = g < M;
      const float scl = live ? __uint_as_float((uint32_t)(127 + s_sigma[g]) << 23) : 0.f;
#pragma unroll
      for (int si = 0; si < kSlices; ++si) {
        const int slice = warp + si * kConsumerWarps;
        const int e0 = slice * (64 / T::kElemBytes) + tq * (16 / T::kElemBytes);  // first element of the lane chunk
#pragma unroll
        for (int j = 0; j < T::kMmasPerSlice; ++j) {
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            const int k0 = e0 + 4 * j + 2 * p;
            uint32_t v = 0u;
            if (live && slice * 64 < row_bytes) {
              const uint32_t pair = *reinterpret_cast<const uint32_t*>(x + (size_t)g * H + k0);
              if constexpr (sizeof(W) == 1) {
                __half2 h2 = __floats2half2_rn(bf16_bits_to_f32(pair & 0xffffu) * scl, bf16_bits_to_f32(pair >> 16) * scl);
                v = *reinterpret_cast<uint32_t*>(&h2);
              } else {
                v = pair;  // bf16 pair as is
              }
            }
            bfrag[si][j][p] = v;
          }
        }
      }
    }

    int64_t it = 0;
    for (int64_t t = t_begin; t < t_end; ++t, ++it) {
      const int s = (int)(it % stages);
      const uint32_t ph = (uint32_t)((it / stages) & 1);
      bool ok = !*(volatile int*)s_poison;
      if (ok && lane == 0) ok = mbar_wait(&full[s], ph);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok && lane == 0 && !*(volatile int*)s_poison) { report(hdr, MOE_ERR_TIMEOUT); atomicExch(s_poison, 1); }
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) {
        const uint8_t* tile = ring + (size_t)s * tile_bytes;
#pragma unroll
        for (int si = 0; si < kSlices; ++si) {
          const int slice = warp + si * kConsumerWarps;
          if (slice * 64 < row_bytes) {
            const uint4 ra = *reinterpret_cast<const uint4*>(tile + (size_t)g * stride + slice * 64 + tq * 16);
            const uint4 rb = *reinterpret_cast<const uint4*>(tile + (size_t)(g + 8) * stride + slice * 64 + tq * 16);
            const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w}, wb[4] = {rb.x, rb.y, rb.z, rb.w};
            if constexpr (sizeof(W) == 1) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t a[4] = {e4m3x2_to_f16x2(wa[j] & 0xffffu), e4m3x2_to_f16x2(wb[j] & 0xffffu),
                                       e4m3x2_to_f16x2(wa[j] >> 16), e4m3x2_to_f16x2(wb[j] >> 16)};
                mma_f16(d, a, bfrag[si][j][0], bfrag[si][j][1]);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t a[4] = {wa[2 * j], wb[2 * j], wa[2 * j + 1], wb[2 * j + 1]};
                mma_bf16(d, a, bfrag[si][j][0], bfrag[si][j][1]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // partial sums -> shared; tokens 2tq and 2tq+1 live in lanes with tq < 2
      float* rb = red + (size_t)(it & 1) * kConsumerWarps * kTileRows * 4;
      if (tq < 2) {
        rb[(warp * kTileRows + g) * 4 + 2 * tq] = d[0];
        rb[(warp * kTileRows + g) * 4 + 2 * tq + 1] = d[1];
        rb[(warp * kTileRows + g + 8) * 4 + 2 * tq] = d[2];
        rb[(warp * kTileRows + g + 8) * 4 + 2 * tq + 1] = d[3];
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32));

      if (warp < M) {
        // one warp per token: lanes 0..15 own one row of the tile each
        const int m = warp;
        const int64_t row = t * kTileRows + lane;
        const bool valid = lane < kTileRows && row < V;
        float v = -FLT_MAX;
        if (valid) {
          float acc = 0.f;
#pragma unroll
          for (int ww = 0; ww < kConsumerWarps; ++ww) acc += rb[(ww * kTileRows + lane) * 4 + m];
          const float rs = row_scale ? row_scale[row] : 1.0f;
          v = acc * rs * __uint_as_float((uint32_t)(127 - s_sigma[m]) << 23);
          if (logits) logits[(size_t)m * V + row] = v;
        }
        // merge into the sorted list: candidates arrive in increasing id order
        Cand* L = lists + m * top_k;
        const Cand worst = L[top_k - 1];
        uint32_t pend = __ballot_sync(0xffffffffu, valid && better(v, (int32_t)row, worst.v, worst.id));
        while (pend) {
          const int src = __ffs(pend) - 1;
          pend &= pend - 1;
          const float cv = __shfl_sync(0xffffffffu, v, src);
          const int32_t cid = (int32_t)(t * kTileRows + src);
          // position = number of entries better than the candidate
          int pos = 0;
          for (int base = 0; base < top_k; base += 32) {
            const int j = base + lane;
            const bool b = j < top_k && better(L[j].v, L[j].id, cv, cid);
            pos += __popc(__ballot_sync(0xffffffffu, b));
          }
          if (pos < top_k) {
            for (int base = ((top_k - 1) / 32) * 32; base >= 0; base -= 32) {
              const int j = base + lane;
              Cand c{};
              const bool mv = j >= pos && j < top_k - 1;
              if (mv) c = L[j];
              __syncwarp();
              if (mv) L[j + 1] = c;
              __syncwarp();
            }
            if (lane == 0) L[pos] = Cand{cv, cid};
            __syncwarp();
          }
        }
      }
    }
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
  if (!*s_last) return;
  __threadfence();

  // ------------------------ last CTA: merge the lists ------------------------
  // One warp per token; each list is sorted, so repeatedly take the best head.
  uint8_t* heads = ring;  // [M][gridDim] list positions (top_k <= 64); the ring is free now
  for (int i = threadIdx.x; i < M * (int)gridDim.x; i += blockDim.x) heads[i] = 0;
  __syncthreads();
  if (warp < M) {
    const int m = warp;
    uint8_t* hm = heads + m * gridDim.x;
    for (int r = 0; r < top_k; ++r) {
      float bv = -FLT_MAX;
      int32_t bid = INT32_MAX;
      int32_t bc = -1;
      for (int c = lane; c < (int)gridDim.x; c += 32) {
        const int hh = hm[c];
        if (hh < top_k) {
          const Cand* cc = cand + ((size_t)c * M + m) * top_k + hh;
          const float cv = __ldcg(&cc->v);
          const int32_t ci = __ldcg(&cc->id);
          if (bc < 0 || better(cv, ci, bv, bid)) { bv = cv; bid = ci; bc = c; }
        }
      }
      // warp-wide best, carrying the list index
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, bid, o);
        const int32_t oc = __shfl_xor_sync(0xffffffffu, bc, o);
        if (oc >= 0 && (bc < 0 || better(ov, oi, bv, bid))) { bv = ov; bid = oi; bc = oc; }
      }
      if (lane == 0) {
        out_ids[m * top_k + r] = bid;
        out_vals[m * top_k + r] = bv;
        if (bc >= 0) hm[bc] = (uint8_t)(hm[bc] + 1);
      }
      __syncwarp();
    }
  }
  __syncthreads();
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

size_t lmhead_smem_bytes(int H, int elem_bytes, int stages) {
  const int stride = padded_stride(H * elem_bytes);
  size_t bytes = (size_t)stages * kTileRows * stride;
  bytes += 2 * kConsumerWarps * kTileRows * 4 * sizeof(float);
  bytes += 4 * 64 * sizeof(Cand);
  bytes += 2 * stages * sizeof(uint64_t) + 8 * sizeof(int);
  return bytes;
}

size_t lmhead_cand_bytes(int grid, int M, int top_k) { return (size_t)grid * M * top_k * sizeof(Cand); }

template <typename W, int kSlices>
static cudaError_t launch_head_t(const uint16_t* x, const W* w, const float* s, int64_t V, int H, int M, int top_k,
                                 float* logits, int32_t* ids, float* vals, WsHeader* hdr, void* cand, int grid,
                                 cudaStream_t st) {
  const int stages = lmhead_stages(H, (int)sizeof(W));
  const size_t smem = lmhead_smem_bytes(H, (int)sizeof(W), stages);
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
