// sample_kernels.cu -- the two small steps that follow the LM head in a
// sampled or speculative decode:
//  * one draw from the head's sorted top-k with temperature and top-p (the
//    sampled workload of the ncijnetwork.com summary, "What are the 3
//    optimizations?": temperature 0.6, top-p 0.95, top-k 29);
//  * greedy acceptance of draft tokens against the verify step's argmaxes
//    (the saipien.org essay, "Draft three tokens, verify four").
// Both touch a few hundred bytes.  They exist so that the whole decode step,
// the choice of the next token included, stays on the device.
#include <cuda_runtime.h>

#include <cfloat>

#include "../../include/moe_gemv.h"

namespace {

constexpr int kMaxSampleK = 64;

// One token per CTA, lane 0 of one warp: k <= 64 values, fp64 throughout, the
// operations in a fixed order (the draw is an integer decided by floating
// point, so the order is part of the definition):
//   p_i = exp((v_i - v_0) / T); total = sum_i p_i in index order;
//   n = the smallest prefix with mass >= top_p * total;
//   the first i < n whose running sum exceeds u * (p_0 + ... + p_{n-1}).
__global__ void sample_topk_kernel(const int32_t* __restrict__ ids, const float* __restrict__ vals, int k,
                                   double temperature, double top_p, const float* __restrict__ uniforms,
                                   int32_t* __restrict__ out) {
  if (threadIdx.x != 0) return;
  const int m = blockIdx.x;
  const float* v = vals + (size_t)m * k;
  double p[kMaxSampleK];
  double total = 0.0;
  const double v0 = (double)v[0];
  for (int i = 0; i < k; ++i) {
    p[i] = exp(((double)v[i] - v0) / temperature);
    total += p[i];
  }
  int n = 0;
  double before = 0.0;
  while (n < k && before < top_p * total) before += p[n++];
  double kept = 0.0;
  for (int i = 0; i < n; ++i) kept += p[i];
  const double r = (double)uniforms[m] * kept;
  int pick = n - 1;
  double cum = 0.0;
  for (int i = 0; i < n; ++i) {
    cum += p[i];
    if (cum > r) {
      pick = i;
      break;
    }
  }
  out[m] = ids[(size_t)m * k + pick];
}

__global__ void mtp_accept_kernel(const int32_t* __restrict__ draft, const int32_t* __restrict__ verify, int D,
                                  int32_t* __restrict__ emitted, int32_t* __restrict__ n_emitted) {
  if (threadIdx.x != 0) return;
  int a = 0;
  while (a < D && draft[a] == verify[a]) {
    emitted[a] = draft[a];
    ++a;
  }
  emitted[a] = verify[a];
  *n_emitted = a + 1;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" moe_status lmhead_sample(const int32_t* topk_ids, const float* topk_vals, int32_t M, int32_t top_k,
                                    float temperature, float top_p, const float* uniforms, int32_t* out_ids,
                                    void* stream) {
  if (!topk_ids || !topk_vals || !uniforms || !out_ids) return MOE_ERR_INVALID_ARG;
  if (M < 1 || M > 65535 || top_k < 1 || top_k > kMaxSampleK) return MOE_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !(temperature <= FLT_MAX) || !(top_p > 0.f) || !(top_p <= 1.f))
    return MOE_ERR_INVALID_ARG;
  if (!aligned4(topk_ids) || !aligned4(topk_vals) || !aligned4(uniforms) || !aligned4(out_ids))
    return MOE_ERR_MISALIGNED;
  sample_topk_kernel<<<M, 32, 0, static_cast<cudaStream_t>(stream)>>>(topk_ids, topk_vals, top_k, temperature, top_p,
                                                                       uniforms, out_ids);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_mtp_accept(const int32_t* draft_ids, const int32_t* verify_ids, int32_t D,
                                     int32_t* emitted_ids, int32_t* n_emitted, void* stream) {
  if (!draft_ids || !verify_ids || !emitted_ids || !n_emitted) return MOE_ERR_INVALID_ARG;
  if (D < 1 || D > 64) return MOE_ERR_INVALID_ARG;
  if (!aligned4(draft_ids) || !aligned4(verify_ids) || !aligned4(emitted_ids) || !aligned4(n_emitted))
    return MOE_ERR_MISALIGNED;
  mtp_accept_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(draft_ids, verify_ids, D, emitted_ids, n_emitted);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
