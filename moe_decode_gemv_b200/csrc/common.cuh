// common.cuh -- device helpers shared by the sm_100a kernels of this library.
//
// Number formats (OCP Microscaling Formats v1.0; OCP 8-bit Floating Point
// Specification): E4M3 codes are widened with the hardware conversion of
// sm_100a (cvt.rn.f16x2.e4m3x2), exact because every E4M3 value is an f16
// value; E2M1 codes of the packed expert banks become E5M2 codes by moving
// bits; E8M0 scales become fp32 by placing the code in the exponent field.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/moe_gemv.h"

namespace moe {

// ---------------------------------------------------------------------------
// Workspace header shared by every kernel: a status word and two counters.
// It sits at the start of each caller-owned workspace.
// ---------------------------------------------------------------------------
struct WsHeader {
  int32_t status;     // 0, or the first moe_status a kernel reported
  uint32_t ticket;    // last-block-done counter (returns to 0 after each use)
  uint32_t barrier;   // grid barrier word (sense-reversing; see grid_arrive)
  uint32_t epoch;     // calls completed on this workspace (tags published values; see moe_layer.cu)
  uint32_t tiles;     // next tile handed out by a counter (returns to 0 after each use)
  uint32_t pad[11];   // keeps what follows on a 64-byte boundary
};
static_assert(sizeof(WsHeader) == 64, "workspace header is 64 bytes");

__device__ __forceinline__ void report(WsHeader* h, moe_status s) {
  atomicCAS(&h->status, 0, (int32_t)s);
}

// Every device-side wait in this library is bounded in time: after
// kWaitLimitNs of waiting a kernel records MOE_ERR_TIMEOUT and returns instead
// of hanging.  A healthy wait here lasts microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Polls `ready()` until it returns true or `limit_ns` have passed, sleeping
// `backoff_ns` between polls so that a waiting warp leaves the issue slots to
// the warps doing the work.  Returns false on timeout.
template <typename F>
__device__ __forceinline__ bool bounded_spin_for(F ready, uint64_t limit_ns, uint32_t backoff_ns = 64) {
  const uint64_t start = global_ns();
  for (;;) {
    if (ready()) return true;
    if (global_ns() - start > limit_ns) return false;
    if (backoff_ns) __nanosleep(backoff_ns);
  }
}

// The same with the library's limit, kWaitLimitNs.
template <typename F>
__device__ __forceinline__ bool bounded_spin(F ready, uint32_t backoff_ns = 64) {
  return bounded_spin_for(ready, kWaitLimitNs, backoff_ns);
}

// ---------------------------------------------------------------------------
// Format conversions.
// ---------------------------------------------------------------------------

// Two E4M3 codes (low byte = lower-index element) -> f16x2, low byte in the low half.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(two_bytes));
  return r;
}

// Two fp32 values -> two E4M3 codes, round to nearest even, saturating to
// +-448.  `lo` lands in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> one byte of two E2M1 codes, round to nearest even,
// saturating to +-6.  `lo` lands in the low nibble.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// The packed expert banks (pack_kernels.cu) place the two E2M1 codes of a
// byte as element 2j: sign|e1 e0 m at bits 7|3 2 1 and element 2j+1 at bits
// 0|6 5 4.  E5M2 s|0 0 0 e1 e0|m 0 carries the E2M1 value times 2^-14 for
// every code (the E2M1 subnormal 0.5 becomes the E5M2 subnormal 2^-15), so
// the even elements of a packed word are E5M2 codes after one mask, and the
// odd ones after two shifts.  Bytes 0..3 of the result hold elements 0, 2,
// 4, 6 (even) or 1, 3, 5, 7 (odd) of the word.
__device__ __forceinline__ uint32_t packed_even_to_e5m2x4(uint32_t w) { return w & 0x8e8e8e8eu; }
__device__ __forceinline__ uint32_t packed_odd_to_e5m2x4(uint32_t w) {
  return ((w >> 3) & 0x0e0e0e0eu) | ((w << 7) & 0x80808080u);
}

// E8M0 code -> fp32 2^(code - 127) by one integer multiply (the FMA pipe, not
// the logic pipe): exact for codes 1..254.  Code 0 gives 0 instead of 2^-127
// (a block at that scale adds less than 2^-116 of its largest product to any
// sum) and code 255 gives +inf instead of NaN, so a block that carries it
// still turns its dot products into NaN when its elements are zero -- as the
// quantiser writes them -- and into +-inf otherwise.
__device__ __forceinline__ float e8m0_to_f32_fast(uint32_t code) { return __uint_as_float(code * 0x800000u); }

// E5M2 (A) x E4M3 (B) -> fp32 tensor-core MMA, m16n8k32.
__device__ __forceinline__ void mma_e5m2_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.f32.e5m2.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f16 x f16 -> fp32 tensor-core MMA, m16n8k16 (A row-major 16x16, B 16x8).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// E4M3 x E4M3 -> fp32 tensor-core MMA, m16n8k32 (A row-major 16x32, B 32x8).
// Not volatile: it has no effect beyond its outputs, so the compiler may
// interleave independent MMAs instead of issuing them in source order.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four fp32 values -> E4M3 parts (byte j of each part belongs to value j):
// p[0] = rne(v), p[1] = rne(v - p[0]), p[2] = rne(v - p[0] - p[1]), ...
// Each part takes the next four significant bits of v as long as the
// remainder stays in E4M3's normal range; the residues are exact in fp32.
template <int kParts>
__device__ __forceinline__ void split_e4m3x4(float a, float b, float c, float d, uint32_t (&p)[kParts]) {
#pragma unroll
  for (int q = 0; q < kParts; ++q) {
    const uint32_t ab = f32x2_to_e4m3x2(a, b), cd = f32x2_to_e4m3x2(c, d);
    p[q] = ab | (cd << 16);
    if (q + 1 < kParts) {
      const uint32_t fab = e4m3x2_to_f16x2(ab), fcd = e4m3x2_to_f16x2(cd);
      const float2 rab = __half22float2(*reinterpret_cast<const __half2*>(&fab));
      const float2 rcd = __half22float2(*reinterpret_cast<const __half2*>(&fcd));
      a -= rab.x; b -= rab.y; c -= rcd.x; d -= rcd.y;
    }
  }
}

// ---------------------------------------------------------------------------
// Warp reductions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Ordering of (value, index) candidates: larger value first, then lower index.
// Branch-free: evaluated with predicates, never a jump.
__device__ __forceinline__ bool better(float va, int32_t ia, float vb, int32_t ib) {
  return (va > vb) | ((va == vb) & (ia < ib));
}

// ---------------------------------------------------------------------------
// Cache-hinted loads for weights that are read once per step.
// ---------------------------------------------------------------------------
// (not volatile: the compiler may batch and reorder these reads of data that
// no kernel writes while they are in flight)
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ float4 ld_stream_f4(const void* p) {
  float4 r;
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (TMA, non-tensor form) helpers.  No multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// try_wait with a suspend-time hint: a thread whose phase is not complete is
// suspended (up to the hint, here 0.1 ms) instead of spinning.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "r"(100000u) : "memory");
  return ok != 0u;
}

// Bounded wait on an mbarrier phase.  Returns false if the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;  // the common case reads no timer
  return bounded_spin([&] { return mbar_try_wait(bar, parity); }, 0);
}

// Orders this thread's view of global memory (made visible to it by an
// acquire) before its later bulk copies, which read through the async proxy.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async;" ::: "memory"); }

// An L2 cache policy that evicts first: for weights read once per step.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// An L2 cache policy that evicts last: for small inputs every CTA reads.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing on `bar` with a transaction count.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_addr(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

}  // namespace moe
