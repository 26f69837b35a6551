// Device helpers for the sm_100a kernels: inline PTX for the bulk-copy engine, mbarriers,
// bounded waits, and the hardware FP4/FP8 conversions.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace fp4q {

// Device-side status word, read back by fp4q_device_status().  Bit 0: a bounded wait ran out.
// One per translation unit (each unit's kernels are a module of their own).
static __device__ unsigned int g_device_status;
constexpr unsigned int kStatusTimeout = 1u;

// A wait on an mbarrier gives up after this many nanoseconds (about one second).
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make the barrier initialisation visible to the bulk-copy (async) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One try: the thread may be suspended in hardware until the phase completes, for at most
// the hint (20 us) before it returns false.  A suspended warp issues nothing, so waiting
// roles (producer, MMA issuer, sign warps, idle epilogue warps) leave the issue slots to the
// warps with work (measured: the headline kernel 8.57 -> 8.41 us per call).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false, and records
// kStatusTimeout, when it has not completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
#pragma unroll 1
  for (int i = 0; i < 32; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_status, kStatusTimeout);
      return false;
    }
  }
}

// Programmatic dependent launch.  launch_dependents lets the next kernel on the stream be
// scheduled while this one runs; wait blocks until every kernel this one depends on has
// finished and its memory is visible (a no-op when launched without the attribute).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bulk copy (no tensor map) global -> shared, completion signalled on an mbarrier as
// transaction bytes.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Ask for `bytes` (a multiple of 16, 16-byte aligned) of global memory to be brought into L2.
// A hint: L2 is the GPU's point of coherence, so later reads still see any write made after it.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void sts128_u4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void stg128(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void stg256(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ void stg64(void* p, uint32_t a, uint32_t b) {
  asm volatile("st.global.v2.b32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// ---- packed fp32 pairs (f32x2 arithmetic on sm_100); the low half is the even element
using f32x2 = unsigned long long;

__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 f2_sub(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// First butterfly stage straight from a bf16 pair word (element 2k in the low half):
// (x[2k] + x[2k+1], x[2k+1] - x[2k]), each rounded once to fp32, as a packed pair.  The
// second entry is the negated difference: the mixed-precision add takes the high bf16 half
// as its bf16 operand and the low half, widened by an integer multiply, as its fp32 operand.
// Callers undo the negation of the odd elements (it commutes with every later stage, which
// treats the two halves of a pair alike).
__device__ __forceinline__ f32x2 bf16_pair_butterfly_oddneg(uint32_t w) {
  float s, d;
  const float lo = __uint_as_float(w * 65536u);
  asm("{\n .reg .b16 lo16, hi16;\n"
      " mov.b32 {lo16, hi16}, %2;\n"
      " add.rn.f32.bf16 %0, hi16, %3;\n"
      " sub.rn.f32.bf16 %1, hi16, %3;\n}"
      : "=f"(s), "=f"(d)
      : "r"(w), "f"(lo));
  return f2_pack(s, d);
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Approximate reciprocal (the hardware's rcp.approx: relative error below 2^-22).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// bf16 pair (element 2k in the low half) -> two exact fp32 values.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight fp32 values -> eight E2M1 codes (round to nearest even, saturating at +-6), packed
// into one word with element 0 in the low nibble.  cvt...e2m1x2 puts its first source
// operand in the high nibble of the byte.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7) {
  uint32_t r;
  asm("{\n .reg .b8 q0, q1, q2, q3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n"
      " cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n"
      " cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n"
      " mov.b32 %0, {q0, q1, q2, q3};\n}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// fp32 (non-negative) -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}

// E4M3 byte -> fp32 (exact, through f16).
__device__ __forceinline__ float e4m3_decode(uint32_t byte) {
  uint32_t h2;
  const uint16_t in = static_cast<uint16_t>(byte & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// E2M1 code (4 bits) -> fp32 value.
__device__ __forceinline__ float e2m1_decode(uint32_t c) {
  const uint32_t k = c & 7u;
  uint32_t bits = k >= 2u ? ((((k >> 1) + 126u) << 23) | ((k & 1u) << 22)) : (k == 1u ? 0x3F000000u : 0u);
  bits |= (c & 8u) << 28;
  return __uint_as_float(bits);
}

}  // namespace fp4q
