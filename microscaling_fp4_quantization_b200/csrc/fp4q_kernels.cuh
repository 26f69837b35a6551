// Fused block-Hadamard rotation + microscaling FP4 quantization kernels for sm_100a.
//
// The tensor is one flat stream of M*K bf16 values: K is a multiple of the Hadamard block
// b and of the scale group g, so blocks and groups never straddle rows and the row-major
// codes and scales are flat arrays in the same order.  The stream is cut into "units" of
// E = max(b, g) consecutive elements; one thread owns a unit at a time, so the whole
// rotation (every butterfly stage of H_b) and every group amax stay inside the thread's
// registers: no shuffles, no second pass.
//
// Data movement, per warp (warps are independent, there is no block-level barrier on the
// data path):
//   * the warp owns a contiguous range of units, cut evenly over all warps of the grid;
//   * lane 0 streams the range through a ring of S shared-memory stages with the bulk-copy
//     engine (cp.async.bulk global->shared, completion counted on one mbarrier per stage);
//     one stage holds 32*R units;
//   * all lanes wait on the stage's barrier (bounded in time), each lane processes R units
//     (lane l takes units l, l+32, ...), then lane 0 refills the stage S ahead;
//   * codes, scales (and the optional fp32 dump) are stored straight to global memory;
//     one warp's stores for a given r are contiguous.
//
// Shared-memory bank conflicts.  A lane reads its unit as E/8 chunks of 16 bytes.  With the
// natural order, lanes of a quarter-warp hit the same banks (units are 2E bytes apart).  Lane l
// therefore reads chunk j ^ tau(l) into register slot j, where tau only flips chunk-index
// bits inside one Hadamard block.  Because H[i, j] = (-1)^popcount(i & j), feeding the
// butterfly an input permuted by XOR with T = 8*tau yields the same outputs with the sign
// of output j flipped when popcount(T & j) is odd — exactly, in floating point, since every
// butterfly stage only swaps the operands of an add (commutative) or negates a subtraction.
// Amaxima are unaffected; the sign is restored by flipping the sign bits of the affected
// packed codes (and of the dumped values).  An exact zero may then carry either sign bit.
#pragma once

#include <cstdint>

#include "fp4q_device.cuh"

namespace fp4q {

enum : int { kMX = 0, kNV = 1 };
enum : int { kRuleFloor = 0, kRuleCeil = 1, kRuleOas = 2, kRuleNvStatic = 3, kRuleNvDynamic = 4 };

constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }
constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }

// fp32 value of 1/sqrt(b) (round-to-nearest of the real number), for b = 1, 2, 4, ..., 128.
__host__ __device__ constexpr float inv_sqrt_block(int b) {
  return b == 1     ? 1.0f
         : b == 2   ? 0.70710678118654752440f
         : b == 4   ? 0.5f
         : b == 8   ? 0.35355339059327376220f
         : b == 16  ? 0.25f
         : b == 32  ? 0.17677669529663688110f
         : b == 64  ? 0.125f
         : b == 128 ? 0.08838834764831844055f
                    : 0.0f;
}

// Compile-time shape of one kernel instance.
template <int FMT, int B, int RULE, bool DUMP>
struct RQConfig {
  static constexpr int kFmt = FMT;
  static constexpr int kBlock = B;
  static constexpr int kRule = RULE;
  static constexpr bool kDump = DUMP;
  static constexpr int kGroup = FMT == kMX ? 32 : 16;
  static constexpr int kE = cmax(B, kGroup);              // elements per unit
  static constexpr int kChunks = kE / 8;                  // 16-byte chunks per unit
  static constexpr int kGroupsPerUnit = kE / kGroup;
  // Units per lane per stage: a stage of about 4 KB (8 KB for E = 128).
  static constexpr int kR = cmax(1, 64 / kE);
  static constexpr int kUnitsPerStage = 32 * kR;
  static constexpr int kStageBytes = kUnitsPerStage * kE * 2;
  static constexpr int kStages = kE >= 128 ? 3 : 4;
  static constexpr int kWarps = 4;                       // warps per CTA
  static constexpr int kThreads = kWarps * 32;
  // Chunk-index XOR (see the file comment): as many low chunk bits as make a quarter-warp
  // conflict-free, but never more than the chunk bits inside one Hadamard block.
  static constexpr int kTauMaxChunks = cmin(kChunks, 8);
  static constexpr int kTauShift = 3 - ilog2(kTauMaxChunks);
  static constexpr int kTauMask = B >= 16 ? cmin(kTauMaxChunks, B / 8) - 1 : 0;
  static constexpr int kBarBytes = 8 * kStages;
  static constexpr int kWarpSmem = kStages * kStageBytes + 128;  // stages + barriers (padded)
  static constexpr int kSmemBytes = kWarps * kWarpSmem;
  static constexpr float kC = inv_sqrt_block(B);
};

struct RQArgs {
  const uint16_t* x;       // bf16 [n_units * E]
  int64_t n_units;
  uint8_t* codes;          // [n_units * E / 2]
  uint8_t* scales;         // [n_units * E / g]
  float* tensor_scale;     // NV: static -> read; dynamic -> written by CTA 0
  const float* partials;   // NV dynamic: per-CTA rotated amaxima from the amax pass
  int n_partials;
  float* y_dump;           // [n_units * E] when dumping
};

// Butterflies of H_B on every B-block of v[0..E) (unnormalised, in place).
template <int B, int E>
__device__ __forceinline__ void fwht_inplace(float (&v)[E]) {
#pragma unroll
  for (int h = 1; h < B; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// Load one unit from shared memory with the chunk XOR, widening bf16 -> fp32.
template <int E>
__device__ __forceinline__ void load_unit(uint32_t saddr, int tau, float (&v)[E]) {
#pragma unroll
  for (int j = 0; j < E / 8; ++j) {
    const uint4 w = lds128(saddr + 16u * static_cast<uint32_t>(j ^ tau));
    v[8 * j + 0] = bf16_lo(w.x);
    v[8 * j + 1] = bf16_hi(w.x);
    v[8 * j + 2] = bf16_lo(w.y);
    v[8 * j + 3] = bf16_hi(w.y);
    v[8 * j + 4] = bf16_lo(w.z);
    v[8 * j + 5] = bf16_hi(w.z);
    v[8 * j + 6] = bf16_lo(w.w);
    v[8 * j + 7] = bf16_hi(w.w);
  }
}

__device__ __forceinline__ uint32_t parity32(uint32_t v) { return __popc(v) & 1u; }

// MX scale byte from the fp32 group amax A >= 0 (see fp4q.h for the rules).
template <int RULE>
__device__ __forceinline__ int mx_scale_byte(float A) {
  const uint32_t bits = __float_as_uint(A);
  const int eb = static_cast<int>(bits >> 23);          // biased exponent (sign is 0)
  const uint32_t man = bits & 0x7FFFFFu;
  int bump = 0;
  if (RULE == kRuleCeil) bump = man > 0x400000u;       // mantissa above 1.5
  if (RULE == kRuleOas) bump = man > 0x600000u;        // mantissa above 1.75
  int byte = eb - 2 + bump;                            // e + 127 with e = floor(log2 A) - 2 + bump
  return byte < 0 ? 0 : (byte > 254 ? 254 : byte);
}

// 2^(127 - byte) as fp32 (byte in [0, 253]).
__device__ __forceinline__ float mx_inv_scale(int byte) {
  return __uint_as_float(static_cast<uint32_t>(254 - byte) << 23);
}

// Quantize one rotated unit v (unnormalised butterfly sums) and store its codes / scales.
template <class Cfg>
__device__ __forceinline__ void quantize_store_unit(float (&v)[Cfg::kE], int64_t unit, int tau, float s_g,
                                                    float nv_den, const RQArgs& a) {
  constexpr int E = Cfg::kE, G = Cfg::kGroup, NG = Cfg::kGroupsPerUnit;
  constexpr float c = Cfg::kC;
  uint32_t words[E / 8];
  uint32_t sbytes[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < G; ++i) m = fmaxf(m, fabsf(v[q * G + i]));
    const float A = m * c;                 // = max |fl(v * c)|: rounding is monotonic
    float mult;
    uint32_t keep = 0xFFFFFFFFu;
    if (Cfg::kFmt == kMX) {
      const int byte = mx_scale_byte<Cfg::kRule>(A);
      sbytes[q] = static_cast<uint32_t>(byte);
      mult = c * mx_inv_scale(byte);      // exact: a power-of-two multiple of c
    } else {
      const float s_b = __fdiv_rn(A, nv_den);
      const uint32_t byte = e4m3_encode(s_b);
      sbytes[q] = byte;
      const float S = e4m3_decode(byte) * s_g;
      if (S == 0.0f) keep = 0u;           // a zero block scale gives zero codes
      mult = S == 0.0f ? 0.0f : c * __frcp_rn(S);
    }
#pragma unroll
    for (int j = 0; j < G / 8; ++j) {
      const int i = q * G + 8 * j;
      uint32_t w = e2m1x8(v[i] * mult, v[i + 1] * mult, v[i + 2] * mult, v[i + 3] * mult, v[i + 4] * mult,
                          v[i + 5] * mult, v[i + 6] * mult, v[i + 7] * mult);
      const int chunk = i / 8;
      if (parity32(static_cast<uint32_t>(tau & chunk))) w ^= 0x88888888u;
      words[chunk] = w & keep;
    }
  }
  // codes: E/2 bytes per unit
  uint8_t* cp = a.codes + unit * (E / 2);
  if constexpr (E == 16) {
    stg64(cp, words[0], words[1]);
  } else if constexpr (E == 32) {
    stg128(cp, words[0], words[1], words[2], words[3]);
  } else {
#pragma unroll
    for (int k = 0; k < E / 32; ++k) stg128(cp + 16 * k, words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]);
  }
  // scales: E/g bytes per unit
  uint8_t* sp = a.scales + unit * NG;
  if constexpr (NG == 1) {
    *sp = static_cast<uint8_t>(sbytes[0]);
  } else if constexpr (NG == 2) {
    *reinterpret_cast<uint16_t*>(sp) = static_cast<uint16_t>(sbytes[0] | (sbytes[1] << 8));
  } else if constexpr (NG == 4) {
    *reinterpret_cast<uint32_t*>(sp) = sbytes[0] | (sbytes[1] << 8) | (sbytes[2] << 16) | (sbytes[3] << 24);
  } else {
    static_assert(NG == 8, "unit holds 1, 2, 4 or 8 groups");
    stg64(sp, sbytes[0] | (sbytes[1] << 8) | (sbytes[2] << 16) | (sbytes[3] << 24),
          sbytes[4] | (sbytes[5] << 8) | (sbytes[6] << 16) | (sbytes[7] << 24));
  }
  if constexpr (Cfg::kDump) {
    float* yp = a.y_dump + unit * E;
#pragma unroll
    for (int j = 0; j < E / 8; ++j) {
      const float sg = parity32(static_cast<uint32_t>(tau & j)) ? -c : c;
      float4 lo = make_float4(v[8 * j] * sg, v[8 * j + 1] * sg, v[8 * j + 2] * sg, v[8 * j + 3] * sg);
      float4 hi = make_float4(v[8 * j + 4] * sg, v[8 * j + 5] * sg, v[8 * j + 6] * sg, v[8 * j + 7] * sg);
      reinterpret_cast<float4*>(yp)[2 * j] = lo;
      reinterpret_cast<float4*>(yp)[2 * j + 1] = hi;
    }
  }
}

// Per-warp streaming skeleton shared by the quantize and the amax kernels.  `body(v, unit,
// tau)` is called once per unit with the rotated (unnormalised) values.  Returns false when
// a bounded wait ran out.
template <class Cfg, class Body>
__device__ __forceinline__ bool stream_units(const uint16_t* __restrict__ x, int64_t n_units, uint8_t* warp_smem,
                                             Body&& body) {
  constexpr int S = Cfg::kStages, SU = Cfg::kUnitsPerStage, E = Cfg::kE;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t total_warps = static_cast<int64_t>(gridDim.x) * Cfg::kWarps;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * Cfg::kWarps + warp;
  const int64_t u0 = (w * n_units) / total_warps;
  const int64_t u1 = ((w + 1) * n_units) / total_warps;
  const int64_t n_stages = (u1 - u0 + SU - 1) / SU;
  const uint32_t bar0 = smem_addr(warp_smem);
  const uint32_t buf0 = smem_addr(warp_smem + 128);
  const int tau = (lane >> Cfg::kTauShift) & Cfg::kTauMask;

  auto issue = [&](int64_t t) {
    const int st = static_cast<int>(t % S);
    const int64_t us = u0 + t * SU;
    const int64_t cnt = (u1 - us) < SU ? (u1 - us) : SU;
    const uint32_t bytes = static_cast<uint32_t>(cnt) * (E * 2);
    const uint32_t bar = bar0 + 8u * st;
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(buf0 + static_cast<uint32_t>(st) * Cfg::kStageBytes, x + us * E, bytes, bar);
  };

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
    fence_mbar_init();
    for (int64_t t = 0; t < S && t < n_stages; ++t) issue(t);
  }
  __syncwarp();

  bool ok = true;
#pragma unroll 1
  for (int64_t t = 0; t < n_stages; ++t) {
    const int st = static_cast<int>(t % S);
    const uint32_t parity = static_cast<uint32_t>((t / S) & 1);
    // Every lane waits (the wait is what makes the copied bytes visible to it); the warp
    // leaves together if any lane's wait ran out.
    const bool mine = mbar_wait_bounded(bar0 + 8u * st, parity);
    if (!__all_sync(0xFFFFFFFFu, mine)) {
      ok = false;
      // Let the copies already issued for the later stages land before the warp leaves.
      for (int64_t t2 = t + 1; t2 < n_stages && t2 < t + S; ++t2)
        mbar_wait_bounded(bar0 + 8u * static_cast<int>(t2 % S), static_cast<uint32_t>((t2 / S) & 1));
      break;
    }
    const int64_t us = u0 + t * SU;
    const int64_t cnt = (u1 - us) < SU ? (u1 - us) : SU;
    const uint32_t sbase = buf0 + static_cast<uint32_t>(st) * Cfg::kStageBytes;
#pragma unroll
    for (int r = 0; r < Cfg::kR; ++r) {
      const int lu = r * 32 + lane;
      if (lu < cnt) {
        float v[E];
        load_unit<E>(sbase + static_cast<uint32_t>(lu) * (E * 2), tau, v);
        fwht_inplace<Cfg::kBlock, E>(v);
        body(v, us + lu, tau);
      }
    }
    __syncwarp();
    if (lane == 0 && t + S < n_stages) {
      fence_proxy_async_smem();
      issue(t + S);
    }
  }
  return ok;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads) rotate_quantize_kernel(RQArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_tensor_scale;
  const int warp = threadIdx.x >> 5;
  float s_g = 1.0f;
  if constexpr (Cfg::kFmt == kNV) {
    if constexpr (Cfg::kRule == kRuleNvDynamic) {
      if (warp == 0) {
        float m = 0.0f;
        for (int i = threadIdx.x; i < a.n_partials; i += 32) m = fmaxf(m, a.partials[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (threadIdx.x == 0) {
          const float sg = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
          s_tensor_scale = sg;
          if (blockIdx.x == 0) *a.tensor_scale = sg;
        }
      }
    } else {
      if (threadIdx.x == 0) s_tensor_scale = *a.tensor_scale;
    }
    __syncthreads();
    s_g = s_tensor_scale;
  }
  const float nv_den = 6.0f * s_g;
  stream_units<Cfg>(a.x, a.n_units, smem + warp * Cfg::kWarpSmem,
                    [&](float (&v)[Cfg::kE], int64_t unit, int tau) {
                      quantize_store_unit<Cfg>(v, unit, tau, s_g, nv_den, a);
                    });
}

// Rotated amax: every CTA writes max |fl(y)| over its warps' ranges to partials[blockIdx.x].
template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads) rotated_amax_kernel(const uint16_t* __restrict__ x, int64_t n_units,
                                                                     float* __restrict__ partials) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_max[Cfg::kWarps];
  const int warp = threadIdx.x >> 5;
  float m = 0.0f;
  stream_units<Cfg>(x, n_units, smem + warp * Cfg::kWarpSmem, [&](float (&v)[Cfg::kE], int64_t, int) {
#pragma unroll
    for (int i = 0; i < Cfg::kE; ++i) m = fmaxf(m, fabsf(v[i]));
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) s_max[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < Cfg::kWarps; ++i) r = fmaxf(r, s_max[i]);
    partials[blockIdx.x] = r * Cfg::kC;
  }
}

// s_g = fp32(max(partials) / 2688), 1 for an all-zero tensor.  One warp.
__global__ void tensor_scale_finalize_kernel(const float* __restrict__ partials, int n, float* __restrict__ out) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += 32) m = fmaxf(m, partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (threadIdx.x == 0) *out = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
}

// Dequantize: one thread per unit of E = max(b, g) elements; optional inverse rotation.
template <int FMT, int B, bool UNROTATE>
__global__ void __launch_bounds__(128) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ scales,
                                                         const float* __restrict__ tensor_scale, int64_t n_units,
                                                         float* __restrict__ out) {
  constexpr int G = FMT == kMX ? 32 : 16;
  constexpr int E = cmax(B, G);
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (unit >= n_units) return;
  const float s_g = FMT == kNV ? *tensor_scale : 1.0f;
  float v[E];
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes + unit * (E / 2));
#pragma unroll
  for (int q = 0; q < E / G; ++q) {
    const uint32_t byte = scales[unit * (E / G) + q];
    float S;
    if (FMT == kMX) {
      S = byte == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);   // 2^(byte - 127)
    } else {
      S = e4m3_decode(byte) * s_g;
    }
#pragma unroll
    for (int j = 0; j < G / 8; ++j) {
      const uint32_t w = cw[(q * G) / 8 + j];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[q * G + 8 * j + k] = e2m1_decode(w >> (4 * k)) * S;
    }
  }
  if (UNROTATE) {
    fwht_inplace<B, E>(v);
    constexpr float c = inv_sqrt_block(B);
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] *= c;
  }
  float4* op = reinterpret_cast<float4*>(out + unit * E);
#pragma unroll
  for (int i = 0; i < E / 4; ++i) op[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

}  // namespace fp4q
