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

enum : int { kMX = 0, kNV = 1, kMBS = 2 };   // kMBS: MXFP4 under MBS-Static macro-block scales
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

// 1/sqrt(b) as an unevaluated sum hi + lo of two fp32 values (hi = RN(1/sqrt(b))).  Then
// fma(s, hi, RN(s lo)) is the correctly rounded s/sqrt(b) except when s/sqrt(b) lies within
// about 2^-48 (relative) of a rounding boundary.
__host__ __device__ constexpr double inv_sqrt_block_f64(int b) {
  return b == 1     ? 1.0
         : b == 2   ? 0.70710678118654752440
         : b == 4   ? 0.5
         : b == 8   ? 0.35355339059327376220
         : b == 16  ? 0.25
         : b == 32  ? 0.17677669529663688110
         : b == 64  ? 0.125
         : b == 128 ? 0.08838834764831844055
                    : 0.0;
}
__host__ __device__ constexpr float inv_sqrt_block_lo(int b) {
  return static_cast<float>(inv_sqrt_block_f64(b) - static_cast<double>(inv_sqrt_block(b)));
}
// 1/sqrt(b) is a power of two for b = 1, 4, 16, 64 (even log2 b).
__host__ __device__ constexpr bool inv_sqrt_block_is_pow2(int b) { return (ilog2(b) & 1) == 0; }

// Correctly rounded m / sqrt(b) (see inv_sqrt_block_lo).
template <int B>
__device__ __forceinline__ float scale_by_inv_sqrt(float m) {
  if constexpr (inv_sqrt_block_is_pow2(B)) {
    return m * inv_sqrt_block(B);
  } else {
    return fmaf(m, inv_sqrt_block(B), m * inv_sqrt_block_lo(B));
  }
}

// Compile-time shape of one kernel instance.  MINU is the smallest unit: 32 when the
// tensor's element count allows it (fewer per-unit costs, 16-byte code stores), else 16.
template <int FMT, int B, int RULE, bool DUMP, int MINU = 32>
struct RQConfig {
  static constexpr int kFmt = FMT;
  static constexpr int kBlock = B;
  static constexpr int kRule = RULE;
  static constexpr bool kDump = DUMP;
  static constexpr int kGroup = FMT == kNV ? 16 : 32;
  static constexpr int kE = cmax(cmax(B, kGroup), MINU);  // elements per unit
  static_assert(FMT != kMBS || kE == 128, "an MBS unit is one 128-element macro block");
  static constexpr int kPairs = kE / 2;                   // packed fp32 pairs per unit
  static constexpr int kChunks = kE / 8;                  // 16-byte chunks per unit
  static constexpr int kGroupsPerUnit = kE / kGroup;
  // Units per lane per stage: a stage of 2 KB (E <= 32), 4 KB (E = 64) or 8 KB (E = 128).
  static constexpr int kR = cmax(1, 32 / kE);
  static constexpr int kUnitsPerStage = 32 * kR;
  static constexpr int kStageBytes = kUnitsPerStage * kE * 2;
  static constexpr int kStages = kE >= 64 ? 3 : 2;
  static constexpr int kWarps = kE >= 128 ? 2 : 4;        // warps per CTA
  static constexpr int kThreads = kWarps * 32;
  // Chunk-index XOR (see the file comment): as many low chunk bits as make a quarter-warp
  // conflict-free, but never more than the chunk bits inside one Hadamard block.
  static constexpr int kTauMaxChunks = cmin(kChunks, 8);
  static constexpr int kTauShift = 3 - ilog2(kTauMaxChunks);
  static constexpr int kTauMask = B >= 16 ? cmin(kTauMaxChunks, B / 8) - 1 : 0;
  static constexpr int kWarpSmem = kStages * kStageBytes + 128;  // stages + barriers (padded)
  static constexpr int kSmemBytes = kWarps * kWarpSmem;
  static constexpr float kC = inv_sqrt_block(B);
};

// Per-channel random signs of a randomised Hadamard rotation (mask == nullptr: none).  Bit
// (k mod 32) of mask[k / 32] set negates channel k; a unit of E elements sits at channel
// (u mod upr) * E of its row, upr = K / E; stage_step = (units per stage) mod upr.
struct ChannelSigns {
  const uint32_t* mask;
  int upr;
  int stage_step;
  int smem_words = 0;   // butterfly kernels: words of the mask to stage in shared memory (0: read it in place)
};

// Most mask words a butterfly CTA stages in shared memory (16 KB: K <= 131072).
constexpr int kSignSmemMaxWords = 4096;

// Butterfly kernels with channel signs: the CTA copies the mask's words behind its stages
// (dynamic shared memory from byte `offset`) and reads them from there; called by every thread
// of the CTA, after the grid dependency (the mask may come from an earlier kernel).
__device__ __forceinline__ ChannelSigns stage_signs_in_smem(ChannelSigns sg, uint8_t* smem, int offset) {
  if (sg.mask == nullptr || sg.smem_words == 0) return sg;
  uint32_t* ms = reinterpret_cast<uint32_t*>(smem + offset);
  for (int w = threadIdx.x; w < sg.smem_words; w += blockDim.x) ms[w] = __ldg(sg.mask + w);
  __syncthreads();
  sg.mask = ms;
  return sg;
}

struct RQArgs {
  const uint16_t* x;       // bf16 [n_units * E]
  int64_t n_units;
  uint8_t* codes;          // [n_units * E / 2]
  uint8_t* scales;         // [n_units * E / g]
  float* tensor_scale;     // NV: static -> read; dynamic -> written by CTA 0
  const float* partials;   // NV dynamic: per-CTA rotated amaxima from the amax pass
  int n_partials;
  float* y_dump;           // [n_units * E] when dumping
  ChannelSigns signs;      // per-channel random signs (mask nullptr: none)
  uint8_t* macro;          // MBS: [n_units] macro-scale bytes
};

// Per-lane constants of the chunk XOR: tau, and for each of tau's (at most three) bits the
// code-word mask that flips the sign bits of a chunk (0x88888888) when that bit is set.
// Output chunk j comes out of the butterfly with its sign flipped when popcount(tau & j) is
// odd, i.e. its mask is the XOR of basis[b] over the bits b of j.
struct LaneXor {
  int tau;
  uint32_t basis[3];
};

template <class Cfg>
__device__ __forceinline__ LaneXor lane_xor(int lane) {
  LaneXor lx;
  lx.tau = (lane >> Cfg::kTauShift) & Cfg::kTauMask;
#pragma unroll
  for (int b = 0; b < 3; ++b) lx.basis[b] = ((lx.tau >> b) & 1) ? 0x88888888u : 0u;
  return lx;
}

// Sign mask for the packed codes of output chunk j: the chunk XOR's flip, and (B >= 2) the
// negated odd elements of the first butterfly stage (high nibbles, 0x80808080).
template <int B>
__device__ __forceinline__ uint32_t chunk_sign_mask(const LaneXor& lx, int j) {
  uint32_t m = B >= 2 ? 0x80808080u : 0u;
  if (j & 1) m ^= lx.basis[0];
  if (j & 2) m ^= lx.basis[1];
  if (j & 4) m ^= lx.basis[2];
  return m;
}

// The unit's E sign bits, as E/32 words (E = 16: the low 16 bits of one word).
template <int E>
struct UnitSigns {
  uint32_t w[E >= 32 ? E / 32 : 1];
};

template <int E>
__device__ __forceinline__ UnitSigns<E> unit_signs(const uint32_t* mask, int cu) {
  UnitSigns<E> m;
  const int c0 = cu * E;
  if constexpr (E >= 32) {
#pragma unroll
    for (int i = 0; i < E / 32; ++i) m.w[i] = mask[(c0 >> 5) + i];   // shared or global memory
  } else {
    m.w[0] = (mask[c0 >> 5] >> (c0 & 31)) & 0xFFFFu;
  }
  return m;
}

// XOR masks that negate the bf16 elements of one 16-byte chunk (8 elements, word i holding
// elements 2i and 2i+1) whose sign bits are set in byte `mb`.
// One multiply places two copies of the byte so that bits 2i and 2i+1 land on bits 15 and 31
// (the two shifted copies occupy disjoint bit ranges, so the sum carries nowhere), and one AND
// keeps those two bits.
__device__ __forceinline__ uint4 chunk_sign_xor(uint32_t mb) {
  const uint32_t b = mb & 0xFFu;
  uint4 r;
  r.x = (b * 0x40008000u) & 0x80008000u;   // b << 15 + b << 30
  r.y = (b * 0x10002000u) & 0x80008000u;   // b << 13 + b << 28
  r.z = (b * 0x04000800u) & 0x80008000u;   // b << 11 + b << 26
  r.w = (b * 0x01000200u) & 0x80008000u;   // b << 9 + b << 24
  return r;
}

// The same four XOR words folded into one: bit 15 - i holds the sign of element 2i and bit
// 31 - i that of element 2i + 1, so word i of the chunk's XOR is (w << i) & 0x80008000.
__device__ __forceinline__ uint32_t chunk_sign_word(uint32_t mb) {
  const uint4 f = chunk_sign_xor(mb);
  return f.x | (f.y >> 1) | (f.z >> 2) | (f.w >> 3);
}

__device__ __forceinline__ uint4 chunk_sign_xor_word(uint32_t w) {
  return make_uint4(w & 0x80008000u, (w << 1) & 0x80008000u, (w << 2) & 0x80008000u, (w << 3) & 0x80008000u);
}

// Sign byte of original chunk q = j ^ tau of a unit (tau only touches the low three bits,
// so the word is one of two known at compile time).
template <int E>
__device__ __forceinline__ uint32_t unit_sign_byte(const UnitSigns<E>& m, int j, int tau) {
  const int q = j ^ tau;
  uint32_t w;
  if constexpr (E >= 64) {
    const uint32_t a = m.w[(j >> 2)], b = m.w[(j >> 2) ^ 1];
    w = ((j ^ q) & 4) ? b : a;
  } else {
    w = m.w[0];
  }
  return (w >> (8 * (q & 3))) & 0xFFu;
}

// Load one unit from shared memory (chunk j read from position j ^ tau), widen bf16 to
// fp32 and run the butterfly of H_B on every B-block (unnormalised sums).  p[k] holds the
// pair (element 2k, element 2k + 1).  The first stage (distance 1) is taken straight from
// the bf16 pair; the others run on packed pairs, pair k against pair k + h/2.  Every element
// sees the same additions, in the same order, as in the scalar butterfly; for B >= 2 the odd
// elements come out negated (see bf16_pair_butterfly_oddneg).
template <int B, int E, bool SIGNED = false>
__device__ __forceinline__ void load_rotate_unit(uint32_t saddr, int tau, f32x2 (&p)[E / 2],
                                                 const UnitSigns<E>* sg = nullptr) {
#pragma unroll
  for (int j = 0; j < E / 8; ++j) {
    uint4 w = lds128(saddr + 16u * static_cast<uint32_t>(j ^ tau));
    if constexpr (SIGNED) {
      const uint4 f = chunk_sign_xor(unit_sign_byte<E>(*sg, j, tau));
      w.x ^= f.x;
      w.y ^= f.y;
      w.z ^= f.z;
      w.w ^= f.w;
    }
    if constexpr (B >= 2) {
      p[4 * j + 0] = bf16_pair_butterfly_oddneg(w.x);
      p[4 * j + 1] = bf16_pair_butterfly_oddneg(w.y);
      p[4 * j + 2] = bf16_pair_butterfly_oddneg(w.z);
      p[4 * j + 3] = bf16_pair_butterfly_oddneg(w.w);
    } else {
      p[4 * j + 0] = f2_pack(bf16_lo(w.x), bf16_hi(w.x));
      p[4 * j + 1] = f2_pack(bf16_lo(w.y), bf16_hi(w.y));
      p[4 * j + 2] = f2_pack(bf16_lo(w.z), bf16_hi(w.z));
      p[4 * j + 3] = f2_pack(bf16_lo(w.w), bf16_hi(w.w));
    }
  }
#pragma unroll
  for (int h = 2; h < B; h <<= 1) {
    const int hp = h / 2;
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      if ((k & hp) == 0) {
        const f32x2 a = p[k], b = p[k + hp];
        p[k] = f2_add(a, b);
        p[k + hp] = f2_sub(a, b);
      }
    }
  }
}

// max |value| over N pairs (N a power of two), with three-input maxima: each step folds
// both values of one pair into a running maximum.
template <int N>
__device__ __forceinline__ float pairs_amax(const f32x2* p) {
  // four independent chains for instruction-level parallelism, merged at the end
  constexpr int C = N >= 4 ? 4 : N;
  float m[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    float lo, hi;
    f2_unpack(p[c], lo, hi);
    m[c] = fmaxf(fabsf(lo), fabsf(hi));
  }
#pragma unroll
  for (int k = C; k < N; ++k) {
    float lo, hi;
    f2_unpack(p[k], lo, hi);
    m[k % C] = fmax3(m[k % C], fabsf(lo), fabsf(hi));
  }
  if constexpr (C == 4) return fmax3(fmaxf(m[0], m[1]), m[2], m[3]);
  if constexpr (C == 2) return fmaxf(m[0], m[1]);
  return m[0];
}

// MX scale byte from the fp32 group amax A >= 0 (see fp4q.h for the rules).
template <int RULE>
__device__ __forceinline__ int mx_scale_byte(float A) {
  const uint32_t bits = __float_as_uint(A);
  const int eb = static_cast<int>(bits >> 23);          // biased exponent (sign is 0)
  const uint32_t man = bits & 0x7FFFFFu;
  int bump = 0;
  if (RULE == kRuleCeil) bump = man > 0x400000u;       // mantissa above 1.5
  if (RULE == kRuleOas) bump = man > 0x600000u;        // mantissa above 1.75
  const int byte = eb - 2 + bump;                      // e + 127 with e = floor(log2 A) - 2 + bump
  return byte < 0 ? 0 : byte;                          // finite A keeps byte <= 253
}

// 2^(127 - byte) as fp32 (byte in [0, 253]).
__device__ __forceinline__ float mx_inv_scale(int byte) {
  return __uint_as_float(static_cast<uint32_t>(254 - byte) << 23);
}

// Correctly rounded a / d from rd = RN(1/d): one Markstein correction step of the product
// a * rd (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  Valid while the quotient and the residual
// stay in the normal range; a quotient below that range rounds to a zero E4M3 scale anyway.
__device__ __forceinline__ float div_rn_markstein(float a, float d, float rd) {
  const float q0 = a * rd;
  const float r = fmaf(-q0, d, a);
  return fmaf(r, rd, q0);
}

// Element quotients v = y / X of N pairs of unnormalised sums s (y = RN(s / sqrt(b))), in the
// pairs' own (raw butterfly) signs.
//
// MX: X = 2^e, so v = s * (c 2^-e), c = fp32(1/sqrt(b)): one product with a power-of-two
// multiple of c.
template <int N>
__device__ __forceinline__ void mx_quotients(const f32x2* s, int byte, float c, f32x2 (&v)[N]) {
  const float mult = c * mx_inv_scale(byte);
  const f32x2 mm = f2_pack(mult, mult);
#pragma unroll
  for (int t = 0; t < N; ++t) v[t] = f2_mul(s[t], mm);
}

// NV: the correctly rounded quotient y / S.  With a power-of-two 1/sqrt(b) it is folded into
// the divisor (exactly): s / (S sqrt(b)); otherwise y is first rounded from s with the
// two-term constant.  Sd is the divisor, rd = RN(1 / Sd).
struct NvDivisor {
  float Sd, rd;
};

template <int B>
__device__ __forceinline__ NvDivisor nv_divisor(float S) {
  const float Sd = inv_sqrt_block_is_pow2(B) ? S * (1.0f / inv_sqrt_block(B)) : S;
  return {Sd, __frcp_rn(Sd)};
}

template <int B, int N>
__device__ __forceinline__ void nv_quotients(const f32x2* s, NvDivisor dv, f32x2 (&v)[N]) {
  const f32x2 rd2 = f2_pack(dv.rd, dv.rd), nSd2 = f2_pack(-dv.Sd, -dv.Sd);
#pragma unroll
  for (int t = 0; t < N; ++t) {
    f32x2 y = s[t];
    if constexpr (!inv_sqrt_block_is_pow2(B)) {
      constexpr float chi = inv_sqrt_block(B), clo = inv_sqrt_block_lo(B);
      y = f2_fma(y, f2_pack(chi, chi), f2_mul(y, f2_pack(clo, clo)));
    }
    const f32x2 q0 = f2_mul(y, rd2);   // Markstein correction, lane-wise
    const f32x2 rem = f2_fma(q0, nSd2, y);
    v[t] = f2_fma(rem, rd2, q0);
  }
}

// E2M1 code word of four pairs (element 0 in the low nibble).
__device__ __forceinline__ uint32_t e2m1x8_pairs(const f32x2 (&v)[4]) {
  float e[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) f2_unpack(v[t], e[2 * t], e[2 * t + 1]);
  return e2m1x8(e[0], e[1], e[2], e[3], e[4], e[5], e[6], e[7]);
}

// MBS-Static macro-scale byte from the fp32 macro-block maximum A_M: with
// fp32(A_M / 6) = 2^E (1 + f), m8 = ceil(256 f) mod 256 (the mantissa rounded up to 8 bits;
// 256 wraps to 0, which is s_M = 2 with every group exponent one higher).  A_M = 0 gives 0.
__device__ __forceinline__ uint32_t mbs_macro_byte(float A_M) {
  const float r = __fdiv_rn(A_M, 6.0f);
  if (r == 0.0f) return 0u;
  uint32_t bits = __float_as_uint(r);
  if (bits < 0x00800000u) bits = __float_as_uint(r * 0x1p64f);   // subnormal: the same mantissa, normalised
  const uint32_t F = bits & 0x7FFFFFu;                            // f = F / 2^23
  return ((F + 0x7FFFu) >> 15) & 0xFFu;
}

// s_M = 1 + m8 / 256 (exact).
__device__ __forceinline__ float mbs_macro_scale(uint32_t m8) { return 1.0f + static_cast<float>(m8) * (1.0f / 256.0f); }

// Quantize one rotated unit (pairs p, unnormalised butterfly sums) and store its codes and
// scales.  `lx` undoes the chunk XOR's sign flips.
template <class Cfg>
__device__ __forceinline__ void quantize_store_unit(const f32x2 (&p)[Cfg::kPairs], int64_t unit, const LaneXor& lx,
                                                    float s_g, float nv_den, float nv_rden, const RQArgs& a) {
  constexpr int E = Cfg::kE, G = Cfg::kGroup, NG = Cfg::kGroupsPerUnit;
  constexpr float c = Cfg::kC;
  uint32_t words[E / 8];
  uint32_t sbytes[NG];
  if constexpr (Cfg::kFmt == kMBS) {
    // the unit is one macro block: y' = RN(y / s_M), then MXFP4 groups on y'
    const float AM = scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<E / 2>(p));
    const uint32_t m8 = mbs_macro_byte(AM);
    a.macro[unit] = static_cast<uint8_t>(m8);
    f32x2 yq[E / 2];
    nv_quotients<Cfg::kBlock, E / 2>(p, nv_divisor<Cfg::kBlock>(mbs_macro_scale(m8)), yq);
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const int byte = mx_scale_byte<Cfg::kRule>(pairs_amax<G / 2>(&yq[q * G / 2]));
      sbytes[q] = static_cast<uint32_t>(byte);
#pragma unroll
      for (int j = 0; j < G / 8; ++j) {
        const int chunk = q * (G / 8) + j;
        f32x2 v[4];
        mx_quotients<4>(&yq[4 * chunk], byte, 1.0f, v);
        words[chunk] = e2m1x8_pairs(v) ^ chunk_sign_mask<Cfg::kBlock>(lx, chunk);
      }
    }
  } else {
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    // group amax of the fp32 rotated values: RN(max |s| / sqrt(b)) = max |RN(s / sqrt(b))|
    const float A = scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<G / 2>(&p[q * G / 2]));
    if constexpr (Cfg::kFmt == kMX) {
      const int byte = mx_scale_byte<Cfg::kRule>(A);
      sbytes[q] = static_cast<uint32_t>(byte);
#pragma unroll
      for (int j = 0; j < G / 8; ++j) {
        const int chunk = q * (G / 8) + j;
        f32x2 v[4];
        mx_quotients<4>(&p[4 * chunk], byte, c, v);
        words[chunk] = e2m1x8_pairs(v) ^ chunk_sign_mask<Cfg::kBlock>(lx, chunk);
      }
    } else {
      const float s_b = div_rn_markstein(A, nv_den, nv_rden);
      const uint32_t byte = e4m3_encode(s_b);
      sbytes[q] = byte;
      const float S = e4m3_decode(byte) * s_g;
      const uint32_t keep = S == 0.0f ? 0u : 0xFFFFFFFFu;   // a zero block scale gives zero codes
      const NvDivisor dv = nv_divisor<Cfg::kBlock>(S);
#pragma unroll
      for (int j = 0; j < G / 8; ++j) {
        const int chunk = q * (G / 8) + j;
        f32x2 v[4];
        nv_quotients<Cfg::kBlock, 4>(&p[4 * chunk], dv, v);
        words[chunk] = (e2m1x8_pairs(v) ^ chunk_sign_mask<Cfg::kBlock>(lx, chunk)) & keep;
      }
    }
  }
  }
  // codes: E/2 bytes per unit
  uint8_t* cp = a.codes + unit * (E / 2);
  if constexpr (E == 16) {
    stg64(cp, words[0], words[1]);
  } else {
#pragma unroll
    for (int k = 0; k < E / 32; ++k)
      stg128(cp + 16 * k, words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]);
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
      const uint32_t msk = chunk_sign_mask<Cfg::kBlock>(lx, j);
      const float se = (msk & 0x08u) ? -c : c;    // even elements: the chunk flip only
      const float so = (msk & 0x80u) ? -c : c;    // odd elements: flip and first-stage negation
      float v[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) f2_unpack(p[4 * j + t], v[2 * t], v[2 * t + 1]);
      reinterpret_cast<float4*>(yp)[2 * j] = make_float4(v[0] * se, v[1] * so, v[2] * se, v[3] * so);
      reinterpret_cast<float4*>(yp)[2 * j + 1] = make_float4(v[4] * se, v[5] * so, v[6] * se, v[7] * so);
    }
  }
}

// Per-warp streaming skeleton shared by the quantize and the amax kernels.  `body(p, unit)`
// is called once per unit with the rotated (unnormalised) pairs.  Returns false when a
// bounded wait ran out.
template <class Cfg, bool SIGNED = false, class Body>
__device__ __forceinline__ bool stream_units(const uint16_t* __restrict__ x, int64_t n_units, uint8_t* warp_smem,
                                             int tau, Body&& body, ChannelSigns sgn = {nullptr, 1, 0}) {
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
  }
  // Before the grid dependency only a hint: ask L2 for this warp's first S stages, so their
  // DRAM traffic overlaps the end of the kernel this one follows.  Nothing below reads or writes
  // global memory before the kernels this one depends on (for example the producer of x) have
  // finished.
  if (lane == 0)
    for (int64_t t = 0; t < S && t < n_stages; ++t) {
      const int64_t us = u0 + t * SU;
      const int64_t cnt = (u1 - us) < SU ? (u1 - us) : SU;
      bulk_prefetch_l2(x + us * E, static_cast<uint32_t>(cnt) * (E * 2));
    }
  pdl_wait();
  if (lane == 0)
    for (int64_t t = 0; t < S && t < n_stages; ++t) issue(t);
  __syncwarp();

  // SIGNED: channel-unit index (u mod upr) of this lane's r-th unit of the current stage
  int cu[Cfg::kR];
  if constexpr (SIGNED) {
#pragma unroll
    for (int r = 0; r < Cfg::kR; ++r) cu[r] = static_cast<int>((u0 + r * 32 + lane) % sgn.upr);
  }
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
    if (cnt == SU) {
      // full stage: no per-unit bounds test, so the R units interleave freely
#pragma unroll
      for (int r = 0; r < Cfg::kR; ++r) {
        const int lu = r * 32 + lane;
        f32x2 p[Cfg::kPairs];
        if constexpr (SIGNED) {
          const UnitSigns<E> m = unit_signs<E>(sgn.mask, cu[r]);
          load_rotate_unit<Cfg::kBlock, E, true>(sbase + static_cast<uint32_t>(lu) * (E * 2), tau, p, &m);
        } else {
          load_rotate_unit<Cfg::kBlock, E>(sbase + static_cast<uint32_t>(lu) * (E * 2), tau, p);
        }
        body(p, us + lu);
      }
    } else {
#pragma unroll
      for (int r = 0; r < Cfg::kR; ++r) {
        const int lu = r * 32 + lane;
        if (lu < cnt) {
          f32x2 p[Cfg::kPairs];
          if constexpr (SIGNED) {
            const UnitSigns<E> m = unit_signs<E>(sgn.mask, cu[r]);
            load_rotate_unit<Cfg::kBlock, E, true>(sbase + static_cast<uint32_t>(lu) * (E * 2), tau, p, &m);
          } else {
            load_rotate_unit<Cfg::kBlock, E>(sbase + static_cast<uint32_t>(lu) * (E * 2), tau, p);
          }
          body(p, us + lu);
        }
      }
    }
    if constexpr (SIGNED) {
#pragma unroll
      for (int r = 0; r < Cfg::kR; ++r) {
        cu[r] += sgn.stage_step;
        if (cu[r] >= sgn.upr) cu[r] -= sgn.upr;
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

// NV tensor scale s_g for every thread of the CTA: read (static rule), or reduced from the
// amax pass's per-CTA partial maxima (dynamic rule; CTA 0 also writes it out).  Contains a
// __syncthreads; every thread of the CTA calls it.
template <class Cfg>
__device__ __forceinline__ float cta_tensor_scale(float* tensor_scale, const float* partials, int n_partials,
                                                  float* s_slot) {
  pdl_wait();   // the tensor scale or the partial maxima come from an earlier kernel
  if constexpr (Cfg::kRule == kRuleNvDynamic) {
    if (threadIdx.x < 32) {
      float m = 0.0f;
      for (int i = threadIdx.x; i < n_partials; i += 32) m = fmaxf(m, partials[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (threadIdx.x == 0) {
        const float sg = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
        *s_slot = sg;
        if (blockIdx.x == 0) *tensor_scale = sg;
      }
    }
  } else {
    if (threadIdx.x == 0) *s_slot = *tensor_scale;
  }
  __syncthreads();
  return *s_slot;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads) rotate_quantize_kernel(RQArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_tensor_scale;
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5;
  const LaneXor lx = lane_xor<Cfg>(threadIdx.x & 31);
  float s_g = 1.0f;
  if constexpr (Cfg::kFmt == kNV) s_g = cta_tensor_scale<Cfg>(a.tensor_scale, a.partials, a.n_partials, &s_tensor_scale);
  const float nv_den = 6.0f * s_g;
  const float nv_rden = __frcp_rn(nv_den);
  auto body = [&](const f32x2 (&p)[Cfg::kPairs], int64_t unit) {
    quantize_store_unit<Cfg>(p, unit, lx, s_g, nv_den, nv_rden, a);
  };
  if (a.signs.mask) {
    pdl_wait();
    const ChannelSigns sg = stage_signs_in_smem(a.signs, smem, Cfg::kSmemBytes);
    stream_units<Cfg, true>(a.x, a.n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body, sg);
  } else
    stream_units<Cfg>(a.x, a.n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body);
}

// ---------------------------------------------------------------- quantization error

// The errors q - v of one pair of quotients v against their E2M1 codes q (round to nearest
// even, saturating at 6): the pair goes to E2M1 and straight back to f16x2 (exact: every E2M1
// value is an f16 value), then each q - v is one mixed-precision subtraction, rounded once to
// fp32.  |q - v| is also |(|v| - |q|)| (E2M1 rounding keeps the sign of v), so the squares are
// the error energies whatever the sign convention.
__device__ __forceinline__ void e2m1_pair_errors(f32x2 v, float& d0, float& d1) {
  float v0, v1;
  f2_unpack(v, v0, v1);
  asm("{\n .reg .b8 q;\n .reg .b32 h;\n .reg .b16 lo, hi;\n"
      " cvt.rn.satfinite.e2m1x2.f32 q, %3, %2;\n"
      " cvt.rn.f16x2.e2m1x2 h, q;\n"
      " mov.b32 {lo, hi}, h;\n"
      " sub.rn.f32.f16 %0, lo, %2;\n"
      " sub.rn.f32.f16 %1, hi, %3;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(v0), "f"(v1));
}

// Error energy of one group of quotients v (= y / X) against their E2M1 codes, and its
// signal energy, both in units of X^2: sum (v - q)^2 and sum v^2 (fp32; even and odd elements
// in separate sums, the signal as packed pairs, the errors as two scalar sums, which leaves
// the two differences where the subtractions put them).
template <int NP>
__device__ __forceinline__ void group_energies(const f32x2 (&v)[NP], float& sig, float& err) {
  f32x2 as = f2_pack(0.0f, 0.0f);
  float e0 = 0.0f, e1 = 0.0f;
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    as = f2_fma(v[t], v[t], as);
    float d0, d1;
    e2m1_pair_errors(v[t], d0, d1);
    e0 = fmaf(d0, d0, e0);
    e1 = fmaf(d1, d1, e1);
  }
  float a0, a1;
  f2_unpack(as, a0, a1);
  sig = a0 + a1;
  err = e0 + e1;
}

// 2^(2(byte - 127)) as fp64: X^2 for an MX scale byte.
__device__ __forceinline__ double mx_scale_sq(int byte) {
  return __longlong_as_double(static_cast<long long>(1023 + 2 * (byte - 127)) << 52);
}

// Signal and error energy of one rotated unit, accumulated into fp64 running sums.  The
// codes are those of quantize_store_unit (the same scale decisions and quotients).
template <class Cfg>
__device__ __forceinline__ void unit_energies(const f32x2 (&p)[Cfg::kPairs], float s_g, float nv_den, float nv_rden,
                                              double& sig, double& err) {
  constexpr int G = Cfg::kGroup, NG = Cfg::kGroupsPerUnit;
  constexpr float c = Cfg::kC;
  if constexpr (Cfg::kFmt == kMBS) {
    constexpr int E = Cfg::kE;
    const uint32_t m8 = mbs_macro_byte(scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<E / 2>(p)));
    const float sM = mbs_macro_scale(m8);
    const double sM2 = static_cast<double>(sM) * static_cast<double>(sM);
    f32x2 yq[E / 2];
    nv_quotients<Cfg::kBlock, E / 2>(p, nv_divisor<Cfg::kBlock>(sM), yq);
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const int byte = mx_scale_byte<Cfg::kRule>(pairs_amax<G / 2>(&yq[q * G / 2]));
      f32x2 v[G / 2];
      mx_quotients<G / 2>(&yq[q * G / 2], byte, 1.0f, v);
      float gs, ge;
      group_energies<G / 2>(v, gs, ge);
      const double X2 = mx_scale_sq(byte) * sM2;
      sig = fma(static_cast<double>(gs), X2, sig);
      err = fma(static_cast<double>(ge), X2, err);
    }
  } else {
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      const f32x2* pg = &p[q * G / 2];
      const float A = scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<G / 2>(pg));
      f32x2 v[G / 2];
      double X2;
      if constexpr (Cfg::kFmt == kMX) {
        const int byte = mx_scale_byte<Cfg::kRule>(A);
        mx_quotients<G / 2>(pg, byte, c, v);
        X2 = mx_scale_sq(byte);
      } else {
        const float s_b = div_rn_markstein(A, nv_den, nv_rden);
        const uint32_t byte = e4m3_encode(s_b);
        const float S = e4m3_decode(byte) * s_g;
        if (S == 0.0f) {
          // a zero block scale: every code is 0, the error is the whole signal
          constexpr double c64 = inv_sqrt_block_f64(Cfg::kBlock);
          double e2 = 0.0;
#pragma unroll
          for (int t = 0; t < G / 2; ++t) {
            float lo, hi;
            f2_unpack(pg[t], lo, hi);
            const double a = lo * c64, b = hi * c64;
            e2 = fma(a, a, fma(b, b, e2));
          }
          sig += e2;
          err += e2;
          continue;
        }
        nv_quotients<Cfg::kBlock, G / 2>(pg, nv_divisor<Cfg::kBlock>(S), v);
        X2 = static_cast<double>(S) * static_cast<double>(S);
      }
      float gs, ge;
      group_energies<G / 2>(v, gs, ge);
      sig = fma(static_cast<double>(gs), X2, sig);
      err = fma(static_cast<double>(ge), X2, err);
    }
  }
}

struct QEArgs {
  const uint16_t* x;
  int64_t n_units;
  float* tensor_scale;      // NV: static -> read; dynamic -> written by CTA 0
  const float* partials;    // NV dynamic: per-CTA rotated amaxima from the amax pass
  int n_partials;
  double* out_partials;     // [gridDim.x][2]: signal, error energy of each CTA
  unsigned int* ticket;     // CTAs done so far; 0 between calls (the last CTA resets it)
  double* out;              // [3]: signal, error, QSNR dB
  ChannelSigns signs;       // per-channel random signs (mask nullptr: none)
};

// out = {signal, error, QSNR in dB} from n per-CTA partial pairs, by one warp in a fixed
// order; +inf dB when the error is 0, -inf when only the signal is.
__device__ __forceinline__ void qe_final_sum(const double* partials, int n, double* out) {
  double s = 0.0, e = 0.0;
  for (int i = threadIdx.x & 31; i < n; i += 32) {
    s += __ldcg(partials + 2 * i);
    e += __ldcg(partials + 2 * i + 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
  }
  if ((threadIdx.x & 31) == 0) {
    out[0] = s;
    out[1] = e;
    out[2] = e == 0.0 ? __longlong_as_double(0x7FF0000000000000LL)
                      : (s > 0.0 ? 10.0 * log10(s / e) : __longlong_as_double(static_cast<long long>(0xFFF0000000000000ULL)));
  }
}

// Every CTA writes the signal and error energy of its warps' ranges to out_partials; the
// last CTA to finish (a ticket counter, as in a threadfence reduction) sums them in CTA order
// and writes out.  The ranges and the order of every sum are fixed by the grid, so the
// result is deterministic.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads) quant_error_kernel(QEArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_tensor_scale;
  __shared__ double s_part[Cfg::kWarps][2];
  __shared__ bool s_last;
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const LaneXor lx = lane_xor<Cfg>(lane);
  float s_g = 1.0f;
  if constexpr (Cfg::kFmt == kNV) s_g = cta_tensor_scale<Cfg>(a.tensor_scale, a.partials, a.n_partials, &s_tensor_scale);
  const float nv_den = 6.0f * s_g;
  const float nv_rden = __frcp_rn(nv_den);
  double sig = 0.0, err = 0.0;
  auto body = [&](const f32x2 (&p)[Cfg::kPairs], int64_t) { unit_energies<Cfg>(p, s_g, nv_den, nv_rden, sig, err); };
  if (a.signs.mask) {
    pdl_wait();
    const ChannelSigns sg = stage_signs_in_smem(a.signs, smem, Cfg::kSmemBytes);
    stream_units<Cfg, true>(a.x, a.n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body, sg);
  } else
    stream_units<Cfg>(a.x, a.n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sig += __shfl_xor_sync(0xFFFFFFFFu, sig, o);
    err += __shfl_xor_sync(0xFFFFFFFFu, err, o);
  }
  if (lane == 0) {
    s_part[warp][0] = sig;
    s_part[warp][1] = err;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double ts = 0.0, te = 0.0;
#pragma unroll
    for (int i = 0; i < Cfg::kWarps; ++i) {
      ts += s_part[i][0];
      te += s_part[i][1];
    }
    a.out_partials[2 * blockIdx.x] = ts;
    a.out_partials[2 * blockIdx.x + 1] = te;
    __threadfence();
    s_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last && warp == 0) {
    __threadfence();
    qe_final_sum(a.out_partials, static_cast<int>(gridDim.x), a.out);
    if (lane == 0) *a.ticket = 0u;
  }
}

// One warp waits on a barrier that nothing arrives on: the bounded wait gives up after
// kWaitLimitNs, records kStatusTimeout and the kernel returns (the failure path's self-test).
static __global__ void wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (threadIdx.x == 0) mbar_init(b, 1);
  __syncwarp();
  mbar_wait_bounded(b, 0u);   // phase 0 never completes
}

// The same result for an empty X (no CTA to finish): {0, 0, +inf}.  One warp.
static __global__ void quant_error_empty_kernel(const double* __restrict__ partials, double* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  qe_final_sum(partials, 0, out);
}

// Rotated amax: every CTA writes max |fl(y)| over its warps' ranges to partials[blockIdx.x], with
// fl(y) = RN(s / sqrt(b)) of the raw butterfly sum s, the value the quantizer takes its decisions on.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads) rotated_amax_kernel(const uint16_t* __restrict__ x, int64_t n_units,
                                                                     float* __restrict__ partials, ChannelSigns signs) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_max[Cfg::kWarps];
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5;
  const LaneXor lx = lane_xor<Cfg>(threadIdx.x & 31);
  float m = 0.0f;
  auto body = [&](const f32x2 (&p)[Cfg::kPairs], int64_t) { m = fmaxf(m, pairs_amax<Cfg::kPairs>(p)); };
  if (signs.mask) {
    pdl_wait();
    const ChannelSigns sg = stage_signs_in_smem(signs, smem, Cfg::kSmemBytes);
    stream_units<Cfg, true>(x, n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body, sg);
  } else
    stream_units<Cfg>(x, n_units, smem + warp * Cfg::kWarpSmem, lx.tau, body);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) s_max[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < Cfg::kWarps; ++i) r = fmaxf(r, s_max[i]);
    // RN(r / sqrt(b)): the correctly rounded scaling is monotone, so this is the maximum of the
    // elements' own fp32 values RN(sum / sqrt(b)), as the quantizer's group maxima are
    partials[blockIdx.x] = scale_by_inv_sqrt<Cfg::kBlock>(r);
  }
}

// s_g = fp32(max(partials) / 2688), 1 for an all-zero tensor.  One warp.
static __global__ void tensor_scale_finalize_kernel(const float* __restrict__ partials, int n, float* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
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
                                                         float* __restrict__ out, ChannelSigns signs,
                                                         const uint8_t* __restrict__ macro) {
  constexpr int G = FMT == kNV ? 16 : 32;
  constexpr int E = FMT == kMBS ? 128 : cmax(B, G);   // MBS: one macro block per unit
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (unit >= n_units) return;
  const float s_g = FMT == kNV ? *tensor_scale : 1.0f;
  float v[E];
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes + unit * (E / 2));
#pragma unroll
  for (int q = 0; q < E / G; ++q) {
    const uint32_t byte = scales[unit * (E / G) + q];
    float S;
    if (FMT != kNV) {
      S = byte == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);   // 2^(byte - 127)
      if (FMT == kMBS) S *= mbs_macro_scale(macro[unit]);                             // exact: 9-bit s_M
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
    if (signs.mask) {
      // the channel signs again, after the block rotation (Q^-1 = Q^T)
      const int c0 = static_cast<int>(unit % signs.upr) * E;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const uint32_t bit = (__ldg(signs.mask + ((c0 + i) >> 5)) >> ((c0 + i) & 31)) & 1u;
        v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (bit << 31));
      }
    }
  }
  float4* op = reinterpret_cast<float4*>(out + unit * E);
#pragma unroll
  for (int i = 0; i < E / 4; ++i) op[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

}  // namespace fp4q
