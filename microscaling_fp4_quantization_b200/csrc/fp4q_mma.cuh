// Tensor-core variant of the fused rotate + FP4 quantize kernel (sm_100a tcgen05).
//
// The flat stream of M*K bf16 values is read as R = M*K/b rows of one Hadamard block each,
// and the rotation is the product Y = X_rows * H_b: an M = 128, N = b, K = b bf16 MMA with
// fp32 accumulation in tensor memory (TMEM).  The products x * (+-1) are exact; the sums
// are accumulated in fp32 by the tensor core.
//
// Work is cut into super-tiles of 128 TMEM columns: 128 / b row-tiles of 128 rows, 16384
// elements, 32 KB of input.  CTAs are persistent (one or two per SM) and take super-tiles
// round-robin.  Roles, per CTA of 2 + 8 + 2 or 2 + 16 + 8 warps:
//   warp 0        producer: for b <= 32 one contiguous bulk copy per stage (left unswizzled,
//                 see MmaConfig::kBulk), else TMA tensor loads (2-D map over the rows, swizzled
//                 K-major layout), into a ring of shared-memory stages, completion on mbarriers;
//   warp 1        TMEM owner (alloc / dealloc of two accumulator buffers) and MMA issuer:
//                 b / 16 MMAs per row-tile into one of the buffers, then tcgen05.commit to free
//                 the stage and to hand the buffer to the epilogue;
//   warps 2..     epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31 (tcgen05.ld), one
//                 column slice of the super-tile each, so each thread owns one row (one rotated
//                 block, or a part of one) and does the amax, scale, E2M1 rounding, packing and
//                 stores of it in its registers; it frees the buffer as soon as its slice is read;
//                 the error pass and the amax pass keep sums or maxima instead of storing;
//   the last 2 or 8 warps   sign warps, for plans with per-channel signs only: they flip the
//                 signs of each landed stage's elements in shared memory (XOR words from a table
//                 staged once per CTA) before the MMA warp may read it.
// All roles wait on the grid dependency (programmatic dependent launch) before touching global
// memory, so the set-up overlaps the end of the kernel this one follows; before it the producer
// only asks L2 to prefetch its first stages.
// H_b is written into shared memory once per CTA, in the same swizzled layout.
// Every wait is bounded in time; a wait that runs out records kStatusTimeout, and the CTA
// lets its issued copies and MMAs land before it frees TMEM and leaves.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"

namespace fp4q {

// QE: the error pass.  The epilogue makes the same scale decisions and codes as the quantizer
// and accumulates the signal and error energies instead of storing anything.
// AMAX: the amax pass of the NVFP4 per-tensor scale.  The epilogue keeps only the largest
// magnitude of the rotated sums and each CTA writes its maximum, scaled by 1/sqrt(b).
template <int FMT, int B, int RULE, bool DUMP, bool QE = false, bool AMAX = false>
struct MmaConfig {
  static constexpr int kFmt = FMT;
  static constexpr int kBlock = B;
  static constexpr int kRule = RULE;
  static constexpr bool kDump = DUMP;
  static constexpr bool kQE = QE;
  static constexpr bool kAmax = AMAX;
  static_assert(!(QE && DUMP), "the error pass stores nothing");
  static_assert(!(AMAX && (QE || DUMP || FMT != kNV)), "the amax pass runs in the NVFP4 configuration alone");
  static constexpr int kGroup = FMT == kNV ? 16 : 32;   // MXFP4 and MBS-Static: 32
  static_assert(B >= 16 && B >= kGroup && B <= 128, "one block holds whole groups");
  // MBS-Static: a 128-element macro block is 128 / b consecutive rows (TMEM lanes of one warp)
  // for b <= 64, and both column halves of one row for b = 128
  static constexpr int kMacroLanes = FMT == kMBS ? (B < 128 ? 128 / B : 1) : 1;
  static constexpr int kKB = B > 64 ? 64 : B;        // K elements per swizzled row (one TMA box row)
  static constexpr int kRB = 2 * kKB;                // bytes per swizzled row
  static constexpr int kHalves = B / kKB;            // K-halves (2 for b = 128)
  static constexpr uint32_t kLayout = kRB == 32 ? 6u : kRB == 64 ? 4u : 2u;   // SW32 / SW64 / SW128
  static constexpr int kSwzBits = kRB == 32 ? 1 : kRB == 64 ? 2 : 3;
  // A super-tile is 128 TMEM columns of 128 rows: 16384 elements, 32 KB of input.
  static constexpr int kSuperCols = 128;
  static constexpr int kRowTiles = kSuperCols / B;   // row-tiles of 128 rows per super-tile
  static constexpr int kRowsPerTile = 128 * kRowTiles;
  static constexpr int kStageBytes = kSuperCols * 256;
  static constexpr int kStages = B >= 128 ? 2 : 3;
  static constexpr int kHBytes = B * B * 2;
  // TMA boxes per stage: up to 256 rows of kKB elements
  static constexpr int kBoxRows = B >= 128 ? 128 : (kRowsPerTile < 256 ? kRowsPerTile : 256);
  static constexpr int kBoxes = B >= 128 ? 2 : kRowsPerTile / kBoxRows;
  static constexpr int kBoxBytes = kBoxRows * kRB;
  // Epilogue warps: kSlices per TMEM lane quarter, each taking kEpiCols of the super-tile's
  // columns.  NVFP4 (the heavier per-element work) gets four per quarter for b <= 64, the others
  // two.  CTAs per SM, from measurement: 1 for NVFP4 b <= 64 (18 warps), else 2.
  static constexpr int kSlices = (FMT == kNV && B <= 64) ? 4 : 2;
  static constexpr int kEpiWarps = 4 * kSlices;
  static constexpr int kEpiCols = kSuperCols / kSlices;   // columns per epilogue warp
  static constexpr int kCtasPerSm = (FMT == kNV && B <= 64) ? 1 : 2;
  // plans with per-channel signs: these warps flip the signs of each landed stage's elements
  // (eight where one CTA has the SM, two beside a second CTA)
  static constexpr int kSignWarps = kCtasPerSm == 1 ? 8 : 2;
  static constexpr int kThreads = 32 * (2 + kEpiWarps + kSignWarps);
  static constexpr int kTmemCols = 2 * kSuperCols;   // two accumulator buffers
  static constexpr float kC = inv_sqrt_block(B);
  // shared memory: [align pad][stages][H][barriers]
  static constexpr int kTableBytes = FMT == kNV ? 256 * 4 : 0;   // NV: element multiplier per E4M3 byte
  // b <= 32: rows of 32 / 64 bytes make TMA tensor boxes slow, so a stage is one contiguous bulk
  // copy, left unswizzled.  Read through the swizzled descriptor, row r's K index comes out
  // XORed with 8 * t(r) (t = (r >> 2) & 1 for 32-byte rows, (r >> 1) & 3 for 64-byte rows), which
  // turns into a sign flip of output column n when popcount(n & 8 t(r)) is odd (H[k ^ T][n] =
  // (-1)^popcount(T & n) H[k][n]); the epilogue undoes it on the packed codes.
  static constexpr bool kBulk = B <= 32;
  static constexpr int kFlipShift = kRB == 32 ? 2 : 1;
  static constexpr int kFlipMask = kRB == 32 ? 1 : 3;
  static constexpr int kBarOffset = kStages * kStageBytes + kHBytes + kTableBytes;
  static constexpr int kMaskOffset = (kBarOffset + 8 * (3 * kStages + 4) + 15) / 16 * 16;
  static constexpr int kSmemBytes = 1024 + kMaskOffset;   // without the staged sign mask
  // Plans with channel signs stage the mask (K / 8 bytes) after the barriers when it fits
  // beside kCtasPerSm CTAs: 228 KB of shared memory per SM, of which each CTA also holds 1 KB
  // reserved by the system and 1 KB of static variables (the kernel's __shared__ scalars,
  // padded to the 1024-byte alignment of the dynamic array that follows them).
  static constexpr int kMaskRoom = (233472 / kCtasPerSm - 2048 - kSmemBytes) / 16 * 16;
  static constexpr int kMaskSmemMax = kMaskRoom < 16384 ? kMaskRoom : 16384;
  static_assert(kMaskSmemMax >= 1024, "room for the sign mask of K <= 8192");
  // Where one CTA has the SM, the sign warps read an expanded table instead of the mask's
  // bits: the four XOR words of every 8-channel chunk of a row (16 bytes each), stored twice
  // over so that a block index below 2 K/b needs no wrap; 4 K bytes, staged when they fit
  // (K <= 16384).
  static constexpr bool kSignTable = kCtasPerSm == 1;
  static constexpr int kSignTableMax = kSignTable ? cmin(kMaskRoom, 65536) : 0;
  static constexpr int kSignSmemMax = cmax(kMaskSmemMax, kSignTableMax);
  // The sign warps' walk over a stage: a region (the whole stage in the bulk layout, one K-half
  // of swizzled 128-byte rows otherwise) holds kSignCpr 16-byte chunks per row; a lane's chunks
  // sit kSignRowStep rows apart, kSignPerLane of them per region.
  static constexpr int kSignCpr = kBulk ? B / 8 : 8;
  static constexpr int kSignRegions = kBulk ? 1 : kHalves;
  static constexpr int kSignLaneStride = 32 * kSignWarps;
  static constexpr int kSignRowStep = kSignLaneStride / kSignCpr;
  static constexpr int kSignPerLane = kStageBytes / kSignRegions / 16 / kSignLaneStride;
  // Where two CTAs share the SM, the sign warps read a word table when it fits: one 32-bit
  // word per 8-channel chunk (bit 15 - i holds the sign of element 2i, bit 31 - i that of
  // element 2i + 1), for blocks 0 .. K/b - 1 + kSignExt, block k >= K/b repeating block
  // k - K/b, so that a lane's chunks of a stage sit at fixed offsets from its first.
  static constexpr int kSignExt = (kSignPerLane - 1) * kSignRowStep;
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(B >> 3) << 17) |
                                     (static_cast<uint32_t>(128 >> 4) << 24);
};

struct MmaArgs {
  const uint16_t* x;       // bf16 [R][b] (the bulk-copy loads)
  int64_t n_rows;          // R = M*K / b
  int64_t n_super;         // super-tiles
  uint8_t* codes;
  uint8_t* scales;
  float* tensor_scale;
  const float* partials;
  int n_partials;
  float* y_dump;
  const uint8_t* sign_bytes;   // per-channel signs (bit k of byte k / 8 negates channel k), or null
  int64_t sign_upr;            // Hadamard blocks per matrix row, K / b
  int sign_smem;               // bytes staged in shared memory (0: the mask is read from global)
  int sign_table;              // those bytes are: 1 the expanded sign table, 2 the word table, 0 the mask's words
  uint8_t* macro;              // MBS-Static: the macro-scale bytes [R * b / 128]
  // error pass only: [gridDim.x][2] per-CTA signal, error energies; the ticket counter (0
  // between calls, reset by the last CTA); out [3] = signal, error, QSNR dB
  double* qe_partials;
  unsigned int* qe_ticket;
  double* qe_out;
  // amax pass only: amax_out[CTA] = RN(max |rotated sum| / sqrt(b)) of the CTA's rows; CTA 0
  // also zeroes amax_out[gridDim.x .. amax_slots), so that a reduction over all the slots
  // sees only this call's maxima
  float* amax_out;
  int amax_slots;
};

// Offset of byte `off` inside a swizzled K-major tile (rows of 32 / 64 / 128 bytes): the
// 16-byte chunk index is XORed with the row bits above it, as the TMA swizzle modes lay
// them out (and as the MMA descriptors' layout types read them).
template <int BITS>
__device__ __forceinline__ uint32_t swizzle_off(uint32_t off) {
  return off ^ (((off >> 7) & ((1u << BITS) - 1u)) << 4);
}

__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t addr, uint32_t sbo_bytes, uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// The box at (x, y) of a 2-D tensor map into L2 (a hint, as bulk_prefetch_l2).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Quantize one group of G rotated sums s (unnormalised, as produced by the MMA): E2M1 code
// words (G / 8) and the scale byte.
template <class Cfg, int G>
__device__ __forceinline__ uint32_t quantize_group(const float (&s)[G], uint32_t (&words)[G / 8], const float* nv_tab,
                                                   float nv_den, float nv_rden) {
  constexpr float c = Cfg::kC;
  f32x2 p[G / 2];
#pragma unroll
  for (int k = 0; k < G / 2; ++k) p[k] = f2_pack(s[2 * k], s[2 * k + 1]);
  const float A = scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<G / 2>(p));
  uint32_t byte;
  if constexpr (Cfg::kFmt == kMX) {
    byte = static_cast<uint32_t>(mx_scale_byte<Cfg::kRule>(A));
    const float mult = c * mx_inv_scale(static_cast<int>(byte));
    const f32x2 mm = f2_pack(mult, mult);
#pragma unroll
    for (int j = 0; j < G / 8; ++j) {
      float v[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) f2_unpack(f2_mul(p[4 * j + t], mm), v[2 * t], v[2 * t + 1]);
      words[j] = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
    }
  } else {
    const float s_b = div_rn_markstein(A, nv_den, nv_rden);
    byte = e4m3_encode(s_b);
    const uint32_t keep = byte == 0u ? 0u : 0xFFFFFFFFu;   // E4M3 byte 0 is the only zero scale
    // Element quotient y / S as the product s * RN(1 / (S sqrt(b))): within about one ulp of
    // the correctly rounded quotient, so an element's code can only move where its exact
    // quotient lies within a few 2^-24 (relative) of an E2M1 rounding midpoint.
    const float rq = nv_tab[byte];
    const f32x2 rq2 = f2_pack(rq, rq);
#pragma unroll
    for (int j = 0; j < G / 8; ++j) {
      float v[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) f2_unpack(f2_mul(p[4 * j + t], rq2), v[2 * t], v[2 * t + 1]);
      words[j] = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]) & keep;
    }
  }
  return byte;
}

// MBS-Static on G rotated sums s of one group, with r = RN(1 / (s_M sqrt(b))): y' = RN(s r),
// within about one ulp of the correctly rounded RN(y / s_M) that the butterfly kernel takes, so a
// decision can move only where its exact value lies within a few 2^-24 (relative) of a rounding
// or scale boundary, inside the flagged set (as for the NVFP4 element quotients).  Then the
// MXFP4 scale byte of y' under the plan's rule (its amax is RN(max |s| r): RN is monotone) and
// the codes of y' / 2^(byte - 127) = RN(s r 2^(127 - byte)) (the power of two is exact).
template <class Cfg, int G>
__device__ __forceinline__ uint32_t quantize_group_mbs(const float (&s)[G], float r, uint32_t (&words)[G / 8]) {
  f32x2 p[G / 2];
#pragma unroll
  for (int k = 0; k < G / 2; ++k) p[k] = f2_pack(s[2 * k], s[2 * k + 1]);
  const int byte = mx_scale_byte<Cfg::kRule>(pairs_amax<G / 2>(p) * r);
  const float m = r * mx_inv_scale(byte);
  const f32x2 mm = f2_pack(m, m);
#pragma unroll
  for (int j = 0; j < G / 8; ++j) {
    f32x2 v[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) v[t] = f2_mul(p[4 * j + t], mm);
    words[j] = e2m1x8_pairs(v);
  }
  return static_cast<uint32_t>(byte);
}

// r = RN(1 / (s_M sqrt(b))) for quantize_group_mbs: one fp64 division, rounded to fp32.
template <int B>
__device__ __forceinline__ float mbs_multiplier(float sM) {
  return static_cast<float>(inv_sqrt_block_f64(B) / static_cast<double>(sM));
}

// The macro-scale byte of MBS-Static for this lane's macro block, from the largest raw sum
// magnitude of the lane's piece (am) and, for b = 128, of the other half of its row
// (am_other); the lanes of one macro block (b <= 64) combine theirs by shuffles, so every
// lane of the warp must call it.
template <class Cfg>
__device__ __forceinline__ uint32_t mbs_lane_macro_byte(float am, float am_other) {
  if constexpr (Cfg::kMacroLanes >= 2) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
  if constexpr (Cfg::kMacroLanes >= 4) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
  if constexpr (Cfg::kBlock == 128) am = fmaxf(am, am_other);
  return mbs_macro_byte(scale_by_inv_sqrt<Cfg::kBlock>(am));
}

template <int N>
__device__ __forceinline__ float abs_max(const float* v) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < N; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

// Error-pass sums of one lane.  For NVFP4 they are kept in fp32 within a super-tile, in units
// that need no per-group scale: the signal as sum s^2 over the raw sums s (y = s / sqrt(b),
// so y^2 = s^2 / b, and 1/b is a power of two), the error as sum (v - q)^2 E4M3(byte)^2
// (X = E4M3(byte) s_g, so X^2 = E4M3(byte)^2 s_g^2); qe_sums_flush converts them to fp64 once
// per super-tile.  The error of a group with a zero block scale (every code 0: the error is
// the whole signal) goes to fp64 at once.  MXFP4, whose scales 2^(byte - 127) span more than
// fp32's range, adds both energies per group in fp64.
struct QeSums {
  f32x2 s2;
  float e_nv;
  double sig, err;
};

__device__ __forceinline__ void qe_sums_init(QeSums& q) {
  q.s2 = f2_pack(0.0f, 0.0f);
  q.e_nv = 0.0f;
  q.sig = q.err = 0.0;
}

template <int B>
__device__ __forceinline__ void qe_sums_flush(QeSums& q, float s_g) {
  constexpr double inv_b = 1.0 / B;
  float a0, a1;
  f2_unpack(q.s2, a0, a1);
  q.sig = fma(static_cast<double>(a0 + a1), inv_b, q.sig);
  const double sg = s_g;
  q.err = fma(static_cast<double>(q.e_nv), sg * sg, q.err);
  q.s2 = f2_pack(0.0f, 0.0f);
  q.e_nv = 0.0f;
}

// One group of G rotated sums s: the same scale byte and quotients as quantize_group (so the
// same codes), then its signal and error into the lane's sums.
template <class Cfg, int G>
__device__ __forceinline__ void group_energy_mma(const float (&s)[G], const float* nv_tab, float nv_den,
                                                 float nv_rden, QeSums& q) {
  constexpr float c = Cfg::kC;
  f32x2 p[G / 2];
#pragma unroll
  for (int k = 0; k < G / 2; ++k) p[k] = f2_pack(s[2 * k], s[2 * k + 1]);
  const float A = scale_by_inv_sqrt<Cfg::kBlock>(pairs_amax<G / 2>(p));
  float mult;
  if constexpr (Cfg::kFmt == kMX) {
    // both energies per group in fp64 (measured: the fp32 signal sum costs MXFP4 b = 128 more
    // registers than it saves)
    const int byte = mx_scale_byte<Cfg::kRule>(A);
    mult = c * mx_inv_scale(byte);
    const f32x2 mm = f2_pack(mult, mult);
    f32x2 v[G / 2];
#pragma unroll
    for (int k = 0; k < G / 2; ++k) v[k] = f2_mul(p[k], mm);
    float gs, ge;
    group_energies<G / 2>(v, gs, ge);
    const double X2 = mx_scale_sq(byte);
    q.sig = fma(static_cast<double>(gs), X2, q.sig);
    q.err = fma(static_cast<double>(ge), X2, q.err);
  } else {
#pragma unroll
    for (int k = 0; k < G / 2; ++k) q.s2 = f2_fma(p[k], p[k], q.s2);
    const uint32_t byte = e4m3_encode(div_rn_markstein(A, nv_den, nv_rden));
    mult = nv_tab[byte];
    if (byte == 0u || mult == 0.0f) {
      f32x2 g2 = f2_pack(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < G / 2; ++k) g2 = f2_fma(p[k], p[k], g2);
      float a0, a1;
      f2_unpack(g2, a0, a1);
      q.err = fma(static_cast<double>(a0 + a1), 1.0 / Cfg::kBlock, q.err);
      return;
    }
    const f32x2 mm = f2_pack(mult, mult);
    f32x2 v[G / 2];
#pragma unroll
    for (int k = 0; k < G / 2; ++k) v[k] = f2_mul(p[k], mm);
    float gs, ge;
    group_energies<G / 2>(v, gs, ge);
    const float dec = e4m3_decode(byte);
    q.e_nv = fmaf(ge, dec * dec, q.e_nv);
  }
}

// One lane's piece of a block: BW codes (BW / 8 code words) from element `off` of block `row`,
// and their BW / g scale bytes.
template <class Cfg, int BW>
__device__ __forceinline__ void store_piece(const MmaArgs& a, int64_t row, int off, const uint32_t (&words)[BW / 8],
                                            const uint32_t (&sbytes)[BW / Cfg::kGroup]) {
  constexpr int B = Cfg::kBlock, G = Cfg::kGroup, NG = BW / G;
  uint8_t* cp = a.codes + row * (B / 2) + off / 2;
  if constexpr (BW == 16) {
    stg64(cp, words[0], words[1]);
  } else {
#pragma unroll
    for (int k = 0; k < BW / 32; ++k)
      stg128(cp + 16 * k, words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]);
  }
  uint8_t* sp = a.scales + row * (B / G) + off / G;
  if constexpr (NG == 1) {
    *sp = static_cast<uint8_t>(sbytes[0]);
  } else if constexpr (NG == 2) {
    *reinterpret_cast<uint16_t*>(sp) = static_cast<uint16_t>(sbytes[0] | (sbytes[1] << 8));
  } else {
    static_assert(NG == 4, "a slice piece holds 1, 2 or 4 groups");
    *reinterpret_cast<uint32_t*>(sp) = sbytes[0] | (sbytes[1] << 8) | (sbytes[2] << 16) | (sbytes[3] << 24);
  }
}

// group_energy_mma for MBS-Static: the quotients and codes of quantize_group_mbs, energies in
// units of X^2 = 2^(2 (byte - 127)) s_M^2 (sM2).
template <class Cfg, int G>
__device__ __forceinline__ void group_energy_mma_mbs(const float (&s)[G], float r, double sM2, double& sig,
                                                     double& err) {
  f32x2 p[G / 2];
#pragma unroll
  for (int k = 0; k < G / 2; ++k) p[k] = f2_pack(s[2 * k], s[2 * k + 1]);
  const int byte = mx_scale_byte<Cfg::kRule>(pairs_amax<G / 2>(p) * r);
  const float m = r * mx_inv_scale(byte);
  const f32x2 mm = f2_pack(m, m);
  f32x2 v[G / 2];
#pragma unroll
  for (int k = 0; k < G / 2; ++k) v[k] = f2_mul(p[k], mm);
  float gs, ge;
  group_energies<G / 2>(v, gs, ge);
  const double X2 = mx_scale_sq(byte) * sM2;
  sig = fma(static_cast<double>(gs), X2, sig);
  err = fma(static_cast<double>(ge), X2, err);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, Cfg::kCtasPerSm)
    rotate_quantize_mma_kernel(const __grid_constant__ CUtensorMap xmap, MmaArgs a) {
  constexpr int B = Cfg::kBlock, G = Cfg::kGroup, S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  __shared__ float s_tensor_scale;
  __shared__ double s_qe[Cfg::kQE ? Cfg::kEpiWarps : 1][2];   // error pass: energies per epilogue warp
  __shared__ bool s_qe_last;
  __shared__ float s_amax[Cfg::kAmax ? Cfg::kEpiWarps : 1];   // amax pass: maximum per epilogue warp
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t stage0 = smem_addr(smem);
  const uint32_t hbase = stage0 + S * Cfg::kStageBytes;
  const uint32_t bars = stage0 + Cfg::kBarOffset;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
  auto tfull_bar = [&](int d) { return bars + 8u * (2 * S + d); };
  auto tempty_bar = [&](int d) { return bars + 8u * (2 * S + 2 + d); };
  auto signed_bar = [&](int s) { return bars + 8u * (2 * S + 4 + s); };

  // H_b, K-major, swizzled like the activation tiles: row n holds H[n][0..b) (H is symmetric)
  uint8_t* hs = smem + S * Cfg::kStageBytes;
  for (int i = tid; i < B * B; i += Cfg::kThreads) {
    const int n = i / B, k = i % B;
    const int h = k / Cfg::kKB, kk = k % Cfg::kKB;
    const uint32_t off = h * (B * Cfg::kRB) + swizzle_off<Cfg::kSwzBits>(n * Cfg::kRB + kk * 2);
    *reinterpret_cast<uint16_t*>(hs + off) = (__popc(n & k) & 1) ? 0xBF80u : 0x3F80u;   // bf16 -1 / +1
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(tfull_bar(d), 1);
      mbar_init(tempty_bar(d), Cfg::kEpiWarps);
    }
    for (int s = 0; s < S; ++s) mbar_init(signed_bar(s), Cfg::kSignWarps);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem_base)),
                 "r"(Cfg::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem_base;
  const int64_t n_super = a.n_super;
  float* nv_tab = reinterpret_cast<float*>(smem + S * Cfg::kStageBytes + Cfg::kHBytes);

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      // Before the grid dependency: ask L2 for this CTA's first S super-tiles, so their DRAM
      // traffic overlaps the end of the kernel this one follows.  Only a hint: the copies below
      // still wait on the dependency, and L2 holds any write that kernel makes meanwhile.
      {
        int64_t i = 0;
        for (int64_t t = blockIdx.x; t < n_super && i < S; t += gridDim.x, ++i) {
          const int64_t row0 = t * Cfg::kRowsPerTile;
          if constexpr (Cfg::kBulk) {
            const int64_t rows = (a.n_rows - row0) < Cfg::kRowsPerTile ? (a.n_rows - row0) : Cfg::kRowsPerTile;
            bulk_prefetch_l2(a.x + row0 * B, static_cast<uint32_t>(rows) * (2 * B));
          } else if constexpr (B >= 128) {
            tma_prefetch_2d(&xmap, 0, static_cast<int>(row0));
            tma_prefetch_2d(&xmap, 64, static_cast<int>(row0));
          } else {
#pragma unroll
            for (int k = 0; k < Cfg::kBoxes; ++k)
              if (row0 + k * Cfg::kBoxRows < a.n_rows) tma_prefetch_2d(&xmap, 0, static_cast<int>(row0 + k * Cfg::kBoxRows));
          }
        }
      }
      pdl_wait();   // x may come from the kernel this one depends on
      int64_t i = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < n_super; t += gridDim.x, ++i) {
        const int s = static_cast<int>(i % S);
        const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
        if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u)) {
          ok = false;
          break;
        }
        const int64_t row0 = t * Cfg::kRowsPerTile;
        const uint32_t dst = stage0 + s * Cfg::kStageBytes;
        if constexpr (Cfg::kBulk) {
          const int64_t rows = (a.n_rows - row0) < Cfg::kRowsPerTile ? (a.n_rows - row0) : Cfg::kRowsPerTile;
          const uint32_t bytes = static_cast<uint32_t>(rows) * (2 * B);
          mbar_arrive_expect_tx(full_bar(s), bytes);
          bulk_g2s(dst, a.x + row0 * B, bytes, full_bar(s));
        } else if constexpr (B >= 128) {
          mbar_arrive_expect_tx(full_bar(s), 2u * Cfg::kBoxBytes);
          tma_load_2d(dst, &xmap, 0, static_cast<int>(row0), full_bar(s));
          tma_load_2d(dst + Cfg::kBoxBytes, &xmap, 64, static_cast<int>(row0), full_bar(s));
        } else {
          int nb = 0;
#pragma unroll
          for (int k = 0; k < Cfg::kBoxes; ++k) nb += (row0 + k * Cfg::kBoxRows < a.n_rows) ? 1 : 0;
          mbar_arrive_expect_tx(full_bar(s), static_cast<uint32_t>(nb) * Cfg::kBoxBytes);
#pragma unroll
          for (int k = 0; k < Cfg::kBoxes; ++k)
            if (row0 + k * Cfg::kBoxRows < a.n_rows)
              tma_load_2d(dst + k * Cfg::kBoxBytes, &xmap, 0, static_cast<int>(row0 + k * Cfg::kBoxRows), full_bar(s));
        }
      }
      // let every issued copy land before the CTA can leave
      const int64_t issued = i;
      for (int64_t j = (issued > S ? issued - S : 0); j < issued; ++j)
        mbar_wait_bounded(full_bar(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1));
      (void)ok;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int64_t i = 0;
      for (int64_t t = blockIdx.x; t < n_super; t += gridDim.x, ++i) {
        const int s = static_cast<int>(i % S);
        const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
        const int d = static_cast<int>(i & 1);
        const uint32_t dph = static_cast<uint32_t>((i >> 1) & 1);
        // with signs, the sign warps' "signed" barrier follows the stage's "full" one
        if (!mbar_wait_bounded(a.sign_bytes ? signed_bar(s) : full_bar(s), ph)) break;
        if (!mbar_wait_bounded(tempty_bar(d), dph ^ 1u)) break;
        tc_fence_after();
        const uint32_t a0 = stage0 + s * Cfg::kStageBytes;
        const uint32_t dcol = tmem_base + d * Cfg::kSuperCols;
#pragma unroll
        for (int j = 0; j < Cfg::kRowTiles; ++j) {
#pragma unroll
          for (int k = 0; k < B / 16; ++k) {
            const int h = (16 * k) / Cfg::kKB, kk = (16 * k) % Cfg::kKB;
            const uint32_t aa = a0 + j * (128 * Cfg::kRB) + h * (128 * Cfg::kRB) + kk * 2;
            const uint32_t ha = hbase + h * (B * Cfg::kRB) + kk * 2;
            umma_bf16(dcol + j * B, umma_smem_desc(aa, 8 * Cfg::kRB, Cfg::kLayout),
                      umma_smem_desc(ha, 8 * Cfg::kRB, Cfg::kLayout), Cfg::kIdesc, k > 0 ? 1u : 0u);
          }
        }
        umma_commit(empty_bar(s));
        umma_commit(tfull_bar(d));
      }
      // the last commits must have landed before TMEM is freed
      if (i > 0) {
        const int64_t j = i - 1;
        mbar_wait_bounded(tfull_bar(static_cast<int>(j & 1)), static_cast<uint32_t>((j >> 1) & 1));
      }
    }
  } else if (warp >= 2 + Cfg::kEpiWarps) {
    // ---------------- sign warps: x_k -> s_k x_k in the landed stage (plans with channel signs)
    // The warps walk the stage's 16-byte chunks in physical order (lane-consecutive addresses:
    // no bank conflicts), kBatch chunks a lane at a time.  A stage region (the whole stage in
    // the bulk layout, one K-half of swizzled 128-byte rows otherwise) holds kCpr chunks per
    // row; a lane's chunks sit kRowStep rows apart and, as kRowStep is a multiple of the
    // 8-row swizzle period, all carry the same logical chunk q of their rows.
    if (a.sign_bytes != nullptr) {
      constexpr int kCpr = Cfg::kSignCpr;                          // chunks per row of a region
      constexpr int kRegions = Cfg::kSignRegions;
      constexpr int kRegionBytes = Cfg::kStageBytes / kRegions;
      constexpr int kLaneStride = Cfg::kSignLaneStride;            // chunks between a lane's chunks
      constexpr int kRowStep = Cfg::kSignRowStep;
      constexpr int kPerLane = Cfg::kSignPerLane;                  // chunks per lane per region
      constexpr int kBatch = Cfg::kCtasPerSm == 1 ? 4 : 8;
      static_assert(kLaneStride % kCpr == 0 && (Cfg::kBulk || kRowStep % 8 == 0), "lane chunk walk");
      static_assert(kPerLane % kBatch == 0, "whole batches per region");
      const int sw = warp - (2 + Cfg::kEpiWarps);
      const int c0 = 32 * sw + lane;                               // lane's first chunk of a region
      const uint32_t row0 = static_cast<uint32_t>(c0 / kCpr);
      const uint32_t pq = static_cast<uint32_t>(c0 % kCpr);
      const uint32_t upr = static_cast<uint32_t>(a.sign_upr);
      const uint32_t row_step = static_cast<uint32_t>(kRowStep) % upr;
      pdl_wait();   // the mask belongs to the caller and may come from an earlier kernel
      // Hadamard block (within its matrix row) of the lane's first row, kept incrementally:
      // super-tile t starts at block (t * kRowsPerTile) mod upr, and t advances by gridDim.x
      const uint32_t tile_step = static_cast<uint32_t>((static_cast<uint64_t>(gridDim.x) * Cfg::kRowsPerTile) % upr);
      const uint32_t row0_kb = row0 % upr;
      uint32_t tile_kb = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x) * Cfg::kRowsPerTile) % upr);
      const uint32_t tab_s = stage0 + Cfg::kMaskOffset;
      // the mask words behind this lane's table entries: word 32 sw + lane + k * kLaneStride
      // (ceil(chunks / 4) words in all), loaded together
      auto load_mask_words = [&](auto& mw, uint32_t chunks) {
        const uint32_t* mg = reinterpret_cast<const uint32_t*>(a.sign_bytes);
        const uint32_t nw = (chunks + 3) / 4;
        constexpr int N = sizeof(mw) / sizeof(mw[0]);
#pragma unroll
        for (int k = 0; k < N; ++k) {
          const uint32_t w = 32u * sw + lane + static_cast<uint32_t>(k * kLaneStride);
          mw[k] = w < nw ? __ldg(mg + w) : 0u;
        }
      };
      if constexpr (Cfg::kSignTable) {
        if (a.sign_table == 1) {
          // the expanded table: entry e (and e + K/8) = the XOR words of mask byte e; every
          // mask word a lane needs is loaded before any is used (one memory latency, not one
          // per word)
          const uint32_t chunks = upr * (B / 8);
          constexpr int kWordsPerLane = (Cfg::kSignTableMax / 32 / 4 + kLaneStride - 1) / kLaneStride;
          uint32_t mw[kWordsPerLane];
          load_mask_words(mw, chunks);
#pragma unroll
          for (int k = 0; k < kWordsPerLane; ++k) {
            const uint32_t e0 = 4u * (32u * sw + lane + static_cast<uint32_t>(k * kLaneStride));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t e = e0 + j;
              if (e < chunks) {
                const uint4 f = chunk_sign_xor((mw[k] >> (8 * j)) & 0xFFu);
                sts128_u4(tab_s + 16u * e, f);
                sts128_u4(tab_s + 16u * (e + chunks), f);
              }
            }
          }
          asm volatile("bar.sync 2, %0;" ::"r"(32 * Cfg::kSignWarps) : "memory");
          static_assert(kRegions == 1 && kPerLane % kBatch == 0, "one region, whole batches");
          // byte offsets, in the table, of the lane's chunks relative to its first: chunk u sits
          // (u * kRowStep) mod upr blocks further on (the same for every lane and stage)
          uint32_t dk[kPerLane];
#pragma unroll
          for (int u = 0; u < kPerLane; ++u)
            dk[u] = static_cast<uint32_t>((static_cast<uint64_t>(u) * row_step) % upr) * (2u * B);
          int64_t i = 0;
          for (int64_t t = blockIdx.x; t < n_super; t += gridDim.x, ++i) {
            const int s = static_cast<int>(i % S);
            const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
            uint32_t kb_first = tile_kb + row0_kb;
            if (kb_first >= upr) kb_first -= upr;
            tile_kb += tile_step;
            if (tile_kb >= upr) tile_kb -= upr;
            // logical chunk of the lane's rows: the bulk layout is unswizzled; a swizzled row's
            // physical chunk is its logical one XOR (row & 7)
            const uint32_t q = Cfg::kBulk ? pq : (pq ^ (row0 & 7u));
            const uint32_t tb = tab_s + kb_first * (2u * B) + 16u * q;
            const uint32_t addr = stage0 + s * Cfg::kStageBytes + 16u * c0;
            const bool mine = mbar_wait_bounded(full_bar(s), ph);
            if (!__all_sync(0xFFFFFFFFu, mine)) break;
#pragma unroll
            for (int j = 0; j < kPerLane; j += kBatch) {
              uint4 w[kBatch], f[kBatch];
#pragma unroll
              for (int u = 0; u < kBatch; ++u) {
                f[u] = lds128(tb + dk[j + u]);
                w[u] = lds128(addr + 16u * kLaneStride * (j + u));
              }
#pragma unroll
              for (int u = 0; u < kBatch; ++u)
                sts128_u4(addr + 16u * kLaneStride * (j + u),
                          make_uint4(w[u].x ^ f[u].x, w[u].y ^ f[u].y, w[u].z ^ f[u].z, w[u].w ^ f[u].w));
            }
            fence_proxy_async_smem();   // the tensor core reads the stage through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(signed_bar(s));
          }
        }
      }
      if constexpr (!Cfg::kSignTable) {
        if (a.sign_table == 2) {
          // the word table: word e = the sign word of mask byte e mod (K/8); the mask words
          // are all loaded first, as for the expanded table
          const uint32_t chunks = upr * (B / 8);
          const uint32_t words = (upr + static_cast<uint32_t>(Cfg::kSignExt)) * (B / 8);
          constexpr int kWordsPerLane = (Cfg::kMaskSmemMax / 4 / 4 + kLaneStride - 1) / kLaneStride;
          uint32_t mw[kWordsPerLane];
          load_mask_words(mw, chunks);
#pragma unroll
          for (int k = 0; k < kWordsPerLane; ++k) {
            const uint32_t e0 = 4u * (32u * sw + lane + static_cast<uint32_t>(k * kLaneStride));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t w = chunk_sign_word((mw[k] >> (8 * j)) & 0xFFu);
              if (e0 + j < chunks)
                for (uint32_t e = e0 + j; e < words; e += chunks) sts32(tab_s + 4u * e, w);
            }
          }
          asm volatile("bar.sync 2, %0;" ::"r"(32 * Cfg::kSignWarps) : "memory");
          constexpr uint32_t kWordStep = 4u * kRowStep * (B / 8);    // table bytes between a lane's chunks
          int64_t i = 0;
          for (int64_t t = blockIdx.x; t < n_super; t += gridDim.x, ++i) {
            const int s = static_cast<int>(i % S);
            const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
            uint32_t kb_first = tile_kb + row0_kb;
            if (kb_first >= upr) kb_first -= upr;
            tile_kb += tile_step;
            if (tile_kb >= upr) tile_kb -= upr;
            const bool mine = mbar_wait_bounded(full_bar(s), ph);
            if (!__all_sync(0xFFFFFFFFu, mine)) break;
#pragma unroll 1
            for (int h = 0; h < kRegions; ++h) {
              // logical chunk of the lane's rows: the bulk layout is unswizzled; a swizzled row's
              // physical chunk is its logical one XOR (row & 7)
              const uint32_t q = Cfg::kBulk ? pq : 8u * h + (pq ^ (row0 & 7u));
              uint32_t tb = tab_s + 4u * (kb_first * (B / 8) + q);
              uint32_t addr = stage0 + s * Cfg::kStageBytes + h * kRegionBytes + 16u * c0;
#pragma unroll 1
              for (int j = 0; j < kPerLane; j += kBatch) {
                uint4 w[kBatch];
                uint32_t m[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                  m[u] = lds32(tb + kWordStep * u);
                  w[u] = lds128(addr + 16u * kLaneStride * u);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                  const uint4 f = chunk_sign_xor_word(m[u]);
                  sts128_u4(addr + 16u * kLaneStride * u,
                            make_uint4(w[u].x ^ f.x, w[u].y ^ f.y, w[u].z ^ f.z, w[u].w ^ f.w));
                }
                tb += kWordStep * kBatch;
                addr += 16u * kLaneStride * kBatch;
              }
            }
            fence_proxy_async_smem();   // the tensor core reads the stage through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(signed_bar(s));
          }
        }
      }
      const uint8_t* mask_g = a.sign_bytes;
      const bool staged = a.sign_smem > 0;
      const uint32_t mask_s = tab_s;
      if (staged && !a.sign_table) {
        // the mask's words, once per CTA, into shared memory (a few hundred bytes to 16 KB)
        uint32_t* ms = reinterpret_cast<uint32_t*>(smem + Cfg::kMaskOffset);
        const uint32_t* mg = reinterpret_cast<const uint32_t*>(a.sign_bytes);
        const int words = static_cast<int>((static_cast<int64_t>(upr) * B + 31) / 32);   // the caller's ceil(K / 32)
        for (int w = 32 * sw + lane; w < words; w += 32 * Cfg::kSignWarps) ms[w] = __ldg(mg + w);
        asm volatile("bar.sync 2, %0;" ::"r"(32 * Cfg::kSignWarps) : "memory");
      }
      int64_t i = 0;
      for (int64_t t = blockIdx.x; a.sign_table == 0 && t < n_super; t += gridDim.x, ++i) {
        const int s = static_cast<int>(i % S);
        const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
        uint32_t kb_first = tile_kb + row0_kb;
        if (kb_first >= upr) kb_first -= upr;
        tile_kb += tile_step;
        if (tile_kb >= upr) tile_kb -= upr;
        const bool mine = mbar_wait_bounded(full_bar(s), ph);
        if (!__all_sync(0xFFFFFFFFu, mine)) break;
#pragma unroll 1
        for (int h = 0; h < kRegions; ++h) {
          // logical chunk of the lane's rows: the bulk layout is unswizzled; a swizzled row's
          // physical chunk is its logical one XOR (row & 7)
          const uint32_t q = Cfg::kBulk ? pq : 8u * h + (pq ^ (row0 & 7u));
          uint32_t kb = kb_first;
          uint32_t addr = stage0 + s * Cfg::kStageBytes + h * kRegionBytes + 16u * c0;
#pragma unroll 1
          for (int j = 0; j < kPerLane; j += kBatch) {
            uint4 w[kBatch];
            uint32_t m[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const uint32_t mi = kb * (B / 8) + q;   // the chunk's mask byte
              m[u] = staged ? lds_u8(mask_s + mi) : static_cast<uint32_t>(__ldg(mask_g + mi));
              kb += row_step;
              if (kb >= upr) kb -= upr;
              w[u] = lds128(addr + 16u * kLaneStride * u);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const uint4 f = chunk_sign_xor(m[u]);
              sts128_u4(addr + 16u * kLaneStride * u,
                        make_uint4(w[u].x ^ f.x, w[u].y ^ f.y, w[u].z ^ f.z, w[u].w ^ f.w));
            }
            addr += 16u * kLaneStride * kBatch;
          }
        }
        fence_proxy_async_smem();   // the tensor core reads the stage through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(signed_bar(s));
      }
    }
  } else {
    // ---------------- epilogue: warps 2.., TMEM lane quarter warp % 4, column slice (warp - 2) / 4
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;                  // slice index, 0 .. kSlices - 1
    const int lane_row = 32 * quarter + lane;
    pdl_wait();   // the tensor scale (or the partial maxima) and the outputs belong to earlier kernels
    float s_g = 1.0f;
    if constexpr (Cfg::kFmt == kNV && !Cfg::kAmax) {
      constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
      if (warp == 2) {
        if constexpr (Cfg::kRule == kRuleNvDynamic) {
          float m = 0.0f;
          for (int i2 = lane; i2 < a.n_partials; i2 += 32) m = fmaxf(m, a.partials[i2]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
          if (lane == 0) {
            const float sg = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
            s_tensor_scale = sg;
            if (blockIdx.x == 0) *a.tensor_scale = sg;
          }
        } else {
          if (lane == 0) s_tensor_scale = *a.tensor_scale;
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
      s_g = s_tensor_scale;
      // for every E4M3 byte: the multiplier that takes a raw MMA sum s to the element quotient,
      // RN(1 / (S sqrt(b))) with S = fp32(E4M3(byte) s_g), from one fp64 division
      for (int byte = tid - 64; byte < 256; byte += kEpiThreads) {
        const float Sv = e4m3_decode(static_cast<uint32_t>(byte & 0x7F)) * s_g;
        nv_tab[byte] = Sv == 0.0f ? 0.0f : static_cast<float>(inv_sqrt_block_f64(B) / static_cast<double>(Sv));
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
    }
    // bulk-copied stages: chunk c of this lane's rows comes out sign-flipped when
    // popcount(c & t) is odd; flip_basis[k] is the code-word mask for bit k of t
    const int flip_t = Cfg::kBulk ? ((lane_row >> Cfg::kFlipShift) & Cfg::kFlipMask) : 0;
    const uint32_t flip_basis0 = (flip_t & 1) ? 0x88888888u : 0u;
    const uint32_t flip_basis1 = (flip_t & 2) ? 0x88888888u : 0u;
    const float nv_den = 6.0f * s_g;
    const float nv_rden = __frcp_rn(nv_den);
    constexpr int EC = Cfg::kEpiCols;                 // 16, 32 or 64 columns
    constexpr int NGW = EC / G;                        // groups per warp slice
    double qe_sig = 0.0, qe_err = 0.0;                 // error pass (MBS): this lane's running energies
    QeSums qe;                                         // error pass (MXFP4, NVFP4): this lane's sums
    qe_sums_init(qe);
    float amax_m = 0.0f;                               // amax pass: this lane's largest |sum|
    int64_t i = 0;
    for (int64_t t = blockIdx.x; t < n_super; t += gridDim.x, ++i) {
      const int d = static_cast<int>(i & 1);
      const uint32_t dph = static_cast<uint32_t>((i >> 1) & 1);
      const bool mine = mbar_wait_bounded(tfull_bar(d), dph);
      if (!__all_sync(0xFFFFFFFFu, mine)) break;
      tc_fence_after();
      const int col0 = half * EC;                      // first column of this warp's slice
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * quarter) << 16) + d * Cfg::kSuperCols + col0;
      if constexpr (Cfg::kFmt == kMBS) {
        // MBS-Static.  Pass 1 keeps only the largest magnitude of each piece (and, for b = 128,
        // of the row's other column half); once the macro byte is known, each group is read
        // again from tensor memory and quantized (or measured).  Few values are live at a time,
        // and the accumulator buffer is released after the second pass.
        constexpr int BWm = B < EC ? B : EC;
        constexpr int PCm = EC / BWm;
        // 32 columns (two loads) per wait
        float am[PCm];
#pragma unroll
        for (int pc = 0; pc < PCm; ++pc) {
          am[pc] = 0.0f;
#pragma unroll
          for (int c32 = 0; c32 < BWm / 32; ++c32) {
            float w0[16], w1[16];
            tmem_ld16(tq + pc * BWm + 32 * c32, w0);
            tmem_ld16(tq + pc * BWm + 32 * c32 + 16, w1);
            tmem_wait_ld();
            am[pc] = fmaxf(am[pc], fmaxf(abs_max<16>(w0), abs_max<16>(w1)));
          }
        }
        float am_other = 0.0f;
        if constexpr (B == 128) {
          const uint32_t tp = tq - col0 + (EC - col0);
#pragma unroll
          for (int c32 = 0; c32 < EC / 32; ++c32) {
            float w0[16], w1[16];
            tmem_ld16(tp + 32 * c32, w0);
            tmem_ld16(tp + 32 * c32 + 16, w1);
            tmem_wait_ld();
            am_other = fmaxf(am_other, fmaxf(abs_max<16>(w0), abs_max<16>(w1)));
          }
        }
#pragma unroll
        for (int pc = 0; pc < PCm; ++pc) {
          const int col = col0 + pc * BWm;
          const int j = col / B, off = col % B;
          const int64_t row = t * Cfg::kRowsPerTile + j * 128 + lane_row;
          const uint32_t m8 = mbs_lane_macro_byte<Cfg>(am[pc], am_other);
          const float sM = mbs_macro_scale(m8);
          const float mr = mbs_multiplier<B>(sM);
          if constexpr (!Cfg::kQE) {
            // the macro byte from the macro block's first lane (b = 128: the first half's warp)
            const bool first = Cfg::kMacroLanes > 1 ? (lane % Cfg::kMacroLanes) == 0 : half == 0;
            if (first && row < a.n_rows) a.macro[row * B / 128] = static_cast<uint8_t>(m8);
          }
#pragma unroll
          for (int q = 0; q < BWm / G; ++q) {
            float gv[G];
            {
              static_assert(G == 32, "an MBS group is two 16-column loads");
              float w0[16], w1[16];
              tmem_ld16(tq + pc * BWm + q * G, w0);
              tmem_ld16(tq + pc * BWm + q * G + 16, w1);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                gv[e] = w0[e];
                gv[16 + e] = w1[e];
              }
            }
            if constexpr (Cfg::kQE) {
              if (row < a.n_rows)
                group_energy_mma_mbs<Cfg, G>(gv, mr, static_cast<double>(sM) * static_cast<double>(sM), qe_sig,
                                             qe_err);
            } else {
              // each group's codes and scale go out as soon as they are made
              uint32_t gw[G / 8];
              uint32_t sb[1];
              sb[0] = quantize_group_mbs<Cfg, G>(gv, mr, gw);
#pragma unroll
              for (int e = 0; e < G / 8; ++e) {
                const int chunk = (off + q * G) / 8 + e;
                if constexpr (Cfg::kBulk) {
                  if (chunk & 1) gw[e] ^= flip_basis0;
                  if (chunk & 2) gw[e] ^= flip_basis1;
                }
              }
              if (row < a.n_rows) store_piece<Cfg, G>(a, row, off + q * G, gw, sb);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(d));
        continue;
      }
      float v[EC];
#pragma unroll
      for (int c16 = 0; c16 < EC / 16; ++c16) {
        float w16[16];
        tmem_ld16(tq + 16 * c16, w16);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[16 * c16 + e] = w16[e];
      }
      tmem_wait_ld();
      // the accumulator buffer can be reused as soon as every epilogue warp has its slice
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(d));
      // The slice holds whole blocks (b < EC), exactly one block (b == EC) or half of one.
      constexpr int BW = B < EC ? B : EC;              // block elements in one slice piece
      constexpr int PIECES = EC / BW;                  // block pieces in the slice
      if constexpr (Cfg::kAmax) {
        // magnitudes only: a column's sign flip from the bulk layout does not change them
#pragma unroll
        for (int pc = 0; pc < PIECES; ++pc) {
          const int j = (col0 + pc * BW) / B;
          const int64_t row = t * Cfg::kRowsPerTile + j * 128 + lane_row;
          if (row < a.n_rows) {
#pragma unroll
            for (int e = 0; e < BW; ++e) amax_m = fmaxf(amax_m, fabsf(v[pc * BW + e]));
          }
        }
        continue;
      }
      if constexpr (Cfg::kQE) {
        // energies only; a column's sign flip from the bulk layout changes neither v^2 nor
        // (v - q)^2 (E2M1 rounds the magnitude)
#pragma unroll
        for (int pc = 0; pc < PIECES; ++pc) {
          const int j = (col0 + pc * BW) / B;
          const int64_t row = t * Cfg::kRowsPerTile + j * 128 + lane_row;
          if (row < a.n_rows) {
#pragma unroll
            for (int q = 0; q < BW / G; ++q) {
              float gv[G];
#pragma unroll
              for (int e = 0; e < G; ++e) gv[e] = v[pc * BW + q * G + e];
              group_energy_mma<Cfg, G>(gv, nv_tab, nv_den, nv_rden, qe);
            }
          }
        }
        qe_sums_flush<B>(qe, s_g);
        continue;
      }
#pragma unroll
      for (int pc = 0; pc < PIECES; ++pc) {
        const int col = col0 + pc * BW;                // column within the super-tile
        const int j = col / B;                         // row-tile = block of this lane
        const int off = col % B;                       // element offset inside the block
        const int64_t row = t * Cfg::kRowsPerTile + j * 128 + lane_row;
        uint32_t words[BW / 8];
        uint32_t sbytes[BW / G];
#pragma unroll
        for (int q = 0; q < BW / G; ++q) {
          float gv[G];
#pragma unroll
          for (int e = 0; e < G; ++e) gv[e] = v[pc * BW + q * G + e];
          uint32_t gw[G / 8];
          sbytes[q] = quantize_group<Cfg, G>(gv, gw, nv_tab, nv_den, nv_rden);
#pragma unroll
          for (int e = 0; e < G / 8; ++e) {
            const int chunk = (off + q * G) / 8 + e;   // 8-column chunk inside the block
            uint32_t w = gw[e];
            if constexpr (Cfg::kBulk) {
              if (chunk & 1) w ^= flip_basis0;
              if (chunk & 2) w ^= flip_basis1;
              // a zero NV block scale gives code 0x0 for every element: the flip above must not
              // turn them into 0x8
              if constexpr (Cfg::kFmt == kNV) w = sbytes[q] == 0u ? 0u : w;
            }
            words[q * (G / 8) + e] = w;
          }
          if constexpr (Cfg::kDump) {
            if (row < a.n_rows) {
              float* yp = a.y_dump + row * B + off + q * G;
#pragma unroll
              for (int e = 0; e < G; e += 4) {
                const int chunk = (off + q * G + e) / 8;
                const float sg = (Cfg::kBulk && (__popc(chunk & flip_t) & 1)) ? -1.0f : 1.0f;
                *reinterpret_cast<float4*>(yp + e) =
                    make_float4(sg * scale_by_inv_sqrt<B>(gv[e]), sg * scale_by_inv_sqrt<B>(gv[e + 1]),
                                sg * scale_by_inv_sqrt<B>(gv[e + 2]), sg * scale_by_inv_sqrt<B>(gv[e + 3]));
              }
            }
          }
        }
        if (row < a.n_rows) store_piece<Cfg, BW>(a, row, off, words, sbytes);
      }
      (void)NGW;
    }
    if constexpr (Cfg::kAmax) {
      constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax_m = fmaxf(amax_m, __shfl_xor_sync(0xFFFFFFFFu, amax_m, o));
      if (lane == 0) s_amax[warp - 2] = amax_m;
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
      if (warp == 2 && lane == 0) {
        float r = 0.0f;
#pragma unroll
        for (int w = 0; w < Cfg::kEpiWarps; ++w) r = fmaxf(r, s_amax[w]);
        // RN(r / sqrt(b)), monotone: the largest of the elements' own RN(sum / sqrt(b))
        a.amax_out[blockIdx.x] = scale_by_inv_sqrt<B>(r);
      }
      if (blockIdx.x == 0)
        for (int i = static_cast<int>(gridDim.x) + (tid - 64); i < a.amax_slots; i += kEpiThreads) a.amax_out[i] = 0.0f;
    }
    if constexpr (Cfg::kQE) {
      // the CTA's energies (epilogue warps in order), then the last CTA to finish sums the
      // per-CTA pairs in CTA order: a fixed order for a fixed grid, so the result is deterministic
      constexpr int kEpiThreads = 32 * Cfg::kEpiWarps;
      qe_sig += qe.sig;
      qe_err += qe.err;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        qe_sig += __shfl_xor_sync(0xFFFFFFFFu, qe_sig, o);
        qe_err += __shfl_xor_sync(0xFFFFFFFFu, qe_err, o);
      }
      if (lane == 0) {
        s_qe[warp - 2][0] = qe_sig;
        s_qe[warp - 2][1] = qe_err;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
      if (warp == 2 && lane == 0) {
        double ts = 0.0, te = 0.0;
#pragma unroll
        for (int w = 0; w < Cfg::kEpiWarps; ++w) {
          ts += s_qe[w][0];
          te += s_qe[w][1];
        }
        a.qe_partials[2 * blockIdx.x] = ts;
        a.qe_partials[2 * blockIdx.x + 1] = te;
        __threadfence();
        s_qe_last = atomicAdd(a.qe_ticket, 1u) == gridDim.x - 1;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
      if (s_qe_last && warp == 2) {
        __threadfence();
        qe_final_sum(a.qe_partials, static_cast<int>(gridDim.x), a.qe_out);
        if (lane == 0) *a.qe_ticket = 0u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Cfg::kTmemCols)
                 : "memory");
  }
}

}  // namespace fp4q
