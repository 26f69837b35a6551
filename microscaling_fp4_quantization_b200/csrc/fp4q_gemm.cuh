// Block-scaled FP4 GEMM on the 5th-generation tensor cores (sm_100a tcgen05):
//   D[M][N] (bf16) = alpha * A[M][K] * B[N][K]^T,
// with A and B in the layout the quantizer writes: packed E2M1 codes [rows][K/2] (element 2j
// in the low nibble) and row-major block scales [rows][K/g] (MXFP4: E8M0, g = 32; NVFP4:
// E4M3, g = 16); alpha is the product of the two NVFP4 tensor scales (1 for MXFP4).  This is
// the product the rotated, quantized activations and weights meet in ("Bridging the Gap
// Between Promise and Performance for Microscaling FP4 Quantization", Technische
// Zusammenfassung, 2. Methodik, GPU-Kernel-Unterstützung).
//
// One MMA is tcgen05.mma.kind::mxf4 (block 32, E8M0 scales) or kind::mxf4nvf4 (block 16, E4M3
// scales) of M = 128, N = 256, K = 64, accumulating in fp32 in tensor memory; the scale
// factors also live in tensor memory.  A CTA owns output tiles of 128 x 256 (persistent,
// round-robin over the tiles, M-tiles innermost so that B tiles are shared through L2) and
// streams K in stages of 256 through a 4-deep shared-memory ring.  Tensor memory holds two
// 48-column scale-factor buffers and the 256-column accumulator (a second accumulator, which
// would let the epilogue overlap the next tile, does not fit next to them at this width;
// measured, the narrower tiles that make room cost more in the mainloop than the overlap
// saves).  Roles (14 warps):
//   warp 0      producer: TMA loads of the A (128 rows x 128 B) and B (256 rows x 128 B) code
//               tiles, 128-byte swizzled, completion on the stage's "full" barrier;
//   warp 1      TMEM owner and MMA issuer: per stage, tcgen05.cp of the stage's scale factors
//               into TMEM (32x128b blocks replicated to the four lane quarters; two buffers),
//               four MMAs, then tcgen05.commit to free the stage; after a tile, commit to the
//               epilogue (issuing a stage's copies a stage earlier measured no faster: the copies
//               and the MMAs share the tensor pipe);
//   warps 2..9  epilogue, two per TMEM lane quarter (warp % 4), each taking half of the 256
//               accumulator columns: tcgen05.ld of the accumulator, times alpha,
//               to bf16, stored straight to D; then frees the accumulator;
//   warps 10..13 scale rearrangers, one per ring slot: each reads the row-major scale bytes of
//               its slot's stages and writes them in the layout tcgen05.cp reads (per MMA and
//               128 rows: 32 rows of 16 bytes, row l = the 4-byte scale words of rows l, l+32,
//               l+64, l+96), then "sf full".  A warp loads its next stage's words before it
//               waits for the slot, so four stages of scale loads are in flight.
// In tensor memory, the scale factor of row r (r < 128) and scale j of one MMA sits in lane
// r mod 32 (and its copies in the other lane quarters), column r / 32, byte j; B's 256 rows
// take 8 columns.  MXFP4's two scales per MMA take half a cell: MMA 2q uses bytes 0-1 of
// cell q (scale-factor id 0) and MMA 2q + 1 bytes 2-3 (id 2).  Every wait is bounded in time;
// a wait that runs out records kStatusTimeout and the CTA lets its issued copies and MMAs land
// before it frees TMEM.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_mma.cuh"

namespace fp4q {

template <int FMT>
struct GemmConfig {
  static constexpr int kFmt = FMT;
  static constexpr int kGroup = FMT == kMX ? 32 : 16;
  static constexpr int kBM = 128, kBN = 256, kBK = 256;   // tile rows, tile columns, K per stage
  static constexpr int kKSteps = kBK / 64;                 // MMAs per stage
  static constexpr int kStages = 4;
  static constexpr int kABytes = kBM * kBK / 2;            // 16 KB of codes
  static constexpr int kBBytes = kBN * kBK / 2;            // 32 KB of codes
  // MXFP4's two scales per MMA share a 32-bit cell with the next MMA's (bytes 0-1 and 2-3,
  // told apart by the scale-factor id), so a cell column serves two MMAs; NVFP4's four fill it
  static constexpr int kMmasPerCell = FMT == kMX ? 2 : 1;
  static constexpr int kCellSteps = kKSteps / kMmasPerCell;   // cell columns per stage and row group
  static constexpr int kSfaBytes = kCellSteps * 512;       // one 32 x 16 B block per cell step
  static constexpr int kSfbBytes = kCellSteps * 1024;      // two per cell step (up to 256 rows)
  static constexpr int kSfPad = (1024 - (kABytes + kBBytes + kSfaBytes + kSfbBytes) % 1024) % 1024;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes + kSfPad;
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned (128-byte swizzle atoms)");
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = 1024 + kBarOffset + 256;
  static constexpr int kSfColsPerStage = kCellSteps * (4 + 8);
  static constexpr int kSfCol0 = 0;                        // two scale-factor buffers, then
  static constexpr int kAccCol0 = 2 * kSfColsPerStage;     // the fp32 accumulator(s) of kBN columns
  static constexpr int kTmemCols = 512;
  // two accumulators (the epilogue of one tile under the MMAs of the next) when they fit
  static constexpr int kAccBufs = kAccCol0 + 2 * kBN <= kTmemCols ? 2 : 1;
  static_assert(kAccCol0 + kAccBufs * kBN <= kTmemCols, "accumulators and two scale buffers fit");
  static_assert(kBN % 16 == 0 && kAccCol0 % 16 == 0, "MMA N and accumulator columns in steps of 16");
  static constexpr int kBRowGroups = kBN / 32;             // 32-row groups of B (2 copy blocks of 4)
  static_assert(kBN % 32 == 0 && kBRowGroups <= 8, "B tile of at most 256 rows in 32-row groups");
  // eight epilogue warps drain the single accumulator twice as fast as four (the MMAs of
  // the next tile wait for it)
  static constexpr int kEpiWarps = 8;
  static constexpr int kEpiWarp0 = 2, kScaleWarp0 = kEpiWarp0 + kEpiWarps;
  static constexpr int kThreads = 32 * (kScaleWarp0 + kStages);
  // instruction descriptor: E2M1 x E2M1 (format 1), K-major A and B, N >> 3, scale format
  // (1 = E8M0, 0 = E4M3), M >> 4; dense, no negation, scale-factor ids 0
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                                     ((FMT == kMX ? 1u : 0u) << 23) | (static_cast<uint32_t>(kBM >> 4) << 24);
};

struct GemmArgs {
  const uint8_t* a_scales;   // [M][K/g]
  const uint8_t* b_scales;   // [N][K/g]
  const float* a_tensor_scale;
  const float* b_tensor_scale;
  uint16_t* d;               // bf16 [M][N]
  int64_t M, N, K;
  int tiles_m, tiles_n, k_stages;
};

__device__ __forceinline__ void utccp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <int FMT>
__device__ __forceinline__ void umma_fp4_block_scaled(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                                      uint32_t tsfa, uint32_t tsfb, uint32_t acc) {
  if constexpr (FMT == kNV) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
        : "memory");
  }
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The 4-byte scale cells of one row for the stage (NVFP4: cell kk = the scales of K elements
// 64 kk .. 64 kk + 63 of the stage; MXFP4: cells 0 and 1, two MMAs each); zero for rows past
// the end.
template <int FMT>
__device__ __forceinline__ uint4 stage_scale_words(const uint8_t* scales, int64_t row, int64_t rows, int64_t K,
                                                   int ks) {
  if (row >= rows) return make_uint4(0u, 0u, 0u, 0u);
  if constexpr (FMT == kNV) {
    // 16 scale bytes: 4 per MMA
    return __ldg(reinterpret_cast<const uint4*>(scales + row * (K / 16) + static_cast<int64_t>(ks) * 16));
  } else {
    // 8 scale bytes: 2 per MMA; word q holds MMAs 2q (bytes 0-1) and 2q + 1 (bytes 2-3)
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(scales + row * (K / 32) + static_cast<int64_t>(ks) * 8));
    return make_uint4(v.x, v.y, 0u, 0u);
  }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, GemmArgs g) {
  constexpr int S = Cfg::kStages, KS = Cfg::kKSteps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t stage0 = smem_addr(smem);
  const uint32_t bars = stage0 + Cfg::kBarOffset;
  auto a_tile = [&](int s) { return stage0 + s * Cfg::kStageBytes; };
  auto b_tile = [&](int s) { return stage0 + s * Cfg::kStageBytes + Cfg::kABytes; };
  auto sfa_blk = [&](int s) { return stage0 + s * Cfg::kStageBytes + Cfg::kABytes + Cfg::kBBytes; };
  auto sfb_blk = [&](int s) { return stage0 + s * Cfg::kStageBytes + Cfg::kABytes + Cfg::kBBytes + Cfg::kSfaBytes; };
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto sfull_bar = [&](int s) { return bars + 8u * (S + s); };
  auto empty_bar = [&](int s) { return bars + 8u * (2 * S + s); };
  auto acc_full = [&](int d) { return bars + 8u * (3 * S + d); };
  auto acc_empty = [&](int d) { return bars + 8u * (3 * S + 2 + d); };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(sfull_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int d = 0; d < 2; ++d) {
      mbar_init(acc_full(d), 1);
      mbar_init(acc_empty(d), Cfg::kEpiWarps);
    }
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
  const int n_tiles = g.tiles_m * g.tiles_n;

  if (warp == 0) {
    // ---------------- producer: TMA loads of the code tiles
    if (lane == 0) {
      pdl_wait();
      int64_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int tm = t % g.tiles_m, tn = t / g.tiles_m;
        for (int ks = 0; ks < g.k_stages; ++ks, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), Cfg::kABytes + Cfg::kBBytes);
          tma_load_2d(a_tile(s), &amap, ks * (Cfg::kBK / 2), tm * Cfg::kBM, full_bar(s));
          tma_load_2d(b_tile(s), &bmap, ks * (Cfg::kBK / 2), tn * Cfg::kBN, full_bar(s));
        }
      }
      // let every issued copy land before the CTA can leave
      for (int64_t j = (it > S ? it - S : 0); j < it; ++j)
        mbar_wait_bounded(full_bar(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1));
    }
  } else if (warp >= Cfg::kScaleWarp0) {
    // ---------------- scale rearrangers: warp kScaleWarp0 + j serves ring slot j
    const int slot = warp - Cfg::kScaleWarp0;
    pdl_wait();
    // this warp's stages, in order: global stage index it = slot, slot + S, ...
    const int64_t total = static_cast<int64_t>((n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                               static_cast<int>(gridDim.x)) * g.k_stages;
    auto load = [&](int64_t it, uint4 (&wa)[4], uint4 (&wb)[8]) {
      const int t = static_cast<int>(blockIdx.x) + static_cast<int>(it / g.k_stages) * static_cast<int>(gridDim.x);
      const int ks = static_cast<int>(it % g.k_stages);
      const int tm = t % g.tiles_m, tn = t / g.tiles_m;
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1)
        wa[r1] = stage_scale_words<Cfg::kFmt>(g.a_scales, static_cast<int64_t>(tm) * Cfg::kBM + lane + 32 * r1, g.M,
                                              g.K, ks);
#pragma unroll
      for (int n1 = 0; n1 < 8; ++n1) {
        const int rt = lane + 32 * n1;   // row within the tile; rows past it belong to the next one
        wb[n1] = n1 < Cfg::kBRowGroups
                     ? stage_scale_words<Cfg::kFmt>(g.b_scales, static_cast<int64_t>(tn) * Cfg::kBN + rt, g.N, g.K, ks)
                     : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    uint4 wa[4], wb[8];
    if (slot < total) load(slot, wa, wb);
    for (int64_t it = slot; it < total; it += S) {
      const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
      const bool mine = mbar_wait_bounded(empty_bar(slot), ph ^ 1u);
      if (!__all_sync(0xFFFFFFFFu, mine)) break;
      // one 16-byte store per lane and block: lane l writes its row of 4 words (conflict-free)
      const uint32_t la = sfa_blk(slot) + lane * 16, lb = sfb_blk(slot) + lane * 16;
      sts128(la + 0 * 512, wa[0].x, wa[1].x, wa[2].x, wa[3].x);
      sts128(la + 1 * 512, wa[0].y, wa[1].y, wa[2].y, wa[3].y);
      sts128(lb + 0 * 1024, wb[0].x, wb[1].x, wb[2].x, wb[3].x);
      sts128(lb + 0 * 1024 + 512, wb[4].x, wb[5].x, wb[6].x, wb[7].x);
      sts128(lb + 1 * 1024, wb[0].y, wb[1].y, wb[2].y, wb[3].y);
      sts128(lb + 1 * 1024 + 512, wb[4].y, wb[5].y, wb[6].y, wb[7].y);
      if constexpr (Cfg::kCellSteps == 4) {
        sts128(la + 2 * 512, wa[0].z, wa[1].z, wa[2].z, wa[3].z);
        sts128(la + 3 * 512, wa[0].w, wa[1].w, wa[2].w, wa[3].w);
        sts128(lb + 2 * 1024, wb[0].z, wb[1].z, wb[2].z, wb[3].z);
        sts128(lb + 2 * 1024 + 512, wb[4].z, wb[5].z, wb[6].z, wb[7].z);
        sts128(lb + 3 * 1024, wb[0].w, wb[1].w, wb[2].w, wb[3].w);
        sts128(lb + 3 * 1024 + 512, wb[4].w, wb[5].w, wb[6].w, wb[7].w);
      }
      fence_proxy_async_smem();   // the tensor core's copy reads these bytes through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(sfull_bar(slot));
      if (it + S < total) load(it + S, wa, wb);   // the next stage's words travel while this one is consumed
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int64_t it = 0;
      int tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++tc) {
        const int d = tc % Cfg::kAccBufs;
        const uint32_t dph = static_cast<uint32_t>((tc / Cfg::kAccBufs) & 1);
        if (!mbar_wait_bounded(acc_empty(d), dph ^ 1u)) break;
        tc_fence_after();
        const uint32_t acc = tmem_base + Cfg::kAccCol0 + d * Cfg::kBN;
        for (int ks = 0; ks < g.k_stages; ++ks, ++it) {
          const int s = static_cast<int>(it % S);
          const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
          if (!mbar_wait_bounded(full_bar(s), ph) || !mbar_wait_bounded(sfull_bar(s), ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tmem_base + Cfg::kSfCol0 + static_cast<uint32_t>(it & 1) * Cfg::kSfColsPerStage;
          constexpr int CS = Cfg::kCellSteps;
#pragma unroll
          for (int c = 0; c < CS; ++c) {
            utccp_32x128b_x4(sf + c * 4, umma_smem_desc(sfa_blk(s) + c * 512, 128, 0));
            utccp_32x128b_x4(sf + 4 * CS + c * 8, umma_smem_desc(sfb_blk(s) + c * 1024, 128, 0));
            utccp_32x128b_x4(sf + 4 * CS + c * 8 + 4, umma_smem_desc(sfb_blk(s) + c * 1024 + 512, 128, 0));
          }
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            // the MMA's scales start at byte `id` of their cells: the id goes in the instruction
            // descriptor and in the top two bits of the TMEM addresses
            const int c = kk / Cfg::kMmasPerCell;
            const uint32_t id = static_cast<uint32_t>((kk % Cfg::kMmasPerCell) * 2);
            const uint32_t idesc = Cfg::kIdesc | (id << 4) | (id << 29);
            umma_fp4_block_scaled<Cfg::kFmt>(acc, umma_smem_desc(a_tile(s) + kk * 32, 1024, 2),
                                             umma_smem_desc(b_tile(s) + kk * 32, 1024, 2), idesc,
                                             (sf + c * 4) | (id << 30), (sf + 4 * CS + c * 8) | (id << 30),
                                             (ks | kk) != 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
        }
        if (!ok) break;
        umma_commit(acc_full(d));
      }
      // the last commits must have landed before TMEM is freed
      if (tc > 0)
        mbar_wait_bounded(acc_full((tc - 1) % Cfg::kAccBufs), static_cast<uint32_t>(((tc - 1) / Cfg::kAccBufs) & 1));
    }
  } else {
    // ---------------- epilogue: warps 2..9, TMEM lane quarter warp % 4, column half (warp - 2) / 4
    const int q = warp & 3;
    constexpr int kColChunks = Cfg::kBN / 16 / (Cfg::kEpiWarps / 4);   // 16-column chunks per warp
    const int c0 = ((warp - Cfg::kEpiWarp0) >> 2) * kColChunks;
    pdl_wait();   // the tensor scales come from earlier kernels, and D may still be read by one
    const float alpha = Cfg::kFmt == kNV ? (*g.a_tensor_scale) * (*g.b_tensor_scale) : 1.0f;
    int tc = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
      const int tm = t % g.tiles_m, tn = t / g.tiles_m;
      const int d = tc % Cfg::kAccBufs;
      const bool mine = mbar_wait_bounded(acc_full(d), static_cast<uint32_t>((tc / Cfg::kAccBufs) & 1));
      if (!__all_sync(0xFFFFFFFFu, mine)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(tm) * Cfg::kBM + 32 * q + lane;
      const uint32_t acc = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + Cfg::kAccCol0 + d * Cfg::kBN;
      static_assert(kColChunks % 2 == 0, "chunks are read in pairs");
#pragma unroll 1
      for (int c = c0; c < c0 + kColChunks; c += 2) {
        float v[2][16];
        tmem_ld16(acc + c * 16, v[0]);   // two 16-column chunks per wait
        tmem_ld16(acc + c * 16 + 16, v[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t col0 = static_cast<int64_t>(tn) * Cfg::kBN + 16 * (c + h);
          if (row < g.M && col0 < g.N) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[h][2 * i] * alpha, v[h][2 * i + 1] * alpha);
            uint16_t* dp = g.d + row * g.N + col0;
            stg128(dp, w[0], w[1], w[2], w[3]);
            stg128(dp + 8, w[4], w[5], w[6], w[7]);
          }
        }
      }
      // the accumulator can be reused once every epilogue warp has read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(d));
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
