// Definitions of the per-configuration launchers declared in fp4q_host.cuh.  Included only
// by the instantiation units (fp4q_inst_*.cu), each of which instantiates the launchers of
// one kernel family explicitly.
#pragma once

#include <cstdio>

#include "fp4q_host.cuh"

namespace fp4q {
namespace host {

template <class Cfg>
fp4q_status launch_rq(RQArgs a, int64_t n_elems, cudaStream_t stream, int64_t K) {
  a.n_units = n_elems / Cfg::kE;
  a.signs = channel_signs<Cfg>(a.signs.mask, K);
  auto kernel = rotate_quantize_kernel<Cfg>;
  KernelInfo ki;
  fp4q_status st = butterfly_kernel_info<Cfg>(kernel, &ki, a.signs.smem_words);
  if (st != FP4Q_OK) return st;
  const int64_t warps_needed = (a.n_units + Cfg::kUnitsPerStage - 1) / Cfg::kUnitsPerStage;
  int64_t ctas = (warps_needed + Cfg::kWarps - 1) / Cfg::kWarps;
  const int64_t max_ctas = static_cast<int64_t>(ki.sm_count) * ki.ctas_per_sm;
  if (ctas > max_ctas) ctas = max_ctas;
  cudaError_t e = launch_pdl(kernel, dim3(static_cast<unsigned>(ctas)), dim3(Cfg::kThreads),
                             Cfg::kSmemBytes + 4 * a.signs.smem_words, stream, a);
  if (e != cudaSuccess) return cuda_fail(e, "rotate_quantize launch");
  return FP4Q_OK;
}

// Tensor-core kernel: a TMA tensor map over the rows of one Hadamard block each.  `a` holds
// the outputs (codes and scales, or the error pass's sums); the rest is filled in here.
// max_ctas caps the persistent grid (the error pass's partial-sum slots), 0 for none.
template <class Cfg>
fp4q_status launch_mma_common(MmaArgs a, const uint16_t* x, int64_t n_elems, const ChannelSigns& signs,
                              cudaStream_t stream, int64_t K, int64_t max_ctas) {
  EncodeTiledFn enc;
  fp4q_status st = encode_fn(&enc);
  if (st != FP4Q_OK) return st;
  a.x = x;
  a.n_rows = n_elems / Cfg::kBlock;
  a.n_super = (a.n_rows + Cfg::kRowsPerTile - 1) / Cfg::kRowsPerTile;
  a.sign_bytes = reinterpret_cast<const uint8_t*>(signs.mask);
  a.sign_upr = signs.mask ? K / Cfg::kBlock : 1;
  // the expanded sign table (4 K bytes) where the configuration has one and it fits, else the
  // mask's words (ceil(K / 32) of them), staged in shared memory when they fit
  const int64_t mask_bytes = signs.mask ? (K + 127) / 128 * 16 : 0;
  const int64_t table_bytes = signs.mask ? 4 * K : 0;
  const int64_t word_bytes = signs.mask ? 4 * (K / Cfg::kBlock + Cfg::kSignExt) * (Cfg::kBlock / 8) : 0;
  a.sign_table = !signs.mask                                                 ? 0
                 : Cfg::kSignTable && table_bytes <= Cfg::kSignTableMax      ? 1
                 : !Cfg::kSignTable && word_bytes <= Cfg::kMaskSmemMax       ? 2
                                                                             : 0;
  a.sign_smem = a.sign_table == 1                 ? static_cast<int>(table_bytes)
                : a.sign_table == 2               ? static_cast<int>(word_bytes)
                : mask_bytes <= Cfg::kMaskSmemMax ? static_cast<int>(mask_bytes)
                                                  : 0;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Cfg::kBlock), static_cast<cuuint64_t>(a.n_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Cfg::kBlock) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(Cfg::kKB), static_cast<cuuint32_t>(Cfg::kBoxRows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = Cfg::kRB == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                : Cfg::kRB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(last_error_buffer(), kLastErrorBytes, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return FP4Q_ERR_CUDA;
  }
  auto kernel = rotate_quantize_mma_kernel<Cfg>;
  KernelInfo ki;
  st = kernel_info(kernel, Cfg::kSmemBytes + Cfg::kSignSmemMax, Cfg::kThreads, &ki);
  if (st != FP4Q_OK) return st;
  // CTAs per SM from measurement (the kernel's CTAs are independent, so a CTA that does not
  // fit next to the others simply starts later); tensor memory holds 512 columns per SM
  int per_sm = Cfg::kCtasPerSm;
  if (per_sm > 512 / Cfg::kTmemCols) per_sm = 512 / Cfg::kTmemCols;
  int64_t ctas = static_cast<int64_t>(ki.sm_count) * per_sm;
  if (ctas > a.n_super) ctas = a.n_super;
  if (max_ctas > 0 && ctas > max_ctas) ctas = max_ctas;
  cudaError_t e = launch_pdl(kernel, dim3(static_cast<unsigned>(ctas)), dim3(Cfg::kThreads),
                             Cfg::kSmemBytes + a.sign_smem, stream, map, a);
  if (e != cudaSuccess) return cuda_fail(e, Cfg::kQE ? "quant_error (tensor core) launch"
                                                     : "rotate_quantize (tensor core) launch");
  return FP4Q_OK;
}

template <class Cfg>
fp4q_status launch_mma(const uint16_t* x, int64_t n_elems, const RQArgs& ra, cudaStream_t stream, int64_t K) {
  MmaArgs a = {};
  a.codes = ra.codes;
  a.scales = ra.scales;
  a.tensor_scale = ra.tensor_scale;
  a.partials = ra.partials;
  a.n_partials = ra.n_partials;
  a.y_dump = ra.y_dump;
  a.macro = ra.macro;
  return launch_mma_common<Cfg>(a, x, n_elems, ra.signs, stream, K, 0);
}

// The error pass on the tensor-core kernel: one partial pair per CTA in qa.out_partials,
// whose slots (max_ctas of them) cap the grid.
template <class Cfg>
fp4q_status launch_mma_qe(const QEArgs& qa, int64_t n_elems, cudaStream_t stream, int64_t K, int max_ctas) {
  MmaArgs a = {};
  a.tensor_scale = qa.tensor_scale;
  a.partials = qa.partials;
  a.n_partials = qa.n_partials;
  a.qe_partials = qa.out_partials;
  a.qe_ticket = qa.ticket;
  a.qe_out = qa.out;
  return launch_mma_common<Cfg>(a, qa.x, n_elems, qa.signs, stream, K, max_ctas);
}

template <class Cfg>
fp4q_status launch_mma_amax(const uint16_t* x, int64_t n_elems, float* partials, int slots, const ChannelSigns& signs,
                            cudaStream_t stream, int64_t K) {
  MmaArgs a = {};
  a.amax_out = partials;
  a.amax_slots = slots;
  return launch_mma_common<Cfg>(a, x, n_elems, signs, stream, K, slots);
}

template <class Cfg>
fp4q_status qe_wave(int* n) {
  KernelInfo ki;
  fp4q_status r = butterfly_kernel_info<Cfg>(quant_error_kernel<Cfg>, &ki);
  *n = ki.sm_count * ki.ctas_per_sm;
  return r;
}

template <class Cfg>
fp4q_status launch_qe(fp4q_plan p, QEArgs a, int64_t n_elems, double* out, cudaStream_t stream) {
  a.n_units = n_elems / Cfg::kE;
  a.signs = channel_signs<Cfg>(p->signs, p->signs_K);
  auto kernel = quant_error_kernel<Cfg>;
  KernelInfo ki;
  fp4q_status st = butterfly_kernel_info<Cfg>(kernel, &ki, a.signs.smem_words);
  if (st != FP4Q_OK) return st;
  const int64_t warps_needed = (a.n_units + Cfg::kUnitsPerStage - 1) / Cfg::kUnitsPerStage;
  int64_t ctas = (warps_needed + Cfg::kWarps - 1) / Cfg::kWarps;
  const int64_t max_ctas = static_cast<int64_t>(ki.sm_count) * ki.ctas_per_sm;
  if (ctas > max_ctas) ctas = max_ctas;
  if (ctas > p->n_err_partials) ctas = p->n_err_partials;
  a.out = out;
  cudaError_t e = launch_pdl(kernel, dim3(static_cast<unsigned>(ctas)), dim3(Cfg::kThreads),
                             Cfg::kSmemBytes + 4 * a.signs.smem_words, stream, a);
  if (e != cudaSuccess) return cuda_fail(e, "quant_error launch");
  return FP4Q_OK;
}

template <class Cfg>
fp4q_status amax_wave(int* n) {
  KernelInfo ki;
  fp4q_status r = butterfly_kernel_info<Cfg>(rotated_amax_kernel<Cfg>, &ki);
  *n = ki.sm_count * ki.ctas_per_sm;
  return r;
}

template <class Cfg>
fp4q_status launch_amax_cfg(const uint16_t* x, int64_t n_elems, float* partials, int n_partials, ChannelSigns sg,
                            cudaStream_t stream, bool pdl) {
  // the attribute for the largest (signed) launch on the current context, as the other
  // butterfly launchers set it
  KernelInfo ki;
  fp4q_status st = butterfly_kernel_info<Cfg>(rotated_amax_kernel<Cfg>, &ki, sg.smem_words);
  if (st != FP4Q_OK) return st;
  cudaError_t e;
  const size_t smem = Cfg::kSmemBytes + 4 * static_cast<size_t>(sg.smem_words);
  if (pdl) {
    e = launch_pdl(rotated_amax_kernel<Cfg>, dim3(n_partials), dim3(Cfg::kThreads), smem, stream, x,
                   n_elems / Cfg::kE, partials, sg);
  } else {
    rotated_amax_kernel<Cfg><<<n_partials, Cfg::kThreads, smem, stream>>>(x, n_elems / Cfg::kE, partials, sg);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  return FP4Q_OK;
}

template <int FMT, int B, bool UNROTATE>
fp4q_status launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t n_units,
                              float* out, ChannelSigns sg, const uint8_t* macro, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((n_units + 127) / 128);
  dequantize_kernel<FMT, B, UNROTATE><<<grid, 128, 0, stream>>>(codes, scales, tensor_scale, n_units, out, sg, macro);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return FP4Q_OK;
}

template <int FMT>
fp4q_status launch_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts, const uint8_t* b_codes,
                        const uint8_t* b_scales, const float* b_ts, int64_t M, int64_t N, int64_t K, uint16_t* d,
                        cudaStream_t stream) {
  using Cfg = GemmConfig<FMT>;
  EncodeTiledFn enc;
  fp4q_status st = encode_fn(&enc);
  if (st != FP4Q_OK) return st;
  // code tiles: bytes [rows][K/2], boxes of 128 bytes (256 E2M1 values) x 128 or 256 rows,
  // 128-byte swizzled; rows past the end read as zeros
  CUtensorMap maps[2];
  const uint8_t* srcs[2] = {a_codes, b_codes};
  const int64_t rows[2] = {M, N};
  const cuuint32_t box_rows[2] = {static_cast<cuuint32_t>(Cfg::kBM), static_cast<cuuint32_t>(Cfg::kBN)};
  for (int i = 0; i < 2; ++i) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows[i])};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(Cfg::kBK / 2), box_rows[i]};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(srcs[i]), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      std::snprintf(last_error_buffer(), kLastErrorBytes, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
      return FP4Q_ERR_CUDA;
    }
  }
  GemmArgs a;
  a.a_scales = a_scales;
  a.b_scales = b_scales;
  a.a_tensor_scale = a_ts;
  a.b_tensor_scale = b_ts;
  a.d = d;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = static_cast<int>((M + Cfg::kBM - 1) / Cfg::kBM);
  a.tiles_n = static_cast<int>((N + Cfg::kBN - 1) / Cfg::kBN);
  a.k_stages = static_cast<int>(K / Cfg::kBK);
  auto kernel = gemm_fp4_kernel<Cfg>;
  KernelInfo ki;
  st = kernel_info(kernel, Cfg::kSmemBytes, Cfg::kThreads, &ki);
  if (st != FP4Q_OK) return st;
  int64_t ctas = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  if (ctas > ki.sm_count) ctas = ki.sm_count;   // one persistent CTA per SM (its shared memory fills the SM)
  cudaError_t e = launch_pdl(kernel, dim3(static_cast<unsigned>(ctas)), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream,
                             maps[0], maps[1], a);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return FP4Q_OK;
}

}  // namespace host
}  // namespace fp4q

// Reader of this translation unit's device status word (see fp4q_host.cuh).
#define FP4Q_DEFINE_STATUS_READER(name)                                        \
  fp4q_status fp4q::host::name(unsigned int* v) {                              \
    unsigned int x = 0, zero = 0;                                              \
    cudaError_t e = cudaMemcpyFromSymbol(&x, fp4q::g_device_status, sizeof(x)); \
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");         \
    if (x) {                                                                   \
      e = cudaMemcpyToSymbol(fp4q::g_device_status, &zero, sizeof(zero));      \
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");         \
    }                                                                          \
    *v |= x;                                                                   \
    return FP4Q_OK;                                                            \
  }

// Explicit instantiation helpers: X(B) for every Hadamard block size.
#define FP4Q_FOR_BLOCKS(X) X(1) X(2) X(4) X(8) X(16) X(32) X(64) X(128)
