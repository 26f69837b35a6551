// Host-side internals shared by the translation units of the library: the plan object,
// launch helpers, and the declarations of the per-configuration launchers.  The launchers
// are defined in fp4q_launch.cuh and explicitly instantiated, one kernel family per
// translation unit (fp4q_inst_*.cu), so that the kernels compile in parallel; the C ABI and
// its dispatch (fp4q.cu) only call them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "fp4q.h"
#include "fp4q_kernels.cuh"
#include "fp4q_mma.cuh"
#include "fp4q_gemm.cuh"

struct fp4q_plan_s {
  uint32_t magic;
  int format, group, block, rule;
  int unit;        // elements per butterfly unit: max(block, group), 128 for MBS
  int device;
  uint64_t context; // identity of the CUDA context its device arrays were allocated in (0: none)
  float* partials; // NV plans: per-CTA rotated amaxima (device)
  int n_partials;
  int kernel;      // fp4q_kernel
  const uint32_t* signs; // per-channel random signs (device, borrowed; null: none)
  int64_t signs_K;       // the row length K the signs are for
  double* err_partials;  // fp4q_quant_error scratch (device; null without a device): per-CTA signal and
                         // error energy, then a ticket counter
  int n_err_partials;    // CTAs those hold room for
};

namespace fp4q {
namespace host {

// Identity of the CUDA context current on the calling thread (cuCtxGetId), binding the
// current device's primary context first when none is current.
fp4q_status bound_context_id(uint64_t* out);

// Records the CUDA error message (fp4q_last_cuda_error) and returns FP4Q_ERR_CUDA.
fp4q_status cuda_fail(cudaError_t e, const char* what);
// The thread's message buffer behind fp4q_last_cuda_error.
char* last_error_buffer();
constexpr int kLastErrorBytes = 512;

// Per (kernel, CUDA context, launch size) one-time set-up: opt in to the dynamic shared memory
// the kernel needs and record how many CTAs of that size fit on one SM.
struct KernelInfo {
  int ctas_per_sm = 0;
  int sm_count = 0;
};
// Occupancy is computed for smem_bytes, the dynamic shared memory of the launch; the kernel
// may be launched with up to max_smem_bytes (when larger), which every call for one kernel
// passes alike.  Results are cached per (kernel, context, smem_bytes, threads).
fp4q_status kernel_info_impl(const void* kernel, int smem_bytes, int threads, KernelInfo* out, int max_smem_bytes);

template <class K>
fp4q_status kernel_info(K kernel, int smem_bytes, int threads, KernelInfo* out, int max_smem_bytes = 0) {
  return kernel_info_impl(reinterpret_cast<const void*>(kernel), smem_bytes, threads, out, max_smem_bytes);
}

// The butterfly kernels (rotate + quantize, error pass, amax) may stage a sign mask of up to
// kSignSmemMaxWords words behind their stages; occupancy is that of a launch staging
// smem_words of them (0: an unsigned launch, or a mask read in place).
template <class Cfg, class K>
fp4q_status butterfly_kernel_info(K kernel, KernelInfo* out, int smem_words = 0) {
  return kernel_info(kernel, Cfg::kSmemBytes + 4 * smem_words, Cfg::kThreads, out,
                     Cfg::kSmemBytes + 4 * kSignSmemMaxWords);
}

// Launch with programmatic stream serialization, so the kernel's start overlaps the tail of
// the previous kernel on the stream (the kernels wait on the dependency before touching
// global memory).
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Call f.template operator()<B>() for the runtime Hadamard block b.
template <class F>
fp4q_status with_block(int b, F&& f) {
  switch (b) {
    case 1: return f.template operator()<1>();
    case 2: return f.template operator()<2>();
    case 4: return f.template operator()<4>();
    case 8: return f.template operator()<8>();
    case 16: return f.template operator()<16>();
    case 32: return f.template operator()<32>();
    case 64: return f.template operator()<64>();
    case 128: return f.template operator()<128>();
    default: return FP4Q_ERR_UNSUPPORTED;
  }
}

// The kernels' view of the plan's channel signs for a configuration with E-element units.
template <class Cfg>
ChannelSigns channel_signs(const uint32_t* mask, int64_t K) {
  if (!mask) return ChannelSigns{nullptr, 1, 0};
  const int upr = static_cast<int>(K / Cfg::kE);
  const int64_t words = (K + 31) / 32;   // the caller's mask, ceil(K / 32) words
  return ChannelSigns{mask, upr, static_cast<int>(Cfg::kUnitsPerStage % upr),
                      words <= kSignSmemMaxWords ? static_cast<int>(words) : 0};
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
// cuTensorMapEncodeTiled from the driver, looked up once.
fp4q_status encode_fn(EncodeTiledFn* out);

template <int B, int MINU>
using AmaxCfg = RQConfig<kNV, B, kRuleNvStatic, false, MINU>;

// ---- launchers (fp4q_launch.cuh), instantiated per kernel family

template <class Cfg>
fp4q_status launch_rq(RQArgs a, int64_t n_elems, cudaStream_t stream, int64_t K = 0);
template <class Cfg>
fp4q_status launch_mma(const uint16_t* x, int64_t n_elems, const RQArgs& ra, cudaStream_t stream, int64_t K);
template <class Cfg>
fp4q_status launch_mma_qe(const QEArgs& qa, int64_t n_elems, cudaStream_t stream, int64_t K, int max_ctas);
// The amax pass on the tensor-core kernel: slots entries of partials, one per CTA of a grid of
// at most that many (the rest zero).
template <class Cfg>
fp4q_status launch_mma_amax(const uint16_t* x, int64_t n_elems, float* partials, int slots, const ChannelSigns& signs,
                            cudaStream_t stream, int64_t K);
template <class Cfg>
fp4q_status launch_qe(fp4q_plan p, QEArgs a, int64_t n_elems, double* out, cudaStream_t stream);
// CTAs of one full wave of a configuration's error kernel / amax kernel.
template <class Cfg>
fp4q_status qe_wave(int* n);
template <class Cfg>
fp4q_status amax_wave(int* n);
// The amax pass over n_partials CTAs (pdl: with programmatic dependent launch).
template <class Cfg>
fp4q_status launch_amax_cfg(const uint16_t* x, int64_t n_elems, float* partials, int n_partials, ChannelSigns sg,
                            cudaStream_t stream, bool pdl);
template <int FMT, int B, bool UNROTATE>
fp4q_status launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t n_units,
                              float* out, ChannelSigns sg, const uint8_t* macro, cudaStream_t stream);
// The block-scaled FP4 GEMM D = alpha A B^T (bf16 D [M][N]); arguments validated by the caller.
template <int FMT>
fp4q_status launch_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts, const uint8_t* b_codes,
                        const uint8_t* b_scales, const float* b_ts, int64_t M, int64_t N, int64_t K, uint16_t* d,
                        cudaStream_t stream);
fp4q_status launch_tensor_scale_finalize(const float* partials, int n, float* out, cudaStream_t stream);
fp4q_status launch_quant_error_empty(const double* partials, double* out, cudaStream_t stream);
// Device address of the no-allocation path's fixed scratch (kNoAllocMaxPartials floats).
constexpr int kNoAllocMaxPartials = 4096;
fp4q_status noalloc_partials_symbol(float** out);

// Each translation unit with kernels has its own copy of the device status word; these read
// and clear it, OR-ing the flags into *v.
fp4q_status status_rq_mx(unsigned int* v);
fp4q_status status_rq_nv(unsigned int* v);
fp4q_status status_mbs(unsigned int* v);
fp4q_status status_qe(unsigned int* v);
fp4q_status status_mma(unsigned int* v);
fp4q_status status_mma_qe(unsigned int* v);
// One warp whose bounded wait runs out (fp4q_selftest_wait_timeout).
fp4q_status launch_wait_timeout_selftest(cudaStream_t stream);
fp4q_status status_dequant(unsigned int* v);
fp4q_status status_gemm(unsigned int* v);

}  // namespace host
}  // namespace fp4q
