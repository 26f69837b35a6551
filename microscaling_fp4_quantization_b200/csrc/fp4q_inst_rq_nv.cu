// Explicit instantiations of the NVFP4 butterfly rotate + quantize kernels, the rotated-amax pass, its finalize kernel and the no-allocation scratch.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_RQ_NV_RULE(B, R, U)                                                                              \
  template fp4q_status launch_rq<RQConfig<kNV, B, R, false, U>>(RQArgs, int64_t, cudaStream_t, int64_t);     \
  template fp4q_status launch_rq<RQConfig<kNV, B, R, true, U>>(RQArgs, int64_t, cudaStream_t, int64_t);
#define FP4Q_RQ_NV(B)                                                                                         \
  FP4Q_RQ_NV_RULE(B, kRuleNvStatic, 16) FP4Q_RQ_NV_RULE(B, kRuleNvStatic, 32)                                 \
  FP4Q_RQ_NV_RULE(B, kRuleNvDynamic, 16) FP4Q_RQ_NV_RULE(B, kRuleNvDynamic, 32)                               \
  template fp4q_status amax_wave<AmaxCfg<B, 16>>(int*);                                                       \
  template fp4q_status amax_wave<AmaxCfg<B, 32>>(int*);                                                       \
  template fp4q_status launch_amax_cfg<AmaxCfg<B, 16>>(const uint16_t*, int64_t, float*, int, ChannelSigns,   \
                                                       cudaStream_t, bool);                                   \
  template fp4q_status launch_amax_cfg<AmaxCfg<B, 32>>(const uint16_t*, int64_t, float*, int, ChannelSigns,   \
                                                       cudaStream_t, bool);
FP4Q_FOR_BLOCKS(FP4Q_RQ_NV)

fp4q_status launch_tensor_scale_finalize(const float* partials, int n, float* out, cudaStream_t stream) {
  cudaError_t e = launch_pdl(tensor_scale_finalize_kernel, dim3(1), dim3(32), 0, stream, partials, n, out);
  if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  return FP4Q_OK;
}

}  // namespace host
}  // namespace fp4q

// Scratch of the no-allocation entry point (the host name below is only a stand-in; kernels
// get the device address from cudaGetSymbolAddress).
static __device__ __align__(256) float g_noalloc_partials[fp4q::host::kNoAllocMaxPartials];

fp4q_status fp4q::host::noalloc_partials_symbol(float** out) {
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_noalloc_partials);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  return FP4Q_OK;
}

FP4Q_DEFINE_STATUS_READER(status_rq_nv)
