// Explicit instantiations of the quantization-error kernels of MXFP4 and NVFP4.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_QE_ONE(CFG)                                                                                       \
  template fp4q_status launch_qe<CFG>(fp4q_plan, QEArgs, int64_t, double*, cudaStream_t);                    \
  template fp4q_status qe_wave<CFG>(int*);
#define FP4Q_QE(B)                                                                                             \
  FP4Q_QE_ONE(RQConfig<kMX FP4Q_COMMA B FP4Q_COMMA kRuleFloor FP4Q_COMMA false>)                               \
  FP4Q_QE_ONE(RQConfig<kMX FP4Q_COMMA B FP4Q_COMMA kRuleCeil FP4Q_COMMA false>)                                \
  FP4Q_QE_ONE(RQConfig<kMX FP4Q_COMMA B FP4Q_COMMA kRuleOas FP4Q_COMMA false>)                                 \
  FP4Q_QE_ONE(RQConfig<kNV FP4Q_COMMA B FP4Q_COMMA kRuleNvStatic FP4Q_COMMA false FP4Q_COMMA 16>)              \
  FP4Q_QE_ONE(RQConfig<kNV FP4Q_COMMA B FP4Q_COMMA kRuleNvStatic FP4Q_COMMA false FP4Q_COMMA 32>)              \
  FP4Q_QE_ONE(RQConfig<kNV FP4Q_COMMA B FP4Q_COMMA kRuleNvDynamic FP4Q_COMMA false FP4Q_COMMA 16>)             \
  FP4Q_QE_ONE(RQConfig<kNV FP4Q_COMMA B FP4Q_COMMA kRuleNvDynamic FP4Q_COMMA false FP4Q_COMMA 32>)
#define FP4Q_COMMA ,
FP4Q_FOR_BLOCKS(FP4Q_QE)

fp4q_status launch_quant_error_empty(const double* partials, double* out, cudaStream_t stream) {
  cudaError_t e = launch_pdl(quant_error_empty_kernel, dim3(1), dim3(32), 0, stream, partials, out);
  if (e != cudaSuccess) return cuda_fail(e, "quant_error launch");
  return FP4Q_OK;
}

fp4q_status launch_wait_timeout_selftest(cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return FP4Q_OK;
}

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_qe)
