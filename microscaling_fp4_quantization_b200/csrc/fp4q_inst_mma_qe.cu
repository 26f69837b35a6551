// Explicit instantiations of the tensor-core (tcgen05) error pass and amax pass: the rotate +
// quantize kernel with the epilogue that accumulates energies, or keeps the largest magnitude.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_MMA_QE_ONE(F, B, R) \
  template fp4q_status launch_mma_qe<MmaConfig<F, B, R, false, true>>(const QEArgs&, int64_t, cudaStream_t, int64_t, int);
#define FP4Q_MMA_QE_MX(B) FP4Q_MMA_QE_ONE(kMX, B, kRuleFloor) FP4Q_MMA_QE_ONE(kMX, B, kRuleCeil) FP4Q_MMA_QE_ONE(kMX, B, kRuleOas)
#define FP4Q_MMA_QE_NV(B) FP4Q_MMA_QE_ONE(kNV, B, kRuleNvStatic) FP4Q_MMA_QE_ONE(kNV, B, kRuleNvDynamic)
#define FP4Q_MMA_QE_MBS(B) \
  FP4Q_MMA_QE_ONE(kMBS, B, kRuleFloor) FP4Q_MMA_QE_ONE(kMBS, B, kRuleCeil) FP4Q_MMA_QE_ONE(kMBS, B, kRuleOas)
FP4Q_MMA_QE_MX(32) FP4Q_MMA_QE_MX(64) FP4Q_MMA_QE_MX(128)
FP4Q_MMA_QE_MBS(32) FP4Q_MMA_QE_MBS(64) FP4Q_MMA_QE_MBS(128)
FP4Q_MMA_QE_NV(16) FP4Q_MMA_QE_NV(32) FP4Q_MMA_QE_NV(64) FP4Q_MMA_QE_NV(128)

// the amax pass (the NVFP4 configuration, epilogue keeping the largest magnitude)
#define FP4Q_MMA_AMAX(B)                                                                                 \
  template fp4q_status launch_mma_amax<MmaConfig<kNV, B, kRuleNvStatic, false, false, true>>(            \
      const uint16_t*, int64_t, float*, int, const ChannelSigns&, cudaStream_t, int64_t);
FP4Q_MMA_AMAX(16) FP4Q_MMA_AMAX(32) FP4Q_MMA_AMAX(64) FP4Q_MMA_AMAX(128)

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_mma_qe)
