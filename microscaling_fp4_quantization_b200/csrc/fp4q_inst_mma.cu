// Explicit instantiations of the tensor-core (tcgen05) rotate + quantize kernels.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_MMA_ONE(F, B, R)                                                                                  \
  template fp4q_status launch_mma<MmaConfig<F, B, R, false>>(const uint16_t*, int64_t, const RQArgs&,         \
                                                             cudaStream_t, int64_t);                          \
  template fp4q_status launch_mma<MmaConfig<F, B, R, true>>(const uint16_t*, int64_t, const RQArgs&, cudaStream_t, \
                                                            int64_t);
#define FP4Q_MMA_MX(B) FP4Q_MMA_ONE(kMX, B, kRuleFloor) FP4Q_MMA_ONE(kMX, B, kRuleCeil) FP4Q_MMA_ONE(kMX, B, kRuleOas)
#define FP4Q_MMA_NV(B) FP4Q_MMA_ONE(kNV, B, kRuleNvStatic) FP4Q_MMA_ONE(kNV, B, kRuleNvDynamic)
// MBS-Static: no dump form
#define FP4Q_MMA_MBS_ONE(B, R)                                                                              \
  template fp4q_status launch_mma<MmaConfig<kMBS, B, R, false>>(const uint16_t*, int64_t, const RQArgs&, \
                                                                cudaStream_t, int64_t);
#define FP4Q_MMA_MBS(B) FP4Q_MMA_MBS_ONE(B, kRuleFloor) FP4Q_MMA_MBS_ONE(B, kRuleCeil) FP4Q_MMA_MBS_ONE(B, kRuleOas)
FP4Q_MMA_MX(32) FP4Q_MMA_MX(64) FP4Q_MMA_MX(128)
FP4Q_MMA_MBS(32) FP4Q_MMA_MBS(64) FP4Q_MMA_MBS(128)
FP4Q_MMA_NV(16) FP4Q_MMA_NV(32) FP4Q_MMA_NV(64) FP4Q_MMA_NV(128)

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_mma)
