// Explicit instantiations of the MBS-Static kernels (rotate + quantize, error pass, dequantize).  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_MBS_RULE(B, R)                                                                                    \
  template fp4q_status launch_rq<RQConfig<kMBS, B, R, false, 128>>(RQArgs, int64_t, cudaStream_t, int64_t);   \
  template fp4q_status launch_qe<RQConfig<kMBS, B, R, false, 128>>(fp4q_plan, QEArgs, int64_t, double*,       \
                                                                   cudaStream_t);                             \
  template fp4q_status qe_wave<RQConfig<kMBS, B, R, false, 128>>(int*);
#define FP4Q_MBS(B)                                                                                            \
  FP4Q_MBS_RULE(B, kRuleFloor) FP4Q_MBS_RULE(B, kRuleCeil) FP4Q_MBS_RULE(B, kRuleOas)                         \
  template fp4q_status launch_dequantize<kMBS, B, true>(const uint8_t*, const uint8_t*, const float*, int64_t,  \
                                                        float*, ChannelSigns, const uint8_t*, cudaStream_t);  \
  template fp4q_status launch_dequantize<kMBS, B, false>(const uint8_t*, const uint8_t*, const float*, int64_t, \
                                                         float*, ChannelSigns, const uint8_t*, cudaStream_t);
FP4Q_FOR_BLOCKS(FP4Q_MBS)

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_mbs)
