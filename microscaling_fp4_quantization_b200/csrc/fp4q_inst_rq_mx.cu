// Explicit instantiations of the MXFP4 butterfly rotate + quantize kernels.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_RQ_MX(B)                                                                                       \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleFloor, false>>(RQArgs, int64_t, cudaStream_t, int64_t); \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleFloor, true>>(RQArgs, int64_t, cudaStream_t, int64_t);  \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleCeil, false>>(RQArgs, int64_t, cudaStream_t, int64_t);  \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleCeil, true>>(RQArgs, int64_t, cudaStream_t, int64_t);   \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleOas, false>>(RQArgs, int64_t, cudaStream_t, int64_t);   \
  template fp4q_status launch_rq<RQConfig<kMX, B, kRuleOas, true>>(RQArgs, int64_t, cudaStream_t, int64_t);
FP4Q_FOR_BLOCKS(FP4Q_RQ_MX)

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_rq_mx)
