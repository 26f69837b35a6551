// Explicit instantiations of the dequantize kernels of MXFP4 and NVFP4.  One kernel family per translation unit, so
// that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

#define FP4Q_DQ_ONE(F, B, U)                                                                                   \
  template fp4q_status launch_dequantize<F, B, U>(const uint8_t*, const uint8_t*, const float*, int64_t, float*, \
                                                  ChannelSigns, const uint8_t*, cudaStream_t);
#define FP4Q_DQ(B) FP4Q_DQ_ONE(kMX, B, true) FP4Q_DQ_ONE(kMX, B, false) FP4Q_DQ_ONE(kNV, B, true) FP4Q_DQ_ONE(kNV, B, false)
FP4Q_FOR_BLOCKS(FP4Q_DQ)

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_dequant)
