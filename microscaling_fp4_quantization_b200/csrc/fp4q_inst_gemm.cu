// Explicit instantiations of the block-scaled FP4 GEMM.  One kernel family per translation
// unit, so that the library's kernels compile in parallel (see fp4q_host.cuh).
#include "fp4q_launch.cuh"

namespace fp4q {
namespace host {

template fp4q_status launch_gemm<kMX>(const uint8_t*, const uint8_t*, const float*, const uint8_t*, const uint8_t*,
                                      const float*, int64_t, int64_t, int64_t, uint16_t*, cudaStream_t);
template fp4q_status launch_gemm<kNV>(const uint8_t*, const uint8_t*, const float*, const uint8_t*, const uint8_t*,
                                      const float*, int64_t, int64_t, int64_t, uint16_t*, cudaStream_t);

}  // namespace host
}  // namespace fp4q

FP4Q_DEFINE_STATUS_READER(status_gemm)
