// bwd_sm100.cu -- placeholder until the tcgen05 backward kernels land.
#include "launch.h"
namespace ra {
cudaError_t launch_bwd_dkdv_sm100(const ra_problem&, const Sm100Maps&, const void*, const void*,
                                  const float*, const float*, const float2*, void*, void*, float*,
                                  const DevCtl&, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_bwd_dq_sm100(const ra_problem&, const Sm100Maps&, const void*, const float*,
                                const float*, const float2*, void*, float*, const DevCtl&,
                                cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace ra
