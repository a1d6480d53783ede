// Per-group implicit GEMM on tcgen05 tensor cores (placeholder until the kernel lands).
#include "internal.cuh"

namespace gconv {

bool igemm_supported(const Conv2d&) { return false; }
size_t igemm_nchw_workspace(const Conv2d&) { return 0; }
cudaError_t launch_igemm_nhwc(const Conv2d&, const void*, const void*, const void*, void*,
                              cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_igemm_nchw(const Conv2d&, const void*, const void*, const void*, void*, void*,
                              cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace gconv
