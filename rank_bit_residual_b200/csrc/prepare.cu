// prepare.cu - placeholder until the randomized-SVD weight split lands.
#include "internal.h"

namespace svdq {

size_t prepare_scratch_bytes(int64_t, int64_t, int32_t, int32_t) { return 256; }

svdq_status run_prepare(const void*, svdq_dtype, int64_t, int64_t, int64_t, const float*, int32_t,
                        svdq_fmt, uint64_t, int32_t, int32_t, void*, size_t, svdq_weight*,
                        cudaStream_t) {
  return SVDQ_EUNSUPPORTED;
}

cudaError_t launch_gemm_nvfp4(const svdq_weight*, const uint8_t*, const uint8_t*, const float*,
                              const void*, int64_t, const void*, void*, svdq_dtype, int64_t,
                              cudaStream_t, bool* bad_args) {
  *bad_args = true;
  return cudaSuccess;
}

}  // namespace svdq
