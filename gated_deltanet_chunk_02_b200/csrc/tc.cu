// tc.cu — tcgen05 tensor-core kernels of libgdn (sm_100a).
#include "common.cuh"
#include "tc.h"

namespace gdn {

bool tc_available() { return false; }

cudaError_t launch_build_A_tc(const void*, const float*, const float*, float*, int64_t, int,
                              cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_neumann_tc(const float*, float*, int64_t, int, int, int, int, cudaStream_t) {
    return cudaErrorNotSupported;
}
cudaError_t launch_wy_tc(const float*, const void*, const void*, const float*, const float*,
                         void*, void*, int64_t, int, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_neumann_i8_tc(const float*, float*, int, int, int8_t*, int32_t*, float*,
                                 int64_t, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_fused_tc(const void*, const void*, const float*, const float*, int, int, int,
                            int, void*, void*, float*, int64_t, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdn
