// ssd_tc.cu -- tensor-core path (placeholder until the tcgen05 kernels land).
#include "ssd_tc.cuh"

namespace ssd {

bool tc_supports(const ssd_shape*, int) { return false; }

cudaError_t launch_tc(const Problem&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace ssd
