// ssd_tc.cuh -- the tensor-core (tcgen05 / TMEM / TMA) path of the chunked SSD forward pass.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

// True when the tensor-core path takes this shape and chunk length.
bool tc_supports(const ssd_shape* s, int chunk);

// Enqueues the tensor-core kernels; the chunk table must already be enqueued.
cudaError_t launch_tc(const Problem& pb, cudaStream_t st);

}  // namespace ssd
