// ssd_tc.cuh -- the tensor-core (tcgen05 / TMEM / TMA) path of the chunked SSD forward pass.
#pragma once

#include <cudaTypedefs.h>

#include "ssd_common.cuh"

namespace ssd {

// True when the tensor-core path takes this shape and chunk length.
bool tc_supports(const ssd_shape* s, int chunk);

// Enqueues the fused tensor-core kernel; for a packed batch the chunk table (which
// gives seq_tiles) must already be enqueued.
cudaError_t launch_tc(const Problem& pb, cudaStream_t st);

// The driver's cuTensorMapEncodeTiled (looked up once), or null.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace ssd
