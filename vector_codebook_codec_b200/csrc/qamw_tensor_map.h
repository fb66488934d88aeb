// qamw_tensor_map.h -- the driver's cuTensorMapEncodeTiled, reached through
// the runtime (no link against libcuda), shared by the kernels that move
// tiles with TMA tensor copies.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

namespace qamw {

// nullptr if the driver does not provide it
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace qamw
