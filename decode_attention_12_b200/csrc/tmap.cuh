// tmap.cuh -- tensor-map (TMA descriptor) encoder shared by the TMA-fed kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace lla {

// cuTensorMapEncodeTiled of the loaded driver, or nullptr when unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

} // namespace lla
