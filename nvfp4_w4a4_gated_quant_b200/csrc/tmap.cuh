// Tensor-map (TMA descriptor) encoding, shared by the kernels that move tiles
// with cp.async.bulk.tensor.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

namespace gdn {

// cuTensorMapEncodeTiled, resolved once through the runtime's driver entry
// point (the library links no libcuda); nullptr when the driver lacks it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace gdn
