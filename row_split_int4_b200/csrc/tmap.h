// tmap.h -- the driver's tensor-map encoder (cuTensorMapEncodeTiled), looked up
// once through the runtime so that libtf.so needs no link against libcuda.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

namespace tf {

// null when the driver offers no encoder
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn();

}  // namespace tf
