// baseline.cu -- uncompressed fp16 / fp8 paged decode (measurement baselines).
#include "common.cuh"
#include "kvarn_internal.h"

namespace kvarn {

cudaError_t launch_baseline(const BaselineArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kvarn
