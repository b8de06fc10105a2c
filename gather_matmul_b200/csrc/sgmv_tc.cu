// tcgen05 tensor-core kernels for segment-grouped (SGMV) shrink and expand.
#include "common.cuh"
#include "internal.h"

namespace lora {

cudaError_t launch_shrink_segment_tc(lora_dtype, const ShrinkArgs&, const SegArgs&,
                                     cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_expand_segment_tc(lora_dtype, const ExpandArgs&, const SegArgs&,
                                     cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lora
