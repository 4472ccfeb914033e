#include "common.cuh"

namespace duo {

cudaError_t launch_prefill(const PrefillParams &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace duo
