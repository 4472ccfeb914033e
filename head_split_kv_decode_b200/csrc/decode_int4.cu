#include "common.cuh"

namespace duo {

cudaError_t decode_int4_config(int, int, DecodeConfig *) { return cudaErrorNotSupported; }
cudaError_t launch_decode_int4(const DecodeParams &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace duo
