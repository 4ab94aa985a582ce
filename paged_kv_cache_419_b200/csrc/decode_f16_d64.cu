// Decode kernels for f16 caches with head_dim 64.
#include "decode_launch.cuh"

namespace pkv {
template cudaError_t launch_decode<__half, 64>(const DecodeArgs&, const DecodeMaps&, int, int,
                                           bool, int, cudaStream_t);
}  // namespace pkv
