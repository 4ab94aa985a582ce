// Decode kernels for bf16 caches with head_dim 128.
#include "decode_launch.cuh"

namespace pkv {
template cudaError_t launch_decode<__nv_bfloat16, 128>(const DecodeArgs&, const DecodeMaps&, int, int,
                                           bool, int, cudaStream_t);
}  // namespace pkv
