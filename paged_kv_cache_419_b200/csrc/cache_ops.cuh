// Host launchers of the cache-write and block-copy kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slots, int32_t num_tokens,
                                     int32_t num_kv_heads, int32_t row_bytes, int32_t block_size,
                                     int32_t num_blocks, int num_sms, unsigned int* err,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                               int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               int num_sms, unsigned int* err, cudaStream_t stream);

}  // namespace pkv
