// Cache write (reshape_and_cache) and copy-on-write block copy for sm_100a.
//
// Both are pure byte movement and are bound by HBM; each thread moves 16-byte
// vectors, consecutive threads touch consecutive vectors (coalesced), and the
// grids are sized in multiples of the SM count.
//
// Cache write: vLLM and PagedAttention slide 11 ("New block only when the last
// fills"): a new token's key and value go into the slot the allocator reserved,
// frame slot / B, offset slot mod B; a negative slot is padding.
// Block copy: slide 13 and the dataarena note section 3.2: a branch about to
// write into a shared, partially filled block first gets a private copy of it.
#include "cache_ops.cuh"
#include "device.cuh"

namespace pkv {

// One 16-byte vector per thread per iteration.  Vector index v enumerates
// (token, kv head, column) with the column fastest, so a warp covers whole rows.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slots, int64_t num_vectors,
    int32_t num_kv_heads, int32_t vec_per_row, int32_t block_size, int64_t num_slots,
    unsigned int* err) {
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * vec_per_row;
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < num_vectors;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = v / per_token;
    const int64_t rem = v - i * per_token;  // = head * vec_per_row + column
    const int64_t slot = __ldg(slots + i);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (rem == 0) set_error(err, PKV_DEVERR_SLOT);
      continue;
    }
    const int64_t frame = slot / block_size;
    const int64_t off = slot - frame * block_size;
    const int64_t head = rem / vec_per_row;
    const int64_t col = rem - head * vec_per_row;
    const int64_t dst = ((frame * num_kv_heads + head) * block_size + off) * vec_per_row + col;
    k_cache[dst] = __ldg(key + v);
    v_cache[dst] = __ldg(value + v);
  }
}

// grid.y = pair, grid.z = 0 (K) / 1 (V); grid.x strides over the frame's vectors.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                          uint4* __restrict__ v_cache,
                                                          const int64_t* __restrict__ pairs,
                                                          int64_t vec_per_block, int32_t num_blocks,
                                                          unsigned int* err) {
  const int pair = blockIdx.y;
  const int64_t src = __ldg(pairs + 2 * pair);
  const int64_t dst = __ldg(pairs + 2 * pair + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) set_error(err, PKV_DEVERR_COPY_PAIR);
    return;
  }
  if (src == dst) return;
  uint4* cache = blockIdx.z == 0 ? k_cache : v_cache;
  const uint4* from = cache + src * vec_per_block;
  uint4* to = cache + dst * vec_per_block;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < vec_per_block;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    to[i] = from[i];
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slots, int32_t num_tokens,
                                     int32_t num_kv_heads, int32_t row_bytes, int32_t block_size,
                                     int32_t num_blocks, int num_sms, unsigned int* err,
                                     cudaStream_t stream) {
  const int32_t vec_per_row = row_bytes / 16;
  const int64_t num_vectors = static_cast<int64_t>(num_tokens) * num_kv_heads * vec_per_row;
  if (num_vectors == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (num_vectors + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  reshape_and_cache_kernel<<<blocks, threads, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slots, num_vectors, num_kv_heads, vec_per_row, block_size,
      static_cast<int64_t>(num_blocks) * block_size, err);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                               int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               unsigned int* err, cudaStream_t stream) {
  if (num_pairs == 0) return cudaSuccess;
  const int64_t vec_per_block = block_bytes / 16;
  const int threads = 256;
  int64_t xblocks = (vec_per_block + threads - 1) / threads;
  if (xblocks > 64) xblocks = 64;
  const dim3 grid(static_cast<unsigned>(xblocks), static_cast<unsigned>(num_pairs), 2);
  copy_blocks_kernel<<<grid, threads, 0, stream>>>(static_cast<uint4*>(k_cache),
                                                   static_cast<uint4*>(v_cache), pairs,
                                                   vec_per_block, num_blocks, err);
  return cudaGetLastError();
}

}  // namespace pkv
