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

// Cache write: CTA iteration j handles tokens j and j + gridDim.x (loads of
// both issued before their stores).  A token's key (and value) is per_token =
// Hkv x vpr 16-byte vectors, contiguous; thread t moves vector t (and t +
// blockDim.x, ...), i.e. head t >> vpr_shift, column t & (vpr - 1) of the row,
// into frame slot / B, offset slot mod B of that head's tile.
constexpr int kReshapeThreads = 128;

__global__ void __launch_bounds__(kReshapeThreads) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slots, int64_t num_tokens,
    int32_t num_kv_heads, int32_t vpr_shift, int32_t block_size, int64_t num_slots,
    unsigned int* err) {
  // A kernel queued behind this one with programmatic dependent launch (the
  // decode call's planning kernel) may become resident now; it waits for this
  // grid to complete before it goes on.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int32_t per_token = num_kv_heads << vpr_shift;
  const int32_t col_mask = (1 << vpr_shift) - 1;
  const int64_t stride = 2 * static_cast<int64_t>(gridDim.x);
  for (int64_t i0 = blockIdx.x; i0 < num_tokens; i0 += stride) {
    const int64_t i1 = i0 + gridDim.x;
    int64_t base[2] = {-1, -1};  // first destination vector of each token's tile row (-1: skip)
    const int64_t tok[2] = {i0, i1};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (tok[u] >= num_tokens) continue;
      const int64_t slot = __ldg(slots + tok[u]);
      if (slot < 0) continue;  // padding
      if (slot >= num_slots) {
        if (threadIdx.x == 0) set_error(err, PKV_DEVERR_SLOT);
        continue;
      }
      const int64_t frame = slot / block_size;
      const int64_t off = slot - frame * block_size;
      base[u] = (frame * num_kv_heads * block_size + off) << vpr_shift;
    }
    const int64_t head_stride = static_cast<int64_t>(block_size) << vpr_shift;
    for (int32_t t = threadIdx.x; t < per_token; t += kReshapeThreads) {
      const int64_t rel = (t >> vpr_shift) * head_stride + (t & col_mask);
      uint4 kv[2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (base[u] >= 0) {
          kv[u][0] = __ldg(key + tok[u] * per_token + t);
          kv[u][1] = __ldg(value + tok[u] * per_token + t);
        }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (base[u] >= 0) {
          k_cache[base[u] + rel] = kv[u][0];
          v_cache[base[u] + rel] = kv[u][1];
        }
    }
  }
}

// Block copy: item = (pair, cache), two per pair; each CTA takes whole items
// (grid-stride) and each thread keeps 4 vectors in flight.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                                   uint4* __restrict__ v_cache,
                                                                   const int64_t* __restrict__ pairs,
                                                                   int32_t num_pairs,
                                                                   int64_t vec_per_block,
                                                                   int32_t num_blocks,
                                                                   unsigned int* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // as in the cache write
  for (int64_t item = blockIdx.x; item < 2 * static_cast<int64_t>(num_pairs); item += gridDim.x) {
    const int64_t pair = item >> 1;
    const int64_t src = __ldg(pairs + 2 * pair);
    const int64_t dst = __ldg(pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if ((item & 1) == 0 && threadIdx.x == 0) set_error(err, PKV_DEVERR_COPY_PAIR);
      continue;
    }
    if (src == dst) continue;
    uint4* cache = (item & 1) == 0 ? k_cache : v_cache;
    const uint4* from = cache + src * vec_per_block;
    uint4* to = cache + dst * vec_per_block;
    for (int64_t b0 = threadIdx.x; b0 < vec_per_block; b0 += kCopyUnroll * kCopyThreads) {
      uint4 r[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = b0 + u * kCopyThreads;
        if (i < vec_per_block) r[u] = from[i];
      }
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = b0 + u * kCopyThreads;
        if (i < vec_per_block) to[i] = r[u];
      }
    }
  }
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slots, int32_t num_tokens,
                                     int32_t num_kv_heads, int32_t row_bytes, int32_t block_size,
                                     int32_t num_blocks, int num_sms, unsigned int* err,
                                     cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int32_t vec_per_row = row_bytes / 16;  // a power of two (head_dim 64 or 128: 8 or 16)
  int32_t shift = 0;
  while ((1 << shift) < vec_per_row) ++shift;
  if ((1 << shift) != vec_per_row) return cudaErrorInvalidValue;
  const int64_t want = (static_cast<int64_t>(num_tokens) + 1) / 2;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  reshape_and_cache_kernel<<<blocks, kReshapeThreads, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slots, num_tokens, num_kv_heads, shift, block_size,
      static_cast<int64_t>(num_blocks) * block_size, err);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs,
                               int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               int num_sms, unsigned int* err, cudaStream_t stream) {
  if (num_pairs == 0) return cudaSuccess;
  const int64_t vec_per_block = block_bytes / 16;
  const int64_t items = 2 * static_cast<int64_t>(num_pairs);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int blocks = static_cast<int>(items < cap ? items : cap);
  copy_blocks_kernel<<<blocks, kCopyThreads, 0, stream>>>(static_cast<uint4*>(k_cache),
                                                         static_cast<uint4*>(v_cache), pairs,
                                                         num_pairs, vec_per_block, num_blocks, err);
  return cudaGetLastError();
}

}  // namespace pkv
