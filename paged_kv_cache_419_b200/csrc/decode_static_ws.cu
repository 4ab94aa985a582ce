// Paged decode attention for callers that cannot allocate device memory.
//
// Some callers have no way to get scratch memory from cudaMalloc or a caching
// allocator at the point where they run decode: an engine that plans all of its
// device memory up front and forbids allocation afterwards, a plugin whose
// enqueue hook must not allocate, or code running where the allocator is owned
// by someone else.  pkv_paged_attention_decode_static serves them: its scratch
// (the per-partition partial results of long contexts) is one fixed array in
// the library's own device memory, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable of PKV_STATIC_WORKSPACE_BYTES.
// Every GPU that loads the library holds it until the process exits.  In host
// code its name is only a host-side stand-in, so its device address is looked up
// with cudaGetSymbolAddress once per device (with that device current) on the
// first call there, and that address is what the kernels receive.
#include <mutex>

#include "pkv.h"

static __device__ __align__(256) unsigned char g_static_scratch[PKV_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_static_scratch on the current device (set up once per device).
pkv_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ECUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return PKV_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PKV_OK;
}

}  // namespace

extern "C" pkv_status pkv_paged_attention_decode_static(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t max_blocks_per_seq, int32_t num_blocks, float scale, int32_t num_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, pkv_dtype dtype,
    int32_t partition_size, cudaStream_t stream) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0) return PKV_EINVAL;
  const int64_t max_ctx = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  if (max_ctx > (1 << 30)) return PKV_EUNSUPPORTED;
  const size_t need = pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
                                                 static_cast<int32_t>(max_ctx), partition_size);
  if (need > PKV_STATIC_WORKSPACE_BYTES) return PKV_EUNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    const pkv_status st = scratch_address(&scratch);
    if (st != PKV_OK) return st;
  }
  // Nothing in the scratch needs clearing: every call's planning kernel writes the
  // work list and zeroes the counters it uses, and the partition merge reads only
  // results written earlier in the same call.
  return pkv_paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                                    max_blocks_per_seq, num_blocks, scale, num_heads, num_kv_heads,
                                    head_dim, block_size, dtype, partition_size, scratch,
                                    need > 0 ? PKV_STATIC_WORKSPACE_BYTES : 0, stream);
}
