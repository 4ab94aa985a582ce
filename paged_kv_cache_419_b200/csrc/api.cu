// C ABI entry points (include/pkv.h): argument checks on the host, then launch.
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "cache_ops.cuh"
#include "decode.cuh"
#include "pkv.h"
#include "prefill.cuh"

namespace pkv {

// Sticky error flags of the kernels on each device (PKV_DEVERR_*).
static __device__ unsigned int g_device_error;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDefaultPartition = 1024;
constexpr int kBalancedMinPartition = 512;

struct DeviceInfo {
  bool ready = false;
  unsigned int* err = nullptr;  // device address of g_device_error
  int num_sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mutex;

// Bounded-wait test hook (pkv_test_set_merge_wait): 0 = the normal bound.
std::atomic<unsigned long long> g_merge_wait_limit_ns{0};
std::atomic<uint32_t> g_merge_wait_extra{0};

// The error of the last CUDA call that made a pkv_* call of this host thread
// return PKV_ECUDA (pkv_last_cuda_error).
thread_local int g_last_cuda_error = 0;

// Records why a call returns PKV_ECUDA: the runtime's pending error of this
// thread (taken, so that it is not blamed on a later launch), else `fallback`.
pkv_status cuda_fail(cudaError_t fallback = cudaErrorUnknown) {
  cudaError_t e = cudaGetLastError();
  g_last_cuda_error = static_cast<int>(e != cudaSuccess ? e : fallback);
  return PKV_ECUDA;
}

pkv_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return PKV_OK;
  g_last_cuda_error = static_cast<int>(e);
  return PKV_ECUDA;
}

// Per-device set-up with that device current: the device address of the error
// flag and the SM count (under a lock: host threads may make their first call
// on a device at the same time).
pkv_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail();
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(g_devices_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return cuda_fail();
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cuda_fail();
    d.err = static_cast<unsigned int*>(p);
    d.num_sms = sms;
    d.ready = true;
  }
  *out = &d;
  return PKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool validate_env() {
  const char* v = getenv("PKV_VALIDATE");
  return v && v[0] && strcmp(v, "0") != 0;
}



bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

int resolve_partition(int32_t partition_size) {
  return partition_size == 0 ? kDefaultPartition : partition_size;
}

// Partition size that bounds the workspace: the requested one, or for the
// default (0) the smallest size the per-call balanced policy picks when a
// context spans several partitions.
int workspace_partition(int32_t partition_size) {
  return partition_size == 0 ? kBalancedMinPartition : partition_size;
}

bool valid_partition(int p) { return p >= kStageTokens && p <= kMaxPartTokens && p % kStageTokens == 0; }

// The partition arguments of a call (a.max_ctx set): the size, whether the
// default size may become the balanced policy at launch, and the workspace's
// partitions per context.  False for an unsupported partition_size.
bool set_partition_args(DecodeArgs& a, int32_t partition_size) {
  const int part = resolve_partition(partition_size);
  if (!valid_partition(part)) return false;
  const int ws_part = workspace_partition(partition_size);
  a.part_tokens = part;
  // default size: the launcher switches to the balanced policy when the batch
  // has fewer (sequence, kv head) pairs than decode CTAs
  a.balanced = partition_size == 0 ? 1 : 0;
  a.max_parts = (a.max_ctx + ws_part - 1) / ws_part;
  if (a.max_parts < 1) a.max_parts = 1;
  return true;
}

int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

// Workspace layout: [work counters | list of multi-partition sequences (S) |
// published partitions per (sequence, kv head) (S x Hkv <= S x Hq) | work
// records (S x P) | partition results (only when P > 1)].
struct WorkspaceLayout {
  int64_t counters, merge, done, records, tmp, total;
};

WorkspaceLayout workspace_layout(int64_t S, int64_t Hq, int64_t D, int64_t max_ctx, int64_t part) {
  int64_t P = (max_ctx + part - 1) / part;
  if (P < 1) P = 1;
  WorkspaceLayout w;
  w.counters = 0;
  w.merge = 256;
  w.done = w.merge + round256(4 * S);
  w.records = w.done + round256(4 * S * Hq);
  w.tmp = w.records + round256(S * P * kRecordBytes);
  w.total = w.tmp + (P > 1 ? round256(S * Hq * P * (D + 2) * 4) : 0);
  return w;
}

size_t workspace_bytes(int64_t S, int64_t Hq, int64_t D, int64_t max_ctx, int64_t part) {
  return static_cast<size_t>(workspace_layout(S, Hq, D, max_ctx, part).total);
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link against
// the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Map of a cache viewed as [planes][rows][head_dim] 16-bit elements: boxes of
// one 128-byte panel x box_rows rows x 1 plane, 128-byte swizzle, zero fill
// outside the tensor, 256-byte L2 promotion (a box reads half of each
// 256-byte row; the other half is the next box).
pkv_status encode_cache_map(CUtensorMap* m, const void* base, pkv_dtype dtype, int head_dim,
                            int64_t rows, int64_t planes, int box_rows) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim),
                              static_cast<cuuint64_t>(rows > 0 ? rows : 1),
                              static_cast<cuuint64_t>(planes > 0 ? planes : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(dims[1]) * head_dim * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t elem_strides[3] = {1u, 1u, 1u};
  const CUresult r =
      fn(m, dtype == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
         const_cast<void*>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_EINVAL;
}

// The four maps of one call (full-chunk and 8-row boxes of K and V).
pkv_status encode_decode_maps(DecodeMaps* m, const DecodeArgs& a, pkv_dtype dtype, int head_dim,
                              int block_size, bool paged) {
  const int64_t rows = paged ? static_cast<int64_t>(a.num_kv_heads) * block_size : a.max_ctx;
  const int64_t planes =
      paged ? a.num_blocks : static_cast<int64_t>(a.num_seqs) * a.num_kv_heads;
  const int ch = chunk_rows(paged, block_size);
  pkv_status st;
  if ((st = encode_cache_map(&m->k, a.k, dtype, head_dim, rows, planes, ch)) != PKV_OK) return st;
  if ((st = encode_cache_map(&m->v, a.v, dtype, head_dim, rows, planes, ch)) != PKV_OK) return st;
  if ((st = encode_cache_map(&m->k_tail, a.k, dtype, head_dim, rows, planes, 8)) != PKV_OK) return st;
  return encode_cache_map(&m->v_tail, a.v, dtype, head_dim, rows, planes, 8);
}

// Shared checks and launch of the paged and contiguous decode.
pkv_status decode_common(DecodeArgs& a, int32_t head_dim, int32_t block_size, pkv_dtype dtype,
                         int32_t partition_size, void* workspace, size_t ws_bytes, bool paged,
                         float scale, cudaStream_t stream) {
  if (a.num_seqs == 0) return PKV_OK;
  if (!set_partition_args(a, partition_size)) return PKV_EINVAL;
  const int ws_part = workspace_partition(partition_size);
  const int group = a.num_heads / a.num_kv_heads;
  const WorkspaceLayout lay = workspace_layout(a.num_seqs, a.num_heads, head_dim, a.max_ctx, ws_part);
  if (!workspace || ws_bytes < static_cast<size_t>(lay.total) || !aligned16(workspace))
    return PKV_EINVAL;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.work = reinterpret_cast<uint32_t*>(ws + lay.counters);
  a.merge_seqs = reinterpret_cast<int32_t*>(ws + lay.merge);
  a.pair_done = reinterpret_cast<uint32_t*>(ws + lay.done);
  a.records = ws + lay.records;
  a.block_size = block_size;
  if (a.max_parts > 1) {
    const int64_t cells = static_cast<int64_t>(a.num_seqs) * a.num_heads * a.max_parts;
    a.tmp_out = reinterpret_cast<float*>(ws + lay.tmp);
    a.tmp_m = a.tmp_out + cells * head_dim;
    a.tmp_l = a.tmp_m + cells;
  } else {
    a.tmp_out = a.tmp_m = a.tmp_l = nullptr;
  }
  a.scale_log2 = scale * 1.4426950408889634f;
  const unsigned long long hook_ns = g_merge_wait_limit_ns.load(std::memory_order_relaxed);
  a.merge_wait_limit_ns = hook_ns ? hook_ns : kWaitLimitNs;
  a.merge_wait_extra = g_merge_wait_extra.load(std::memory_order_relaxed);
  DeviceInfo* dev = nullptr;
  pkv_status st = device_info(&dev);
  if (st != PKV_OK) return st;
  a.err = dev->err;
  const int sms = dev->num_sms;
  DecodeMaps maps;
  st = encode_decode_maps(&maps, a, dtype, head_dim, block_size, paged);
  if (st != PKV_OK) return st;
  cudaError_t e;
  if (dtype == PKV_F16)
    e = head_dim == 64 ? launch_decode<__half, 64>(a, maps, group, block_size, paged, sms, stream)
                       : launch_decode<__half, 128>(a, maps, group, block_size, paged, sms, stream);
  else
    e = head_dim == 64
            ? launch_decode<__nv_bfloat16, 64>(a, maps, group, block_size, paged, sms, stream)
            : launch_decode<__nv_bfloat16, 128>(a, maps, group, block_size, paged, sms, stream);
  return from_cuda(e);
}

pkv_status check_heads(int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, pkv_dtype dtype) {
  if (num_heads <= 0 || num_kv_heads <= 0) return PKV_EINVAL;
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EUNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PKV_EUNSUPPORTED;
  if (num_heads % num_kv_heads != 0 || !supported_group(num_heads / num_kv_heads))
    return PKV_EUNSUPPORTED;
  return PKV_OK;
}

// PKV_VALIDATE=1: copy the tables and lengths back and check every entry the
// kernel would read.
pkv_status validate_decode_tables(const int32_t* tables, const int32_t* lens, int32_t S,
                                  int32_t MB, int32_t N, int32_t B, cudaStream_t stream) {
  std::vector<int32_t> h_lens(S), h_tab(static_cast<size_t>(S) * MB);
  if (cudaMemcpyAsync(h_lens.data(), lens, sizeof(int32_t) * S, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(h_tab.data(), tables, sizeof(int32_t) * h_tab.size(), cudaMemcpyDeviceToHost,
                      stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return cuda_fail();
  for (int32_t s = 0; s < S; ++s) {
    const int64_t L = h_lens[s];
    if (L < 0 || L > static_cast<int64_t>(MB) * B) return PKV_ERANGE;
    for (int64_t j = 0; j < (L + B - 1) / B; ++j) {
      const int32_t p = h_tab[static_cast<size_t>(s) * MB + j];
      if (p < 0 || p >= N) return PKV_ERANGE;
    }
  }
  return PKV_OK;
}

// PKV_VALIDATE=1 check of a copy list (host copy): every frame in range, and the
// pairs independent of their order (all run concurrently): distinct
// destinations, and no destination that is also the source of another pair.
pkv_status validate_copy_pairs(const int64_t* pairs, int32_t n, int32_t num_blocks) {
  std::vector<uint8_t> role(static_cast<size_t>(num_blocks), 0);  // bit 0: source, bit 1: destination
  for (int32_t i = 0; i < n; ++i) {
    const int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return PKV_ERANGE;
  }
  for (int32_t i = 0; i < n; ++i) {
    const int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src == dst) continue;  // no-op pair
    role[static_cast<size_t>(src)] |= 1u;
    if (role[static_cast<size_t>(dst)] & 2u) return PKV_EINVAL;  // two pairs write one frame
    role[static_cast<size_t>(dst)] |= 2u;
  }
  for (int32_t i = 0; i < n; ++i) {
    const int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src != dst && (role[static_cast<size_t>(dst)] & 1u)) return PKV_EINVAL;  // read and written
  }
  return PKV_OK;
}

// Map of q viewed as [total_q][Hq][head_dim] 16-bit elements: boxes of one
// 128-byte panel x 1 head x 128 query rows, 128-byte swizzle (the K-major
// layout the tensor cores read), zero fill past the last row.
pkv_status encode_query_map(CUtensorMap* m, const void* q, pkv_dtype dtype, int head_dim,
                            int64_t num_heads, int64_t total_q) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_heads),
                              static_cast<cuuint64_t>(total_q > 0 ? total_q : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                 static_cast<cuuint64_t>(num_heads) * head_dim * 2};
  const cuuint32_t box[3] = {64u, 1u, static_cast<cuuint32_t>(kPrefillTileM)};
  const cuuint32_t elem_strides[3] = {1u, 1u, 1u};
  const CUresult r =
      fn(m, dtype == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
         const_cast<void*>(q), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_EINVAL;
}

// PKV_VALIDATE=1 check of a prefill batch (host copies of the query offsets,
// context lengths and block tables).
pkv_status validate_prefill(const int32_t* query_start, const int32_t* lens, const int32_t* tables,
                            int32_t S, int32_t max_query_len, int32_t total_q, int32_t MB,
                            int32_t N, int32_t B, cudaStream_t stream) {
  std::vector<int32_t> qs(static_cast<size_t>(S) + 1), h_lens(S), h_tab(static_cast<size_t>(S) * MB);
  if (cudaMemcpyAsync(qs.data(), query_start, sizeof(int32_t) * qs.size(), cudaMemcpyDeviceToHost,
                      stream) != cudaSuccess ||
      cudaMemcpyAsync(h_lens.data(), lens, sizeof(int32_t) * S, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(h_tab.data(), tables, sizeof(int32_t) * h_tab.size(), cudaMemcpyDeviceToHost,
                      stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return cuda_fail();
  for (int32_t s = 0; s < S; ++s) {
    const int64_t T = static_cast<int64_t>(qs[s + 1]) - qs[s];
    const int64_t L = h_lens[s];
    if (qs[s] < 0 || T < 0 || qs[s + 1] > total_q || T > max_query_len) return PKV_ERANGE;
    if (L < T || L > static_cast<int64_t>(MB) * B) return PKV_ERANGE;
    for (int64_t j = 0; j < (L + B - 1) / B; ++j) {
      const int32_t p = h_tab[static_cast<size_t>(s) * MB + j];
      if (p < 0 || p >= N) return PKV_ERANGE;
    }
  }
  return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(pkv_status status) {
  switch (status) {
    case PKV_OK: return "PKV_OK";
    case PKV_EINVAL: return "PKV_EINVAL: invalid argument";
    case PKV_EUNSUPPORTED: return "PKV_EUNSUPPORTED: unsupported shape or dtype";
    case PKV_ECUDA: return "PKV_ECUDA: CUDA runtime error";
    case PKV_ENOMEM: return "PKV_ENOMEM: block pool exhausted";
    case PKV_ERANGE: return "PKV_ERANGE: index out of range";
  }
  return "unknown pkv_status";
}

int pkv_last_cuda_error(void) { return g_last_cuda_error; }

const char* pkv_cuda_error_name(int error) {
  return cudaGetErrorName(static_cast<cudaError_t>(error));
}

pkv_status pkv_device_error(unsigned int* flags_out, int clear, cudaStream_t stream) {
  if (!flags_out) return PKV_EINVAL;
  DeviceInfo* dev = nullptr;
  pkv_status st = device_info(&dev);
  if (st != PKV_OK) return st;
  unsigned int h = 0;
  if (cudaMemcpyAsync(&h, dev->err, sizeof h, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return cuda_fail();
  if (clear && cudaMemsetAsync(dev->err, 0, sizeof h, stream) != cudaSuccess) return cuda_fail();
  if (cudaStreamSynchronize(stream) != cudaSuccess) return cuda_fail();
  *flags_out = h;
  return PKV_OK;
}

pkv_status pkv_test_set_merge_wait(uint64_t limit_ns, uint32_t extra) {
  g_merge_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  g_merge_wait_extra.store(extra, std::memory_order_relaxed);
  return PKV_OK;
}

pkv_status pkv_test_partitions(const int32_t* context_lens, int32_t num_seqs, int32_t num_kv_heads,
                               int32_t max_context_len, int32_t block_size, int32_t partition_size,
                               int32_t grid_ctas, int32_t* n_parts, int32_t* n_big, int32_t* p_big,
                               int32_t* p_small) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_context_len < 0 || grid_ctas <= 0 ||
      (block_size != 8 && block_size != 16 && block_size != 32))
    return PKV_EINVAL;
  if (num_seqs == 0) return PKV_OK;
  if (!context_lens || !n_parts || !n_big || !p_big || !p_small) return PKV_EINVAL;
  DecodeArgs a = {};
  a.num_seqs = num_seqs;
  a.num_kv_heads = num_kv_heads;
  a.max_ctx = max_context_len;
  if (!set_partition_args(a, partition_size)) return PKV_EINVAL;
  apply_partition_policy(a, grid_ctas, block_size, true);
  unsigned long long U = 0;  // the batch's token-heads, as the kernels sum them
  for (int32_t s = 0; s < num_seqs; ++s)
    U += static_cast<unsigned long long>(clamp_len(context_lens[s], a.max_ctx));
  U *= static_cast<unsigned long long>(num_kv_heads);
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int L = clamp_len(context_lens[s], a.max_ctx);
    int n = 0, nb = 0, pb = 0, ps = 0;
    if (round_robin(a)) {
      partition_rr(L, a, U, nb, n, pb, ps);
    } else {
      partition_for(L, a, U, n, pb);
      nb = n;
      ps = pb;
    }
    n_parts[s] = n;
    n_big[s] = nb;
    p_big[s] = pb;
    p_small[s] = ps;
  }
  return PKV_OK;
}

size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                  int32_t max_context_len, int32_t partition_size) {
  const int part = resolve_partition(partition_size);
  if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      !valid_partition(part))
    return 0;
  return workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                         workspace_partition(partition_size));
}

pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* context_lens, int32_t num_seqs,
                                      int32_t max_blocks_per_seq, int32_t num_blocks, float scale,
                                      int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, pkv_dtype dtype, int32_t partition_size,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return PKV_EINVAL;
  pkv_status st = check_heads(num_heads, num_kv_heads, head_dim, dtype);
  if (st != PKV_OK) return st;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_EUNSUPPORTED;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_EINVAL;
  const int64_t max_ctx = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  if (max_ctx > (1 << 30)) return PKV_EUNSUPPORTED;
  if (validate_env()) {
    st = validate_decode_tables(block_tables, context_lens, num_seqs, max_blocks_per_seq,
                                num_blocks, block_size, stream);
    if (st != PKV_OK) return st;
  }
  DecodeArgs a{};
  a.out = out;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.tables = block_tables;
  a.lens = context_lens;
  a.num_seqs = num_seqs;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.max_ctx = static_cast<int32_t>(max_ctx);
  return decode_common(a, head_dim, block_size, dtype, partition_size, workspace, workspace_bytes,
                       true, scale, stream);
}

pkv_status pkv_contiguous_attention_decode(void* out, const void* q, const void* k, const void* v,
                                           const int32_t* context_lens, int32_t num_seqs,
                                           int32_t max_context_len, float scale, int32_t num_heads,
                                           int32_t num_kv_heads, int32_t head_dim, pkv_dtype dtype,
                                           int32_t partition_size, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream) {
  if (num_seqs < 0 || max_context_len < 0) return PKV_EINVAL;
  pkv_status st = check_heads(num_heads, num_kv_heads, head_dim, dtype);
  if (st != PKV_OK) return st;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !k || !v || !context_lens) return PKV_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return PKV_EINVAL;
  if (max_context_len > (1 << 30)) return PKV_EUNSUPPORTED;
  if (validate_env()) {
    std::vector<int32_t> h(num_seqs);
    if (cudaMemcpyAsync(h.data(), context_lens, sizeof(int32_t) * num_seqs,
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return cuda_fail();
    for (int32_t L : h)
      if (L < 0 || L > max_context_len) return PKV_ERANGE;
  }
  DecodeArgs a{};
  a.out = out;
  a.q = q;
  a.k = k;
  a.v = v;
  a.lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.max_ctx = max_context_len;
  return decode_common(a, head_dim, 32, dtype, partition_size, workspace, workspace_bytes, false,
                       scale, stream);
}

pkv_status pkv_paged_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* query_start,
                             const int32_t* context_lens, int32_t num_seqs, int32_t max_query_len,
                             int32_t total_query_tokens, int32_t max_blocks_per_seq,
                             int32_t num_blocks, float scale, int32_t num_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                             pkv_dtype dtype, cudaStream_t stream) {
  if (num_seqs < 0 || max_query_len < 0 || total_query_tokens < 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0 || num_heads <= 0 || num_kv_heads <= 0)
    return PKV_EINVAL;
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EUNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PKV_EUNSUPPORTED;
  if (num_heads % num_kv_heads != 0) return PKV_EUNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_EUNSUPPORTED;
  if (num_seqs > 65535 || num_heads > 65535) return PKV_EUNSUPPORTED;
  if (static_cast<int64_t>(max_blocks_per_seq) * block_size > (1 << 30)) return PKV_EUNSUPPORTED;
  if (num_seqs == 0 || max_query_len == 0 || total_query_tokens == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !query_start || !context_lens)
    return PKV_EINVAL;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_EINVAL;
  if (validate_env()) {
    const pkv_status vs = validate_prefill(query_start, context_lens, block_tables, num_seqs,
                                           max_query_len, total_query_tokens, max_blocks_per_seq,
                                           num_blocks, block_size, stream);
    if (vs != PKV_OK) return vs;
  }
  DeviceInfo* dev = nullptr;
  pkv_status st = device_info(&dev);
  if (st != PKV_OK) return st;
  PrefillArgs a{};
  a.out = out;
  a.tables = block_tables;
  a.query_start = query_start;
  a.lens = context_lens;
  a.num_seqs = num_seqs;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.block_size = block_size;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.total_q = total_query_tokens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.err = dev->err;
  PrefillMaps maps;
  if ((st = encode_query_map(&maps.q, q, dtype, head_dim, num_heads, total_query_tokens)) != PKV_OK)
    return st;
  const int64_t rows = static_cast<int64_t>(num_kv_heads) * block_size;
  if ((st = encode_cache_map(&maps.k, k_cache, dtype, head_dim, rows, num_blocks, block_size)) != PKV_OK)
    return st;
  if ((st = encode_cache_map(&maps.v, v_cache, dtype, head_dim, rows, num_blocks, block_size)) != PKV_OK)
    return st;
  cudaError_t e;
  if (dtype == PKV_F16)
    e = head_dim == 64 ? launch_prefill<__half, 64>(a, maps, max_query_len, stream)
                       : launch_prefill<__half, 128>(a, maps, max_query_len, stream);
  else
    e = head_dim == 64 ? launch_prefill<__nv_bfloat16, 64>(a, maps, max_query_len, stream)
                       : launch_prefill<__nv_bfloat16, 128>(a, maps, max_query_len, stream);
  return from_cuda(e);
}

pkv_status pkv_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                                 const int64_t* slot_mapping, int32_t num_tokens,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t num_blocks, pkv_dtype dtype, cudaStream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return PKV_EINVAL;
  if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_EUNSUPPORTED;
  const int32_t row_bytes = head_dim * 2;
  // rows move as 16-byte vectors, a power of two of them per row
  if (row_bytes % 16 != 0 || ((row_bytes / 16) & (row_bytes / 16 - 1)) != 0) return PKV_EUNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_EINVAL;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_EINVAL;
  if (validate_env()) {
    std::vector<int64_t> h(num_tokens);
    if (cudaMemcpyAsync(h.data(), slot_mapping, sizeof(int64_t) * num_tokens,
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return cuda_fail();
    for (int64_t s : h)
      if (s >= static_cast<int64_t>(num_blocks) * block_size) return PKV_ERANGE;
  }
  DeviceInfo* dev = nullptr;
  pkv_status st = device_info(&dev);
  if (st != PKV_OK) return st;
  return from_cuda(launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                            num_kv_heads, row_bytes, block_size, num_blocks,
                                            dev->num_sms, dev->err, stream));
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs,
                           int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                           cudaStream_t stream) {
  if (num_pairs < 0 || block_bytes <= 0 || num_blocks <= 0) return PKV_EINVAL;
  if (block_bytes % 16 != 0) return PKV_EINVAL;
  if (num_pairs > 65535) return PKV_EUNSUPPORTED;
  if (num_pairs == 0) return PKV_OK;
  if (!k_cache || !v_cache || !src_dst_pairs) return PKV_EINVAL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_EINVAL;
  if (validate_env()) {
    std::vector<int64_t> h(2 * static_cast<size_t>(num_pairs));
    if (cudaMemcpyAsync(h.data(), src_dst_pairs, sizeof(int64_t) * h.size(), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return cuda_fail();
    const pkv_status vs = validate_copy_pairs(h.data(), num_pairs, num_blocks);
    if (vs != PKV_OK) return vs;
  }
  DeviceInfo* dev = nullptr;
  pkv_status st = device_info(&dev);
  if (st != PKV_OK) return st;
  return from_cuda(launch_copy_blocks(k_cache, v_cache, src_dst_pairs, num_pairs, block_bytes,
                                      num_blocks, dev->num_sms, dev->err, stream));
}

}  // extern "C"
