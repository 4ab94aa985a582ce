// Host launchers for the decode kernels; included by one file per (dtype, head_dim).
#pragma once

#include <atomic>

#include "decode.cuh"

namespace pkv {

// Persistent grid size of one decode instantiation on the current device:
// SM count x resident CTAs per SM (set up once per device).
// Two host threads making their first call at once may both run the set-up; it
// is idempotent and the atomic store publishes the same value.
template <typename T, int D, int G, int B, bool PAGED>
cudaError_t decode_grid(int num_sms, int* grid) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  static std::atomic<int> blocks_per_sm[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int per_sm = blocks_per_sm[dev].load(std::memory_order_acquire);
  if (per_sm == 0) {
    auto kern = decode_kernel<T, D, G, B, PAGED>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kDecodeThreads, Tr::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    per_sm = n > 0 ? n : 1;
    blocks_per_sm[dev].store(per_sm, std::memory_order_release);
  }
  *grid = num_sms * per_sm;
  return cudaSuccess;
}

// Launch of the merge grid behind the decode grid (programmatic dependent
// launch): at most one wave (the CTAs one SM holds of this instantiation, times
// the SMs), so that no merge CTA waits for a slot behind one that is parked at
// its final grid wait.
template <typename T, int D, int G, int NREG>
cudaError_t launch_merge(const DecodeArgs& a, int num_sms, cudaStream_t stream) {
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, merge_kernel<T, D, G, NREG>, kMergeThreads, 0) !=
            cudaSuccess ||
        n < 1) {
      (void)cudaGetLastError();
      n = 1;
    }
    return n;
  }();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int64_t pairs = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads;
  const int64_t want = static_cast<int64_t>(num_sms) * per_sm;
  cfg.gridDim = dim3(static_cast<unsigned>(pairs < want ? pairs : want));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, merge_kernel<T, D, G, NREG>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D, int G, int B, bool PAGED>
cudaError_t launch_decode_one(const DecodeArgs& args, const DecodeMaps& maps, int num_sms,
                              cudaStream_t stream) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  int grid = 0;
  cudaError_t e = decode_grid<T, D, G, B, PAGED>(num_sms, &grid);
  if (e != cudaSuccess) return e;
  DecodeArgs a = args;
  apply_partition_policy(a, grid, B, PAGED);
  // All three grids use programmatic dependent launch: each may become resident
  // while its predecessor runs.  The plan waits in-kernel for its predecessor
  // (whatever the caller queued before the call) to complete before it lets the
  // decode grid launch, so the kernels behind it may read their inputs as soon
  // as they start; decode and merge wait in-kernel for their predecessors before
  // touching anything those write.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, plan_kernel, a);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = Tr::SMEM_BYTES;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<T, D, G, B, PAGED>, a, maps);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess || a.max_parts <= 1) return e;
  // Partition merge, also behind its predecessor: its CTAs become resident as
  // decode CTAs retire and merge each pair once the decode grid has published
  // it.
  constexpr int slices = kMergeThreads / (G * D / 4);
  const int need = (a.max_parts + slices - 1) / slices;  // partials per thread for one load round
  if (need <= 2) return launch_merge<T, D, G, 2>(a, num_sms, stream);
  if (need <= 4) return launch_merge<T, D, G, 4>(a, num_sms, stream);
  if (need <= 8) return launch_merge<T, D, G, 8>(a, num_sms, stream);
  return launch_merge<T, D, G, kMergeMaxRegs>(a, num_sms, stream);
}


template <typename T, int D, int B, bool PAGED>
cudaError_t launch_decode_group(const DecodeArgs& a, const DecodeMaps& m, int group, int num_sms,
                               cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode_one<T, D, 1, B, PAGED>(a, m, num_sms, stream);
    case 2: return launch_decode_one<T, D, 2, B, PAGED>(a, m, num_sms, stream);
    case 4: return launch_decode_one<T, D, 4, B, PAGED>(a, m, num_sms, stream);
    case 8: return launch_decode_one<T, D, 8, B, PAGED>(a, m, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, int group, int block_size,
                          bool paged, int num_sms, cudaStream_t stream) {
  if (!paged) return launch_decode_group<T, D, 32, false>(a, m, group, num_sms, stream);
  switch (block_size) {
    case 8: return launch_decode_group<T, D, 8, true>(a, m, group, num_sms, stream);
    case 16: return launch_decode_group<T, D, 16, true>(a, m, group, num_sms, stream);
    case 32: return launch_decode_group<T, D, 32, true>(a, m, group, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pkv
