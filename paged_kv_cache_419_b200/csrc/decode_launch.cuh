// Host launchers for the decode kernels; included by one file per (dtype, head_dim).
#pragma once

#include "decode.cuh"

namespace pkv {

template <typename T, int D, int G, int B, bool PAGED>
cudaError_t launch_decode_one(const DecodeArgs& a, cudaStream_t stream) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  auto kern = decode_kernel<T, D, G, B, PAGED>;
  // The opt-in shared-memory size is a per-device function attribute; set it
  // once per device.
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const dim3 grid(a.max_parts, a.num_kv_heads, a.num_seqs);
  kern<<<grid, kDecodeThreads, Tr::SMEM_BYTES, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.max_parts > 1) {
    merge_partitions_kernel<T, D><<<dim3(a.num_heads, a.num_seqs), D, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

template <typename T, int D, int B, bool PAGED>
cudaError_t launch_decode_group(const DecodeArgs& a, int group, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode_one<T, D, 1, B, PAGED>(a, stream);
    case 2: return launch_decode_one<T, D, 2, B, PAGED>(a, stream);
    case 4: return launch_decode_one<T, D, 4, B, PAGED>(a, stream);
    case 8: return launch_decode_one<T, D, 8, B, PAGED>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
cudaError_t launch_decode(const DecodeArgs& a, int group, int block_size, bool paged,
                          cudaStream_t stream) {
  if (!paged) return launch_decode_group<T, D, 32, false>(a, group, stream);
  switch (block_size) {
    case 8: return launch_decode_group<T, D, 8, true>(a, group, stream);
    case 16: return launch_decode_group<T, D, 16, true>(a, group, stream);
    case 32: return launch_decode_group<T, D, 32, true>(a, group, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pkv
