// Paged prefill attention: launch arguments and tile sizes (the kernel and its
// design are in prefill.cu).
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include <type_traits>

#include "device.cuh"

namespace pkv {

struct PrefillArgs {
  void* out;                  // [total_q, Hq, D]
  const int32_t* tables;      // [S, MB]
  const int32_t* query_start; // [S + 1]
  const int32_t* lens;        // [S]: p0 + T, context length after the chunk
  int32_t num_seqs;
  int32_t max_blocks;
  int32_t num_blocks;
  int32_t block_size;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t total_q;
  float scale_log2;
  unsigned int* err;
};

// Tensor maps: q viewed as [total_q][Hq][D] (box 64 x 1 x 128 rows), the caches
// as [N][Hkv * B][D] (box 64 x B x 1), all with the 128-byte swizzle.
struct PrefillMaps {
  CUtensorMap q, k, v;
};

constexpr int kPrefillThreads = 576;  // TMA, MMA, 2 x 8 softmax warps
constexpr int kPrefillTileM = 128;  // query rows per CTA
constexpr int kPrefillTileN = 128;  // keys per tile
constexpr int kPrefillStages = 2;
constexpr uint32_t kPrefillTmemCols = 512;

template <int D>
struct PrefillTraits {
  static constexpr int ND = D / 64;                       // 128-byte panels per row
  static constexpr int PANEL = kPrefillTileM * 128;       // one panel of 128 rows
  static constexpr int TILE = ND * PANEL;                 // Q, K or V tile
  static constexpr int OFF_Q = 0;                         // two query tiles
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + kPrefillStages * TILE;
  static constexpr int OFF_RED = OFF_V + kPrefillStages * TILE;  // [2 tiles][2 halves][128] maxima, then sums
  static constexpr int OFF_BAR = OFF_RED + 8 * kPrefillTileM * 4;
  // q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], s_full[2], p_full[2][2] (per query
  // tile and chunk of P), pv_done[2], o_final
  static constexpr int NUM_BARS = 1 + 4 * kPrefillStages + 8 + 1;
  static constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_USED = OFF_TMEM + 16;
  // SMEM_USED + 1024 bytes of slack for the 1024-byte aligned base, and never
  // less than 117 KB: two CTAs never share an SM, so the second never waits in
  // tcgen05.alloc for the first one's 512 tensor-memory columns.
  static constexpr int SMEM_BYTES = SMEM_USED + 1024 > 117 * 1024 ? SMEM_USED + 1024 : 117 * 1024;
  // tensor memory: query tile t has its scores at colS(t) (128 columns; P of
  // keys 64 h .. 64 h + 63 over columns 64 h .. 64 h + 31 of them) and its
  // output accumulator at colO(t) (D columns)
  static constexpr uint32_t colS(int t) { return 256u * static_cast<uint32_t>(t); }
  static constexpr uint32_t colO(int t) { return 256u * static_cast<uint32_t>(t) + 128u; }
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Launch of the prefill grid (instantiated in prefill.cu for fp16 / bf16 and
// head_dim 64 / 128): per sequence, one CTA per pair of 128-row query tiles
// (two heads of a kv group on the same rows when Hq / Hkv is even, else two
// consecutive row tiles of one head).
template <typename T, int D>
cudaError_t launch_prefill(const PrefillArgs& a, const PrefillMaps& m, int max_query_len,
                           cudaStream_t stream);

}  // namespace pkv
