// Paged decode attention for sm_100a.
//
// Method (vLLM and PagedAttention slides 9-10; dataarena note section 2): one
// query token per sequence attends over keys and values that sit in blocks of B
// tokens at arbitrary frames of a pool, found through the sequence's block table.
// Attention is softmax(scale q K^T) V, accumulated in fp32.
//
// Kernel design (B200): single-token decode is a bandwidth-bound GEMV, so the
// kernel is built to keep HBM busy, not to feed tensor cores.
//  * One CTA per (sequence, kv head, context partition of `part_tokens` tokens);
//    all query heads of the kv head's group (G = Hq/Hkv) share one K/V fetch.
//  * Warp 4 (the producer) preloads the partition's block-table entries into
//    shared memory, then one lane streams K and V into a ring of STAGES shared
//    memory stages with 1-D bulk copies (the copy engine, no register staging):
//    a (frame, kv head) tile is contiguous in the [N, Hkv, B, D] layout, so one
//    copy per block of K and one of V.  Full/empty mbarriers hand stages between
//    the producer and the four consumer warps.
//  * Stage = TS = 32 logical tokens; consumer warp w owns tokens 8w..8w+7 of
//    every stage and keeps its own online-softmax state (running max, partial
//    sum, fp32 accumulator) for the G heads.  Scores: LPT lanes cooperate on one
//    token (16-byte shared loads, packed fp32 FMA, shuffle reduction).  PV: each
//    lane owns D/32 output dims of all G heads.
//  * The four warps' states are merged through shared memory at the end; a
//    single-partition sequence writes `out` directly, otherwise the partition's
//    normalised output, max and sum go to the workspace and a second kernel
//    merges the partitions (log-sum-exp).
//  * Scores are kept in base-2 units (q is pre-scaled by scale * log2 e) so the
//    exponentials are single ex2 instructions.
#pragma once

#include <math_constants.h>

#include "device.cuh"

namespace pkv {

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* tables;  // paged: [S, MB]
  const int32_t* lens;    // [S]
  int32_t num_seqs;
  int32_t max_blocks;     // paged: MB
  int32_t num_blocks;     // paged: N
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t max_ctx;        // capacity in tokens: MB * B (paged) or the contiguous stride
  int32_t part_tokens;
  int32_t max_parts;      // ceil(max_ctx / part_tokens)
  float scale_log2;       // scale * log2(e)
  float* tmp_out;         // [S, Hq, P, D]
  float* tmp_m;           // [S, Hq, P]
  float* tmp_l;           // [S, Hq, P]
  unsigned int* err;
};

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxPartTokens = 8192;

template <typename T, int D_, int G_, int B_, bool PAGED_>
struct DecodeTraits {
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr int B = B_;
  static constexpr bool PAGED = PAGED_;
  static constexpr int LPT = (G * D / 8 <= 64) ? 8 : 16;  // lanes per token (scores)
  static constexpr int EPL = D / LPT;                     // row elements per lane (scores)
  static constexpr int VPL = EPL / 8;                     // 16-byte vectors per lane (scores)
  static constexpr int TPR = 32 / LPT;                    // tokens per warp round
  static constexpr int TPW = 8;                           // tokens per warp per stage
  static constexpr int ROUNDS = TPW / TPR;
  static constexpr int TS = kConsumerWarps * TPW;         // tokens per stage
  static constexpr int CH = PAGED ? (B < TS ? B : TS) : TS;  // tokens per bulk copy
  static constexpr int NCH = TS / CH;
  static constexpr int STAGES = 4;
  static constexpr int DPL = D / 32;                      // output dims per lane (PV)
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int TILE_BYTES = TS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int MAX_TABLE = PAGED ? kMaxPartTokens / B : 4;
  // shared memory carve-up (bytes)
  static constexpr int OFF_BARS = STAGES * STAGE_BYTES;
  static constexpr int OFF_TABLE = OFF_BARS + 2 * STAGES * 8;
  static constexpr int OFF_P = OFF_TABLE + MAX_TABLE * 4;
  static constexpr int OFF_M = OFF_P + kConsumerWarps * TPW * G * 4;
  static constexpr int OFF_L = OFF_M + kConsumerWarps * G * 4;
  static constexpr int SMEM_BYTES = OFF_L + kConsumerWarps * G * 4;
  static constexpr int MERGE_BYTES = kConsumerWarps * G * D * 4;  // reuses the stage ring

  static_assert(D % 64 == 0, "head_dim must be 64 or 128");
  static_assert(EPL % 8 == 0 && VPL >= 1, "score vectors are 16 bytes");
  static_assert(G <= LPT, "one lane per head inside a token group");
  static_assert(TPW % TPR == 0, "whole rounds per stage");
  static_assert(TS % CH == 0, "whole copies per stage");
  static_assert(MERGE_BYTES <= STAGES * STAGE_BYTES, "merge buffer fits in the ring");
  static_assert(DPL == 2 || DPL == 4, "PV reads 4 or 8 bytes per lane");
};

template <typename T, int D, int G, int B, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeArgs a) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  constexpr int STAGES = Tr::STAGES, TS = Tr::TS, LPT = Tr::LPT, TPR = Tr::TPR;
  constexpr int TPW = Tr::TPW, ROUNDS = Tr::ROUNDS, VPL = Tr::VPL, DPL = Tr::DPL;

  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  const int s = blockIdx.z;

  int L = __ldg(a.lens + s);
  if (L < 0 || L > a.max_ctx) {
    if (part == 0 && kvh == 0 && threadIdx.x == 0) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : a.max_ctx;
  }
  const int n_parts = L == 0 ? 1 : (L + a.part_tokens - 1) / a.part_tokens;
  if (part >= n_parts) return;
  const int t_begin = part * a.part_tokens;
  const int n_tok = min(L - t_begin, a.part_tokens);  // 0 only when L == 0
  const int n_stages = (n_tok + TS - 1) / TS;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BARS);
  uint64_t* empty = full + STAGES;
  int32_t* s_table = reinterpret_cast<int32_t*>(smem + Tr::OFF_TABLE);
  float* s_p = reinterpret_cast<float*>(smem + Tr::OFF_P);
  float* s_m = reinterpret_cast<float*>(smem + Tr::OFF_M);
  float* s_l = reinterpret_cast<float*>(smem + Tr::OFF_L);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  // ---------------------------------------------------------------- producer
  if (warp == kConsumerWarps) {
    int n_blk = 0;
    if constexpr (PAGED) {
      // The partition starts on a block boundary (part_tokens % 32 == 0, B | 32).
      const int first_blk = t_begin / B;
      n_blk = (n_tok + B - 1) / B;
      const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks + first_blk;
      for (int j = lane; j < n_blk; j += 32) {
        int32_t p = __ldg(row + j);
        if (p < 0 || p >= a.num_blocks) {
          set_error(a.err, PKV_DEVERR_TABLE_ENTRY);
          p = 0;
        }
        s_table[j] = p;
      }
      __syncwarp();
    }
    if (lane != 0) return;
    const uint8_t* kbase = static_cast<const uint8_t*>(a.k);
    const uint8_t* vbase = static_cast<const uint8_t*>(a.v);
    int issued = 0;
    for (int i = 0; i < n_stages; ++i) {
      const int st = i % STAGES;
      if (i >= STAGES && !mbar_wait_bounded(&empty[st], ((i / STAGES) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        break;
      }
      const int t0 = i * TS;  // relative to the partition start
      uint32_t bytes = 0;
#pragma unroll
      for (int c = 0; c < Tr::NCH; ++c) {
        const int tc = t0 + c * Tr::CH;
        if (tc < n_tok) bytes += min(Tr::CH, n_tok - tc) * Tr::ROW_BYTES;
      }
      mbar_arrive_expect_tx(&full[st], 2 * bytes);
      uint8_t* sk = smem + st * Tr::STAGE_BYTES;
      uint8_t* sv = sk + Tr::TILE_BYTES;
#pragma unroll
      for (int c = 0; c < Tr::NCH; ++c) {
        const int tc = t0 + c * Tr::CH;
        if (tc < n_tok) {
          const uint32_t nbytes = min(Tr::CH, n_tok - tc) * Tr::ROW_BYTES;
          int64_t row;
          if constexpr (PAGED) {
            const int64_t frame = s_table[tc / B];
            row = (frame * a.num_kv_heads + kvh) * B + (tc % B);
          } else {
            row = (static_cast<int64_t>(s) * a.num_kv_heads + kvh) * a.max_ctx + t_begin + tc;
          }
          bulk_load(sk + c * Tr::CH * Tr::ROW_BYTES, kbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
          bulk_load(sv + c * Tr::CH * Tr::ROW_BYTES, vbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
        }
      }
      ++issued;
    }
    // Never leave the CTA with copies in flight: wait (bounded) until the
    // last use of every stage has landed.
    for (int i = max(0, issued - STAGES); i < issued; ++i) {
      if (!mbar_wait_bounded(&full[i % STAGES], (i / STAGES) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int tg = lane / LPT;  // token group inside a round
  const int li = lane % LPT;  // lane inside the token group
  const int h0 = kvh * G;

  // q of the G heads, pre-scaled into base-2 score units, in the score-step layout:
  // vector c of lane li covers row elements [(c * LPT + li) * 8, +8).
  float2 qf[G][VPL][4];
  {
    const T* qrow = static_cast<const T*>(a.q) + (static_cast<int64_t>(s) * a.num_heads + h0) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + g * D + (c * LPT + li) * 8));
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack2<T>(w4[j]);
          qf[g][c][j] = make_float2(f.x * a.scale_log2, f.y * a.scale_log2);
        }
      }
    }
  }

  float m_run[G];
  float2 acc[G][DPL / 2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -CUDART_INF_F;
#pragma unroll
    for (int k = 0; k < DPL / 2; ++k) acc[g][k] = make_float2(0.f, 0.f);
  }
  float l_lane = 0.f;  // partial softmax sum of head li (lanes li < G)

  float* p_warp = s_p + warp * TPW * G;
  const int w_tok0 = warp * TPW;

  for (int i = 0; i < n_stages; ++i) {
    const int st = i % STAGES;
    if (!mbar_wait_bounded(&full[st], (i / STAGES) & 1)) {
      set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
      break;
    }
    const T* sK = reinterpret_cast<const T*>(smem + st * Tr::STAGE_BYTES);
    const T* sV = sK + TS * D;
    const int nv = min(TS, n_tok - i * TS);

    // scores of this warp's tokens
    float sc[ROUNDS][G];
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
      const int tok = w_tok0 + r * TPR + tg;
      const T* krow = sK + tok * D;
      float2 part2[G];
#pragma unroll
      for (int g = 0; g < G; ++g) part2[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(krow + (c * LPT + li) * 8);
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 kf = unpack2<T>(w4[j]);
#pragma unroll
          for (int g = 0; g < G; ++g) part2[g] = ffma2(qf[g][c][j], kf, part2[g]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = part2[g].x + part2[g].y;
#pragma unroll
        for (int o = LPT / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        sc[r][g] = tok < nv ? x : -CUDART_INF_F;
      }
    }

    // online softmax: new running max per head over the warp's tokens
    bool rescale = false;
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = sc[0][g];
#pragma unroll
      for (int r = 1; r < ROUNDS; ++r) mx = fmaxf(mx, sc[r][g]);
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_run[g], mx);
      alpha[g] = (m_new == m_run[g]) ? 1.f : fast_exp2(m_run[g] - m_new);
      rescale |= (m_new != m_run[g]);
      m_run[g] = m_new;
    }

    // probabilities: lane li < G computes head li of its token
    {
      float m_mine = m_run[0], a_mine = alpha[0];
#pragma unroll
      for (int g = 1; g < G; ++g)
        if (li == g) {
          m_mine = m_run[g];
          a_mine = alpha[g];
        }
      l_lane *= a_mine;
#pragma unroll
      for (int r = 0; r < ROUNDS; ++r) {
        float s_mine = sc[r][0];
#pragma unroll
        for (int g = 1; g < G; ++g)
          if (li == g) s_mine = sc[r][g];
        const float p = (s_mine == -CUDART_INF_F) ? 0.f : fast_exp2(s_mine - m_mine);
        if (li < G) {
          p_warp[(r * TPR + tg) * G + li] = p;
          l_lane += p;
        }
      }
    }
    __syncwarp();

    if (rescale) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float2 a2 = make_float2(alpha[g], alpha[g]);
#pragma unroll
        for (int k = 0; k < DPL / 2; ++k) acc[g][k] = fmul2(acc[g][k], a2);
      }
    }

    // PV over this warp's valid tokens
#pragma unroll
    for (int j = 0; j < TPW; ++j) {
      if (w_tok0 + j >= nv) break;
      float pj[G];
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int g = 0; g < G; g += 4) {
          const float4 p4 = *reinterpret_cast<const float4*>(p_warp + j * G + g);
          pj[g] = p4.x; pj[g + 1] = p4.y; pj[g + 2] = p4.z; pj[g + 3] = p4.w;
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) pj[g] = p_warp[j * G + g];
      }
      const T* vrow = sV + (w_tok0 + j) * D + lane * DPL;
      float2 vf[DPL / 2];
      if constexpr (DPL == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(vrow);
        vf[0] = unpack2<T>(raw.x);
        vf[1] = unpack2<T>(raw.y);
      } else {
        vf[0] = unpack2<T>(*reinterpret_cast<const uint32_t*>(vrow));
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float2 p2 = make_float2(pj[g], pj[g]);
#pragma unroll
        for (int k = 0; k < DPL / 2; ++k) acc[g][k] = ffma2(p2, vf[k], acc[g][k]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ------------------------------------------------------- merge the 4 warps
  // sum of probabilities of head li over the warp's token groups
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);

  named_barrier_sync(1, kConsumerWarps * 32);  // every warp is done with the ring
  float* s_acc = reinterpret_cast<float*>(smem);  // [warps][G][D]
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int k = 0; k < DPL / 2; ++k)
      *reinterpret_cast<float2*>(s_acc + (warp * G + g) * D + lane * DPL + 2 * k) = acc[g][k];
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) s_m[warp * G + g] = m_run[g];
  }
  if (tg == 0 && li < G) s_l[warp * G + li] = l_lane;
  named_barrier_sync(1, kConsumerWarps * 32);

  const bool single = (n_parts == 1);
  for (int idx = threadIdx.x; idx < G * D; idx += kConsumerWarps * 32) {
    const int g = idx / D;
    const int d = idx % D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_m[w * G + g]);
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = s_m[w * G + g];
      const float f = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
      lsum += f * s_l[w * G + g];
      o += f * s_acc[(w * G + g) * D + d];
    }
    const int h = h0 + g;
    if (single) {
      const float val = lsum > 0.f ? o / lsum : 0.f;
      static_cast<T*>(a.out)[(static_cast<int64_t>(s) * a.num_heads + h) * D + d] = from_float<T>(val);
    } else {
      const int64_t cell = (static_cast<int64_t>(s) * a.num_heads + h) * a.max_parts + part;
      a.tmp_out[cell * D + d] = o / lsum;
      if (d == 0) {
        a.tmp_m[cell] = M;
        a.tmp_l[cell] = lsum;
      }
    }
  }
}

// Second pass: merge the partitions of every (sequence, query head) whose
// context spans more than one partition.  One CTA of D threads per pair.
template <typename T, int D>
__global__ void __launch_bounds__(D) merge_partitions_kernel(const DecodeArgs a) {
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  int L = __ldg(a.lens + s);
  L = L < 0 ? 0 : (L > a.max_ctx ? a.max_ctx : L);
  const int n_parts = L == 0 ? 1 : (L + a.part_tokens - 1) / a.part_tokens;
  if (n_parts <= 1) return;
  const int64_t base = (static_cast<int64_t>(s) * a.num_heads + h) * a.max_parts;
  float M = -CUDART_INF_F;
  for (int p = 0; p < n_parts; ++p) M = fmaxf(M, a.tmp_m[base + p]);
  float lsum = 0.f, o = 0.f;
  const int d = threadIdx.x;
  for (int p = 0; p < n_parts; ++p) {
    const float w = a.tmp_l[base + p] * fast_exp2(a.tmp_m[base + p] - M);
    lsum += w;
    o += w * a.tmp_out[(base + p) * D + d];
  }
  static_cast<T*>(a.out)[(static_cast<int64_t>(s) * a.num_heads + h) * D + d] =
      from_float<T>(lsum > 0.f ? o / lsum : 0.f);
}

// Host-side launcher, instantiated per (dtype, head_dim) in its own file.
template <typename T, int D>
cudaError_t launch_decode(const DecodeArgs& a, int group, int block_size, bool paged,
                          cudaStream_t stream);

}  // namespace pkv
