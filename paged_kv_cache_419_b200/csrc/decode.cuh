// Paged decode attention for sm_100a.
//
// Method (vLLM and PagedAttention slides 9-10; dataarena note section 2): one
// query token per sequence attends over keys and values that sit in blocks of B
// tokens at arbitrary frames of a pool, found through the sequence's block table.
// Attention is softmax(scale q K^T) V, accumulated in fp32.
//
// Kernel design (B200).  Single-token decode is a bandwidth-bound GEMV, so the
// kernels are built to keep HBM busy, not to feed tensor cores.
//
//  * Work item = (sequence, kv head, context partition).  A context of L tokens
//    is cut into n = ceil(L / part_tokens) near-equal partitions whose sizes are
//    multiples of 32 tokens.  All G = Hq/Hkv query heads of the kv head share one
//    K/V fetch.
//  * plan_kernel (one CTA) lists the items, largest first, and zeroes the work
//    counter and the per-(sequence, kv head) merge counters in the workspace.
//  * decode_kernel is persistent: (SM count x occupancy) CTAs, launched with
//    programmatic dependent launch so that their set-up overlaps the plan.  Each
//    CTA takes items from the list with an atomic counter until it runs dry.
//  * Inside a CTA, warp 4 is the producer: it takes the next item, copies its q
//    rows into an item slot and streams the item's K and V through a ring of
//    STAGES shared-memory stages with 1-D bulk copies (one copy per block of K
//    and of V: a (frame, kv head) tile is contiguous in [N, Hkv, B, D]).  It runs
//    ahead across items, so the next item's data arrives while the consumers
//    finish the current one.  mbarriers hand stages and item slots over.
//  * Stage = 32 logical tokens; consumer warp w owns tokens 8w..8w+7 of each
//    stage with its own online-softmax state.  Scores: LPT lanes share a token
//    (16-byte shared loads, packed fp32 FMA), then a reduce-scatter across the
//    LPT lanes leaves every lane holding the finished score of one head.  PV:
//    each lane owns D/32 output dims of all G heads.
//  * Epilogue per item: the four warps merge in shared memory.  A one-partition
//    context writes `out`; otherwise the partition's normalised output, max and
//    sum go to the workspace, and the CTA that completes the last partition of a
//    (sequence, kv head) merges them (log-sum-exp) and writes `out`.
//  * Scores are kept in base-2 units (q is pre-scaled by scale * log2 e), so the
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
  int32_t part_tokens;    // maximum tokens per partition (multiple of 32)
  int32_t max_parts;      // ceil(max_ctx / part_tokens): upper bound of partitions per context
  float scale_log2;       // scale * log2(e)
  uint32_t* work;         // [0] next item, [1] item count
  uint32_t* merge_cnt;    // [S * Hkv] partitions finished
  int2* items;            // [S * max_parts] (sequence, partition), largest first
  float* tmp_out;         // [S, Hq, max_parts, D]
  float* tmp_m;           // [S, Hq, max_parts]
  float* tmp_l;           // [S, Hq, max_parts]
  unsigned int* err;
};

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxPartTokens = 4096;
constexpr int kPlanThreads = 1024;
constexpr int kItemSlots = 2;

// Partitioning of a context of L tokens (L already clamped to [0, max_ctx]):
// n partitions of `size` tokens (a multiple of 32), the last one shorter.
__device__ __forceinline__ void partition_of(int L, int part_tokens, int& n, int& size) {
  if (L <= 0) {
    n = 1;
    size = 0;
    return;
  }
  const int n0 = (L + part_tokens - 1) / part_tokens;
  size = ((L + n0 - 1) / n0 + 31) & ~31;
  n = (L + size - 1) / size;
}

__device__ __forceinline__ int clamp_len(int L, int max_ctx) {
  return L < 0 ? 0 : (L > max_ctx ? max_ctx : L);
}

template <typename T, int D_, int G_, int B_, bool PAGED_>
struct DecodeTraits {
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr int B = B_;
  static constexpr bool PAGED = PAGED_;
  static constexpr int LPT = (G * D / 8 <= 64) ? 8 : 16;  // lanes per token (scores)
  static constexpr int LPH = LPT / G;                     // lanes holding one head's score
  static constexpr int EPL = D / LPT;                     // row elements per lane (scores)
  static constexpr int VPL = EPL / 8;                     // 16-byte vectors per lane (scores)
  static constexpr int TPR = 32 / LPT;                    // tokens per warp round
  static constexpr int TPW = 8;                           // tokens per warp per stage
  static constexpr int ROUNDS = TPW / TPR;
  static constexpr int TS = kConsumerWarps * TPW;         // tokens per stage
  static constexpr int CH = PAGED ? (B < TS ? B : TS) : TS;  // tokens per bulk copy
  static constexpr int NCH = TS / CH;
  static constexpr int STAGES = 3;
  static constexpr int DPL = D / 32;                      // output dims per lane (PV)
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int TILE_BYTES = TS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int MAX_TABLE = PAGED ? kMaxPartTokens / B : 4;
  // shared memory carve-up (bytes, 16-byte aligned pieces)
  static constexpr int OFF_Q = STAGES * STAGE_BYTES;
  static constexpr int OFF_ACC = OFF_Q + kItemSlots * Q_BYTES;          // [warps][G][D] f32
  static constexpr int OFF_P = OFF_ACC + kConsumerWarps * G * D * 4;    // [warps][TPW][G] (p, p)
  static constexpr int OFF_TABLE = OFF_P + kConsumerWarps * TPW * G * 8;
  static constexpr int OFF_STAT = OFF_TABLE + MAX_TABLE * 4;            // m, l per warp and head
  static constexpr int OFF_ITEM = OFF_STAT + 2 * kConsumerWarps * G * 4 + 16;
  static constexpr int OFF_BARS = OFF_ITEM + kItemSlots * 32;
  static constexpr int SMEM_BYTES = OFF_BARS + (2 * STAGES + 2 * kItemSlots) * 8;

  static_assert(D % 64 == 0, "head_dim must be 64 or 128");
  static_assert(EPL % 8 == 0 && VPL >= 1, "score vectors are 16 bytes");
  static_assert(G <= LPT && LPT % G == 0, "reduce-scatter leaves one head per lane group");
  static_assert(TPW % TPR == 0, "whole rounds per stage");
  static_assert(TS % CH == 0 && NCH <= 32, "whole copies per stage, one lane each");
  static_assert(DPL == 2 || DPL == 4, "PV reads 4 or 8 bytes per lane");
  static_assert(OFF_BARS % 8 == 0, "mbarriers are 8-byte aligned");
};

// Item slot handed from the producer to the consumers.
struct ItemInfo {
  int s, kvh, part, n_parts, t_begin, n_tok;
};

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- plan
// One CTA: clamp the context lengths, list every (sequence, partition) in
// decreasing order of size (counting sort on 32-token size classes), and zero
// the work counter and the merge counters.
static __global__ void __launch_bounds__(kPlanThreads) plan_kernel(const DecodeArgs a) {
  constexpr int kMaxClasses = kMaxPartTokens / 32 + 2;
  __shared__ uint32_t count[kMaxClasses];
  __shared__ uint32_t cursor[kMaxClasses];
  __shared__ uint32_t total;
  const int classes = a.part_tokens / 32 + 2;  // class c: size in (part - 32(c+1), part - 32c]; last: empty
  for (int c = threadIdx.x; c < classes; c += blockDim.x) count[c] = 0;
  if (threadIdx.x == 0) total = 0;
  const int cnt_len = a.num_seqs * a.num_kv_heads;
  for (int i = threadIdx.x; i < cnt_len; i += blockDim.x) a.merge_cnt[i] = 0;
  __syncthreads();
  auto size_class = [&](int sz) {
    return sz == 0 ? classes - 1 : (a.part_tokens - sz) / 32;
  };
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int raw = a.lens[s];
    if (raw < 0 || raw > a.max_ctx) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    const int L = clamp_len(raw, a.max_ctx);
    int n, size;
    partition_of(L, a.part_tokens, n, size);
    for (int p = 0; p < n; ++p) atomicAdd(&count[size_class(min(size, L - p * size))], 1u);
    atomicAdd(&total, static_cast<uint32_t>(n));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t run = 0;
    for (int c = 0; c < classes; ++c) {
      cursor[c] = run;
      run += count[c];
    }
  }
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int L = clamp_len(a.lens[s], a.max_ctx);
    int n, size;
    partition_of(L, a.part_tokens, n, size);
    for (int p = 0; p < n; ++p) {
      const uint32_t pos = atomicAdd(&cursor[size_class(min(size, L - p * size))], 1u);
      a.items[pos] = make_int2(s, p);
    }
  }
  if (threadIdx.x == 0) {
    a.work[0] = 0;
    a.work[1] = total * static_cast<uint32_t>(a.num_kv_heads);
  }
  __threadfence();
  __syncthreads();
  allow_dependent_launch();
}

// ---------------------------------------------------------------- decode
template <typename T, int D, int G, int B, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeArgs a) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  constexpr int STAGES = Tr::STAGES, TS = Tr::TS, LPT = Tr::LPT, LPH = Tr::LPH, TPR = Tr::TPR;
  constexpr int TPW = Tr::TPW, ROUNDS = Tr::ROUNDS, VPL = Tr::VPL, DPL = Tr::DPL;
  constexpr int NW = kConsumerWarps;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BARS);
  uint64_t* empty = full + STAGES;
  uint64_t* item_full = empty + STAGES;
  uint64_t* item_empty = item_full + kItemSlots;
  ItemInfo* items = reinterpret_cast<ItemInfo*>(smem + Tr::OFF_ITEM);
  int32_t* s_table = reinterpret_cast<int32_t*>(smem + Tr::OFF_TABLE);
  float* s_acc = reinterpret_cast<float*>(smem + Tr::OFF_ACC);
  float2* s_p = reinterpret_cast<float2*>(smem + Tr::OFF_P);
  float* s_m = reinterpret_cast<float*>(smem + Tr::OFF_STAT);
  float* s_l = s_m + NW * G;
  int* s_flag = reinterpret_cast<int*>(s_l + NW * G);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], NW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  // Everything below reads what the plan kernel wrote.
  grid_dependency_wait();

  // ================================================================ producer
  if (warp == NW) {
    const uint8_t* kbase = static_cast<const uint8_t*>(a.k);
    const uint8_t* vbase = static_cast<const uint8_t*>(a.v);
    const uint32_t n_items = *reinterpret_cast<volatile uint32_t*>(a.work + 1);
    uint32_t stage_iter = 0;
    bool ok = true;
    for (uint32_t item_iter = 0;; ++item_iter) {
      uint32_t idx = 0;
      if (lane == 0) idx = atomicAdd(a.work, 1u);
      idx = __shfl_sync(0xffffffffu, idx, 0);
      const int slot = item_iter % kItemSlots;
      if (item_iter >= kItemSlots && lane == 0 &&
          !mbar_wait_bounded(&item_empty[slot], ((item_iter / kItemSlots) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (idx >= n_items) {
        if (lane == 0) {
          items[slot].s = -1;  // no more work
          mbar_arrive(&item_full[slot]);
        }
        break;
      }
      const int2 it = __ldcg(a.items + idx / a.num_kv_heads);
      const int kvh = idx % a.num_kv_heads;
      const int s = it.x, part = it.y;
      const int L = clamp_len(__ldg(a.lens + s), a.max_ctx);
      int n_parts, psize;
      partition_of(L, a.part_tokens, n_parts, psize);
      const int t_begin = part * psize;
      const int n_tok = min(L - t_begin, psize);  // 0 only when L == 0
      if constexpr (PAGED) {
        const int first_blk = t_begin / B;
        const int n_blk = (n_tok + B - 1) / B;
        const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks + first_blk;
        for (int j = lane; j < n_blk; j += 32) {
          int32_t p = __ldg(row + j);
          if (p < 0 || p >= a.num_blocks) {
            set_error(a.err, PKV_DEVERR_TABLE_ENTRY);
            p = 0;
          }
          s_table[j] = p;
        }
      }
      if (lane == 0) {
        ItemInfo& info = items[slot];
        info.s = s;
        info.kvh = kvh;
        info.part = part;
        info.n_parts = n_parts;
        info.t_begin = t_begin;
        info.n_tok = n_tok;
        mbar_arrive_expect_tx(&item_full[slot], Tr::Q_BYTES);
        const uint8_t* qsrc = static_cast<const uint8_t*>(a.q) +
                              (static_cast<int64_t>(s) * a.num_heads + kvh * G) * Tr::ROW_BYTES;
        bulk_load(smem + Tr::OFF_Q + slot * Tr::Q_BYTES, qsrc, Tr::Q_BYTES, &item_full[slot]);
      }
      __syncwarp();
      const int n_stages = (n_tok + TS - 1) / TS;
      for (int i = 0; i < n_stages; ++i, ++stage_iter) {
        const int st = stage_iter % STAGES;
        if (lane == 0 && stage_iter >= STAGES &&
            !mbar_wait_bounded(&empty[st], ((stage_iter / STAGES) - 1) & 1)) {
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
          ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const int t0 = i * TS;  // relative to the partition start (block aligned)
        if (lane == 0) {
          const int rows = min(TS, n_tok - t0);
          mbar_arrive_expect_tx(&full[st], 2u * rows * Tr::ROW_BYTES);
        }
        __syncwarp();
        const int tc = t0 + lane * Tr::CH;
        if (lane < Tr::NCH && tc < n_tok) {
          const uint32_t nbytes = min(Tr::CH, n_tok - tc) * Tr::ROW_BYTES;
          int64_t row;
          if constexpr (PAGED) {
            const int64_t frame = s_table[tc / B];
            row = (frame * a.num_kv_heads + kvh) * B + (t_begin + tc) % B;
          } else {
            row = (static_cast<int64_t>(s) * a.num_kv_heads + kvh) * a.max_ctx + t_begin + tc;
          }
          uint8_t* sk = smem + st * Tr::STAGE_BYTES + lane * Tr::CH * Tr::ROW_BYTES;
          bulk_load(sk, kbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
          bulk_load(sk + Tr::TILE_BYTES, vbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
        }
        __syncwarp();
      }
      if (!ok) break;  // the consumers time out on their next wait and stop too
    }
    // Never leave the CTA with copies in flight: wait (bounded) until the last
    // use of every stage has landed.
    if (lane == 0) {
      const uint32_t first = stage_iter > STAGES ? stage_iter - STAGES : 0;
      for (uint32_t i = first; i < stage_iter; ++i)
        if (!mbar_wait_bounded(&full[i % STAGES], (i / STAGES) & 1))
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    return;
  }

  // ================================================================ consumers
  // Exits are decided together (barrier-OR over the consumer warps) so that no
  // warp is ever left waiting at a named barrier.
  const int tg = lane / LPT;       // token group inside a round
  const int li = lane % LPT;       // lane inside the token group
  const int my_h = li / LPH;       // head whose score this lane holds after the reduce-scatter
  const bool p_writer = (li % LPH) == 0;
  const int w_tok0 = warp * TPW;
  float2* p_warp = s_p + warp * TPW * G;
  uint32_t stage_iter = 0;

  for (uint32_t item_iter = 0;; ++item_iter) {
    const int slot = item_iter % kItemSlots;
    const bool arrived = mbar_wait_bounded(&item_full[slot], (item_iter / kItemSlots) & 1);
    if (!arrived && lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    const ItemInfo info = items[slot];
    if (named_barrier_or(1, NW * 32, !arrived || info.s < 0)) break;
    const int h0 = info.kvh * G;

    // q of the G heads, scaled into base-2 score units, in the score-step layout:
    // vector c of lane li covers row elements [(c * LPT + li) * 8, +8).
    float2 qf[G][VPL][4];
    {
      const T* sq = reinterpret_cast<const T*>(smem + Tr::OFF_Q + slot * Tr::Q_BYTES);
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
          const uint4 raw = *reinterpret_cast<const uint4*>(sq + g * D + (c * LPT + li) * 8);
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = unpack2<T>(w4[j]);
            qf[g][c][j] = make_float2(f.x * a.scale_log2, f.y * a.scale_log2);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[slot]);

    float m_run = -CUDART_INF_F;  // running max of head my_h
    float l_lane = 0.f;           // partial softmax sum of head my_h (p_writer lanes)
    float2 acc[G][DPL / 2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int k = 0; k < DPL / 2; ++k) acc[g][k] = make_float2(0.f, 0.f);

    const int n_stages = (info.n_tok + TS - 1) / TS;
    bool ok = true;
    for (int i = 0; i < n_stages; ++i, ++stage_iter) {
      const int st = stage_iter % STAGES;
      if (!mbar_wait_bounded(&full[st], (stage_iter / STAGES) & 1)) {
        if (lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
        break;
      }
      const T* sK = reinterpret_cast<const T*>(smem + st * Tr::STAGE_BYTES);
      const T* sV = sK + TS * D;
      const int nv = min(TS, info.n_tok - i * TS);

      // ---- scores: every lane ends with the score of head my_h of its token
      float sc[ROUNDS];
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
        float x[G];
#pragma unroll
        for (int g = 0; g < G; ++g) x[g] = part2[g].x + part2[g].y;
        // reduce-scatter: each halving step keeps half of the heads
#pragma unroll
        for (int cnt = G, m = LPT / 2; cnt > 1; cnt >>= 1, m >>= 1) {
          const bool upper = (li & m) != 0;
#pragma unroll
          for (int j = 0; j < cnt / 2; ++j) {
            const float send = upper ? x[j] : x[j + cnt / 2];
            const float keep = upper ? x[j + cnt / 2] : x[j];
            x[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
        }
        // the lanes of one head's group finish with a plain reduction
#pragma unroll
        for (int m = LPH / 2; m > 0; m >>= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], m);
        sc[r] = tok < nv ? x[0] : -CUDART_INF_F;
      }

      // ---- online softmax for head my_h
      float mx = sc[0];
#pragma unroll
      for (int r = 1; r < ROUNDS; ++r) mx = fmaxf(mx, sc[r]);
#pragma unroll
      for (int m = LPT; m < 32; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      const float m_new = fmaxf(m_run, mx);
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float alpha = m_new == m_run ? 1.f : fast_exp2(m_run - m_new);  // 0 when m_run = -inf
        l_lane *= alpha;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float ag = __shfl_sync(0xffffffffu, alpha, g * LPH);
          const float2 a2 = make_float2(ag, ag);
#pragma unroll
          for (int k = 0; k < DPL / 2; ++k) acc[g][k] = fmul2(acc[g][k], a2);
        }
        m_run = m_new;
      }
#pragma unroll
      for (int r = 0; r < ROUNDS; ++r) {
        const float p = sc[r] == -CUDART_INF_F ? 0.f : fast_exp2(sc[r] - m_run);
        if (p_writer) {
          p_warp[(r * TPR + tg) * G + my_h] = make_float2(p, p);
          l_lane += p;
        }
      }
      __syncwarp();

      // ---- PV over this warp's valid tokens
#pragma unroll
      for (int j = 0; j < TPW; ++j) {
        if (w_tok0 + j >= nv) break;
        float2 pj[G];
        if constexpr (G % 2 == 0) {
#pragma unroll
          for (int g = 0; g < G; g += 2) {
            const float4 p4 = *reinterpret_cast<const float4*>(p_warp + j * G + g);
            pj[g] = make_float2(p4.x, p4.y);
            pj[g + 1] = make_float2(p4.z, p4.w);
          }
        } else {
          pj[0] = p_warp[j * G];
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
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int k = 0; k < DPL / 2; ++k) acc[g][k] = ffma2(pj[g], vf[k], acc[g][k]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- merge the four warps of this item
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, m);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int k = 0; k < DPL / 2; ++k)
        *reinterpret_cast<float2*>(s_acc + (warp * G + g) * D + lane * DPL + 2 * k) = acc[g][k];
    if (tg == 0 && p_writer) {
      s_m[warp * G + my_h] = m_run;
      s_l[warp * G + my_h] = l_lane;
    }
    if (named_barrier_or(1, NW * 32, !ok)) break;  // a timed-out stage: stop, output invalid

    const int s = info.s;
    const bool single = info.n_parts == 1;
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
      const int g = idx / D, d = idx % D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m[w * G + g]);
      float lsum = 0.f, o = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = s_m[w * G + g];
        const float f = mw == -CUDART_INF_F ? 0.f : fast_exp2(mw - M);
        lsum += f * s_l[w * G + g];
        o += f * s_acc[(w * G + g) * D + d];
      }
      if (single) {
        static_cast<T*>(a.out)[(static_cast<int64_t>(s) * a.num_heads + h0 + g) * D + d] =
            from_float<T>(lsum > 0.f ? o / lsum : 0.f);
      } else {
        const int64_t cell = (static_cast<int64_t>(s) * a.num_heads + h0 + g) * a.max_parts + info.part;
        __stcg(a.tmp_out + cell * D + d, o / lsum);
        if (d == 0) {
          __stcg(a.tmp_m + cell, M);
          __stcg(a.tmp_l + cell, lsum);
        }
      }
    }
    if (!single) __threadfence();
    named_barrier_sync(1, NW * 32);  // s_acc, s_m, s_l are free again
    if (single) continue;

    if (threadIdx.x == 0) {
      const uint32_t done = atomicAdd(a.merge_cnt + s * a.num_kv_heads + info.kvh, 1u);
      *s_flag = (done == static_cast<uint32_t>(info.n_parts - 1));
    }
    named_barrier_sync(1, NW * 32);
    if (!*s_flag) continue;

    // Last partition of this (sequence, kv head) to finish: merge all partitions,
    // out = sum_p w_p o_p with w_p = l_p 2^(m_p - M) / sum_q l_q 2^(m_q - M), in
    // partition order.
    __threadfence();
    constexpr int kChunk = NW * D;  // partitions per pass; s_acc holds G * kChunk weights
    constexpr int kPer = (G * D + NW * 32 - 1) / (NW * 32);
    const int np = info.n_parts;
    float o_reg[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) o_reg[k] = 0.f;
    float* s_w = s_acc;
    for (int p0 = 0; p0 < np; p0 += kChunk) {
      const int pc = min(kChunk, np - p0);
      for (int g = warp; g < G; g += NW) {
        const int64_t base = (static_cast<int64_t>(s) * a.num_heads + h0 + g) * a.max_parts;
        float M = -CUDART_INF_F;
        for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldcg(a.tmp_m + base + p));
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
        float lsum = 0.f;
        for (int p = lane; p < np; p += 32)
          lsum += __ldcg(a.tmp_l + base + p) * fast_exp2(__ldcg(a.tmp_m + base + p) - M);
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, m);
        const float inv = 1.f / lsum;
        for (int p = lane; p < pc; p += 32)
          s_w[g * kChunk + p] =
              __ldcg(a.tmp_l + base + p0 + p) * fast_exp2(__ldcg(a.tmp_m + base + p0 + p) - M) * inv;
      }
      named_barrier_sync(1, NW * 32);
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int idx = threadIdx.x + k * NW * 32;
        if (idx < G * D) {
          const int g = idx / D, d = idx % D;
          const int64_t base = (static_cast<int64_t>(s) * a.num_heads + h0 + g) * a.max_parts + p0;
          float o = o_reg[k];
          for (int p = 0; p < pc; ++p) o += s_w[g * kChunk + p] * __ldcg(a.tmp_out + (base + p) * D + d);
          o_reg[k] = o;
        }
      }
      named_barrier_sync(1, NW * 32);
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = threadIdx.x + k * NW * 32;
      if (idx < G * D) {
        const int g = idx / D, d = idx % D;
        static_cast<T*>(a.out)[(static_cast<int64_t>(s) * a.num_heads + h0 + g) * D + d] =
            from_float<T>(o_reg[k]);
      }
    }
  }
}

// Host-side launcher, instantiated per (dtype, head_dim) in its own file.
template <typename T, int D>
cudaError_t launch_decode(const DecodeArgs& a, int group, int block_size, bool paged, int num_sms,
                          cudaStream_t stream);

}  // namespace pkv
