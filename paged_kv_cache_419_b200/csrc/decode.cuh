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
//  * plan_kernel (one CTA) lists the items, largest first, lists the contexts
//    that span several partitions, and resets the work counter.
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
//    sum go to the workspace, and merge_kernel (launched behind the decode grid)
//    merges the partitions of each such context (log-sum-exp) into `out`.
//  * Scores are kept in base-2 units (q is pre-scaled by scale * log2 e), so the
//    exponentials are single ex2 instructions.
#pragma once

#include <math_constants.h>

#include <type_traits>

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
  int32_t block_size;     // paged: B
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t max_ctx;        // capacity in tokens: MB * B (paged) or the contiguous stride
  int32_t part_tokens;    // maximum tokens per partition (multiple of 32)
  int32_t max_parts;      // ceil(max_ctx / part_tokens): upper bound of partitions per context
  float scale_log2;       // scale * log2(e)
  int32_t grid_ctas;      // decode CTAs; the first 3 * grid_ctas items are assigned statically
  uint32_t* work;         // [0] next item, [1] item count, [2] multi-partition sequences
  int32_t* merge_seqs;    // [S] sequences whose context spans more than one partition
  uint8_t* records;       // [S * max_parts] work records, largest partition first (32 B each)
  float* tmp_out;         // [S, Hq, max_parts, D]
  float* tmp_m;           // [S, Hq, max_parts]
  float* tmp_l;           // [S, Hq, max_parts]
  unsigned int* err;
};

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxPartTokens = 2048;
constexpr int kPlanThreads = 1024;
constexpr int kItemSlots = 2;
constexpr int kRecSlots = 4;   // records of items k .. k+3 (copied two items ahead)
constexpr int kStageTokens = 64;
// Work record of one (sequence, partition): int32 s, part, n_parts, t_begin,
// n_tok, L, 0, 0.
constexpr int kRecordBytes = 32;

// Partitioning of a context of L tokens (L already clamped to [0, max_ctx]):
// n partitions of `size` tokens (a multiple of the 64-token stage), the last
// one shorter.  part_tokens is a multiple of 64, so size <= part_tokens.
__device__ __forceinline__ void partition_of(int L, int part_tokens, int& n, int& size) {
  if (L <= 0) {
    n = 1;
    size = 0;
    return;
  }
  const int n0 = (L + part_tokens - 1) / part_tokens;
  size = ((L + n0 - 1) / n0 + kStageTokens - 1) & ~(kStageTokens - 1);
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
  static constexpr int TPW = kStageTokens / kConsumerWarps;  // tokens per warp per stage
  static constexpr int ROUNDS = TPW / TPR;
  static constexpr int TS = kConsumerWarps * TPW;         // tokens per stage
  static constexpr int CH = PAGED ? (B < TS ? B : TS) : TS;  // tokens per bulk copy
  static constexpr int NCH = TS / CH;
  static constexpr int STAGES = 2;
  static constexpr int DPL = D / 32;                      // output dims per lane (PV)
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int TILE_BYTES = TS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int Q_BYTES = G * D * 2;
  static constexpr int MAX_TABLE = PAGED ? kMaxPartTokens / B : 4;  // table entries of one item
  // shared memory carve-up (bytes, 16-byte aligned pieces)
  static constexpr int OFF_Q = STAGES * STAGE_BYTES;
  static constexpr int HG = G > 1 ? G / 2 : 1;                          // heads per merge round
  static constexpr int OFF_ACC = OFF_Q + kItemSlots * Q_BYTES;          // [warps][HG][D] f32
  static constexpr int OFF_P = OFF_ACC + kConsumerWarps * HG * D * 4;   // [warps][TPW][G] (p, p)
  static constexpr int OFF_REC = OFF_P + kConsumerWarps * TPW * G * 8;  // record slots
  static constexpr int OFF_TAB = OFF_REC + kRecSlots * kRecordBytes;    // 2 table buffers
  static constexpr int OFF_STAT = OFF_TAB + 2 * MAX_TABLE * 4;          // m, l per warp and head
  static constexpr int OFF_ITEM = OFF_STAT + 2 * kConsumerWarps * G * 4 + 16;
  static constexpr int OFF_BARS = OFF_ITEM + kItemSlots * 32;
  static constexpr int SMEM_BYTES = OFF_BARS + (2 * STAGES + 2 * kItemSlots + kRecSlots + 2) * 8;

  static_assert(D % 64 == 0, "head_dim must be 64 or 128");
  static_assert(EPL % 8 == 0 && VPL >= 1, "score vectors are 16 bytes");
  static_assert(G <= LPT && LPT % G == 0, "reduce-scatter leaves one head per lane group");
  static_assert(TPW % TPR == 0, "whole rounds per stage");
  static_assert(TS == kStageTokens, "stage = partition granule");
  static_assert(TS % CH == 0 && NCH <= 32, "whole copies per stage, one lane each");
  static_assert(DPL == 2 || DPL == 4, "PV reads 4 or 8 bytes per lane");
  static_assert(OFF_BARS % 8 == 0 && OFF_STAT % 16 == 0, "alignment");
  // three CTAs per SM (228 KB of shared memory, 1 KB reserved per CTA) up to G = 4
  static_assert(G > 4 || 3 * (SMEM_BYTES + 1024) <= 228 * 1024, "3 CTAs per SM");
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
// One CTA: clamp the context lengths, write one work record per (sequence,
// partition) in decreasing order of partition size (counting sort on 32-token
// size classes), list the sequences that span several partitions (for the
// merge kernel), and reset the work counter.  Every global read is issued by
// all threads at once (one round trip); the lengths are kept in shared memory
// for the second pass.
constexpr int kPlanSmemSeqs = 8192;

static __global__ void __launch_bounds__(kPlanThreads) plan_kernel(const DecodeArgs a) {
  // The decode grid may start its set-up now; it waits for this grid to finish
  // before it reads anything written here.  This grid itself starts behind its
  // predecessor on the stream and waits for it before reading any input.
  allow_dependent_launch();
  grid_dependency_wait();
  constexpr int kMaxClasses = kMaxPartTokens / 32 + 2;
  __shared__ uint32_t count[kMaxClasses];
  __shared__ uint32_t cursor[kMaxClasses];
  __shared__ uint32_t total, n_multi;
  __shared__ int s_len[kPlanSmemSeqs];
  const int classes = a.part_tokens / 32 + 2;  // class c: size in (part - 32(c+1), part - 32c]; last: empty
  const bool cached = a.num_seqs <= kPlanSmemSeqs;
  for (int c = threadIdx.x; c < classes; c += blockDim.x) count[c] = 0;
  if (threadIdx.x == 0) total = n_multi = 0;
  __syncthreads();
  auto size_class = [&](int sz) { return sz == 0 ? classes - 1 : (a.part_tokens - sz) / 32; };
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int raw = a.lens[s];
    if (raw < 0 || raw > a.max_ctx) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    const int L = clamp_len(raw, a.max_ctx);
    if (cached) s_len[s] = L;
    int n, size;
    partition_of(L, a.part_tokens, n, size);
    for (int p = 0; p < n; ++p) atomicAdd(&count[size_class(min(size, L - p * size))], 1u);
    atomicAdd(&total, static_cast<uint32_t>(n));
    if (n > 1) a.merge_seqs[atomicAdd(&n_multi, 1u)] = s;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // exclusive scan of the class counts, one warp
    const int lane = threadIdx.x;
    constexpr int kPerLane = (kMaxClasses + 31) / 32;
    uint32_t v[kPerLane], run = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int c = lane * kPerLane + i;
      v[i] = c < classes ? count[c] : 0u;
      run += v[i];
    }
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    uint32_t base = incl - run;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int c = lane * kPerLane + i;
      if (c < classes) cursor[c] = base;
      base += v[i];
    }
  }
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int L = cached ? s_len[s] : clamp_len(a.lens[s], a.max_ctx);
    int n, size;
    partition_of(L, a.part_tokens, n, size);
    for (int p = 0; p < n; ++p) {
      const int t_begin = p * size;
      const int n_tok = min(size, L - t_begin);
      const uint32_t pos = atomicAdd(&cursor[size_class(n_tok)], 1u);
      int4* rec = reinterpret_cast<int4*>(a.records + static_cast<int64_t>(pos) * kRecordBytes);
      rec[0] = make_int4(s, p, n, t_begin);
      rec[1] = make_int4(n_tok, L, 0, 0);
    }
  }
  if (threadIdx.x == 0) {
    a.work[0] = 3u * static_cast<uint32_t>(a.grid_ctas);  // items below are pre-assigned
    a.work[1] = total * static_cast<uint32_t>(a.num_kv_heads);
    a.work[2] = n_multi;
  }
}

// ---------------------------------------------------------------- decode
template <typename T, int D, int G, int B, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads, (G <= 4 ? 3 : 2)) decode_kernel(const DecodeArgs a) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  constexpr int STAGES = Tr::STAGES, TS = Tr::TS, LPT = Tr::LPT, LPH = Tr::LPH, TPR = Tr::TPR;
  constexpr int TPW = Tr::TPW, ROUNDS = Tr::ROUNDS, VPL = Tr::VPL, DPL = Tr::DPL;
  constexpr int NW = kConsumerWarps;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BARS);
  uint64_t* empty = full + STAGES;
  uint64_t* item_full = empty + STAGES;
  uint64_t* item_empty = item_full + kItemSlots;
  uint64_t* rec_bar = item_empty + kItemSlots;  // [kRecSlots]
  uint64_t* tab_bar = rec_bar + kRecSlots;       // [2]
  ItemInfo* items = reinterpret_cast<ItemInfo*>(smem + Tr::OFF_ITEM);
  float* s_acc = reinterpret_cast<float*>(smem + Tr::OFF_ACC);
  float2* s_p = reinterpret_cast<float2*>(smem + Tr::OFF_P);
  float* s_m = reinterpret_cast<float*>(smem + Tr::OFF_STAT);
  float* s_l = s_m + NW * G;

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
    for (int i = 0; i < kRecSlots; ++i) mbar_init(&rec_bar[i], 1);
    mbar_init(&tab_bar[0], 32);  // one asynchronous arrival per producer lane
    mbar_init(&tab_bar[1], 32);
    fence_barrier_init();
  }
  __syncthreads();
  // Everything below reads what the plan kernel wrote.
  grid_dependency_wait();

  // ================================================================ producer
  // Item j (the j-th item this CTA takes): its index is taken three items ahead,
  // its 32-byte record is bulk-copied two items ahead into record slot j % 4, and
  // its block-table entries are fetched one item ahead with cp.async into table
  // buffer j % 2.  So while item k's stages are issued, nothing the producer
  // waits for was requested less than one item ago.
  if (warp == NW) {
    const uint8_t* kbase = static_cast<const uint8_t*>(a.k);
    const uint8_t* vbase = static_cast<const uint8_t*>(a.v);
    const uint32_t n_items = *reinterpret_cast<volatile uint32_t*>(a.work + 1);
    const uint32_t Hkv = static_cast<uint32_t>(a.num_kv_heads);
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem + Tr::OFF_TAB);
    auto rec_slot = [&](uint32_t j) {
      return reinterpret_cast<const int32_t*>(smem + Tr::OFF_REC + (j % kRecSlots) * kRecordBytes);
    };
    // Outstanding copies nobody waited for yet (error exits drain them): bit r of
    // rec_pending / rec_parity = record slot r and the parity of its open phase;
    // likewise for the two table buffers.
    uint32_t rec_pending = 0, rec_parity = 0, tab_pending = 0, tab_parity = 0;
    auto copy_record = [&](uint32_t j, uint32_t idx) {  // lane 0
      const uint32_t r = j % kRecSlots;
      mbar_arrive_expect_tx(&rec_bar[r], kRecordBytes);
      bulk_load(smem + Tr::OFF_REC + r * kRecordBytes,
                a.records + static_cast<int64_t>(idx / Hkv) * kRecordBytes, kRecordBytes, &rec_bar[r]);
      rec_pending |= 1u << r;
      rec_parity = (rec_parity & ~(1u << r)) | (((j / kRecSlots) & 1u) << r);
    };
    // Every lane waits for record j (all lanes read it).
    auto wait_record = [&](uint32_t j) {
      const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&rec_bar[j % kRecSlots], (j / kRecSlots) & 1));
      if (lane == 0) {
        if (!got) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        rec_pending &= ~(1u << (j % kRecSlots));
      }
      return got;
    };
    // Block-table entries of item j (its record has landed) into buffer j % 2.
    auto fetch_table = [&](uint32_t j) {
      if constexpr (PAGED) {
        const int32_t* rec = rec_slot(j);
        const int s = rec[0], t_begin = rec[3], n_tok = rec[4];
        const int nb = (n_tok + B - 1) / B;
        const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks + t_begin / B;
        int32_t* dst = s_tab + (j & 1) * Tr::MAX_TABLE;
        for (int e = lane; e < nb; e += 32) cp_async_4(dst + e, row + e);
        cp_async_arrive_noinc(&tab_bar[j & 1]);
        tab_pending |= 1u << (j & 1);
        tab_parity = (tab_parity & ~(1u << (j & 1))) | (((j >> 1) & 1u) << (j & 1));
      }
    };
    auto wait_table = [&](uint32_t j) {
      if constexpr (PAGED) {
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&tab_bar[j & 1], (j >> 1) & 1));
        if (!got && lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        tab_pending &= ~(1u << (j & 1));
        return got;
      }
      return true;
    };

    uint32_t idx0 = 0, idx1 = 0, idx2 = 0;  // items k, k + 1, k + 2 (lane 0)
    bool ok = true;
    if (lane == 0) {
      // CTA c starts with items c, c + G, c + 2G (G = grid size) of the
      // largest-first list, then takes more from the counter.
      idx0 = blockIdx.x;
      idx1 = blockIdx.x + gridDim.x;
      idx2 = blockIdx.x + 2 * gridDim.x;
      if (idx0 < n_items) copy_record(0, idx0);
      if (idx1 < n_items) copy_record(1, idx1);
    }
    if (__shfl_sync(0xffffffffu, idx0, 0) < n_items) {
      ok = wait_record(0);
      if (ok) fetch_table(0);
    }
    uint32_t issued = 0, st = 0, ph = 0;  // stages issued; ring slot and use parity of the next
    for (uint32_t k = 0; ok; ++k) {
      const int slot = k & (kItemSlots - 1);
      const uint32_t cur = __shfl_sync(0xffffffffu, idx0, 0);
      const uint32_t nx1 = __shfl_sync(0xffffffffu, idx1, 0);
      if (lane == 0 && k >= kItemSlots &&
          !mbar_wait_bounded(&item_empty[slot], ((k / kItemSlots) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (cur >= n_items) {
        if (lane == 0) {
          items[slot].s = -1;  // no more work
          mbar_arrive(&item_full[slot]);
        }
        break;
      }
      uint32_t idx3 = 0;
      if (lane == 0) {
        if (idx2 < n_items) {
          fence_proxy_async_smem();  // this record slot was last read two items ago
          copy_record(k + 2, idx2);
        }
        idx3 = atomicAdd(a.work, 1u);
      }
      if (nx1 < n_items) {
        // record k + 1 was requested one item ago; fetch its table now
        if (!wait_record(k + 1)) break;
        fetch_table(k + 1);
      }
      if (!wait_table(k)) break;  // requested one item ago
      const int32_t* rec = rec_slot(k);
      const int s = rec[0], part = rec[1], n_parts = rec[2], t_begin = rec[3], n_tok = rec[4];
      const int kvh = static_cast<int>(cur % Hkv);
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
      const int32_t* tab = s_tab + (k & 1) * Tr::MAX_TABLE;
      const int n_stages = (n_tok + TS - 1) / TS;
      for (int i = 0; i < n_stages; ++i) {
        if (lane == 0 && issued >= STAGES && !mbar_wait_bounded(&empty[st], ph ^ 1)) {
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
          ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const int t0 = i * TS;  // relative to the partition start (block aligned)
        if (lane == 0) mbar_arrive_expect_tx(&full[st], 2u * min(TS, n_tok - t0) * Tr::ROW_BYTES);
        __syncwarp();
        const int tc = t0 + lane * Tr::CH;
        if (lane < Tr::NCH && tc < n_tok) {
          const uint32_t nbytes = min(Tr::CH, n_tok - tc) * Tr::ROW_BYTES;
          int64_t row;
          if constexpr (PAGED) {
            int32_t f = tab[tc / B];
            if (f < 0 || f >= a.num_blocks) {
              set_error(a.err, PKV_DEVERR_TABLE_ENTRY);
              f = 0;
            }
            row = (static_cast<int64_t>(f) * a.num_kv_heads + kvh) * B + tc % B;
          } else {
            row = (static_cast<int64_t>(s) * a.num_kv_heads + kvh) * a.max_ctx + t_begin + tc;
          }
          uint8_t* sk = smem + st * Tr::STAGE_BYTES + lane * Tr::CH * Tr::ROW_BYTES;
          bulk_load(sk, kbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
          bulk_load(sk + Tr::TILE_BYTES, vbase + row * Tr::ROW_BYTES, nbytes, &full[st]);
        }
        __syncwarp();
        ++issued;
        if (++st == STAGES) {
          st = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;  // the consumers time out on their next wait and stop too
      idx0 = idx1;
      idx1 = idx2;
      idx2 = idx3;
    }
    // Never leave the CTA with copies in flight: wait (bounded) until the last
    // use of every stage, and every record and table copy, have landed.
    if (lane == 0) {
      const uint32_t first = issued > STAGES ? issued - STAGES : 0;
      for (uint32_t i = first; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % STAGES], (i / STAGES) & 1))
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    for (int r = 0; r < kRecSlots; ++r)
      if (lane == 0 && ((rec_pending >> r) & 1u) &&
          !mbar_wait_bounded(&rec_bar[r], (rec_parity >> r) & 1u))
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    for (int b = 0; b < 2; ++b)
      if (((tab_pending >> b) & 1u) && !mbar_wait_bounded(&tab_bar[b], (tab_parity >> b) & 1u) &&
          lane == 0)
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
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
  uint32_t st = 0, ph = 0;  // ring slot and use parity of the next stage

  for (uint32_t k = 0;; ++k) {
    const int slot = k & (kItemSlots - 1);
    const bool arrived = mbar_wait_bounded(&item_full[slot], (k / kItemSlots) & 1);
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
      for (int kk = 0; kk < DPL / 2; ++kk) acc[g][kk] = make_float2(0.f, 0.f);

    // One stage: scores of this warp's TPW tokens, online softmax, PV.  FULL
    // stages (all TS tokens valid) skip the masking and the early exits.
    auto stage = [&](const T* sK, const T* sV, int nv, auto full_tag) {
      constexpr bool FULL = decltype(full_tag)::value;
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
        if constexpr (FULL)
          sc[r] = x[0];
        else
          sc[r] = tok < nv ? x[0] : -CUDART_INF_F;
      }

      // online softmax for head my_h
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
          for (int kk = 0; kk < DPL / 2; ++kk) acc[g][kk] = fmul2(acc[g][kk], a2);
        }
        m_run = m_new;
      }
#pragma unroll
      for (int r = 0; r < ROUNDS; ++r) {
        float p;
        if constexpr (FULL)
          p = fast_exp2(sc[r] - m_run);
        else
          p = sc[r] == -CUDART_INF_F ? 0.f : fast_exp2(sc[r] - m_run);
        if (p_writer) {
          p_warp[(r * TPR + tg) * G + my_h] = make_float2(p, p);
          l_lane += p;
        }
      }
      __syncwarp();

      // PV over this warp's valid tokens
#pragma unroll
      for (int j = 0; j < TPW; ++j) {
        if constexpr (!FULL) {
          if (w_tok0 + j >= nv) break;
        }
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
          for (int kk = 0; kk < DPL / 2; ++kk) acc[g][kk] = ffma2(pj[g], vf[kk], acc[g][kk]);
      }
    };

    const int n_stages = (info.n_tok + TS - 1) / TS;
    bool ok = true;
    for (int i = 0; i < n_stages; ++i) {
      if (!mbar_wait_bounded(&full[st], ph)) {
        if (lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
        break;
      }
      const T* sK = reinterpret_cast<const T*>(smem + st * Tr::STAGE_BYTES);
      const T* sV = sK + TS * D;
      const int nv = info.n_tok - i * TS;
      if (nv >= TS)
        stage(sK, sV, TS, std::true_type{});
      else
        stage(sK, sV, nv, std::false_type{});
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == STAGES) {
        st = 0;
        ph ^= 1;
      }
    }

    // ---- merge the four warps of this item, HG heads per round
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, m);
    if (tg == 0 && p_writer) {
      s_m[warp * G + my_h] = m_run;
      s_l[warp * G + my_h] = l_lane;
    }
    if (named_barrier_or(1, NW * 32, !ok)) break;  // a timed-out stage: stop, output invalid

    const int s = info.s;
    const bool single = info.n_parts == 1;
    constexpr int HG = Tr::HG;
#pragma unroll
    for (int r = 0; r < G / HG; ++r) {
      if (r > 0) named_barrier_sync(1, NW * 32);  // previous round's reads are done
#pragma unroll
      for (int gg = 0; gg < HG; ++gg)
#pragma unroll
        for (int kk = 0; kk < DPL / 2; ++kk)
          *reinterpret_cast<float2*>(s_acc + (warp * HG + gg) * D + lane * DPL + 2 * kk) = acc[r * HG + gg][kk];
      named_barrier_sync(1, NW * 32);
      for (int idx = threadIdx.x; idx < HG * D; idx += NW * 32) {
        const int gg = idx / D, d = idx % D;
        const int g = r * HG + gg;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m[w * G + g]);
        float lsum = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float mw = s_m[w * G + g];
          const float f = mw == -CUDART_INF_F ? 0.f : fast_exp2(mw - M);
          lsum += f * s_l[w * G + g];
          o += f * s_acc[(w * HG + gg) * D + d];
        }
        if (single) {
          static_cast<T*>(a.out)[(static_cast<int64_t>(s) * a.num_heads + h0 + g) * D + d] =
              from_float<T>(lsum > 0.f ? o / lsum : 0.f);
        } else {
          const int64_t cell = (static_cast<int64_t>(s) * a.num_heads + h0 + g) * a.max_parts + info.part;
          a.tmp_out[cell * D + d] = o / lsum;
          if (d == 0) {
            a.tmp_m[cell] = M;
            a.tmp_l[cell] = lsum;
          }
        }
      }
    }
    named_barrier_sync(1, NW * 32);  // s_acc, s_m, s_l are free again
  }
}

// ---------------------------------------------------------------- merge
// Contexts that span several partitions: out = sum_p w_p o_p with
// w_p = l_p 2^(m_p - M) / sum_q l_q 2^(m_q - M), M = max_p m_p, summed in
// partition order.  One CTA of 128 threads per (sequence, kv head) pair listed
// by the plan kernel (grid-stride when there are more pairs than CTAs).  The
// outputs of the first kPre partitions are loaded into registers up front, so
// with up to kPre partitions a pair costs about one memory round trip.
// Launched behind the decode grid (programmatic dependent launch): it waits for
// the whole decode grid before reading its results.
constexpr int kMergeThreads = 128;
constexpr int kMergeStat = 64;  // partitions per statistics round
constexpr int kPre = 8;         // partitions per output round

template <typename T, int D, int G>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const DecodeArgs a) {
  __shared__ float s_m[G][kMergeStat], s_l[G][kMergeStat], s_w[G][kPre];
  __shared__ float s_M[G], s_L[G];
  grid_dependency_wait();
  constexpr int kPer = (G * D + kMergeThreads - 1) / kMergeThreads;
  const uint32_t Hkv = static_cast<uint32_t>(a.num_kv_heads);
  const uint32_t n_tasks = a.work[2] * Hkv;
  for (uint32_t t = blockIdx.x; t < n_tasks; t += gridDim.x) {
    const int s = a.merge_seqs[t / Hkv];
    const int h0 = static_cast<int>(t % Hkv) * G;
    int np, psize;
    partition_of(clamp_len(a.lens[s], a.max_ctx), a.part_tokens, np, psize);
    const int64_t base0 = (static_cast<int64_t>(s) * a.num_heads + h0) * a.max_parts;
    auto cell = [&](int g, int p) { return base0 + static_cast<int64_t>(g) * a.max_parts + p; };

    float pre[kPre][kPer];  // outputs of partitions 0 .. kPre-1
#pragma unroll
    for (int p = 0; p < kPre; ++p)
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int idx = threadIdx.x + k * kMergeThreads;
        pre[p][k] = (p < np && idx < G * D) ? a.tmp_out[cell(idx / D, p) * D + idx % D] : 0.f;
      }

    // M and the normaliser per head, online over rounds of kMergeStat partitions
    if (threadIdx.x < G) {
      s_M[threadIdx.x] = -CUDART_INF_F;
      s_L[threadIdx.x] = 0.f;
    }
    for (int c0 = 0; c0 < np; c0 += kMergeStat) {
      const int cn = min(kMergeStat, np - c0);
      for (int i = threadIdx.x; i < G * cn; i += kMergeThreads) {
        const int g = i / cn, p = i % cn;
        s_m[g][p] = a.tmp_m[cell(g, c0 + p)];
        s_l[g][p] = a.tmp_l[cell(g, c0 + p)];
      }
      __syncthreads();
      if (threadIdx.x < G) {
        const int g = threadIdx.x;
        float M = s_M[g];
        for (int p = 0; p < cn; ++p) M = fmaxf(M, s_m[g][p]);
        float L = s_L[g] * fast_exp2(s_M[g] - M);  // 0 on the first round
        for (int p = 0; p < cn; ++p) L += s_l[g][p] * fast_exp2(s_m[g][p] - M);
        s_M[g] = M;
        s_L[g] = L;
      }
      __syncthreads();
    }

    float o_reg[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) o_reg[k] = 0.f;
    for (int p0 = 0; p0 < np; p0 += kPre) {
      const int pc = min(kPre, np - p0);
      if (threadIdx.x < G * pc) {
        const int g = threadIdx.x / pc, p = threadIdx.x % pc;
        s_w[g][p] = a.tmp_l[cell(g, p0 + p)] * fast_exp2(a.tmp_m[cell(g, p0 + p)] - s_M[g]) / s_L[g];
      }
      if (p0 > 0) {
#pragma unroll
        for (int p = 0; p < kPre; ++p)
#pragma unroll
          for (int k = 0; k < kPer; ++k) {
            const int idx = threadIdx.x + k * kMergeThreads;
            pre[p][k] = (p < pc && idx < G * D) ? a.tmp_out[cell(idx / D, p0 + p) * D + idx % D] : 0.f;
          }
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int idx = threadIdx.x + k * kMergeThreads;
        if (idx < G * D) {
          const int g = idx / D;
          float o = o_reg[k];
#pragma unroll
          for (int p = 0; p < kPre; ++p)
            if (p < pc) o += s_w[g][p] * pre[p][k];
          o_reg[k] = o;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int idx = threadIdx.x + k * kMergeThreads;
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
