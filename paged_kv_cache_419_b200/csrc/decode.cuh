// Paged decode attention for sm_100a.
//
// Method (vLLM and PagedAttention slides 9-10; dataarena note section 2): one
// query token per sequence attends over keys and values that sit in blocks of B
// tokens at arbitrary frames of a pool, found through the sequence's block table.
// Attention is softmax(scale q K^T) V, accumulated in fp32.
//
// Kernel design (B200).  The kernels are built to keep HBM busy; the
// contractions of the G query heads that share a kv head run as small
// tensor-core tiles only so that issuing them never holds the loads back.
//
//  * Work item = (sequence, kv head, context partition).  A context of L tokens
//    is cut into n = ceil(L / part_tokens) near-equal partitions whose sizes are
//    multiples of 64 tokens.  All G = Hq/Hkv query heads of the kv head share one
//    K/V fetch.
//  * plan_kernel (one CTA; it may become resident while the work before it on
//    the stream finishes, and waits for that work in-kernel) lists the items, largest first,
//    lists the contexts that span several partitions and zeroes their
//    completion counters.  Partition 0 of the first grid/Hkv sequences is not
//    listed: decode CTA c starts with it (sequence c / Hkv, kv head c % Hkv),
//    described from the context length alone, while the plan still runs.
//  * decode_kernel is persistent: (SM count x occupancy) CTAs, launched behind
//    the plan with programmatic dependent launch.  After its first item each
//    CTA takes items from the list with an atomic counter until it runs dry.
//  * Inside a CTA, warp 4 is the producer: it takes the next item, copies its q
//    rows into an item slot and streams the item's K and V through a ring of
//    two 64-token stages with TMA tensor copies (one 128-byte panel of a block
//    per box, 128-byte swizzle; the ragged end of a context in 8-row boxes).
//    It runs ahead across items, so the next item's data arrives while the
//    consumers finish the current one.  mbarriers hand stages (K and V halves
//    separately) and item slots over.
//  * Consumer warp w owns tokens 16w..16w+15 of each stage with its own
//    online-softmax state.  Scores: S^T = Q K^T as mma.sync m16n8k16 tiles (fp32
//    accumulation), K fragments read with ldmatrix from the swizzled stage, Q
//    fragments read from the item slot in every stage (rows padded against bank
//    conflicts; held in registers for the whole item they made the consumers
//    spill at their 128-register budget).  PV:
//    O^T += V^T P^T, P^T taken from the score accumulators as they lie (as two
//    16-bit parts, hi + lo, so that the weights keep about 16 significant bits),
//    V^T read with transposing ldmatrix.
//  * Epilogue per item: the four warps merge through shared memory in a fixed
//    order (bit-reproducible).  A one-partition context writes `out`; otherwise
//    the partition's normalised output, max and sum go to the workspace.  Each
//    multi-partition item is published as soon as it is written (a release
//    increment of its (sequence, kv head) counter), and merge_kernel, which runs
//    in the decode grid's tail, merges each such context (log-sum-exp) into
//    `out` as soon as its count is complete.
//  * Scores are kept in base-2 units (scale * log2 e folded into one multiply),
//    so the exponentials are single ex2 instructions.
#pragma once

#include <cuda.h>
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
  int32_t part_tokens;    // maximum tokens per partition (multiple of 64)
  int32_t max_parts;      // upper bound of partitions per context (workspace stride)
  int32_t balanced;       // 1: partitions sized per call from the batch's total work
  float scale_log2;       // scale * log2(e)
  int32_t grid_ctas;      // decode CTAs; item c (c < grid_ctas) is CTA c's first item
  uint32_t* work;         // [0] next item, [1] item count, [2] multi-partition sequences,
                          // [4..5] (balanced) the batch's token-heads U as a uint64
  uint32_t* pair_done;    // [S * Hkv] partitions published per (sequence, kv head)
  int32_t* merge_seqs;    // [S] sequences whose context spans more than one partition
  uint8_t* records;       // [S * max_parts] work records, largest partition first (32 B each)
  float* tmp_out;         // [S, Hq, max_parts, D]
  float* tmp_m;           // [S, Hq, max_parts]
  float* tmp_l;           // [S, Hq, max_parts]
  unsigned int* err;
  // Bound of the merge grid's wait for a pair's partitions, and extra
  // publications it waits for beyond the partition count (0 except under the
  // bounded-wait test hook, which makes the wait run out on purpose).
  unsigned long long merge_wait_limit_ns;
  uint32_t merge_wait_extra;
};

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxPartTokens = 2048;  // largest partition_size a caller may ask for
// Block-table entries of one item (a shared-memory buffer of the producer): the
// balanced policy's partitions reach kMaxTableEntries x block_size tokens
// (2048 at 8-token blocks, 8192 at 32).
constexpr int kMaxTableEntries = 256;
constexpr int kMaxBalancedPartTokens = kMaxTableEntries * 32;
constexpr int kPlanThreads = 1024;
constexpr int kItemSlots = 2;
constexpr int kRecSlots = 2;   // records of items k and k+1
constexpr int kStageTokens = 64;
// Multi-partition items a CTA has finished and not yet published to the merge
// grid: at most one (it is published at the start of the next item, or at exit).
constexpr int kPubSlots = 2;
// Work record of one (sequence, partition): int32 s, part, n_parts, t_begin,
// n_tok, L, 0, 0.
constexpr int kRecordBytes = 32;

// Partitioning of a context of L tokens (L already clamped to [0, max_ctx]):
// n partitions of `size` tokens (a multiple of the 64-token stage), the last
// one shorter.  part_tokens is a multiple of 64, so size <= part_tokens.
__host__ __device__ __forceinline__ void partition_of(int L, int part_tokens, int& n, int& size) {
  if (L <= 0) {
    n = 1;
    size = 0;
    return;
  }
  const int n0 = (L + part_tokens - 1) / part_tokens;
  size = ((L + n0 - 1) / n0 + kStageTokens - 1) & ~(kStageTokens - 1);
  n = (L + size - 1) / size;
}

// Balanced partitioning, for batches with fewer (sequence, kv head) pairs than
// decode CTAs: there, fixed-size partitions leave a last wave of a few items
// on an otherwise idle grid.  The batch's U = Hkv x sum L token-heads are cut
// into at most k x grid items of near-equal size (k whole waves of the grid):
// k = round(U / (grid x 2048)), raised to the fewest waves whose items fit in
// max_part tokens, and at least 1.  One item per CTA while a CTA's share stays
// below ~3 K tokens: an item boundary costs a CTA about 2 us of its streaming
// time, more than a finer split recovers in balance.  A context of L tokens
// gets n = floor(L k grid / U) partitions (so the batch makes at most k x grid
// items), at least ceil(L / max_part), at most max_parts and ceil(L / 64), of
// equal size rounded up to a multiple of 64 (the last one shorter).  Integer
// arithmetic only: the plan, the statically started CTAs and the merge agree.
// k of the balanced rule: round(U / (grid x 2048)), raised to the fewest waves
// whose items fit in max_part tokens, at least 1.
__host__ __device__ __forceinline__ long long balanced_waves(long long uu, long long g, long long max_part) {
  long long k = (uu + g * 1024) / (g * 2048);
  const long long k_fit = (uu + g * max_part - 1) / (g * max_part);
  if (k < k_fit) k = k_fit;
  return k < 1 ? 1 : k;
}

__host__ __device__ __forceinline__ void partition_balanced(int L, unsigned long long U, int grid,
                                                            int max_parts, int max_part, int& n,
                                                            int& size) {
  if (L <= 0 || U == 0) {
    n = 1;
    size = L > 0 ? L : 0;
    return;
  }
  const long long g = grid, uu = static_cast<long long>(U);
  const long long k = balanced_waves(uu, g, max_part);
  long long nn = static_cast<long long>(L) * k * g / uu;
  const long long lo = (L + max_part - 1) / max_part;
  const long long by_stage = (L + 63) / 64;
  const long long hi = max_parts < by_stage ? max_parts : by_stage;
  nn = nn < lo ? lo : nn;
  nn = nn > hi ? hi : nn;
  if (nn < 1) nn = 1;
  size = ((L + static_cast<int>(nn) - 1) / static_cast<int>(nn) + kStageTokens - 1) & ~(kStageTokens - 1);
  n = (L + size - 1) / size;
}

// Partitions of a context of L tokens under this call's policy (U: the batch's
// token-heads, used by the balanced policy only).
__host__ __device__ __forceinline__ void partition_for(int L, const DecodeArgs& a,
                                                       unsigned long long U, int& n, int& size) {
  if (a.balanced)
    partition_balanced(L, U, a.grid_ctas, a.max_parts, a.part_tokens, n, size);
  else
    partition_of(L, a.part_tokens, n, size);
}

// Partitions of the round-robin schedule, two sizes.  With one static item
// per CTA the grid's finishing times spread with the SMs' streaming rates (per
// SM mean item time 55-70 us on the long batch), and the last CTAs stream alone.
// So each context is cut into "big" partitions of p_big ~ 7/8 of a CTA's
// share, U / (k grid) token-heads, rounded up to a multiple of 64 (at most
// floor(7/8 L / p_big) of them, so the batch has at most k x grid big items,
// handed out round-robin), followed by "small" partitions of p_small ~ p_big / 4
// for the rest, which CTAs claim one at a time from a counter near the end of
// their current item: the fast SMs take more of them.  The split applies when
// p_small would reach 256 tokens; then p_small grows if needed so that a
// context keeps within max_parts partitions.  Otherwise, and off the round-robin
// schedule, every partition is a big one by the balanced rule (n_big = n).
// Partition p < n_big covers tokens [p p_big, (p + 1) p_big); partition
// n_big + q covers [n_big p_big + q p_small, ...), the last one shorter.  Per
// sequence and from U alone: the plan, the decode grid and the merge agree.
constexpr int kBigNum = 14, kBigDen = 16, kSmallDiv = 4, kMinSmallTokens = 256;
constexpr int kClaimLead = 3;
__host__ __device__ __forceinline__ void partition_rr(int L, const DecodeArgs& a,
                                                      unsigned long long U, int& n_big, int& n,
                                                      int& p_big, int& p_small) {
  const long long g = a.grid_ctas, uu = static_cast<long long>(U);
  const long long k = uu > 0 ? balanced_waves(uu, g, a.part_tokens) : 1;
  long long pb = uu > 0 ? (uu * kBigNum + k * g * kBigDen - 1) / (k * g * kBigDen) : 0;
  pb = (pb + kStageTokens - 1) & ~static_cast<long long>(kStageTokens - 1);
  if (pb > a.part_tokens) pb = a.part_tokens;
  long long ps = (pb / kSmallDiv + kStageTokens - 1) & ~static_cast<long long>(kStageTokens - 1);
  if (L <= 0 || uu == 0 || ps < kMinSmallTokens) {  // one size: the balanced rule
    int size = 0;
    partition_balanced(L, U, a.grid_ctas, a.max_parts, a.part_tokens, n, size);
    n_big = n;
    p_big = p_small = size;
    return;
  }
  const long long nb = static_cast<long long>(L) * kBigNum / (kBigDen * pb);
  const long long rest = L - nb * pb;
  long long ns = (rest + ps - 1) / ps;
  if (nb + ns > a.max_parts) {  // fewer, larger small partitions (max_parts > nb here)
    const long long room = a.max_parts - nb > 0 ? a.max_parts - nb : 1;
    ps = (((rest + room - 1) / room) + kStageTokens - 1) & ~static_cast<long long>(kStageTokens - 1);
    ns = (rest + ps - 1) / ps;
  }
  n_big = static_cast<int>(nb);
  n = static_cast<int>(nb + (ns > 0 ? ns : 0));
  if (n < 1) n = 1;  // L > 0 here, so rest > 0 when nb = 0
  p_big = static_cast<int>(pb);
  p_small = static_cast<int>(ps);
}

// Round-robin schedule: under the balanced policy the items are near-equal by
// construction, so no largest-first list is needed.  With at most
// kRoundRobinSeqs sequences (two per lane of a warp), each decode CTA c takes
// items c, c + grid, c + 2 grid, ... of the enumeration (sequence, partition,
// kv head), kv head fastest, which it computes from the context lengths alone:
// no CTA waits for the planning kernel's list.
constexpr int kRoundRobinSeqs = 64;
__host__ __device__ __forceinline__ bool round_robin(const DecodeArgs& a) {
  return a.balanced && a.num_seqs <= kRoundRobinSeqs;
}

// The call's partition policy once the decode grid is known (host, at launch):
// the default size becomes the balanced policy when the batch has fewer
// (sequence, kv head) pairs than CTAs (then every pair's partition 0 is a
// static first item, and a partition may take a whole table buffer:
// kMaxTableEntries blocks, part_tokens = its largest size).
inline void apply_partition_policy(DecodeArgs& a, int grid, int block_size, bool paged) {
  a.grid_ctas = grid;
  if (a.balanced) {
    a.balanced = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads < grid ? 1 : 0;
    if (a.balanced) a.part_tokens = paged ? kMaxTableEntries * block_size : kMaxPartTokens;
  }
}

// Sequences whose partition 0 runs as a static first item: decode CTA c
// (c < this * Hkv) starts with partition 0 of sequence c / Hkv, kv head c % Hkv,
// computed from the inputs alone, so it does not wait for the plan; the plan
// lists every other (sequence, partition).
__device__ __forceinline__ int static_first_seqs(const int num_seqs, const int grid_ctas, const int Hkv) {
  const int n = grid_ctas / Hkv;
  return n < num_seqs ? n : num_seqs;
}

__host__ __device__ __forceinline__ int clamp_len(int L, int max_ctx) {
  return L < 0 ? 0 : (L > max_ctx ? max_ctx : L);
}

// Rows of a full box: one cache block (paged, blocks up to a stage long) or a
// whole stage (contiguous).
constexpr int chunk_rows(bool paged, int block_size) {
  return paged ? (block_size < kStageTokens ? block_size : kStageTokens) : kStageTokens;
}

// Tensor maps of the K and V caches, built on the host for each call.  A cache
// is viewed as [planes][rows][D] (paged: [N][Hkv * B][D]; contiguous:
// [S * Hkv][max_ctx][D]).  A box is one 128-byte panel (64 elements) of D wide
// and stored with the 128-byte swizzle: 16-byte chunk c of tile row r lands at
// chunk c ^ (r % 8) of that row.  `k`, `v` copy a full chunk of CH rows;
// `k_tail`, `v_tail` 8 rows, for the ragged end of a context.
struct DecodeMaps {
  CUtensorMap k, v, k_tail, v_tail;
};

template <typename T, int D_, int G_, int B_, bool PAGED_>
struct DecodeTraits {
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr int B = B_;
  static constexpr bool PAGED = PAGED_;
  static constexpr int TS = kStageTokens;                    // tokens per stage
  static constexpr int TPW = TS / kConsumerWarps;            // tokens per warp per stage
  static constexpr int KS = D / 16;                          // k-steps of the score tile
  static constexpr int MT = D / 16;                          // 16-dim m-tiles of the output tile
  static constexpr int ND = D / 64;                          // 128-byte panels per row
  static constexpr int CH = chunk_rows(PAGED, B);            // rows per full box
  static constexpr int NCH = TS / CH;
  static constexpr int STAGES = 2;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int PANEL_BYTES = TS * 128;               // one panel of a stage tile
  static constexpr int TILE_BYTES = ND * PANEL_BYTES;        // K (or V) of one stage
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int Q_BYTES = G * D * 2;
  // Q slot in shared memory: one row per head, rows 16 bytes apart beyond
  // their 2D bytes, so that the 8 heads' 32-bit reads of one instruction fall
  // in different banks.
  static constexpr int Q_PITCH = ROW_BYTES + 16;
  static constexpr int Q_SLOT = G * Q_PITCH;
  static constexpr int ACC_PITCH = D + 4;                    // floats per head row of a merge slot
  static constexpr int HG = G <= 2 ? G : G / 2;              // heads per merge round
  static constexpr int MAX_TABLE = PAGED ? kMaxTableEntries : 4;  // table entries of one item
  // shared memory carve-up (bytes from a 1024-byte aligned base)
  static constexpr int OFF_Q = STAGES * STAGE_BYTES;
  static constexpr int OFF_ACC = OFF_Q + kItemSlots * Q_SLOT;          // [warps][HG][ACC_PITCH] f32
  static constexpr int OFF_REC = OFF_ACC + kConsumerWarps * HG * ACC_PITCH * 4;  // record slots
  static constexpr int OFF_TAB = OFF_REC + kRecSlots * kRecordBytes;    // 2 table buffers
  static constexpr int OFF_STAT = OFF_TAB + 2 * MAX_TABLE * 4;          // m, l per warp and head
  static constexpr int OFF_ITEM = OFF_STAT + 2 * kConsumerWarps * G * 4 + 16;
  static constexpr int OFF_PUB = OFF_ITEM + kItemSlots * 32;           // pairs awaiting publication
  static constexpr int OFF_BARS = OFF_PUB + (kPubSlots + 2) * 4;
  static constexpr int SMEM_USED = OFF_BARS + (4 * STAGES + 2 * kItemSlots + kRecSlots + 2) * 8;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base

  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static_assert(G <= 8, "one 8-column n-tile holds the heads of a group");
  static_assert(TPW == 16, "a warp's tokens are one 16-deep k-step of the output tile");
  static_assert(CH % 8 == 0 && TS % CH == 0 && NCH * ND <= 32, "one copier lane per box");
  static_assert(STAGE_BYTES % 1024 == 0 && PANEL_BYTES % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(OFF_BARS % 8 == 0 && OFF_STAT % 16 == 0 && OFF_ACC % 16 == 0, "alignment");
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
constexpr int kPlanDirect = 8;   // partitions a thread writes itself
constexpr int kPlanWide = 512;   // sequences listed for warp-wide record writing

static __global__ void __launch_bounds__(kPlanThreads) plan_kernel(const DecodeArgs a) {
  // This grid may be launched while its predecessor on the stream still runs
  // (programmatic dependent launch): wait here until the predecessor has
  // completed and its writes are visible.  Then the decode grid may start: its
  // static first items read only inputs, and it waits for this grid before it
  // touches anything written here.
  grid_dependency_wait();
  allow_dependent_launch();
  const int n_static = static_first_seqs(a.num_seqs, a.grid_ctas, a.num_kv_heads);
  constexpr int kMaxClasses = kMaxBalancedPartTokens / 32 + 2;
  __shared__ uint32_t count[kMaxClasses];
  __shared__ uint32_t cursor[kMaxClasses];
  __shared__ uint32_t total, n_multi, n_wide;
  __shared__ int4 s_wide[kPlanWide];  // (sequence, first full-size slot, last slot, first listed partition)
  __shared__ int s_len[kPlanSmemSeqs];
  __shared__ unsigned long long s_U;
  const int classes = a.part_tokens / 32 + 2;  // class c: size in (part - 32(c+1), part - 32c]; last: empty
  const bool cached = a.num_seqs <= kPlanSmemSeqs;
  for (int c = threadIdx.x; c < classes; c += blockDim.x) count[c] = 0;
  if (threadIdx.x == 0) {
    total = n_multi = n_wide = 0;
    s_U = 0ull;
  }
  __syncthreads();
  // Balanced policy: the batch's token-heads first (the merge grid reads them too).
  unsigned long long U = 0;
  if (a.balanced) {
    unsigned long long mine = 0;
    for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x)
      mine += static_cast<unsigned long long>(clamp_len(a.lens[s], a.max_ctx));
    atomicAdd(&s_U, mine);
    __syncthreads();
    U = s_U * static_cast<unsigned long long>(a.num_kv_heads);
    if (threadIdx.x == 0) *reinterpret_cast<unsigned long long*>(a.work + 4) = U;
  }
  auto size_class = [&](int sz) { return sz == 0 ? classes - 1 : (a.part_tokens - sz) / 32; };
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int raw = a.lens[s];
    if (raw < 0 || raw > a.max_ctx) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    const int L = clamp_len(raw, a.max_ctx);
    if (cached) s_len[s] = L;
    int n, size;
    if (round_robin(a)) {  // no list: only the merge's sequences and counters
      int n_big, p_big, p_small;
      partition_rr(L, a, U, n_big, n, p_big, p_small);
    } else {
      partition_for(L, a, U, n, size);
      // listed partitions: skip .. n-1 (partition 0 of a static sequence is not
      // listed); partitions below n-1 have `size` tokens, the last one the rest
      const int skip = s < n_static ? 1 : 0;
      const int n_full = n - 1 - skip;
      if (n_full > 0) atomicAdd(&count[size_class(size)], static_cast<uint32_t>(n_full));
      if (n - 1 >= skip) atomicAdd(&count[size_class(L - (n - 1) * size)], 1u);
      atomicAdd(&total, static_cast<uint32_t>(n - skip));
    }
    if (n > 1) {
      a.merge_seqs[atomicAdd(&n_multi, 1u)] = s;
      for (int h = 0; h < a.num_kv_heads; ++h) a.pair_done[s * a.num_kv_heads + h] = 0u;
    }
  }
  __syncthreads();
  if (round_robin(a)) {  // every item is taken statically: no list to write
    if (threadIdx.x == 0) {
      a.work[0] = 0u;
      a.work[1] = 0u;
      a.work[2] = n_multi;
    }
    return;
  }
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
  // Records: one reservation per size class and sequence (its full-size
  // partitions take consecutive slots).  A sequence with more than
  // kPlanDirect partitions has its records written by a whole warp afterwards
  // (one lane per partition) instead of by one thread in a loop.  The first
  // records of the list (about one item per decode CTA: record r holds items
  // r * Hkv .. r * Hkv + Hkv - 1) are taken within microseconds of the start,
  // so their block-table entries are prefetched into L2 here.
  const uint32_t first_wave_records =
      (static_cast<uint32_t>(a.grid_ctas) + a.num_kv_heads - 1) / a.num_kv_heads;
  auto write_record = [&](int s, int p, int n, int size, int L, uint32_t pos) {
    const int t_begin = p * size;
    const int n_tok = min(size, L - t_begin);
    int4* rec = reinterpret_cast<int4*>(a.records + static_cast<int64_t>(pos) * kRecordBytes);
    rec[0] = make_int4(s, p, n, t_begin);
    rec[1] = make_int4(n_tok, L, 0, 0);
    if (a.tables != nullptr && pos < first_wave_records && n_tok > 0) {
      const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks + t_begin / a.block_size;
      const int nb = (n_tok + a.block_size - 1) / a.block_size;
      for (int e = 0; e < nb; e += 32) prefetch_l2(row + e);  // one per 128-byte line
      prefetch_l2(row + nb - 1);                                // the line of the last entry
    }
  };
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int L = cached ? s_len[s] : clamp_len(a.lens[s], a.max_ctx);
    int n, size;
    partition_for(L, a, U, n, size);
    const int last = L - (n - 1) * size;
    const int skip = s < n_static ? 1 : 0;
    const int n_full = n - 1 - skip;
    const uint32_t base = n_full > 0 ? atomicAdd(&cursor[size_class(size)], static_cast<uint32_t>(n_full)) : 0u;
    const uint32_t last_pos = n - 1 >= skip ? atomicAdd(&cursor[size_class(last)], 1u) : 0u;
    if (n > kPlanDirect) {
      const uint32_t i = atomicAdd(&n_wide, 1u);
      if (i < kPlanWide) {
        s_wide[i] = make_int4(s, static_cast<int>(base), static_cast<int>(last_pos), skip);
        continue;
      }
    }
    for (int p = skip; p < n; ++p)
      write_record(s, p, n, size, L, p < n - 1 ? base + static_cast<uint32_t>(p - skip) : last_pos);
  }
  __syncthreads();
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_w = min(static_cast<int>(n_wide), kPlanWide);
    for (int i = warp; i < n_w; i += kPlanThreads / 32) {
      const int4 e = s_wide[i];
      const int s = e.x;
      const int L = cached ? s_len[s] : clamp_len(a.lens[s], a.max_ctx);
      int n, size;
      partition_for(L, a, U, n, size);
      for (int p = e.w + lane; p < n; p += 32)
        write_record(s, p, n, size, L,
                     p < n - 1 ? static_cast<uint32_t>(e.y + p - e.w) : static_cast<uint32_t>(e.z));
    }
  }
  if (threadIdx.x == 0) {
    a.work[0] = 0u;  // next list item
    a.work[1] = total * static_cast<uint32_t>(a.num_kv_heads);
    a.work[2] = n_multi;
  }
}

// ---------------------------------------------------------------- decode
template <typename T, int D, int G, int B, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads, (G <= 4 ? 3 : 2))
    decode_kernel(const DecodeArgs a, const __grid_constant__ DecodeMaps maps) {
  using Tr = DecodeTraits<T, D, G, B, PAGED>;
  constexpr int STAGES = Tr::STAGES, TS = Tr::TS, TPW = Tr::TPW, KS = Tr::KS, MT = Tr::MT;
  constexpr int ND = Tr::ND;
  constexpr int NW = kConsumerWarps;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Swizzled tiles need a 1024-byte aligned base; the launch reserves the slack.
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  // K and V halves of a stage have their own barriers: K is released after the
  // scores, V after PV, so a half is refilled as soon as it is no longer read.
  uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BARS);
  uint64_t* full_v = full_k + STAGES;
  uint64_t* empty_k = full_v + STAGES;
  uint64_t* empty_v = empty_k + STAGES;
  uint64_t* item_full = empty_v + STAGES;
  uint64_t* item_empty = item_full + kItemSlots;
  uint64_t* rec_bar = item_empty + kItemSlots;  // [kRecSlots]
  uint64_t* tab_bar = rec_bar + kRecSlots;       // [2]
  ItemInfo* items = reinterpret_cast<ItemInfo*>(smem + Tr::OFF_ITEM);
  float* s_acc = reinterpret_cast<float*>(smem + Tr::OFF_ACC);
  float* s_m = reinterpret_cast<float*>(smem + Tr::OFF_STAT);
  float* s_l = s_m + NW * G;
  uint32_t* s_pub = reinterpret_cast<uint32_t*>(smem + Tr::OFF_PUB);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&full_v[i], 1);
      mbar_init(&empty_k[i], NW);
      mbar_init(&empty_v[i], NW);
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
  // The plan grid was launched in plain stream order and let this grid start,
  // so every input is ready here; what the plan writes (work list, counters) is
  // read only after grid_dependency_wait (plan_wait below).

  // ================================================================ producer
  // Item k (the k-th item this CTA takes).  CTAs below static_first_seqs * Hkv
  // start with partition 0 of sequence blockIdx.x / Hkv (kv head blockIdx.x %
  // Hkv), described from the inputs alone, while the plan is still running.
  // Every other item comes from the largest-first list through the work
  // counter, taken while the previous item streams: right after that item's
  // first stage is issued (a stage is in flight while the atomic returns), its
  // 32-byte record is bulk-copied; after the second stage (or at the end of a
  // one-stage item) the record has landed and its block-table entries are
  // fetched with cp.async.  Only one item is ever reserved ahead, so the end of
  // the list stays dynamic.
  if (warp == NW) {
    if (lane < 4) prefetch_tensor_map(&maps.k + lane);
    const uint32_t Hkv = static_cast<uint32_t>(a.num_kv_heads);
    uint32_t n_items = 0;
    bool plan_done = false;
    // Wait for the plan grid (its list and counters), then let the merge grid
    // launch: it also reads what the plan wrote.
    auto plan_wait = [&]() {
      if (!plan_done) {
        grid_dependency_wait();
        allow_dependent_launch();
        if (!round_robin(a)) n_items = *reinterpret_cast<volatile uint32_t*>(a.work + 1);
        plan_done = true;
      }
    };
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem + Tr::OFF_TAB);
    auto rec_slot = [&](uint32_t j) {
      return reinterpret_cast<const int32_t*>(smem + Tr::OFF_REC + (j & 1) * kRecordBytes);
    };
    // Outstanding copies nobody waited for yet (error exits drain them): bit r of
    // rec_pending / rec_parity = record slot r and the parity of its open phase;
    // likewise for the two table buffers.
    uint32_t rec_pending = 0, rec_parity = 0, tab_pending = 0, tab_parity = 0;
    auto copy_record = [&](uint32_t j, uint32_t idx) {  // lane 0; record j -> slot j % 2
      const uint32_t r = j & 1;
      fence_proxy_async_smem();  // this slot was last read two items ago
      mbar_arrive_expect_tx(&rec_bar[r], kRecordBytes);
      bulk_load(smem + Tr::OFF_REC + r * kRecordBytes,
                a.records + static_cast<int64_t>(idx / Hkv) * kRecordBytes, kRecordBytes, &rec_bar[r]);
      rec_pending |= 1u << r;
      rec_parity = (rec_parity & ~(1u << r)) | (((j >> 1) & 1u) << r);
    };
    auto wait_record = [&](uint32_t j) {  // every lane reads the record, so every lane waits
      const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&rec_bar[j & 1], (j >> 1) & 1));
      if (lane == 0) {
        if (!got) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        rec_pending &= ~(1u << (j & 1));
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

    bool ok = true;
    const bool rr = round_robin(a);
    // Round-robin schedule (see round_robin and partition_rr): lane l describes
    // sequences l and l + 32: length, big and small partition counts, and the
    // index of its first big and first small (sequence, partition) pair in the
    // enumeration, all big pairs first.  Items (pair, kv head) below
    // n_items_big are taken round-robin, the rest from the claim counter.
    int rr_L[2] = {0, 0}, rr_nb[2] = {0, 0}, rr_ns[2] = {0, 0}, rr_fb[2] = {0, 0}, rr_fs[2] = {0, 0};
    int rr_pb[2] = {0, 0}, rr_ps[2] = {0, 0};  // big and small partition sizes
    uint32_t n_items_big = 0;
    auto rr_record = [&](uint32_t j, uint32_t idx) {  // whole warp; record of item idx -> slot j % 2
      const bool big = idx < n_items_big;
      const int pair = static_cast<int>((big ? idx : idx - n_items_big) / Hkv);
      int own = -1;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int f = big ? rr_fb[h] : rr_fs[h], c = big ? rr_nb[h] : rr_ns[h];
        if (pair >= f && pair < f + c) own = h;
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, own >= 0);
      const int src = __ffs(mask) - 1;  // exactly one lane owns the pair
      const int h = __shfl_sync(0xffffffffu, own, src);
      const int L = __shfl_sync(0xffffffffu, h ? rr_L[1] : rr_L[0], src);
      const int nb = __shfl_sync(0xffffffffu, h ? rr_nb[1] : rr_nb[0], src);
      const int ns = __shfl_sync(0xffffffffu, h ? rr_ns[1] : rr_ns[0], src);
      const int first = __shfl_sync(0xffffffffu, big ? (h ? rr_fb[1] : rr_fb[0]) : (h ? rr_fs[1] : rr_fs[0]), src);
      const int pbig = __shfl_sync(0xffffffffu, h ? rr_pb[1] : rr_pb[0], src);
      const int psmall = __shfl_sync(0xffffffffu, h ? rr_ps[1] : rr_ps[0], src);
      if (lane == 0) {
        int32_t* r = reinterpret_cast<int32_t*>(smem + Tr::OFF_REC + (j & 1) * kRecordBytes);
        const int q = pair - first;
        const int p = big ? q : nb + q;
        const int t_begin = big ? q * pbig : nb * pbig + q * psmall;
        r[0] = src + 32 * h;
        r[1] = p;
        r[2] = nb + ns;
        r[3] = t_begin;
        r[4] = min(big ? pbig : psmall, L - t_begin);
        r[5] = L;
        // complete the slot's barrier phase as a copy would have
        mbar_arrive(&rec_bar[j & 1]);
      }
      __syncwarp();
    };
    if (rr) {
      unsigned long long U = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = lane + 32 * h;
        rr_L[h] = t < a.num_seqs ? clamp_len(a.lens[t], a.max_ctx) : 0;
        U += static_cast<unsigned long long>(rr_L[h]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) U += __shfl_xor_sync(0xffffffffu, U, o);
      U *= static_cast<unsigned long long>(a.num_kv_heads);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = lane + 32 * h;
        int nb, n, pb, ps;
        partition_rr(rr_L[h], a, U, nb, n, pb, ps);
        rr_nb[h] = t < a.num_seqs ? nb : 0;  // 0 past the last sequence: no pair maps there
        rr_ns[h] = t < a.num_seqs ? n - nb : 0;
        rr_pb[h] = pb;
        rr_ps[h] = ps;
      }
      // exclusive prefixes of the big and small counts in sequence order
      // (sequences 0..31 on lanes 0..31, then 32..63)
      int b0 = rr_nb[0], b1 = rr_nb[1], s0 = rr_ns[0], s1 = rr_ns[1];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x0 = __shfl_up_sync(0xffffffffu, b0, o), x1 = __shfl_up_sync(0xffffffffu, b1, o);
        const int y0 = __shfl_up_sync(0xffffffffu, s0, o), y1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
          b0 += x0;
          b1 += x1;
          s0 += y0;
          s1 += y1;
        }
      }
      const int tb0 = __shfl_sync(0xffffffffu, b0, 31), ts0 = __shfl_sync(0xffffffffu, s0, 31);
      rr_fb[0] = b0 - rr_nb[0];
      rr_fb[1] = tb0 + b1 - rr_nb[1];
      rr_fs[0] = s0 - rr_ns[0];
      rr_fs[1] = ts0 + s1 - rr_ns[1];
      const uint32_t big_pairs = static_cast<uint32_t>(tb0 + __shfl_sync(0xffffffffu, b1, 31));
      const uint32_t small_pairs = static_cast<uint32_t>(ts0 + __shfl_sync(0xffffffffu, s1, 31));
      n_items_big = big_pairs * Hkv;
      n_items = (big_pairs + small_pairs) * Hkv;
    }
    // Next item under the round-robin schedule: the CTA's next big item, or a
    // claimed small one (the plan zeroed the claim counter: wait for it first).
    auto rr_next = [&](uint32_t after_big) {
      if (after_big < n_items_big) return after_big;
      plan_wait();
      uint32_t c = 0;
      if (lane == 0) c = n_items_big + atomicAdd(a.work, 1u);
      return __shfl_sync(0xffffffffu, c, 0);
    };
    const bool static_first =
        !rr &&
        blockIdx.x < static_cast<uint32_t>(static_first_seqs(a.num_seqs, a.grid_ctas, a.num_kv_heads)) * Hkv;
    uint32_t cur = 0;  // list index of the current item (items after a static first one)
    if (rr) {
      cur = rr_next(blockIdx.x);
      if (cur < n_items) {
        rr_record(0, cur);
        ok = wait_record(0);
        if (ok) fetch_table(0);
      }
    } else if (static_first) {
      const int s = static_cast<int>(blockIdx.x / Hkv);
      if constexpr (PAGED) {
        // The table entries are requested together with the context length, one
        // memory round trip for both: every entry partition 0 can use (at most
        // part_tokens / B, and never past the row), whatever the length turns
        // out to be.  Entries past the context are fetched but never used.
        const int cap = min(a.part_tokens / B, a.max_blocks);
        const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks;
        for (int e = lane; e < cap; e += 32) cp_async_4(s_tab + e, row + e);
        cp_async_arrive_noinc(&tab_bar[0]);
        tab_pending |= 1u;  // buffer 0, phase 0
      }
      // Balanced policy: the batch's token-heads, summed by the warp (a batch
      // with static items for every sequence has fewer than grid / Hkv of them).
      unsigned long long U = 0;
      if (a.balanced) {
        for (int t = lane; t < a.num_seqs; t += 32)
          U += static_cast<unsigned long long>(clamp_len(a.lens[t], a.max_ctx));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) U += __shfl_xor_sync(0xffffffffu, U, o);
        U *= static_cast<unsigned long long>(a.num_kv_heads);
      }
      if (lane == 0) {  // record of partition 0 of sequence blockIdx.x / Hkv, in slot 0
        int32_t* r = reinterpret_cast<int32_t*>(smem + Tr::OFF_REC);
        const int L = clamp_len(a.lens[s], a.max_ctx);
        int n, size;
        partition_for(L, a, U, n, size);
        r[0] = s;
        r[1] = 0;
        r[2] = n;
        r[3] = 0;
        r[4] = min(size, L);
        r[5] = L;
        // Complete phase 0 of the slot's barrier as a copy would have: slot 0
        // is next used by item 2, which waits for phase 1.
        mbar_arrive(&rec_bar[0]);
      }
      __syncwarp();
    } else {
      plan_wait();
      if (lane == 0) cur = atomicAdd(a.work, 1u);
      cur = __shfl_sync(0xffffffffu, cur, 0);
      if (cur < n_items) {
        if (lane == 0) copy_record(0, cur);
        ok = wait_record(0);
        if (ok) fetch_table(0);
      }
    }
    uint32_t issued = 0, st = 0, ph = 0;  // stages issued; ring slot and use parity of the next
    for (uint32_t k = 0; ok; ++k) {
      const int slot = k & (kItemSlots - 1);
      if (lane == 0 && k >= kItemSlots &&
          !mbar_wait_bounded(&item_empty[slot], ((k / kItemSlots) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const bool is_static = k == 0 && static_first;
      if (!is_static && cur >= n_items) {
        if (lane == 0) {
          items[slot].s = -1;  // no more work
          mbar_arrive(&item_full[slot]);
        }
        break;
      }
      if (!wait_table(k)) break;  // fetched while the previous item streamed
      const int32_t* rec = rec_slot(k);
      const int s = rec[0], part = rec[1], n_parts = rec[2], t_begin = rec[3], n_tok = rec[4];
      const int kvh = static_cast<int>((is_static ? blockIdx.x : cur) % Hkv);  // rr: cur = item
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
#pragma unroll
        for (int g = 0; g < G; ++g)
          bulk_load(smem + Tr::OFF_Q + slot * Tr::Q_SLOT + g * Tr::Q_PITCH, qsrc + g * Tr::ROW_BYTES,
                    Tr::ROW_BYTES, &item_full[slot]);
      }
      const int32_t* tab = s_tab + (k & 1) * Tr::MAX_TABLE;
      const int n_stages = (n_tok + TS - 1) / TS;
      uint32_t nxt = n_items;     // next item (lane 0 knows it after the first stage)
      bool next_ready = false;    // its record waited for and its table requested
      auto prepare_next = [&](int step) {
        if (step == 0) {
          if (!rr) plan_wait();
          if (rr) {
            nxt = rr_next(cur < n_items_big ? cur + gridDim.x : n_items_big);
            if (nxt < n_items) rr_record(k + 1, nxt);
          } else {
            if (lane == 0) {
              nxt = atomicAdd(a.work, 1u);
              if (nxt < n_items) copy_record(k + 1, nxt);
            }
            nxt = __shfl_sync(0xffffffffu, nxt, 0);
          }
        } else if (!next_ready) {
          next_ready = true;
          if (nxt < n_items) {
            if (!wait_record(k + 1)) return false;
            fetch_table(k + 1);
          }
        }
        return true;
      };
      // A claimed next item is claimed near the end of this one (kClaimLead
      // stages before it), so that a CTA takes more items the faster it streams;
      // a listed or round-robin one is prepared at once.
      const int prep_at = rr && cur + gridDim.x >= n_items_big ? max(0, n_stages - kClaimLead) : 0;
      for (int i = 0; i < n_stages; ++i) {
        const int t0 = i * TS;  // relative to the partition start (block aligned)
        // Boxes: full chunks of CH rows, the ragged end in 8-row boxes, so a
        // stage moves its valid rows rounded up to 8, per panel.
        const int nvs = min(TS, n_tok - t0);
        const uint32_t half_bytes = static_cast<uint32_t>((nvs + 7) & ~7) * Tr::ROW_BYTES;
        const int c = lane / ND, h = lane % ND;  // copier lane: chunk and panel
        const int tc = t0 + c * Tr::CH;
        const bool copier = c < Tr::NCH && tc < n_tok;
        int rows = 0, y = 0, z = 0;
        if (copier) {
          rows = min(Tr::CH, n_tok - tc);
          if constexpr (PAGED) {
            int32_t f = tab[tc / B];
            if (f < 0 || f >= a.num_blocks) {
              set_error(a.err, PKV_DEVERR_TABLE_ENTRY);
              f = 0;
            }
            y = kvh * B + tc % B;
            z = f;
          } else {
            y = t_begin + tc;
            z = s * static_cast<int>(Hkv) + kvh;
          }
        }
        uint8_t* dst = smem + st * Tr::STAGE_BYTES + h * Tr::PANEL_BYTES + c * Tr::CH * 128;
        auto issue = [&](uint8_t* d, const CUtensorMap* full, const CUtensorMap* tail, uint64_t* bar) {
          if (!copier) return;
          if (rows == Tr::CH) {
            tma_load_3d(d, full, h * 64, y, z, bar);
          } else {
            for (int r = 0; r < rows; r += 8) tma_load_3d(d + r * 128, tail, h * 64, y + r, z, bar);
          }
        };
        // K half: free once the consumers' scores of this slot's last use are done
        if (lane == 0 && issued >= STAGES && !mbar_wait_bounded(&empty_k[st], ph ^ 1)) {
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
          ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&full_k[st], half_bytes);
        __syncwarp();
        issue(dst, &maps.k, &maps.k_tail, &full_k[st]);
        __syncwarp();
        // V half: free once their PV is done
        if (lane == 0 && issued >= STAGES && !mbar_wait_bounded(&empty_v[st], ph ^ 1)) {
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
          ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&full_v[st], half_bytes);
        __syncwarp();
        issue(dst + Tr::TILE_BYTES, &maps.v, &maps.v_tail, &full_v[st]);
        __syncwarp();
        ++issued;
        if (++st == STAGES) {
          st = 0;
          ph ^= 1;
        }
        if ((i == prep_at || i == prep_at + 1) && !prepare_next(i - prep_at)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;  // the consumers time out on their next wait and stop too
      if (n_stages == 0 && !prepare_next(0)) break;
      if (!prepare_next(1)) break;  // one-stage (or empty) items: finish preparing now
      // The next item (or the end of the work) is handed over only after the
      // plan has finished: its counter reset precedes every publication.  (On
      // the list schedule prepare_next waited already; the round-robin schedule
      // reaches here first with its first item's stages in flight.)
      plan_wait();
      cur = nxt;
    }
    // Never leave the CTA with copies in flight: wait (bounded) until the last
    // use of every stage, and every record and table copy, have landed.
    if (lane == 0) {
      const uint32_t first = issued > STAGES ? issued - STAGES : 0;
      for (uint32_t i = first; i < issued; ++i)
        if (!mbar_wait_bounded(&full_k[i % STAGES], (i / STAGES) & 1) ||
            !mbar_wait_bounded(&full_v[i % STAGES], (i / STAGES) & 1))
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    for (int r = 0; r < 2; ++r)
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
  // Warp w owns tokens [16 w, 16 w + 16) of every stage, with its own online
  // softmax state per head; the tiles run on the tensor cores (mma.sync
  // m16n8k16, fp32 accumulation):
  //   scores  S^T (16 x 16) = Q (16 x D, rows >= G zero) K^T: two 8-token
  //           n-tiles, K read with ldmatrix straight from the swizzled stage;
  //   output  O^T (D x 8) += V^T (D x 16) P^T (16 x 8): V read with transposing
  //           ldmatrix, P^T taken from the score accumulators as they lie
  //           (their C layout is the B layout of the next product), as a hi
  //           and a lo 16-bit part, one product each.
  // Exits are decided together (barrier-OR over the consumer warps) so that no
  // warp is ever left waiting at a named barrier.
  const int quad = lane >> 2;  // score tile: head row; output tile: dim row
  const int qc = lane & 3;     // score tile: token pair; output tile: head pair
  const int w_tok0 = warp * TPW;
  // ldmatrix addressing: lane supplies row (lane & 7) of matrix (lane >> 3).
  // Swizzled offset of 16-byte chunk j of tile row r: r * 128 + ((j ^ (r & 7)) << 4);
  // the part of j that varies per call is applied with one xor.
  const int mrow = lane & 7, mat = lane >> 3;
  // K, matrix i of k-step pair kp: token w_tok0 + 8 nt + mrow, chunk 4 (kp & 1) + i
  // of panel kp / 2.
  const uint32_t k_lane = static_cast<uint32_t>((w_tok0 + mrow) * 128 + ((mat ^ mrow) << 4));
  // V, matrix i of m-tile mt: token w_tok0 + 8 (i >> 1) + mrow, chunk
  // 2 (mt & 3) + (i & 1) of panel mt / 4.
  const uint32_t v_lane =
      static_cast<uint32_t>((w_tok0 + 8 * (mat >> 1) + mrow) * 128 + (((mat & 1) ^ mrow) << 4));
  uint32_t st = 0, ph = 0;  // ring slot and use parity of the next stage
  // Publication (thread 0): the partial result of a multi-partition item is
  // announced to the merge grid by one gpu-scope release increment of its
  // (sequence, kv head) counter, right after the named barrier at the start of
  // the next item (or at exit), which orders every consumer thread's write-out
  // of the item before it.  Publishing each item as soon as it is written lets
  // the merge of a context start as soon as its last partition is done.
  // s_pub[kPubSlots] holds the count (thread 0 alone touches the list).
  // The plan grid zeroes the counters while this grid already runs (under the
  // round-robin schedule nothing else here waits for it), so thread 0 waits for
  // the plan to complete before its first increment; by then it has, one item
  // after the start.
  if (threadIdx.x == 0) s_pub[kPubSlots] = 0u;
  bool plan_seen = false;  // thread 0: the plan grid has completed
  auto publish = [&]() {
    const uint32_t n = s_pub[kPubSlots];
    if (n > 0 && !plan_seen) {
      grid_dependency_wait();
      plan_seen = true;
    }
    for (uint32_t i = 0; i < n; ++i) red_add_release_gpu(&a.pair_done[s_pub[i]], 1u);
    s_pub[kPubSlots] = 0u;
  };

  for (uint32_t k = 0;; ++k) {
    const int slot = k & (kItemSlots - 1);
    const bool arrived = mbar_wait_bounded(&item_full[slot], (k / kItemSlots) & 1);
    if (!arrived && lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    const ItemInfo info = items[slot];
    // Every consumer thread has finished the previous item's write-out here.
    if (named_barrier_or(1, NW * 32, !arrived || info.s < 0)) break;
    if (threadIdx.x == 0) publish();
    const int h0 = info.kvh * G;

    // Q as the A operand, read from the item's Q slot in each stage (the slot is
    // released after the item's last stage): lane holds head `quad`, dims
    // 16 ks + 2 qc (+1) and the same + 8 (zero for rows >= G).
    const uint8_t* sq = smem + Tr::OFF_Q + slot * Tr::Q_SLOT + quad * Tr::Q_PITCH + 2 * qc * 2;

    float m_run = -CUDART_INF_F;  // running max of head `quad` over this warp's tokens (base 2)
    float l_lane = 0.f;           // sum of this lane's probabilities of head `quad`
    // O^T accumulators: acc[mt][0], [1] = dim 16 mt + quad of heads 2 qc, 2 qc + 1;
    // acc[mt][2], [3] = the same for dim + 8.
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // One stage.  FULL stages (all TS tokens valid) skip the masking.
    auto stage = [&](uint32_t sK, uint8_t* pV, int nv, auto full_tag) -> bool {
      constexpr bool FULL = decltype(full_tag)::value;
      const uint32_t sV = sK + Tr::TILE_BYTES;
      // ---- scores, one accumulation chain per 8-token n-tile
      float sacc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t kb[4];
          ldmatrix_x4(kb, sK + (kp >> 1) * Tr::PANEL_BYTES + nt * 1024 + (k_lane ^ ((kp & 1) << 6)));
          const uint32_t q00 = quad < G ? *reinterpret_cast<const uint32_t*>(sq + 2 * kp * 32) : 0u;
          const uint32_t q01 = quad < G ? *reinterpret_cast<const uint32_t*>(sq + 2 * kp * 32 + 16) : 0u;
          const uint32_t q10 = quad < G ? *reinterpret_cast<const uint32_t*>(sq + 2 * kp * 32 + 32) : 0u;
          const uint32_t q11 = quad < G ? *reinterpret_cast<const uint32_t*>(sq + 2 * kp * 32 + 48) : 0u;
          const uint32_t a0[4] = {q00, 0u, q01, 0u};
          const uint32_t a1[4] = {q10, 0u, q11, 0u};
          mma_16816<T>(sacc[nt], a0, kb[0], kb[1]);
          mma_16816<T>(sacc[nt], a1, kb[2], kb[3]);
        }
      }
      // x[nt][e]: head quad, token w_tok0 + 8 nt + 2 qc + e, in base-2 units
      float x[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          x[nt][e] = sacc[nt][e] * a.scale_log2;
          if constexpr (!FULL) {
            if (w_tok0 + 8 * nt + 2 * qc + e >= nv) x[nt][e] = -CUDART_INF_F;
          }
        }
      // this warp is done reading the K half
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_k[st]);

      // ---- online softmax, per head over the quad's lanes
      float mx = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float alpha = m_new == m_run ? 1.f : fast_exp2(m_run - m_new);  // 0 when m_run = -inf
        l_lane *= alpha;
        // this lane's output columns are heads 2 qc and 2 qc + 1
        const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * qc);
        const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * qc + 4);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          acc[mt][0] *= a_lo;
          acc[mt][1] *= a_hi;
          acc[mt][2] *= a_lo;
          acc[mt][3] *= a_hi;
        }
        m_run = m_new;
      }
      float p[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if constexpr (FULL)
            p[nt][e] = fast_exp2(x[nt][e] - m_run);
          else
            p[nt][e] = x[nt][e] == -CUDART_INF_F ? 0.f : fast_exp2(x[nt][e] - m_run);
          l_lane += p[nt][e];
        }
      // P^T as the B operand (k = token, n = head), split into two 16-bit parts:
      // hi = p rounded to the input type, lo = the rest (p - hi, exact in fp32)
      // rounded again.  Two products with the same V fragments then carry p to
      // about 16 significant bits, so the weights that multiply V agree with the
      // fp32 weights the normaliser sums.
      const uint32_t pb0 = pack2<T>(p[0][0], p[0][1]);
      const uint32_t pb1 = pack2<T>(p[1][0], p[1][1]);
      const float2 h0 = unpack2<T>(pb0), h1 = unpack2<T>(pb1);
      const uint32_t pl0 = pack2<T>(p[0][0] - h0.x, p[0][1] - h0.y);
      const uint32_t pl1 = pack2<T>(p[1][0] - h1.x, p[1][1] - h1.y);
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_v[st], ph))) return false;
      if constexpr (!FULL) {
        // V rows past the end of the context hold whatever the pool or an
        // earlier stage left there; zero them so that 0 * row stays 0.
        const int r0 = max(nv, w_tok0);
        const int n_zero = (w_tok0 + TPW - r0) * ND * 8;  // 16-byte chunks
        for (int e = lane; e < n_zero; e += 32) {
          const int row = r0 + e / (ND * 8), rem = e % (ND * 8);
          *reinterpret_cast<uint4*>(pV + (rem >> 3) * Tr::PANEL_BYTES + row * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      // ---- O^T += V^T P^T over this warp's 16 tokens
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t va[4];
        ldmatrix_x4_trans(va, sV + (mt >> 2) * Tr::PANEL_BYTES + (v_lane ^ ((mt & 3) << 5)));
        mma_16816<T>(acc[mt], va, pb0, pb1);
        mma_16816<T>(acc[mt], va, pl0, pl1);
      }
      // the zeroing stores must be ordered before the next bulk copy into this half
      if constexpr (!FULL) fence_proxy_async_smem();
      return true;
    };

    const int n_stages = (info.n_tok + TS - 1) / TS;
    bool ok = true;
    for (int i = 0; i < n_stages; ++i) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full_k[st], ph))) {
        if (lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
        break;
      }
      uint8_t* pK = smem + st * Tr::STAGE_BYTES;
      const uint32_t sK = smem_addr(pK);
      const int nv = info.n_tok - i * TS;
      const bool v_ok = nv >= TS ? stage(sK, pK + Tr::TILE_BYTES, TS, std::true_type{})
                                 : stage(sK, pK + Tr::TILE_BYTES, nv, std::false_type{});
      if (!v_ok) {
        if (lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_v[st]);
      if (++st == STAGES) {
        st = 0;
        ph ^= 1;
      }
    }
    // every read of this item's Q slot is done: the producer may refill it
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[slot]);

    // ---- combine the four warps: weight of warp w for head g is
    // 2^(m_w - M) / L with M = max_w m_w and L = sum_w 2^(m_w - M) l_w.
    l_lane += __shfl_xor_sync(0xffffffffu, l_lane, 1);
    l_lane += __shfl_xor_sync(0xffffffffu, l_lane, 2);
    if (qc == 0 && quad < G) {
      s_m[warp * G + quad] = m_run;
      s_l[warp * G + quad] = l_lane;
    }
    if (named_barrier_or(1, NW * 32, !ok)) break;  // a timed-out stage: stop, output invalid

    const int s = info.s;
    const bool single = info.n_parts == 1;
    if (threadIdx.x == 0 && !single)
      s_pub[s_pub[kPubSlots]++] = static_cast<uint32_t>(s * a.num_kv_heads + info.kvh);
    float f_own = 0.f;  // this warp's weight for head `quad`
    if (quad < G) {
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m[w * G + quad]);
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = s_m[w * G + quad];
        L += mw == -CUDART_INF_F ? 0.f : fast_exp2(mw - M) * s_l[w * G + quad];
      }
      if (L > 0.f && m_run != -CUDART_INF_F) f_own = fast_exp2(m_run - M) / L;
      if (!single && warp == 0 && qc == 0) {
        const int64_t cell =
            (static_cast<int64_t>(s) * a.num_heads + h0 + quad) * a.max_parts + info.part;
        a.tmp_m[cell] = M;
        a.tmp_l[cell] = L;
      }
    }
    const float f_lo = __shfl_sync(0xffffffffu, f_own, 8 * qc);
    const float f_hi = __shfl_sync(0xffffffffu, f_own, 8 * qc + 4);
    // Rounds of HG heads: each warp stores its weighted partial output into its
    // own slot, then the slots are summed in warp order (the same order every
    // run) and written out, four dims per thread.
    constexpr int HG = Tr::HG;
    float* my_slot = s_acc + warp * HG * Tr::ACC_PITCH;
#pragma unroll
    for (int r = 0; r < G / HG; ++r) {
      if (r > 0) named_barrier_sync(1, NW * 32);  // the previous round's slots are read
      const int g_lo = 2 * qc - r * HG;          // this lane's heads, relative to the round
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int gg = g_lo + j;
        if (2 * qc + j < G && gg >= 0 && gg < HG) {
          const float f = j ? f_hi : f_lo;
          float* row = my_slot + gg * Tr::ACC_PITCH + quad;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            row[16 * mt] = acc[mt][j] * f;
            row[16 * mt + 8] = acc[mt][2 + j] * f;
          }
        }
      }
      named_barrier_sync(1, NW * 32);
      for (int e = threadIdx.x; e < HG * D / 4; e += NW * 32) {
        const int gg = e / (D / 4), d = (e % (D / 4)) * 4;
        const int g = r * HG + gg;
        float4 o = *reinterpret_cast<const float4*>(s_acc + gg * Tr::ACC_PITCH + d);
#pragma unroll
        for (int w = 1; w < NW; ++w) {
          const float4 t = *reinterpret_cast<const float4*>(s_acc + (w * HG + gg) * Tr::ACC_PITCH + d);
          o.x += t.x;
          o.y += t.y;
          o.z += t.z;
          o.w += t.w;
        }
        if (single) {
          const uint2 packed = make_uint2(pack2<T>(o.x, o.y), pack2<T>(o.z, o.w));
          *reinterpret_cast<uint2*>(static_cast<T*>(a.out) +
                                    (static_cast<int64_t>(s) * a.num_heads + h0 + g) * D + d) = packed;
        } else {
          const int64_t cell =
              (static_cast<int64_t>(s) * a.num_heads + h0 + g) * a.max_parts + info.part;
          *reinterpret_cast<float4*>(a.tmp_out + cell * D + d) = o;
        }
      }
    }
    // The slots and s_m / s_l are rewritten only after the next item's first
    // barrier, which every thread reaches after its reads here.
  }
  // Every loop exit follows a barrier that all consumer threads passed after
  // their last write-out (or a stage timeout, whose item is not listed).
  if (threadIdx.x == 0) publish();
  // The merge grid may launch once every thread of every CTA has passed the
  // plan (the producer did so before its first list access).
  grid_dependency_wait();
  allow_dependent_launch();
}

// ---------------------------------------------------------------- merge
// Contexts that span several partitions: out = sum_p w_p o_p with
// w_p = l_p 2^(m_p - M) / sum_q l_q 2^(m_q - M), M = max_p m_p.  One CTA of
// kMergeThreads threads per (sequence, kv head) pair listed by the plan kernel
// (grid-stride when there are more pairs than CTAs).  Thread t owns float4 group
// t % NV of the pair's G x D output and the partitions p with p % SLICES ==
// t / NV, so a pair's partial outputs are all requested at once; the slices are
// summed in shared memory (fixed order) at the end.  Statistics are read in
// chunks of kMergeChunk partitions (one chunk for up to 64).
// The grid launches while the decode grid still runs: each pair waits for the
// decode grid's per-pair count, and its partials are read from L2.  A pair of
// at most NREG * SLICES (and kMergeChunk) partitions, the common case, issues
// every load at once when it becomes ready: the thread's partials into NREG
// registers together with the statistics into shared memory, so the merge
// costs one memory round trip after the pair's last partition, not one for the
// statistics and more for the partials behind them.  The launcher picks the
// smallest NREG in {2, 4, 8, 16} that covers the call's partition count: the
// register footprint, and with it the number of merge CTAs an SM holds, follows
// what the call needs.
constexpr int kMergeThreads = 256;
constexpr int kMergeChunk = 64;
constexpr int kMergeMaxRegs = 16;  // largest NREG

template <typename T, int D, int G, int NREG>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const DecodeArgs a) {
  constexpr int NV = G * D / 4;  // float4 groups of one pair's output
  static_assert(NV <= kMergeThreads && kMergeThreads % NV == 0, "whole slices");
  constexpr int SLICES = kMergeThreads / NV;
  constexpr int NWARP = kMergeThreads / 32;
  constexpr int FAST_PARTS = NREG * SLICES < kMergeChunk ? NREG * SLICES : kMergeChunk;
  __shared__ float s_m[G][kMergeChunk], s_w[G][kMergeChunk];
  __shared__ float s_M[G], s_L[G];
  __shared__ float4 s_part[SLICES > 1 ? SLICES - 1 : 1][NV];
  __shared__ int s_ready;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int v = tid % NV, slice = tid / NV;
  const int vg = v / (D / 4), vd = (v % (D / 4)) * 4;  // head and first dim of this thread's group
  const uint32_t Hkv = static_cast<uint32_t>(a.num_kv_heads);
  // The plan finished before the decode grid let this grid launch.
  const uint32_t n_tasks = __ldcg(a.work + 2) * Hkv;
  const unsigned long long U =
      a.balanced ? __ldcg(reinterpret_cast<const unsigned long long*>(a.work + 4)) : 0ull;
  for (uint32_t t = blockIdx.x; t < n_tasks; t += gridDim.x) {
    const int s = __ldcg(a.merge_seqs + t / Hkv);
    const int kvh = static_cast<int>(t % Hkv);
    const int h0 = kvh * G;
    int np, psize;
    if (round_robin(a)) {
      int n_big, p_small;
      partition_rr(clamp_len(a.lens[s], a.max_ctx), a, U, n_big, np, psize, p_small);
    } else {
      partition_for(clamp_len(a.lens[s], a.max_ctx), a, U, np, psize);
    }
    const int64_t base0 = (static_cast<int64_t>(s) * a.num_heads + h0) * a.max_parts;
    auto cell = [&](int g, int p) { return base0 + static_cast<int64_t>(g) * a.max_parts + p; };
    // Wait (bounded) until the decode grid has published all np partitions of
    // this pair; their results are then read from L2 (__ldcg), never from a
    // possibly stale L1 line.
    if (tid == 0) {
      s_ready = wait_counter_bounded(a.pair_done + static_cast<int64_t>(s) * Hkv + kvh,
                                     static_cast<uint32_t>(np) + a.merge_wait_extra, a.err,
                                     a.merge_wait_limit_ns);
      if (!s_ready) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    __syncthreads();
    if (!s_ready) {  // uniform: results of this pair stay unwritten
      __syncthreads();  // every thread has read s_ready before thread 0 rewrites it
      continue;
    }

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (np <= FAST_PARTS) {
      const float* src = a.tmp_out + cell(vg, 0) * D + vd;
      // ---- every load at once: partials p = slice, slice + SLICES, ... into
      // registers, the statistics into shared memory
      float4 part[NREG];
#pragma unroll
      for (int i = 0; i < NREG; ++i) {
        const int p = slice + i * SLICES;
        if (p < np) part[i] = __ldcg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(p) * D));
      }
      for (int i = tid; i < G * np; i += kMergeThreads) {
        const int g = i / np, p = i % np;
        s_m[g][p] = __ldcg(a.tmp_m + cell(g, p));
        s_w[g][p] = __ldcg(a.tmp_l + cell(g, p));  // l for now
      }
      __syncthreads();
      // M and L per head (warp g reduces head g)
      for (int g = warp; g < G; g += NWARP) {
        float mc = -CUDART_INF_F;
        for (int p = lane; p < np; p += 32) mc = fmaxf(mc, s_m[g][p]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
        float lc = 0.f;
        for (int p = lane; p < np; p += 32) lc += s_w[g][p] * fast_exp2(s_m[g][p] - mc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lc += __shfl_xor_sync(0xffffffffu, lc, o);
        if (lane == 0) {
          s_M[g] = mc;
          s_L[g] = lc;
        }
      }
      __syncthreads();
      // weights, in place of l: l_p 2^(m_p - M) / L
      for (int i = tid; i < G * np; i += kMergeThreads) {
        const int g = i / np, p = i % np;
        s_w[g][p] = s_w[g][p] * fast_exp2(s_m[g][p] - s_M[g]) / s_L[g];
      }
      __syncthreads();
      const float* wrow = s_w[vg];
#pragma unroll
      for (int i = 0; i < NREG; ++i) {
        const int p = slice + i * SLICES;
        if (p < np) {
          const float wp = wrow[p];
          acc.x += wp * part[i].x;
          acc.y += wp * part[i].y;
          acc.z += wp * part[i].z;
          acc.w += wp * part[i].w;
        }
      }
    } else {
      // ---- M and L per head (warp g reduces head g; online across chunks)
      float M = -CUDART_INF_F, L = 0.f;  // valid in warp g < G
      for (int c0 = 0; c0 < np; c0 += kMergeChunk) {
        const int cn = min(kMergeChunk, np - c0);
        if (c0 > 0) __syncthreads();  // the previous chunk's s_m / s_w are no longer read
        for (int i = tid; i < G * cn; i += kMergeThreads) {
          const int g = i / cn, p = i % cn;
          s_m[g][p] = __ldcg(a.tmp_m + cell(g, c0 + p));
          s_w[g][p] = __ldcg(a.tmp_l + cell(g, c0 + p));  // l for now
        }
        __syncthreads();
        for (int g = warp; g < G; g += NWARP) {
          float mc = -CUDART_INF_F;
          for (int p = lane; p < cn; p += 32) mc = fmaxf(mc, s_m[g][p]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
          const float Mn = fmaxf(M, mc);
          float lc = 0.f;
          for (int p = lane; p < cn; p += 32) lc += s_w[g][p] * fast_exp2(s_m[g][p] - Mn);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) lc += __shfl_xor_sync(0xffffffffu, lc, o);
          L = L * fast_exp2(M - Mn) + lc;  // M = -inf on the first chunk: the old sum is 0
          M = Mn;
        }
      }
      if (warp < G && lane == 0) {
        s_M[warp] = M;
        s_L[warp] = L;
      }
      __syncthreads();

      // ---- weighted sum of the partial outputs
      for (int c0 = 0; c0 < np; c0 += kMergeChunk) {
        const int cn = min(kMergeChunk, np - c0);
        // One chunk: its statistics are still in s_m / s_w from the pass above.
        // Several: that pass left the last chunk there, so every chunk (the first
        // included) is loaded again.
        if (np > kMergeChunk) {
          if (c0 > 0) __syncthreads();  // the previous chunk's weights are no longer read
          for (int i = tid; i < G * cn; i += kMergeThreads) {
            const int g = i / cn, p = i % cn;
            s_m[g][p] = __ldcg(a.tmp_m + cell(g, c0 + p));
            s_w[g][p] = __ldcg(a.tmp_l + cell(g, c0 + p));
          }
          __syncthreads();
        }
        // weights, in place of l: l_p 2^(m_p - M) / L
        for (int i = tid; i < G * cn; i += kMergeThreads) {
          const int g = i / cn, p = i % cn;
          s_w[g][p] = s_w[g][p] * fast_exp2(s_m[g][p] - s_M[g]) / s_L[g];
        }
        __syncthreads();
        const float* wrow = s_w[vg];
        const float* src = a.tmp_out + cell(vg, c0) * D + vd;
#pragma unroll 8
        for (int p = slice; p < cn; p += SLICES) {
          const float4 o = __ldcg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(p) * D));
          const float wp = wrow[p];
          acc.x += wp * o.x;
          acc.y += wp * o.y;
          acc.z += wp * o.z;
          acc.w += wp * o.w;
        }
      }
    }
    // ---- slices 1.. hand their sums to slice 0, which adds them in order
    if (SLICES > 1) {
      if (slice > 0) s_part[slice - 1][v] = acc;
      __syncthreads();
      if (slice == 0) {
#pragma unroll
        for (int j = 0; j < SLICES - 1; ++j) {
          const float4 o = s_part[j][v];
          acc.x += o.x;
          acc.y += o.y;
          acc.z += o.z;
          acc.w += o.w;
        }
      }
    }
    if (slice == 0) {
      const uint2 packed = make_uint2(pack2<T>(acc.x, acc.y), pack2<T>(acc.z, acc.w));
      *reinterpret_cast<uint2*>(static_cast<T*>(a.out) +
                                (static_cast<int64_t>(s) * a.num_heads + h0 + vg) * D + vd) = packed;
    }
    __syncthreads();  // shared state is reused by the next pair
  }
  // Complete only after the decode grid: work behind this grid on the stream
  // then sees every output row, including the single-partition ones.
  grid_dependency_wait();
}

// Host-side launcher, instantiated per (dtype, head_dim) in its own file.
template <typename T, int D>
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& m, int group, int block_size,
                          bool paged, int num_sms, cudaStream_t stream);

}  // namespace pkv
