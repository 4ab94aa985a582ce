// Paged prefill attention for sm_100a (tcgen05 tensor cores, TMEM accumulators).
//
// Method (vLLM and PagedAttention slide 3: the prompt is processed in parallel
// before decoding starts; dataarena note section 4, step 3: a scheduled request
// runs its prefill; slides 9-10: attention reads keys and values block by block
// through the block table).  A sequence s gets T new tokens at positions
// p0 .. p0 + T - 1 (a whole prompt when p0 = 0, a later chunk of it otherwise);
// their keys and values are already in the paged cache, written by the cache
// write.  New token i attends causally over positions 0 .. p0 + i:
//   out[i, h, :] = sum_{t <= p0 + i} softmax_t(scale q[i, h, :] . K[t, :]) V[t, :]
// with kv head h / (Hq / Hkv).  Unlike the single-query decode, this is a dense
// contraction (T x D by D x L), so it runs on the tensor cores.
//
// Kernel design (B200).
//  * One CTA per pair of 128-row query tiles of one sequence: two heads of a
//    kv group on the same rows when Hq / Hkv is even (both tiles read the same
//    K/V tiles and do the same work), else two consecutive row tiles of one
//    head.  576 threads, one CTA per SM (197 KB of shared memory at head_dim
//    128).  Query tiles with more keys are scheduled first.
//  * Warp 0 loads: both tiles' Q rows once (TMA, 128-byte swizzle), then the K
//    and V tiles of 128 keys through a ring of two stages, one TMA box per
//    cache block and 128-byte panel, with the frames taken from the block table.
//  * Warp 1 holds the tensor memory (512 columns: per query tile a 128-column
//    score buffer and a D-column output accumulator) and one of its threads
//    issues the tcgen05.mma instructions.  Per key tile j and query tile t:
//    S_t(j) = Q_t K_j^T (Q, K K-major in shared memory), then O_t += P_t(j) V_j
//    with P_t(j) read from tensor memory and V used as it lies in the cache
//    tile, as an MN-major operand.  While the softmax of one query tile runs,
//    the tensor cores work on the other tile.  Completion is signalled to
//    mbarriers with tcgen05.commit.
//  * Warps 2-9 (tile 0) and 10-17 (tile 1) hold two threads per query row
//    (tensor-memory lane = row), each with half of the tile's 128 keys in
//    registers.  Each half takes its max, with the causal mask applied by
//    select (so garbage keys past the context never reach a sum); the halves
//    exchange maxima through shared memory at a named barrier of the tile's
//    256 threads, and each rescales its half of the row of O in tensor memory
//    when the max grows.  Then each reloads its scores 32 at a time, turns
//    them into P (base-2 exponentials, rounded to the input type, two per
//    32-bit column) and stores P over the first 32 of its own 64 score
//    columns (so neither half overwrites scores the other still reads).  The
//    sum is taken over the rounded weights, so the output is an exact convex
//    combination of V rows.  In the last key tile they zero the V rows past
//    the context (0 x NaN would be NaN).
//  * The next scores of a tile overwrite its P, so they are issued only after
//    the product reading P has completed (tcgen05.mma orders only products
//    into the same accumulator).
//  * Epilogue: out = O / l, rounded to the input type, written per row.
//  * Every mbarrier wait is bounded; on expiry the kernel sets
//    PKV_DEVERR_WAIT_TIMEOUT and moves on.  Before the tensor memory is freed,
//    the MMA thread's last tcgen05.commit (which covers every product it issued)
//    is waited for, and every copy the loader issued has landed.
#include "prefill.cuh"

namespace pkv {

// ------------------------------------------------------------ tcgen05 helpers
// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (all >> 4), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with fp32 accumulation: A and B of the
// same 16-bit type (f16 = 0, bf16 = 1), A K-major, B K-major (0) or MN-major
// (1), shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16(uint32_t ab_format, uint32_t b_mn_major,
                                                      uint32_t M, uint32_t N) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_mn_major << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
        "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
        "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]);

// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16f(uint32_t taddr, const float (&v)[16]) {
  uint32_t u[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i]);
  tmem_st16(taddr, u);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
      : "memory");
}

// One product S = A B^T over K = 16 NK (NK = 4 or 8) as one block of
// instructions, so that nothing else of the issuing thread sits between the
// steps (an MMA is accepted about when the previous one starts, so any delay
// in issuing the next one idles the tensor cores).  Both operands K-major with
// 128-byte rows in panels of 128 rows: K step k at descriptor offset
// (k / 4) * 1024 + (k % 4) * 2 (16-byte units).  The first step overwrites D.
template <int NK>
__device__ __forceinline__ void umma_ss_steps(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  static_assert(NK == 4 || NK == 8, "4 or 8 K steps");
#define PKV_SS_STEP(OFF)                                                                  \
  "add.s64 a1, %1, " #OFF ";\n\tadd.s64 b1, %2, " #OFF ";\n\t"                              \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, p;\n\t"
  if constexpr (NK == 4) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 a1, b1;\n\t"
        "setp.ne.b32 p, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "setp.eq.b32 p, %3, %3;\n\t"
        PKV_SS_STEP(2) PKV_SS_STEP(4) PKV_SS_STEP(6) "}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 a1, b1;\n\t"
        "setp.ne.b32 p, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "setp.eq.b32 p, %3, %3;\n\t"
        PKV_SS_STEP(2) PKV_SS_STEP(4) PKV_SS_STEP(6)
        PKV_SS_STEP(1024) PKV_SS_STEP(1026) PKV_SS_STEP(1028) PKV_SS_STEP(1030) "}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc)
        : "memory");
  }
#undef PKV_SS_STEP
}

// One chunk of O += P V, A (P) from tensor memory, B (V) MN-major in shared
// memory, as one block of instructions: K steps 2c, 2c + 1, 2c + 4, 2c + 5
// (keys 32 c .. 32 c + 31 of each half of the key tile).  `a` is the tensor-
// memory address of step 2c's P (the others at + 8, + 64, + 72 columns), `b`
// the V descriptor of step 2c (the others at + 128, + 512, + 640 in 16-byte
// units: 16 keys of 128-byte rows per step).  The first step accumulates
// only if `acc` != 0.
__device__ __forceinline__ void umma_ts_chunk(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                              uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 a1;\n\t.reg .b64 b1;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "setp.eq.b32 p, %3, %3;\n\t"
      "add.s32 a1, %1, 8;\n\tadd.s64 b1, %2, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, p;\n\t"
      "add.s32 a1, %1, 64;\n\tadd.s64 b1, %2, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, p;\n\t"
      "add.s32 a1, %1, 72;\n\tadd.s64 b1, %2, 640;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, p;\n\t}"
      ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// tcgen05.wait::ld that takes the loaded registers as operands, so that no use
// of them can be scheduled before the wait (for a load left in flight while
// other work runs; elsewhere the plain wait directly follows its loads).
__device__ __forceinline__ void tmem_wait_ld_tied(float (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
                 "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]),
                 "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]), "+f"(v[19]), "+f"(v[20]),
                 "+f"(v[21]), "+f"(v[22]), "+f"(v[23]), "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]),
                 "+f"(v[28]), "+f"(v[29]), "+f"(v[30]), "+f"(v[31])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// max (min) of N values, three at a time (three-input max.f32 / min.f32).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
template <int N>
__device__ __forceinline__ float max3_tree(const float (&x)[N]) {
  // four independent chains, then combined
  float r[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
  for (int e = 4; e + 8 <= N; e += 8) {
    r[0] = fmax3(r[0], x[e], x[e + 1]);
    r[1] = fmax3(r[1], x[e + 2], x[e + 3]);
    r[2] = fmax3(r[2], x[e + 4], x[e + 5]);
    r[3] = fmax3(r[3], x[e + 6], x[e + 7]);
  }
#pragma unroll
  for (int e = 4 + ((N - 4) / 8) * 8; e < N; ++e) r[e & 3] = fmaxf(r[e & 3], x[e]);
  return fmaxf(fmax3(r[0], r[1], r[2]), r[3]);
}
template <int N>
__device__ __forceinline__ float min3_tree(const float (&x)[N]) {
  float r[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
  for (int e = 4; e + 8 <= N; e += 8) {
    r[0] = fmin3(r[0], x[e], x[e + 1]);
    r[1] = fmin3(r[1], x[e + 2], x[e + 3]);
    r[2] = fmin3(r[2], x[e + 4], x[e + 5]);
    r[3] = fmin3(r[3], x[e + 6], x[e + 7]);
  }
#pragma unroll
  for (int e = 4 + ((N - 4) / 8) * 8; e < N; ++e) r[e & 3] = fminf(r[e & 3], x[e]);
  return fminf(fmin3(r[0], r[1], r[2]), r[3]);
}

// Lag of a row's reference max behind its true running max (base-2 units)
// before the output row is rescaled: weights stay below 2^8.
constexpr float kLazy = 8.f;

// Coefficients c_0 .. c_n of p(f) ~ 2^f on |f| <= 1/2, minimax in relative
// error (fitted by exp2_poly_fit.py beside this file): degree 3, error 2^-13.7,
// for bf16 weights (8 significant bits); degree 4, error 2^-18.5, for fp16 (11).
__device__ constexpr float kExp2Deg3[4] = {0.9999280571937561f, 0.6932609677314758f, 0.2426111400127411f,
                                           0.055171627551317215f};
__device__ constexpr float kExp2Deg4[5] = {0.9999992847442627f, 0.6931217908859253f, 0.240247443318367f,
                                           0.05591786280274391f, 0.009570096619427204f};

// 2^y for a pair, on the FMA pipe instead of MUFU (which takes 16 per clock per
// SM): Cody-Waite range reduction y = j + f, j = rint(y) by the 1.5 * 2^23
// rounding shift, |f| <= 1/2; then p(f) by Horner and j added to p's exponent
// field.  y is clamped at -125, so that the result is a normal number (p(f)
// >= 2^-1/2 puts the field at >= 1); a row's largest weight is at least 1, so
// only negligible weights are clamped.
template <typename T>
__device__ __forceinline__ float2 exp2_poly2(float2 y) {
  y.x = fmaxf(y.x, -125.f);
  y.y = fmaxf(y.y, -125.f);
  const float2 t = __fadd2_rn(y, make_float2(12582912.f, 12582912.f));
  const float2 j = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(j, make_float2(-1.f, -1.f), y);  // y - j, exact
  float2 p;
  if constexpr (std::is_same<T, __half>::value) {
    p = make_float2(kExp2Deg4[4], kExp2Deg4[4]);
#pragma unroll
    for (int k = 3; k >= 0; --k) p = __ffma2_rn(p, f, make_float2(kExp2Deg4[k], kExp2Deg4[k]));
  } else {
    p = make_float2(kExp2Deg3[3], kExp2Deg3[3]);
#pragma unroll
    for (int k = 2; k >= 0; --k) p = __ffma2_rn(p, f, make_float2(kExp2Deg3[k], kExp2Deg3[k]));
  }
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// ------------------------------------------------------------ kernel
// Query tile t in {0, 1} of a CTA: head h_t, rows i0_t .. i0_t + 127 of the
// chunk.  Two heads of one kv group share the rows when Hq / Hkv is even (the
// tiles read the same K/V tiles and do the same work); otherwise one head
// takes two consecutive row tiles.
// 96 registers: the register file is split between the SM's four schedulers
// (16 K registers each) and 18 warps put five on two of them, 5 x 32 x 96 <=
// 16 K; more registers per thread and the launch fails for lack of resources.
template <typename T, int D>
__global__ void __maxnreg__(96)
    prefill_kernel(const PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using Tr = PrefillTraits<D>;
  constexpr int ND = Tr::ND;
  constexpr int KSTEPS = D / 16;               // k-steps of S = Q K^T
  static_assert(kPrefillTileN == 128, "O += P V in two chunks of K steps: {0, 1, 4, 5} and {2, 3, 6, 7}");
  constexpr uint32_t AB_FMT = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t IDESC_S = umma_idesc_f16(AB_FMT, 0u, kPrefillTileM, kPrefillTileN);
  constexpr uint32_t IDESC_O = umma_idesc_f16(AB_FMT, 1u, kPrefillTileM, D);

  const int G = a.num_heads / a.num_kv_heads;
  const bool head_pair = (G & 1) == 0;
  const int s = blockIdx.z;
  const int q0 = __ldg(a.query_start + s);
  const int n_new = __ldg(a.query_start + s + 1) - q0;  // T, the chunk's tokens
  const int rows_per_cta = head_pair ? kPrefillTileM : 2 * kPrefillTileM;
  const int cap = a.max_blocks * a.block_size;
  if (q0 < 0 || n_new < 0 || q0 + n_new > a.total_q ||
      n_new > static_cast<int>(gridDim.y) * rows_per_cta || n_new > cap) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    return;
  }
  const int base_row = static_cast<int>(gridDim.y - 1 - blockIdx.y) * rows_per_cta;
  if (base_row >= n_new) return;  // uniform over the CTA, before any set-up
  int L = __ldg(a.lens + s);
  if (L < n_new || L > cap) {
    if (threadIdx.x == 0) set_error(a.err, PKV_DEVERR_CONTEXT_LEN);
    L = L < n_new ? n_new : cap;
  }
  const int p0 = L - n_new;
  int h_t[2], i0_t[2], nkv_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    h_t[t] = head_pair ? 2 * static_cast<int>(blockIdx.x) + t : static_cast<int>(blockIdx.x);
    i0_t[t] = head_pair ? base_row : base_row + t * kPrefillTileM;
    // key tiles this query tile needs (0 when its rows are past the chunk)
    nkv_t[t] = i0_t[t] < n_new ? (p0 + min(i0_t[t] + kPrefillTileM - 1, n_new - 1)) / kPrefillTileN + 1 : 0;
  }
  const int n_kv = max(nkv_t[0], nkv_t[1]);
  const int kvh = h_t[0] / G;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kPrefillStages;
  uint64_t* k_empty = v_full + kPrefillStages;
  uint64_t* v_empty = k_empty + kPrefillStages;
  uint64_t* s_full = v_empty + kPrefillStages;   // [2]: scores of tile t ready
  uint64_t* p_full = s_full + 2;                 // [2][2]: chunk c of P of tile t in tensor memory
  uint64_t* pv_done = p_full + 4;                // [2]: O_t += P_t V done (P_t may be overwritten)
  uint64_t* o_final = pv_done + 2;               // every product done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_TMEM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kPrefillStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[2 * t], 8);  // one arrival per softmax warp of the tile
      mbar_init(&p_full[2 * t + 1], 8);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(o_final, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kPrefillTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  const uint32_t sQ = smem_addr(smem + Tr::OFF_Q);
  const uint32_t sK = smem_addr(smem + Tr::OFF_K);
  const uint32_t sV = smem_addr(smem + Tr::OFF_V);

  if (warp == 0) {
    // ============================================================ loads
    const int B = a.block_size;
    const int32_t* row = a.tables + static_cast<int64_t>(s) * a.max_blocks;
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(2 * Tr::TILE));
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int pn = 0; pn < ND; ++pn)
          tma_load_3d(smem + Tr::OFF_Q + t * Tr::TILE + pn * Tr::PANEL, &maps.q, pn * 64, h_t[t],
                      q0 + i0_t[t], q_full);
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < n_kv && ok; ++j) {
      const int st = j % kPrefillStages;
      const int k_lo = j * kPrefillTileN;
      const int k_hi = min(k_lo + kPrefillTileN, L);
      const int nb = (k_hi - k_lo + B - 1) / B;
      const int blk = lane / ND, pn = lane % ND;
      int frame = 0;
      const bool copier = blk < nb;
      if (copier) {
        frame = __ldg(row + k_lo / B + blk);
        if (frame < 0 || frame >= a.num_blocks) {
          set_error(a.err, PKV_DEVERR_TABLE_ENTRY);
          frame = 0;
        }
      }
      const uint32_t bytes = static_cast<uint32_t>(nb * ND * B * 128);
      const int off = pn * Tr::PANEL + blk * B * 128;
      if (lane == 0 && j >= kPrefillStages &&
          !mbar_wait_bounded(&k_empty[st], ((j / kPrefillStages) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&k_full[st], bytes);
      __syncwarp();
      if (copier)
        tma_load_3d(smem + Tr::OFF_K + st * Tr::TILE + off, &maps.k, pn * 64, kvh * B, frame, &k_full[st]);
      ++issued_k;
      if (lane == 0 && j >= kPrefillStages &&
          !mbar_wait_bounded(&v_empty[st], ((j / kPrefillStages) - 1) & 1)) {
        set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&v_full[st], bytes);
      __syncwarp();
      if (copier)
        tma_load_3d(smem + Tr::OFF_V + st * Tr::TILE + off, &maps.v, pn * 64, kvh * B, frame, &v_full[st]);
      ++issued_v;
    }
    if (lane == 0) {
      if (!mbar_wait_bounded(q_full, 0)) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
      for (int j = max(0, issued_k - kPrefillStages); j < issued_k; ++j)
        if (!mbar_wait_bounded(&k_full[j % kPrefillStages], (j / kPrefillStages) & 1))
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
      for (int j = max(0, issued_v - kPrefillStages); j < issued_v; ++j)
        if (!mbar_wait_bounded(&v_full[j % kPrefillStages], (j / kPrefillStages) & 1))
          set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    // ============================================================ tensor cores
    // Order of the products: S_0(0), S_1(0); then for each key tile j:
    // O_0 += P_0(j) V_j, S_0(j+1), O_1 += P_1(j) V_j, S_1(j+1).  P_t(j) lives in
    // tensor memory inside the columns of S_t(j), so S_t(j+1) is issued
    // only once the product that reads P_t(j) has completed (the hardware orders
    // a thread's products into the same accumulator, not these).  The fixed
    // order keeps the two tiles half a step apart: while one tile's softmax
    // runs, the tensor cores work on the other tile.  (Issuing whichever
    // tile's step is ready first, polling both, measured 17 % slower: both
    // softmaxes then tend to run at the same time.)
    if (lane == 0) {
      bool ok = mbar_wait_bounded(q_full, 0) && mbar_wait_bounded(&k_full[0], 0);
      auto issue_s = [&](int t, int st) {  // S_t = Q_t K^T of the key tile in stage st
        umma_ss_steps<KSTEPS>(tmem + Tr::colS(t), umma_desc(sQ + t * Tr::TILE, 16, 1024),
                              umma_desc(sK + st * Tr::TILE, 16, 1024), IDESC_S);
        umma_commit(&s_full[t]);
      };
      if (ok) {
        tmem_fence_after_sync();
        for (int t = 0; t < 2; ++t)
          if (nkv_t[t] > 0) issue_s(t, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % kPrefillStages, st1 = (j + 1) % kPrefillStages;
        const bool more = j + 1 < n_kv;
        if (!mbar_wait_bounded(&v_full[st], (j / kPrefillStages) & 1) ||
            (more && !mbar_wait_bounded(&k_full[st1], ((j + 1) / kPrefillStages) & 1))) {
          ok = false;
          break;
        }
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= nkv_t[t]) continue;
          // The first chunk of P (keys 0..31 of each half: K steps 0, 1, 4, 5)
          // is multiplied while the softmax computes the second (2, 3, 6, 7).
          bool got = true;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (!mbar_wait_bounded(&p_full[2 * t + c], j & 1)) {
              got = false;
              break;
            }
            tmem_fence_after_sync();
            umma_ts_chunk(tmem + Tr::colO(t), tmem + Tr::colS(t) + 16 * c,
                          umma_desc(sV + st * Tr::TILE + 2 * c * 2048, Tr::PANEL, 1024), IDESC_O,
                          j > 0 || c > 0);
          }
          if (!got) {
            ok = false;
            break;
          }
          umma_commit(&pv_done[t]);
          if (j + 1 < nkv_t[t]) {
            if (!mbar_wait_bounded(&pv_done[t], j & 1)) {
              ok = false;
              break;
            }
            tmem_fence_after_sync();
            issue_s(t, st1);
          }
        }
        umma_commit(&v_empty[st]);
        if (more) umma_commit(&k_empty[st1]);
      }
      if (!ok) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
      // o_final: every product issued above (all of them on the normal path)
      // has finished; the softmax warps read O after it, and the CTA frees the
      // tensor and shared memory only after it.
      umma_commit(o_final);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax rows
    // Query tile t has 8 warps, two threads per query row (tensor-memory lane =
    // row): half hf holds keys 64 hf .. 64 hf + 63 of every key tile, and output
    // columns hf D/2 .. hf D/2 + D/2 - 1.  The two halves of a row combine their
    // maxima through shared memory at a named barrier of the two warps that hold
    // the row's lanes (one per half), so a warp waits only for its partner, not
    // for the slowest of the tile's 8 warps; at the end the sums meet at a
    // barrier of the tile's 256 threads.  A failed wait is carried by these
    // barriers; a warp pair that stops leaves the tensor-core thread without its
    // weights, so every wait of the tile runs out and all of its threads reach
    // the final barrier.
    const int t = (warp - 2) >> 3;                // query tile of this warp group
    const int hf = ((warp - 2) >> 2) & 1;         // half of the keys / output columns
    const int quarter = warp & 3;                 // tensor-memory lanes 32 quarter ..
    const int r = quarter * 32 + lane;            // this thread's query row of the tile
    const int i = i0_t[t] + r;                    // its token index in the chunk
    const bool valid = i < n_new;
    const int limit = valid ? p0 + i : L - 1;     // last key this row may see
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t cS = lane_base + Tr::colS(t) + 64 * hf;          // this half's scores
    const uint32_t cP = lane_base + Tr::colS(t) + 64 * hf;          // its P columns
    const uint32_t cO = lane_base + Tr::colO(t) + hf * (D / 2);     // its output columns
    float* red = reinterpret_cast<float*>(smem + Tr::OFF_RED) + t * 2 * kPrefillTileM;
    float* red_l = reinterpret_cast<float*>(smem + Tr::OFF_RED) + (4 + t * 2) * kPrefillTileM;
    const int bar_id = 1 + t;
    const int pair_bar = 3 + 4 * t + quarter;     // the two warps of these 32 rows
    // Running state of the row, in base-2 units: m is the max the weights are
    // taken against (at most kLazy below the true running max, see below) and
    // l this half's sum of the rounded weights.
    const float sl = a.scale_log2;
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv_t[t]; ++j) {
      const int k0 = j * kPrefillTileN + 64 * hf;  // first key of this half
      ok = ok && mbar_wait_bounded(&s_full[t], j & 1);
      const bool wok = __all_sync(0xffffffffu, ok);
      tmem_fence_after_sync();
      // Keys past this row's limit count as -inf (by select); only tiles on
      // the diagonal (or past the context) need that, and a warp takes the
      // masked path only when one of its rows needs it.  The max of scale * s
      // is scale * max s for scale >= 0 (scale * min s otherwise).
      const bool masked = __any_sync(0xffffffffu, k0 + 63 > limit);
      const bool pos = sl >= 0.f;
      float part = pos ? -CUDART_INF_F : CUDART_INF_F;
      if (wok) {
        float x[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[32];
          tmem_ld32(cS + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = v[e];
        }
        tmem_wait_ld();
        if (pos) {
          if (masked) {
#pragma unroll
            for (int e = 0; e < 64; ++e) x[e] = k0 + e <= limit ? x[e] : -CUDART_INF_F;
          }
          part = max3_tree<64>(x);
        } else {
          if (masked) {
#pragma unroll
            for (int e = 0; e < 64; ++e) x[e] = k0 + e <= limit ? x[e] : CUDART_INF_F;
          }
          part = min3_tree<64>(x);
        }
      }
      red[hf * kPrefillTileM + r] = part;
      // Both halves of these rows have read their scores after this barrier, so
      // the P writes below (over score columns) cannot race with a read.
      if (named_barrier_or(pair_bar, 64, !wok)) {
        ok = false;
        break;
      }
      const float other = red[(1 - hf) * kPrefillTileM + r];
      const float mx = (pos ? fmaxf(part, other) : fminf(part, other)) * sl;
      // Lazy rescale: the weights are 2^(x - m) with m allowed to lag the true
      // running max by up to kLazy (weights up to 2^kLazy, exact in the input
      // type's range and in fp32), so O and l are rescaled only when the max
      // outgrows that.  The product of the previous key tile ran before S_t(j),
      // so O_t holds it.  tcgen05.ld / st are warp-wide (.sync.aligned): the
      // whole warp takes the branch, rows that need no rescale multiply by 1.
      // Both halves decide alike (they see the same max).
      const bool grow = mx > m + kLazy;
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        const float alpha = grow ? fast_exp2(m - mx) : 1.f;
        l *= alpha;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {  // this half's D/2 columns, 16 at a time
          float v[16];
          tmem_ld16(cO + c * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] *= alpha;
          tmem_st16f(cO + c * 16, v);
        }
      }
      if (grow) m = mx;
      // The key tile that reaches past the context: zero the V rows of the keys
      // past it (whatever the stage held there, 0 x it must be 0).  The two
      // threads of a row zero half of its 16-byte chunks each, in both query
      // tiles' warps, before each tile's product (the two tiles' products may
      // run in either order); later writes are zeros over zeros.
      if (j * kPrefillTileN + kPrefillTileN > L) {
        const int st = j % kPrefillStages;
        ok = ok && mbar_wait_bounded(&v_full[st], (j / kPrefillStages) & 1);
        if (ok && j * kPrefillTileN + r >= L) {
          uint8_t* vrow = smem + Tr::OFF_V + st * Tr::TILE + r * 128;
#pragma unroll
          for (int pn = 0; pn < ND; ++pn)
#pragma unroll
            for (int ch = 4 * hf; ch < 4 * hf + 4; ++ch)
              *reinterpret_cast<uint4*>(vrow + pn * Tr::PANEL + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      // P = 2^(x - m) rounded to the input type, two keys per 32-bit column,
      // over the first 32 of this half's 64 score columns (the product's K
      // step k, keys 16 k .. 16 k + 15, reads columns 64 (k / 4) + 8 (k % 4));
      // the sum is over the rounded weights, in packed pairs of partial sums.
      // Each chunk of 32 keys is handed to the tensor cores as soon as it is
      // stored (p_full of the chunk); the second 32 scores are loaded while the
      // first 32 are turned into P.
      float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float xa[32], xb[32];
      tmem_ld32(cS, xa);
      tmem_wait_ld_tied(xa);
      tmem_ld32(cS + 32, xb);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float xv[32];
        if (c == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) xv[e] = xa[e];
        } else {
          tmem_wait_ld_tied(xb);
#pragma unroll
          for (int e = 0; e < 32; ++e) xv[e] = xb[e];
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int ee = c * 32 + e;
          const float2 y = __ffma2_rn(make_float2(xv[e], xv[e + 1]), make_float2(sl, sl), make_float2(-m, -m));
          // One pair in eight on the FMA pipe (keys 14, 15 of every 16: the same
          // keys whatever the rows' mask, so that a row's weights do not depend
          // on which other rows share its warp).
          float p0v, p1v;
          if ((e >> 1) % 8 == 8 - 1) {
            const float2 pe = exp2_poly2<T>(y);
            p0v = pe.x;
            p1v = pe.y;
          } else {
            p0v = fast_exp2(y.x);
            p1v = fast_exp2(y.y);
          }
          if (masked) {
            p0v = k0 + ee <= limit ? p0v : 0.f;
            p1v = k0 + ee + 1 <= limit ? p1v : 0.f;
          }
          pk[e / 2] = pack2<T>(p0v, p1v);
          sum2[(e >> 1) & 1] = __fadd2_rn(sum2[(e >> 1) & 1], unpack2<T>(pk[e / 2]));
        }
        tmem_st16(cP + c * 16, pk);
        tmem_wait_st();
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[2 * t + c]);
      }
      l += (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
    }
    // ---- epilogue: out = O / (l_half0 + l_half1), this half's columns
    ok = ok && (nkv_t[t] == 0 || mbar_wait_bounded(o_final, 0));
    red_l[hf * kPrefillTileM + r] = l;
    if (named_barrier_or(bar_id, 2 * kPrefillTileM, !__all_sync(0xffffffffu, ok))) {
      if (lane == 0) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
    } else if (nkv_t[t] > 0) {
      tmem_fence_after_sync();
      const float lr = red_l[r] + red_l[kPrefillTileM + r];
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      T* orow = static_cast<T*>(a.out) + (static_cast<int64_t>(q0 + i) * a.num_heads + h_t[t]) * D +
                hf * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        float v[32];
        tmem_ld32(cO + c * 32, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const uint4 w = make_uint4(pack2<T>(v[e] * inv, v[e + 1] * inv), pack2<T>(v[e + 2] * inv, v[e + 3] * inv),
                                       pack2<T>(v[e + 4] * inv, v[e + 5] * inv), pack2<T>(v[e + 6] * inv, v[e + 7] * inv));
            *reinterpret_cast<uint4*>(orow + c * 32 + e) = w;
          }
        }
      }
    }
  }
  // Nothing of the tensor cores or the copies is in flight past here: the MMA
  // thread's final commit covers every product, and it is waited for below
  // before the tensor memory is freed.
  if (warp == 1 && lane == 0 && !mbar_wait_bounded(o_final, 0)) set_error(a.err, PKV_DEVERR_WAIT_TIMEOUT);
  tmem_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tmem_fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kPrefillTmemCols)
                 : "memory");
  }
}

template <typename T, int D>
cudaError_t launch_prefill(const PrefillArgs& a, const PrefillMaps& m, int max_query_len,
                           cudaStream_t stream) {
  using Tr = PrefillTraits<D>;
  auto kern = prefill_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const bool head_pair = ((a.num_heads / a.num_kv_heads) & 1) == 0;
  const int rows = head_pair ? kPrefillTileM : 2 * kPrefillTileM;
  const dim3 grid(static_cast<unsigned>(head_pair ? a.num_heads / 2 : a.num_heads),
                  static_cast<unsigned>((max_query_len + rows - 1) / rows),
                  static_cast<unsigned>(a.num_seqs));
  kern<<<grid, kPrefillThreads, Tr::SMEM_BYTES, stream>>>(a, m);
  return cudaGetLastError();
}

template cudaError_t launch_prefill<__half, 64>(const PrefillArgs&, const PrefillMaps&, int, cudaStream_t);
template cudaError_t launch_prefill<__half, 128>(const PrefillArgs&, const PrefillMaps&, int, cudaStream_t);
template cudaError_t launch_prefill<__nv_bfloat16, 64>(const PrefillArgs&, const PrefillMaps&, int, cudaStream_t);
template cudaError_t launch_prefill<__nv_bfloat16, 128>(const PrefillArgs&, const PrefillMaps&, int, cudaStream_t);

}  // namespace pkv
