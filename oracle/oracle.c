/*
 * Plain CPU oracle for paged decode attention, the paged cache write and the
 * copy-on-write block copy, and for paged prefill attention (the definition a
 * prefill kernel would be checked against).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The CUDA library never
 * links, includes or calls it, and it shares no source with the CUDA library.
 *
 * Everything here is written from the plain definitions, in fp64, with no
 * blocking, no online softmax and no partitioning:
 *
 *  - vLLM and PagedAttention slides, slide 9 ("attention block by block",
 *    keys and values fetched from non-contiguous blocks by address) and slide
 *    10 (block table, logical to physical); the dataarena note "High-Throughput
 *    Serving with vLLM & PagedAttention", section 2 (logical blocks of B
 *    tokens, a pool of block frames, a block table mapping logical blocks to
 *    arbitrary physical frames, worked example tokens 0-15 / 16-31 / 32-41 ->
 *    frames 7 / 2 / 11).  Token t of a sequence lives in logical block t / B at
 *    offset t mod B; its physical frame is table[t / B].
 *  - Attention itself is the textbook softmax(scale * q K^T) V; the pages name
 *    no other formula.  Query head h reads kv head h / (Hq / Hkv) (contiguous
 *    grouped-query groups; the pages are silent on grouping).
 *  - Slides 11 and 13 (a new token goes into the free slot of the last block,
 *    else into a new frame; only the last, partially filled block is ever
 *    copied on write): the cache write scatters each new row to
 *    frame slot / B, offset slot mod B; a negative slot is padding and is
 *    skipped; a block copy duplicates a whole frame of K and of V.
 *
 * Storage layouts (the same definitions the C ABI states):
 *   q        [S, Hq, D]                     fp16 or bf16 bit patterns
 *   k_cache  [N, Hkv, B, D]                 ditto (v_cache the same)
 *   tables   [S, max_blocks] int32          logical -> physical frame
 *   dense k  [S, Hkv, max_ctx, D]           contiguous cache (baseline form)
 *   out      [S, Hq, D] double
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F16 = 0, OR_BF16 = 1 };
enum { OR_OK = 0, OR_EINVAL = -1, OR_ERANGE = -2, OR_ENOMEM = -4 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h) {
  int sign = h >> 15;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: 0.f * 2^-14 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f | 0x400), e - 25); /* 1.f * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE 754 binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double to_double(uint16_t bits, int dtype) {
  return dtype == OR_F16 ? oracle_f16_to_double(bits) : oracle_bf16_to_double(bits);
}

/*
 * Round a double to the nearest value of a binary format with `sig` significand
 * bits (implicit bit included), exponent bias `bias` and all-ones exponent field
 * `emax_field` (infinity / NaN), ties to the value whose last significand bit is
 * 0 (IEEE 754 roundTiesToEven), and return its bit pattern.  This is the
 * rounding the outputs are stored with ("RNE to the output dtype").
 *   x = f * 2^(e - sig + 1) with f an integer in [2^(sig-1), 2^sig) when normal;
 *   below the smallest normal exponent 1 - bias the quantum is fixed at
 *   2^(1 - bias - sig + 1) (subnormals).  Scaling by a power of two is exact in
 *   fp64 here, so the only rounding is the explicit integer rounding.
 */
static uint16_t round_to_format(double v, int sig, int bias, int emax_field) {
  const int frac_bits = sig - 1;
  const uint16_t sign = signbit(v) ? 0x8000u : 0u; /* bit 15 in both 16-bit formats */
  const uint16_t inf_bits = (uint16_t)(emax_field << frac_bits);
  if (isnan(v)) return (uint16_t)(inf_bits | (1u << (frac_bits - 1))); /* quiet NaN */
  double x = fabs(v);
  if (isinf(x)) return sign | inf_bits;
  if (x == 0.0) return sign;
  int E;
  frexp(x, &E);              /* x = m 2^E, m in [0.5, 1): leading bit at 2^(E-1) */
  int e = E - 1;             /* unbiased exponent of the leading bit */
  const int emin = 1 - bias; /* smallest normal exponent */
  const int qexp = (e >= emin ? e : emin) - frac_bits;  /* exponent of one quantum */
  const double q = ldexp(x, -qexp);                     /* exact */
  double f = floor(q);
  const double r = q - f;                               /* exact: q < 2^sig */
  if (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
  /* re-normalise: f may have reached 2^sig (carry into the exponent) */
  int field;
  long mant;
  if (e < emin) {            /* subnormal range: field 0, f counts quanta (f = 2^frac_bits: smallest normal) */
    if (f >= ldexp(1.0, frac_bits)) {
      field = 1;
      mant = (long)(f - ldexp(1.0, frac_bits));
    } else {
      field = 0;
      mant = (long)f;
    }
  } else {
    if (f >= ldexp(1.0, sig)) {
      f = ldexp(1.0, frac_bits);
      e += 1;
    }
    field = e + bias;
    mant = (long)(f - ldexp(1.0, frac_bits));
  }
  if (field >= emax_field) return sign | inf_bits;  /* overflow rounds to infinity */
  return sign | (uint16_t)((field << frac_bits) | mant);
}

/* IEEE binary16: 11 significand bits, bias 15. */
uint16_t oracle_double_to_f16(double v) { return round_to_format(v, 11, 15, 31); }

/* bfloat16: 8 significand bits, bias 127 (the upper half of a binary32). */
uint16_t oracle_double_to_bf16(double v) { return round_to_format(v, 8, 127, 255); }

/* Element-wise rounding of n doubles to fp16 (dtype 0) or bf16 (dtype 1) bits. */
int oracle_round_array(uint16_t* out, const double* in, int64_t n, int32_t dtype) {
  if (n < 0 || (dtype != OR_F16 && dtype != OR_BF16)) return OR_EINVAL;
  for (int64_t i = 0; i < n; ++i)
    out[i] = dtype == OR_F16 ? oracle_double_to_f16(in[i]) : oracle_double_to_bf16(in[i]);
  return OR_OK;
}

/*
 * softmax(scale * K q) V over n rows given in logical order.
 *   x_t = scale * sum_d q_d K_{t,d}          (summed in order of d)
 *   m   = max_t x_t,  w_t = exp(x_t - m),  Z = sum_t w_t
 *   out = sum_t (w_t / Z) V_t
 * n == 0 gives out = 0.  weights (may be NULL) receives w_t / Z.
 */
static void attend(double* out, double* weights, double* x, const double* q, const double* K,
                   const double* V, int64_t n, int D, double scale) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (n == 0) return;
  for (int64_t t = 0; t < n; ++t) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * K[t * D + d];
    x[t] = scale * dot;
  }
  double m = x[0];
  for (int64_t t = 1; t < n; ++t)
    if (x[t] > m) m = x[t];
  double Z = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    x[t] = exp(x[t] - m);
    Z += x[t];
  }
  for (int64_t t = 0; t < n; ++t) {
    double p = x[t] / Z;
    if (weights) weights[t] = p;
    for (int d = 0; d < D; ++d) out[d] += p * V[t * D + d];
  }
}

/* Gather kv head g of sequence s into K, V (n x D doubles) through the block table. */
static int gather_paged(double* K, double* V, const uint16_t* kc, const uint16_t* vc,
                        const int32_t* table_row, int64_t n, int g, int Hkv, int D, int B,
                        int N, int dtype) {
  for (int64_t t = 0; t < n; ++t) {
    int32_t p = table_row[t / B];
    int64_t o = t % B;
    if (p < 0 || p >= N) return OR_ERANGE;
    int64_t base = (((int64_t)p * Hkv + g) * B + o) * D;
    for (int d = 0; d < D; ++d) {
      K[t * D + d] = to_double(kc[base + d], dtype);
      V[t * D + d] = to_double(vc[base + d], dtype);
    }
  }
  return OR_OK;
}

static int check_heads(int Hq, int Hkv, int D) {
  if (Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return OR_EINVAL;
  return OR_OK;
}

/*
 * Paged decode for sequences [s_begin, s_end): out[s, h, :] for every query head.
 * Rows of other sequences are left untouched.  Returns OR_ERANGE if a table
 * entry that the context needs is outside [0, N), or if the context needs more
 * than max_blocks entries.
 */
int oracle_paged_decode(double* out, const uint16_t* q, const uint16_t* k_cache,
                        const uint16_t* v_cache, const int32_t* tables, int32_t max_blocks,
                        const int32_t* context_lens, int32_t s_begin, int32_t s_end, double scale,
                        int32_t Hq, int32_t Hkv, int32_t D, int32_t B, int32_t N, int32_t dtype) {
  if (check_heads(Hq, Hkv, D) || B <= 0 || max_blocks < 0) return OR_EINVAL;
  int G = Hq / Hkv;
  int rc = OR_OK;
  for (int32_t s = s_begin; s < s_end && rc == OR_OK; ++s) {
    int64_t n = context_lens[s];
    if (n < 0 || (n + B - 1) / B > max_blocks) return OR_ERANGE;
    size_t cells = (size_t)(n > 0 ? n : 1) * D;
    double* K = malloc(cells * sizeof(double));
    double* V = malloc(cells * sizeof(double));
    double* x = malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double* qd = malloc((size_t)D * sizeof(double));
    if (!K || !V || !x || !qd) rc = OR_ENOMEM;
    for (int g = 0; g < Hkv && rc == OR_OK; ++g) {
      rc = gather_paged(K, V, k_cache, v_cache, tables + (int64_t)s * max_blocks, n, g, Hkv, D,
                        B, N, dtype);
      for (int h = g * G; h < (g + 1) * G && rc == OR_OK; ++h) {
        const uint16_t* qrow = q + ((int64_t)s * Hq + h) * D;
        for (int d = 0; d < D; ++d) qd[d] = to_double(qrow[d], dtype);
        attend(out + ((int64_t)s * Hq + h) * D, NULL, x, qd, K, V, n, D, scale);
      }
    }
    free(K);
    free(V);
    free(x);
    free(qd);
  }
  return rc;
}

/*
 * Softmax weights w_t / Z of one (sequence, query head) over its context, in
 * logical token order (length context_lens[s]).
 */
/*
 * Paged prefill of one sequence: the prefill phase of the vLLM and
 * PagedAttention slides (slide 3: the prompt is processed in parallel before
 * decoding) over the paged cache of slides 9-10.  T new tokens sit at positions
 * p0 .. p0 + T - 1 and their keys and values are already in the cache; query
 * token i attends causally over positions 0 .. p0 + i (itself and everything
 * before it), softmax(scale q K^T) V per query head as in the decode.
 *   q          [T, Hq, D] fp16/bf16 bits     out [T, Hq, D] double
 *   table_row  [max_blocks] int32, the sequence's block table row
 * Returns OR_ERANGE if a table entry that the context p0 + T needs is outside
 * [0, N), or if that context needs more than max_blocks entries.
 */
int oracle_paged_prefill(double* out, const uint16_t* q, const uint16_t* k_cache,
                         const uint16_t* v_cache, const int32_t* table_row, int32_t max_blocks,
                         int32_t p0, int32_t T, double scale, int32_t Hq, int32_t Hkv, int32_t D,
                         int32_t B, int32_t N, int32_t dtype) {
  if (check_heads(Hq, Hkv, D) || B <= 0 || max_blocks < 0 || p0 < 0 || T < 0) return OR_EINVAL;
  const int64_t n = (int64_t)p0 + T;
  if ((n + B - 1) / B > max_blocks) return OR_ERANGE;
  if (T == 0) return OR_OK;
  const int G = Hq / Hkv;
  double* K = malloc((size_t)n * D * sizeof(double));
  double* V = malloc((size_t)n * D * sizeof(double));
  double* x = malloc((size_t)n * sizeof(double));
  double* qd = malloc((size_t)D * sizeof(double));
  int rc = (!K || !V || !x || !qd) ? OR_ENOMEM : OR_OK;
  for (int g = 0; g < Hkv && rc == OR_OK; ++g) {
    rc = gather_paged(K, V, k_cache, v_cache, table_row, n, g, Hkv, D, B, N, dtype);
    for (int32_t i = 0; i < T && rc == OR_OK; ++i) {
      for (int h = g * G; h < (g + 1) * G; ++h) {
        const uint16_t* qrow = q + ((int64_t)i * Hq + h) * D;
        for (int d = 0; d < D; ++d) qd[d] = to_double(qrow[d], dtype);
        attend(out + ((int64_t)i * Hq + h) * D, NULL, x, qd, K, V, (int64_t)p0 + i + 1, D, scale);
      }
    }
  }
  free(K);
  free(V);
  free(x);
  free(qd);
  return rc;
}

int oracle_attention_weights(double* weights, const uint16_t* q, const uint16_t* k_cache,
                             const uint16_t* v_cache, const int32_t* tables, int32_t max_blocks,
                             const int32_t* context_lens, int32_t s, int32_t h, double scale,
                             int32_t Hq, int32_t Hkv, int32_t D, int32_t B, int32_t N,
                             int32_t dtype) {
  if (check_heads(Hq, Hkv, D) || B <= 0 || h < 0 || h >= Hq) return OR_EINVAL;
  int64_t n = context_lens[s];
  if (n < 0 || (n + B - 1) / B > max_blocks) return OR_ERANGE;
  size_t cells = (size_t)(n > 0 ? n : 1) * D;
  double* K = malloc(cells * sizeof(double));
  double* V = malloc(cells * sizeof(double));
  double* x = malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
  double* qd = malloc((size_t)D * sizeof(double));
  double* o = malloc((size_t)D * sizeof(double));
  int rc = (!K || !V || !x || !qd || !o) ? OR_ENOMEM : OR_OK;
  if (rc == OR_OK)
    rc = gather_paged(K, V, k_cache, v_cache, tables + (int64_t)s * max_blocks, n, h / (Hq / Hkv),
                      Hkv, D, B, N, dtype);
  if (rc == OR_OK) {
    const uint16_t* qrow = q + ((int64_t)s * Hq + h) * D;
    for (int d = 0; d < D; ++d) qd[d] = to_double(qrow[d], dtype);
    attend(o, weights, x, qd, K, V, n, D, scale);
  }
  free(K);
  free(V);
  free(x);
  free(qd);
  free(o);
  return rc;
}

/*
 * Decode over a contiguous cache [S, Hkv, max_ctx, D]: the pre-paging layout in
 * which every request owns a max-length reservation (slides 6-7).
 */
int oracle_dense_decode(double* out, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* context_lens, int32_t s_begin, int32_t s_end,
                        int32_t max_ctx, double scale, int32_t Hq, int32_t Hkv, int32_t D,
                        int32_t dtype) {
  if (check_heads(Hq, Hkv, D) || max_ctx < 0) return OR_EINVAL;
  int G = Hq / Hkv;
  int rc = OR_OK;
  for (int32_t s = s_begin; s < s_end && rc == OR_OK; ++s) {
    int64_t n = context_lens[s];
    if (n < 0 || n > max_ctx) return OR_ERANGE;
    size_t cells = (size_t)(n > 0 ? n : 1) * D;
    double* K = malloc(cells * sizeof(double));
    double* V = malloc(cells * sizeof(double));
    double* x = malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double* qd = malloc((size_t)D * sizeof(double));
    if (!K || !V || !x || !qd) rc = OR_ENOMEM;
    for (int g = 0; g < Hkv && rc == OR_OK; ++g) {
      int64_t base = ((int64_t)s * Hkv + g) * max_ctx * D;
      for (int64_t i = 0; i < n * D; ++i) {
        K[i] = to_double(k[base + i], dtype);
        V[i] = to_double(v[base + i], dtype);
      }
      for (int h = g * G; h < (g + 1) * G; ++h) {
        const uint16_t* qrow = q + ((int64_t)s * Hq + h) * D;
        for (int d = 0; d < D; ++d) qd[d] = to_double(qrow[d], dtype);
        attend(out + ((int64_t)s * Hq + h) * D, NULL, x, qd, K, V, n, D, scale);
      }
    }
    free(K);
    free(V);
    free(x);
    free(qd);
  }
  return rc;
}

/*
 * Cache write: for every token i with slot = slots[i] >= 0, copy the row
 * key[i, g, :] to k_cache[slot / B, g, slot mod B, :] for each kv head g (and
 * the same for value / v_cache).  Byte copies, so the result is exact.
 * A slot at or beyond N * B is an error (nothing is written for it).
 */
int oracle_reshape_and_cache(uint8_t* k_cache, uint8_t* v_cache, const uint8_t* key,
                             const uint8_t* value, const int64_t* slots, int32_t T, int32_t Hkv,
                             int32_t D, int32_t B, int32_t elt_bytes, int32_t N) {
  if (T < 0 || Hkv <= 0 || D <= 0 || B <= 0 || elt_bytes <= 0 || N < 0) return OR_EINVAL;
  int rc = OR_OK;
  size_t row = (size_t)D * elt_bytes;
  for (int32_t i = 0; i < T; ++i) {
    int64_t slot = slots[i];
    if (slot < 0) continue;
    if (slot >= (int64_t)N * B) {
      rc = OR_ERANGE;
      continue;
    }
    int64_t frame = slot / B, off = slot % B;
    for (int g = 0; g < Hkv; ++g) {
      size_t dst = (size_t)(((frame * Hkv + g) * B + off)) * row;
      size_t src = ((size_t)i * Hkv + g) * row;
      memcpy(k_cache + dst, key + src, row);
      memcpy(v_cache + dst, value + src, row);
    }
  }
  return rc;
}

/*
 * Block copy: for each pair (src, dst) in order, frame dst of k_cache and of
 * v_cache becomes a copy of frame src (block_bytes = Hkv * B * D * elt each).
 */
int oracle_copy_blocks(uint8_t* k_cache, uint8_t* v_cache, const int64_t* pairs, int32_t n,
                       int64_t block_bytes, int32_t N) {
  if (n < 0 || block_bytes <= 0 || N < 0) return OR_EINVAL;
  for (int32_t i = 0; i < n; ++i) {
    int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= N || dst < 0 || dst >= N) return OR_ERANGE;
    if (src == dst) continue;
    memcpy(k_cache + dst * block_bytes, k_cache + src * block_bytes, (size_t)block_bytes);
    memcpy(v_cache + dst * block_bytes, v_cache + src * block_bytes, (size_t)block_bytes);
  }
  return OR_OK;
}
