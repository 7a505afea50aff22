/*
 * rpk_oracle.c -- plain, slow, fp64 CPU oracle for fused QK RoPE with a paged
 * KV cache and ragged causal grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header, table or helper with the CUDA kernels.
 *
 * Every function is the plain definition written out as loops, in fp64, in the
 * order the pages state it; no blocking, fusion or online (streaming) form,
 * except rpko_flash_step, which exists only to reproduce the pages' worked
 * online-softmax example.
 *
 * Sources (page title, section):
 *  - Mojo "generic_fused_qk_rope_bshd_paged_ragged_kernel_api" (Args, Parameters):
 *    ragged rows by input_row_offsets, RoPE on Q into output and on K into the
 *    paged cache, interleaved vs half pairing, per-token position_ids,
 *    M-RoPE sections, freqs_cis table indexed by position.
 *  - aria_kernel crate index (Functions: rope, rope_half, rope_half_partial):
 *    interleaved pairs, rotate-half pairs, partial rotary_dim.
 *  - algenta "Attention variant kernels" (transformer_attention: scaled score
 *    q.k/sqrt(d), stable softmax, causal mask; positional_encoding:
 *    rope_rotation_angle theta = pos * base^(-2i/d); flash_attention: running
 *    max / sum / output).
 *  - NumKong "Matrix Kernels" (Attention with a Pre-Packed KV-Cache): query row
 *    r of q rows over k keys sits at position r + k - q, sees keys_before keys
 *    before it and keys_after after; rows that see no key are zeros.
 *  - NumKong "NumKong for Python" (conversion policy): narrowing rounds to
 *    nearest, ties to even; (low-precision scalar types): e4m3 is 1 sign,
 *    4 exponent and 3 mantissa bits, range +-448, no infinity, with NaN.
 *  - Mojo "generic_fused_qk_rope_bshd_paged_ragged_kernel_api" (Parameters:
 *    cache_dtype; Args: kv_collection with a scale dtype and a quantization
 *    granularity): the cache may hold a narrower type than q with scales.
 *
 * Readings where the pages are silent (the same list is kept in the design
 * notes): freqs_cis is fp32 [max_position, rotary_dim] with (cos, sin) per
 * pair; the frequency of pair j is base^(-2j/rotary_dim); the rotation is
 * multiplication by e^{i theta}: (a, b) -> (a cos - b sin, b cos + a sin);
 * M-RoPE sections count rotary pairs and pair j takes its section's position;
 * a window w > 0 means w keys including the row's own (keys_before = w - 1);
 * masked keys are left out of the softmax (not given -1e9); an e4m3 cache
 * holds code = e4m3(x / scale) with one fp32 scale per KV head for K and one
 * for V (stored value = code * scale), values beyond the largest finite
 * saturating to +-448.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define RPKO_F32 0
#define RPKO_BF16 1
#define RPKO_E4M3 2

#define RPKO_OK 0
#define RPKO_ERR_ARG 1
#define RPKO_ERR_POSITION 2
#define RPKO_ERR_PAGE 3

/* ---------------------------------------------------------------- numbers */

/* bf16 bits -> fp64: the bf16 pattern is the top half of an fp32 pattern. */
double rpko_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* fp64 -> bf16 bits, one rounding, to nearest with ties to even.
 * bf16 = 1 sign, 8 exponent, 7 mantissa bits (NumKong scalar-type table), so
 * it has fp32's exponent range: normals down to 2^-126, subnormal spacing
 * 2^-133, largest finite (2 - 2^-7) * 2^127. The value is scaled so that one
 * bf16 unit in the last place is 1, rounded with rint (the C default rounding
 * mode is to nearest, ties to even) and scaled back; both scalings are exact
 * powers of two. */
uint16_t rpko_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isinf(a)) return sign | 0x7F80;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);                 /* a = m * 2^e2, m in [0.5, 1): leading bit 2^(e2-1) */
  int lead = e2 - 1;
  if (lead < -126) lead = -126;  /* subnormal range: fixed spacing 2^-133 */
  double ulp = ldexp(1.0, lead - 7);
  double r = rint(a / ulp) * ulp;
  if (r >= ldexp(1.0, 128)) return sign | 0x7F80;   /* rounds past the largest finite */
  float f = (float)r;            /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

/* e4m3 code -> fp64. The code is 1 sign bit, a 4-bit exponent with bias 7
 * and a 3-bit mantissa (E4M3 without infinities): exponent 0 holds the
 * subnormals m * 2^-9, exponent 15 with mantissa 7 is NaN, so the largest
 * finite value is 1.75 * 2^8 = 448. */
double rpko_e4m3_to_f64(uint8_t c) {
  int e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return (c & 0x80) ? -v : v;
}

/* fp64 -> e4m3 code, one rounding to nearest with ties to even. Magnitudes
 * from 448 up (including infinities) saturate to +-448: a value between 448
 * and 464 rounds to 448, 464 is a tie that goes to the even 448, and
 * anything larger has no finite code. NaN stays NaN. The value is scaled so
 * that one unit in the last place at its binade (2^-9 below the normals) is
 * 1, rounded with rint and scaled back, as for bf16. */
uint8_t rpko_f64_to_e4m3(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);
  int lead = e2 - 1;             /* a in [2^lead, 2^(lead+1)) */
  if (lead < -6) lead = -6;      /* below the normals: fixed spacing 2^-9 */
  double ulp = ldexp(1.0, lead - 3);
  double units = rint(a / ulp);  /* whole units in the last place, ties to even */
  double r = units * ulp;
  if (r < ldexp(1.0, -6)) return sign | (uint8_t)(r * 512.0);  /* subnormal code m */
  double mant = frexp(r, &e2);   /* r = mant * 2^e2, mant in [0.5, 1) */
  int E = e2 - 1 + 7;            /* biased exponent, 1 .. 15 */
  int M = (int)((mant * 2.0 - 1.0) * 8.0);  /* exact: r has at most 4 significant bits */
  return sign | (uint8_t)((E << 3) | M);
}

/* fp64 -> fp32 with one rounding to nearest, ties to even (C conversion). */
static float f64_to_f32(double x) { return (float)x; }

static double load_elt(const void* base, int dtype, size_t idx) {
  if (dtype == RPKO_F32) return (double)((const float*)base)[idx];
  return rpko_bf16_to_f64(((const uint16_t*)base)[idx]);
}

static void store_elt(void* base, int dtype, size_t idx, double v) {
  if (dtype == RPKO_F32) ((float*)base)[idx] = f64_to_f32(v);
  else ((uint16_t*)base)[idx] = rpko_f64_to_bf16(v);
}

static void copy_elt(void* dst, const void* src, int dtype, size_t di, size_t si) {
  if (dtype == RPKO_F32) ((float*)dst)[di] = ((const float*)src)[si];
  else ((uint16_t*)dst)[di] = ((const uint16_t*)src)[si];
}

/* Round n fp64 values to dtype (bf16 bits or fp32). */
void rpko_round(const double* x, size_t n, int dtype, void* out) {
  for (size_t i = 0; i < n; ++i) store_elt(out, dtype, i, x[i]);
}

/* Widen n dtype values to fp64. */
void rpko_widen(const void* x, size_t n, int dtype, double* out) {
  for (size_t i = 0; i < n; ++i) out[i] = load_elt(x, dtype, i);
}

/* ------------------------------------------------------------ RoPE table */

/* freqs_cis[p][2j] = cos(p * base^(-2j/R)), freqs_cis[p][2j+1] = sin(...),
 * evaluated in fp64 and rounded once to fp32. (algenta rope_rotation_angle:
 * theta = position * base^(-2i/d_model), with d_model read as rotary_dim.) */
int rpko_freqs_cis(int32_t max_position, int32_t rotary_dim, double base, float* out) {
  if (max_position < 0 || rotary_dim <= 0 || (rotary_dim & 1) || !(base > 0.0) || !out)
    return RPKO_ERR_ARG;
  int half = rotary_dim / 2;
  for (int32_t p = 0; p < max_position; ++p) {
    for (int j = 0; j < half; ++j) {
      double omega = pow(base, -2.0 * (double)j / (double)rotary_dim);
      double angle = (double)p * omega;
      out[(size_t)p * rotary_dim + 2 * j] = f64_to_f32(cos(angle));
      out[(size_t)p * rotary_dim + 2 * j + 1] = f64_to_f32(sin(angle));
    }
  }
  return RPKO_OK;
}

/* p-RoPE table (algenta "Attention variant kernels", rope_half_proportional:
 * the first factor * head_dim / 2 pairs of the rotate-half layout turn, the
 * other pairs are left as they are, and the frequencies take the full
 * head_dim as denominator). Width head_dim, read with rotary_dim = head_dim
 * in the half layout, so pair j is (x[j], x[j + head_dim/2]):
 *   j <  rotated_pairs: (cos, sin)(p * base^(-2j/head_dim)), fp64 rounded once;
 *   j >= rotated_pairs: (1, 0), the identity. */
int rpko_freqs_cis_proportional(int32_t max_position, int32_t head_dim, int32_t rotated_pairs,
                                double base, float* out) {
  if (max_position < 0 || head_dim <= 0 || (head_dim & 1) || !(base > 0.0) || !out)
    return RPKO_ERR_ARG;
  int half = head_dim / 2;
  if (rotated_pairs < 0 || rotated_pairs > half) return RPKO_ERR_ARG;
  for (int32_t p = 0; p < max_position; ++p) {
    for (int j = 0; j < half; ++j) {
      double c = 1.0, s = 0.0;
      if (j < rotated_pairs) {
        double omega = pow(base, -2.0 * (double)j / (double)head_dim);
        c = cos((double)p * omega);
        s = sin((double)p * omega);
      }
      out[(size_t)p * head_dim + 2 * j] = f64_to_f32(c);
      out[(size_t)p * head_dim + 2 * j + 1] = f64_to_f32(s);
    }
  }
  return RPKO_OK;
}

/* ---------------------------------------------------------------- RoPE */

/* Sequence that owns row t: the b with off[b] <= t < off[b+1]. */
static int owner_of(const int32_t* off, int32_t batch, int32_t t) {
  for (int32_t b = 0; b < batch; ++b)
    if (off[b] <= t && t < off[b + 1]) return b;
  return -1;
}

/* M-RoPE section of pair j: sections are consecutive runs of rotary pairs. */
static int section_of(const int32_t* mrope_section, int j) {
  if (!mrope_section) return 0;
  int acc = 0;
  for (int s = 0; s < 3; ++s) {
    acc += mrope_section[s];
    if (j < acc) return s;
  }
  return 2;
}

/*
 * Rotate every head row of x ([T, n_heads, head_dim], dtype) and return the
 * exact fp64 results in out ([T, n_heads, head_dim]).
 *   position of row t (sequence b, index i = t - off[b]):
 *     position_ids == NULL : cache_lens[b] + i
 *     no M-RoPE            : position_ids[t]
 *     M-RoPE               : position_ids[s * T + t] for pair j in section s
 *   pair j < R/2: interleaved -> (x[2j], x[2j+1]); half -> (x[j], x[j + R/2])
 *   (a, b) -> (a c - b s, b c + a s), c, s = freqs_cis[pos][2j], [2j+1]
 *   channels not in any pair are copied.
 */
int rpko_rope(const void* x, int dtype, int32_t T, int32_t n_heads, int32_t head_dim,
              const int32_t* row_offsets, int32_t batch, const int32_t* cache_lens,
              const int32_t* position_ids, const int32_t* mrope_section,
              const float* freqs_cis, int32_t max_position, int interleaved,
              int32_t rotary_dim, double* out) {
  if (!x || !row_offsets || !freqs_cis || !out) return RPKO_ERR_ARG;
  if (rotary_dim <= 0 || (rotary_dim & 1) || rotary_dim > head_dim) return RPKO_ERR_ARG;
  if (!position_ids && !cache_lens) return RPKO_ERR_ARG;
  if (mrope_section) {
    if (!position_ids) return RPKO_ERR_ARG;
    if (mrope_section[0] + mrope_section[1] + mrope_section[2] != rotary_dim / 2)
      return RPKO_ERR_ARG;
  }
  int half = rotary_dim / 2;
  for (int32_t t = 0; t < T; ++t) {
    int b = owner_of(row_offsets, batch, t);
    if (b < 0) return RPKO_ERR_ARG;
    int32_t i = t - row_offsets[b];
    for (int32_t h = 0; h < n_heads; ++h) {
      size_t base = ((size_t)t * n_heads + h) * head_dim;
      for (int32_t c = 0; c < head_dim; ++c) out[base + c] = load_elt(x, dtype, base + c);
      for (int j = 0; j < half; ++j) {
        int32_t pos;
        if (!position_ids) pos = cache_lens[b] + i;
        else if (!mrope_section) pos = position_ids[t];
        else pos = position_ids[(size_t)section_of(mrope_section, j) * T + t];
        if (pos < 0 || pos >= max_position) return RPKO_ERR_POSITION;
        double c = (double)freqs_cis[(size_t)pos * rotary_dim + 2 * j];
        double s = (double)freqs_cis[(size_t)pos * rotary_dim + 2 * j + 1];
        int i1 = interleaved ? 2 * j : j;
        int i2 = interleaved ? 2 * j + 1 : j + half;
        double a = load_elt(x, dtype, base + i1);
        double bb = load_elt(x, dtype, base + i2);
        out[base + i1] = a * c - bb * s;
        out[base + i2] = bb * c + a * s;
      }
    }
  }
  return RPKO_OK;
}

/* ----------------------------------------------------------- cache image */

/*
 * Write the new tokens into the paged pools ([num_pages, P, n_kv_heads, d]):
 * token i of sequence b goes to slot cache_lens[b] + i, i.e. page
 * block_table[b][slot / P], row slot % P. K comes from k_rot (fp64, rounded
 * once to the cache dtype), V is copied bit for bit from v_new.
 */
int rpko_cache_image(const double* k_rot, const void* v_new, int dtype, int32_t T,
                     int32_t n_kv_heads, int32_t head_dim, const int32_t* row_offsets,
                     int32_t batch, const int32_t* cache_lens, const int32_t* block_table,
                     int32_t max_pages_per_seq, int32_t num_pages, int32_t page_size,
                     void* k_pages, void* v_pages) {
  if (!k_rot || !v_new || !row_offsets || !cache_lens || !block_table || !k_pages || !v_pages)
    return RPKO_ERR_ARG;
  for (int32_t t = 0; t < T; ++t) {
    int b = owner_of(row_offsets, batch, t);
    if (b < 0) return RPKO_ERR_ARG;
    int32_t slot = cache_lens[b] + (t - row_offsets[b]);
    int32_t pi = slot / page_size;
    if (pi >= max_pages_per_seq) return RPKO_ERR_PAGE;
    int32_t page = block_table[(size_t)b * max_pages_per_seq + pi];
    if (page < 0 || page >= num_pages) return RPKO_ERR_PAGE;
    int32_t row = slot % page_size;
    for (int32_t kh = 0; kh < n_kv_heads; ++kh) {
      size_t src = ((size_t)t * n_kv_heads + kh) * head_dim;
      size_t dst = (((size_t)page * page_size + row) * n_kv_heads + kh) * head_dim;
      for (int32_t c = 0; c < head_dim; ++c) {
        store_elt(k_pages, dtype, dst + c, k_rot[src + c]);
        copy_elt(v_pages, v_new, dtype, dst + c, src + c);
      }
    }
  }
  return RPKO_OK;
}

/*
 * The same write into an e4m3 cache: K code = e4m3(k_rot / k_scale[kvh]) and
 * V code = e4m3(v / v_scale[kvh]), v widened exactly from dtype (bf16 or
 * fp32), each quotient formed in fp64 and rounded once.
 */
int rpko_cache_image_e4m3(const double* k_rot, const void* v_new, int dtype, int32_t T,
                          int32_t n_kv_heads, int32_t head_dim, const int32_t* row_offsets,
                          int32_t batch, const int32_t* cache_lens, const int32_t* block_table,
                          int32_t max_pages_per_seq, int32_t num_pages, int32_t page_size,
                          const float* k_scale, const float* v_scale, uint8_t* k_pages,
                          uint8_t* v_pages) {
  if (!k_rot || !v_new || !row_offsets || !cache_lens || !block_table || !k_pages || !v_pages ||
      !k_scale || !v_scale)
    return RPKO_ERR_ARG;
  for (int32_t t = 0; t < T; ++t) {
    int b = owner_of(row_offsets, batch, t);
    if (b < 0) return RPKO_ERR_ARG;
    int32_t slot = cache_lens[b] + (t - row_offsets[b]);
    int32_t pi = slot / page_size;
    if (pi >= max_pages_per_seq) return RPKO_ERR_PAGE;
    int32_t page = block_table[(size_t)b * max_pages_per_seq + pi];
    if (page < 0 || page >= num_pages) return RPKO_ERR_PAGE;
    int32_t row = slot - pi * page_size;
    for (int32_t kh = 0; kh < n_kv_heads; ++kh) {
      size_t src = ((size_t)t * n_kv_heads + kh) * head_dim;
      size_t dst = (((size_t)page * page_size + row) * n_kv_heads + kh) * head_dim;
      for (int32_t c = 0; c < head_dim; ++c) {
        k_pages[dst + c] = rpko_f64_to_e4m3(k_rot[src + c] / (double)k_scale[kh]);
        v_pages[dst + c] = rpko_f64_to_e4m3(load_elt(v_new, dtype, src + c) / (double)v_scale[kh]);
      }
    }
  }
  return RPKO_OK;
}

/* ------------------------------------------------------------- attention */

/* Visible key range of row r of a sequence with q_len rows and k_len keys:
 * the row sits at p = r + k_len - q_len; keys [lo, p] with lo = p - (w - 1)
 * under a window w > 0, else 0; clipped to [0, k_len). Empty when hi < lo. */
void rpko_band(int32_t r, int32_t q_len, int32_t k_len, int32_t window, int32_t* lo,
               int32_t* hi) {
  int64_t p = (int64_t)r + k_len - q_len;
  int64_t l = window > 0 ? p - (window - 1) : 0;
  if (l < 0) l = 0;
  int64_t h = p < (int64_t)k_len - 1 ? p : (int64_t)k_len - 1;
  *lo = (int32_t)l;
  *hi = (int32_t)h;
}

/* Key j is visible to row r (StreamingLLM attention sinks with a window,
 * algenta "Attention variant kernels", sparse_attention
 * streaming_llm_sink_score: the first `sinks` keys plus the recent window):
 * j <= p, and, under a window w > 0, either j >= p - (w - 1) or j < sinks.
 * sinks = 0 is the plain band of rpko_band. */
int rpko_visible(int32_t r, int32_t q_len, int32_t k_len, int32_t window, int32_t sinks,
                 int32_t j) {
  int64_t pos = (int64_t)r + k_len - q_len;
  if (j < 0 || j >= k_len || j > pos) return 0;
  if (window <= 0) return 1;
  return j >= pos - (window - 1) || j < sinks;
}

typedef struct {
  const void* q;
  int dtype;
  const int32_t* q_offsets;
  const int32_t* kv_lens;
  int32_t batch, T, n_heads, n_kv_heads, head_dim;
  const void* k_pages;
  const void* v_pages;
  int cache_dtype;        /* dtype of the pools: q's dtype, or RPKO_E4M3 with scales */
  const float* k_scale;   /* [n_kv_heads] for RPKO_E4M3 */
  const float* v_scale;
  int32_t page_size, num_pages, max_pages_per_seq;
  const int32_t* block_table;
  double scale;
  int32_t window;
  int32_t sinks;
  const int32_t* rows; /* pairs (t, h), or NULL for all */
  int64_t n_rows;
  double* out;         /* [n_rows, head_dim] */
  double* lse;         /* [n_rows] or NULL */
  int status;
} attn_job;

typedef struct {
  attn_job* job;
  int64_t begin, end;
  int status;
} attn_slice;

/* One output row: two passes over the visible keys (max, then weights).
 * With lse != NULL also its natural log-sum-exp of the scores, ln sum_j e^{s_j}
 * = m + ln sum_j e^{s_j - m} (NumKong attention_packed's log_sum_exp output);
 * -inf for a row that sees no key (an empty sum). */
/* Element idx of a pool of KV head kvh as the key or value it stands for. */
static double load_cache(const attn_job* J, const void* pool, const float* scale, int kvh,
                         size_t idx) {
  if (J->cache_dtype == RPKO_E4M3)
    return rpko_e4m3_to_f64(((const uint8_t*)pool)[idx]) * (double)scale[kvh];
  return load_elt(pool, J->cache_dtype, idx);
}

static int attention_row(const attn_job* J, int32_t t, int32_t h, double* o, double* w,
                         double* lse) {
  int d = J->head_dim;
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (lse) *lse = -INFINITY;
  int b = owner_of(J->q_offsets, J->batch, t);
  if (b < 0 || h < 0 || h >= J->n_heads) return RPKO_ERR_ARG;
  int32_t q_len = J->q_offsets[b + 1] - J->q_offsets[b];
  int32_t k_len = J->kv_lens[b];
  int32_t r = t - J->q_offsets[b];
  int32_t lo, hi;
  rpko_band(r, q_len, k_len, J->window, &lo, &hi);
  (void)lo; /* the sinks may reach below the window's first key */
  if (hi < 0) return RPKO_OK; /* no visible key: zeros */
  int group = J->n_heads / J->n_kv_heads;
  int kvh = h / group;
  size_t qbase = ((size_t)t * J->n_heads + h) * d;
  /* scores s_j = scale * sum_c q_c k_jc of the visible keys, in key order */
  double m = -INFINITY;
  int64_t n = 0;
  for (int32_t j = 0; j <= hi; ++j) {
    if (!rpko_visible(r, q_len, k_len, J->window, J->sinks, j)) continue;
    int32_t pi = j / J->page_size;
    if (pi >= J->max_pages_per_seq) return RPKO_ERR_PAGE;
    int32_t page = J->block_table[(size_t)b * J->max_pages_per_seq + pi];
    if (page < 0 || page >= J->num_pages) return RPKO_ERR_PAGE;
    size_t kbase = (((size_t)page * J->page_size + j % J->page_size) * J->n_kv_heads + kvh) * d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c)
      acc += load_elt(J->q, J->dtype, qbase + c) * load_cache(J, J->k_pages, J->k_scale, kvh,
                                                              kbase + c);
    double s = J->scale * acc;
    w[n++] = s;
    if (s > m) m = s;
  }
  if (n == 0) return RPKO_OK;
  /* weights e^{s_j - m} / sum e^{s - m}, then out = sum_j w_j v_j */
  double den = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    w[i] = exp(w[i] - m);
    den += w[i];
  }
  if (lse) *lse = m + log(den);
  int64_t i = 0;
  for (int32_t j = 0; j <= hi; ++j) {
    if (!rpko_visible(r, q_len, k_len, J->window, J->sinks, j)) continue;
    double wj = w[i++] / den;
    int32_t page = J->block_table[(size_t)b * J->max_pages_per_seq + j / J->page_size];
    size_t vbase = (((size_t)page * J->page_size + j % J->page_size) * J->n_kv_heads + kvh) * d;
    for (int c = 0; c < d; ++c) o[c] += wj * load_cache(J, J->v_pages, J->v_scale, kvh, vbase + c);
  }
  return RPKO_OK;
}

static int32_t max_kv(const attn_job* J) {
  int32_t m = 1;
  for (int32_t b = 0; b < J->batch; ++b)
    if (J->kv_lens[b] > m) m = J->kv_lens[b];
  return m;
}

static void* attention_worker(void* arg) {
  attn_slice* S = (attn_slice*)arg;
  const attn_job* J = S->job;
  double* w = (double*)malloc(sizeof(double) * (size_t)max_kv(J));
  if (!w) { S->status = RPKO_ERR_ARG; return NULL; }
  S->status = RPKO_OK;
  for (int64_t i = S->begin; i < S->end && S->status == RPKO_OK; ++i) {
    int32_t t, h;
    if (J->rows) { t = J->rows[2 * i]; h = J->rows[2 * i + 1]; }
    else { t = (int32_t)(i / J->n_heads); h = (int32_t)(i % J->n_heads); }
    S->status = attention_row(J, t, h, J->out + (size_t)i * J->head_dim, w,
                              J->lse ? J->lse + i : NULL);
  }
  free(w);
  return NULL;
}

/*
 * Ragged causal (optionally windowed, optionally with attention sinks)
 * grouped-query attention over the paged pools; the visible keys of a row are
 * those of rpko_visible. Query head h reads KV head h / (n_heads / n_kv_heads). Row r of
 * sequence b (q_len rows, kv_lens[b] keys) sees keys [lo, p], p = r + kv_len -
 * q_len (rpko_band). Output fp64, one row of head_dim per requested (t, h),
 * in the order given (rows == NULL: all T * n_heads rows, t-major), and, when
 * lse != NULL, each row's natural log-sum-exp of its scores (-inf when empty).
 * The pools hold q's dtype, or (cache_dtype RPKO_E4M3) e4m3 codes whose key
 * or value is code * k_scale[kvh] or code * v_scale[kvh], formed in fp64.
 * n_threads > 1 splits the rows over POSIX threads.
 */
int rpko_attention_cache(const void* q, int dtype, const int32_t* q_offsets,
                         const int32_t* kv_lens, int32_t batch, int32_t T, int32_t n_heads,
                         int32_t n_kv_heads, int32_t head_dim, const void* k_pages,
                         const void* v_pages, int cache_dtype, const float* k_scale,
                         const float* v_scale, int32_t page_size, int32_t num_pages,
                         const int32_t* block_table, int32_t max_pages_per_seq, double scale,
                         int32_t window, int32_t sinks, const int32_t* rows, int64_t n_rows,
                         double* out, double* lse, int n_threads) {
  if (!q || !q_offsets || !kv_lens || !k_pages || !v_pages || !block_table || !out)
    return RPKO_ERR_ARG;
  if (n_kv_heads <= 0 || n_heads % n_kv_heads != 0 || head_dim <= 0 || page_size <= 0)
    return RPKO_ERR_ARG;
  if (cache_dtype != dtype && !(cache_dtype == RPKO_E4M3 && k_scale && v_scale))
    return RPKO_ERR_ARG;
  attn_job J = {q, dtype, q_offsets, kv_lens, batch, T, n_heads, n_kv_heads, head_dim,
                k_pages, v_pages, cache_dtype, k_scale, v_scale, page_size, num_pages,
                max_pages_per_seq, block_table,
                scale, window, sinks, rows, rows ? n_rows : (int64_t)T * n_heads, out, lse, RPKO_OK};
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > J.n_rows) n_threads = J.n_rows > 0 ? (int)J.n_rows : 1;
  attn_slice slices[256];
  pthread_t tids[256];
  int64_t per = (J.n_rows + n_threads - 1) / n_threads;
  for (int i = 0; i < n_threads; ++i) {
    slices[i].job = &J;
    slices[i].begin = (int64_t)i * per;
    slices[i].end = slices[i].begin + per < J.n_rows ? slices[i].begin + per : J.n_rows;
    slices[i].status = RPKO_OK;
  }
  if (n_threads == 1) {
    attention_worker(&slices[0]);
  } else {
    for (int i = 0; i < n_threads; ++i) pthread_create(&tids[i], NULL, attention_worker, &slices[i]);
    for (int i = 0; i < n_threads; ++i) pthread_join(tids[i], NULL);
  }
  for (int i = 0; i < n_threads; ++i)
    if (slices[i].status != RPKO_OK) return slices[i].status;
  return RPKO_OK;
}

/* rpko_attention_cache with the pools in q's dtype. */
int rpko_attention(const void* q, int dtype, const int32_t* q_offsets, const int32_t* kv_lens,
                   int32_t batch, int32_t T, int32_t n_heads, int32_t n_kv_heads,
                   int32_t head_dim, const void* k_pages, const void* v_pages,
                   int32_t page_size, int32_t num_pages, const int32_t* block_table,
                   int32_t max_pages_per_seq, double scale, int32_t window, int32_t sinks,
                   const int32_t* rows, int64_t n_rows, double* out, double* lse,
                   int n_threads) {
  return rpko_attention_cache(q, dtype, q_offsets, kv_lens, batch, T, n_heads, n_kv_heads,
                              head_dim, k_pages, v_pages, dtype, NULL, NULL, page_size,
                              num_pages, block_table, max_pages_per_seq, scale, window, sinks,
                              rows, n_rows, out, lse, n_threads);
}

/* --------------------------------------------------------- gradients */

/*
 * Gradients of rpko_attention_cache's output (NumKong "Attention with a
 * Pre-Packed KV-Cache": attention_packed_gradients turns the output gradient
 * into query, key and value gradients under the same band). For each row i
 * (token t, head h) and each key j it sees, written out from the definition
 * of softmax attention: s_ij = scale q_i.k_j, P_ij = e^{s_ij} / sum_j' e^{s_ij'}
 * (two-pass, as the forward oracle), dP_ij = dO_i.v_j, D_i = sum_j P_ij dP_ij,
 * dS_ij = P_ij (dP_ij - D_i); then dQ_i = scale sum_j dS_ij k_j,
 * dK_j += scale dS_ij q_i and dV_j += P_ij dO_i, summed over every row and
 * query head that sees key j. dK and dV have the pools' shape
 * [num_pages, page_size, n_kv_heads, head_dim] and are zero where no row
 * looks; dQ is [T, n_heads, head_dim]; d_out is [T, n_heads, head_dim] of
 * dtype (q's). All fp64, single-threaded.
 */
int rpko_attention_backward(const void* q, const void* d_out, int dtype, const int32_t* q_offsets,
                            const int32_t* kv_lens, int32_t batch, int32_t T, int32_t n_heads,
                            int32_t n_kv_heads, int32_t head_dim, const void* k_pages,
                            const void* v_pages, int cache_dtype, const float* k_scale,
                            const float* v_scale, int32_t page_size, int32_t num_pages,
                            const int32_t* block_table, int32_t max_pages_per_seq, double scale,
                            int32_t window, int32_t sinks, double* d_q, double* d_k, double* d_v) {
  if (!q || !d_out || !q_offsets || !kv_lens || !k_pages || !v_pages || !block_table || !d_q ||
      !d_k || !d_v)
    return RPKO_ERR_ARG;
  if (n_kv_heads <= 0 || n_heads % n_kv_heads != 0 || head_dim <= 0 || page_size <= 0)
    return RPKO_ERR_ARG;
  if (cache_dtype != dtype && !(cache_dtype == RPKO_E4M3 && k_scale && v_scale))
    return RPKO_ERR_ARG;
  attn_job J = {q, dtype, q_offsets, kv_lens, batch, T, n_heads, n_kv_heads, head_dim,
                k_pages, v_pages, cache_dtype, k_scale, v_scale, page_size, num_pages,
                max_pages_per_seq, block_table, scale, window, sinks, NULL, 0, NULL, NULL,
                RPKO_OK};
  const int d = head_dim;
  const size_t pool = (size_t)num_pages * page_size * n_kv_heads * d;
  for (size_t e = 0; e < pool; ++e) d_k[e] = d_v[e] = 0.0;
  for (size_t e = 0; e < (size_t)T * n_heads * d; ++e) d_q[e] = 0.0;
  const int group = n_heads / n_kv_heads;
  int32_t maxk = max_kv(&J);
  double* p = (double*)malloc(sizeof(double) * (size_t)maxk);
  double* dp = (double*)malloc(sizeof(double) * (size_t)maxk);
  size_t* base = (size_t*)malloc(sizeof(size_t) * (size_t)maxk);
  if (!p || !dp || !base) { free(p); free(dp); free(base); return RPKO_ERR_ARG; }
  int status = RPKO_OK;
  for (int32_t t = 0; t < T && status == RPKO_OK; ++t) {
    int b = owner_of(q_offsets, batch, t);
    if (b < 0) { status = RPKO_ERR_ARG; break; }
    int32_t q_len = q_offsets[b + 1] - q_offsets[b];
    int32_t k_len = kv_lens[b];
    int32_t r = t - q_offsets[b];
    for (int32_t h = 0; h < n_heads && status == RPKO_OK; ++h) {
      int kv_head = h / group;
      size_t qb = ((size_t)t * n_heads + h) * d;
      /* visible keys: scores, then weights */
      int64_t n = 0;
      double m = -INFINITY;
      for (int32_t j = 0; j < k_len; ++j) {
        if (!rpko_visible(r, q_len, k_len, window, sinks, j)) continue;
        int32_t pi = j / page_size;
        if (pi >= max_pages_per_seq) { status = RPKO_ERR_PAGE; break; }
        int32_t page = block_table[(size_t)b * max_pages_per_seq + pi];
        if (page < 0 || page >= num_pages) { status = RPKO_ERR_PAGE; break; }
        base[n] = (((size_t)page * page_size + j % page_size) * n_kv_heads + kv_head) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
          acc += load_elt(q, dtype, qb + c) * load_cache(&J, k_pages, k_scale, kv_head, base[n] + c);
        p[n] = scale * acc;
        if (p[n] > m) m = p[n];
        ++n;
      }
      if (status != RPKO_OK || n == 0) continue;
      double den = 0.0;
      for (int64_t i = 0; i < n; ++i) {
        p[i] = exp(p[i] - m);
        den += p[i];
      }
      double D = 0.0;
      for (int64_t i = 0; i < n; ++i) {
        p[i] /= den;
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
          acc += load_elt(d_out, dtype, qb + c) * load_cache(&J, v_pages, v_scale, kv_head, base[i] + c);
        dp[i] = acc;
        D += p[i] * dp[i];
      }
      for (int64_t i = 0; i < n; ++i) {
        double ds = p[i] * (dp[i] - D);
        for (int c = 0; c < d; ++c) {
          d_q[qb + c] += scale * ds * load_cache(&J, k_pages, k_scale, kv_head, base[i] + c);
          d_k[base[i] + c] += scale * ds * load_elt(q, dtype, qb + c);
          d_v[base[i] + c] += p[i] * load_elt(d_out, dtype, qb + c);
        }
      }
    }
  }
  free(p);
  free(dp);
  free(base);
  return status;
}

/* ------------------------------------------------- online-softmax state */

/*
 * One step of the flash-style running state (algenta flash_attention:
 * flash_block_max, flash_block_sum_exp, flash_block_output), per key with
 * score s and value v: m' = max(m, s); l' = l e^{m - m'} + e^{s - m'};
 * o' = o e^{m - m'} + e^{s - m'} v. The final output is o / l
 * (flash_final_normalize). Used only to reproduce the pages' worked example
 * and to cross-check the two-pass definition above.
 */
void rpko_flash_step(double* m, double* l, double* o, double s, double v) {
  double m_new = *m > s ? *m : s;
  double alpha = exp(*m - m_new);
  double p = exp(s - m_new);
  *l = *l * alpha + p;
  *o = *o * alpha + p * v;
  *m = m_new;
}
