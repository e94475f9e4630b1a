/*
 * qkv_oracle.c -- plain, slow, fp64 CPU statement of the decode hot path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. The CUDA library never calls it, links
 * it or shares a header, helper or constant with it.
 *
 * Sources (page title, section):
 *   [YARN]  mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
 *           hybrid paged attention for Qwen3.5-Next long-context serving",
 *           section 1 "YaRN rope scaling for the Qwen3.5 partial rotary":
 *           llama.cpp-style corr_dims ramp from beta_fast 32 / beta_slow 1,
 *           net table scale 1 + 0.1 ln(factor) (1.0199427025 at 1.220703125).
 *   [AUTO]  ignis "context-and-speculation", flag --model-rope-scaling: YaRN
 *           factor = max_context / 262,144; the attention factor applies to
 *           queries and keys alike.
 *   [F4]    same mistral.rs PR, section 2 "4-bit F4 KV cache": symmetric
 *           4-bit values (nibble - 8) * scale, 32 values per 16-byte cell.
 *   [SPLIT] same PR section 2 (v1/v2 paged_attention, inline dequant) and
 *           FreeToken issue #568 "Serving ...'s 1M-token window on one 24 GB
 *           card", proposed solution item 2: partials folded by
 *           log2-sum-exp.
 *   [GATHER] same PR section 2: gather_kv_cache gains an F4 path (the paged
 *           cache read back into contiguous rows for prefill attention).
 *   [CHUNK] same PR section 5: paged prefill runs in chunks of 2048 tokens.
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): amax/7 scale rounded once to fp16 (RNE, saturating at 65504);
 * codes by round-half-to-even of x/scale, clamped to [-8, 7]; even element in
 * the low nibble; NEOX rotate-half on the first rot_dim dims; the table scale
 * multiplies cos and sin; softmax scale 1/sqrt(head_dim).
 *
 * Everything is computed in double. No blocking, fusion or reordering beyond
 * the definitions; the attention loop parallelises over independent
 * (sequence, query head) rows only.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Number formats. bf16 = top half of an IEEE binary32; fp16 = IEEE binary16. */

double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);               /* subnormal */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp(1.0 + m / 1024.0, e - 15);
  return sign ? -v : v;
}

/* Round a double to a binary format with `mbits` stored mantissa bits and
 * exponent bias `bias`, ties to even, no saturation (overflow gives inf).
 * Returns the bit pattern without the sign. */
static uint32_t round_to_format(double a, int mbits, int bias, int ebits) {
  const int emax = (1 << ebits) - 2 - bias; /* largest normal exponent */
  const int emin = 1 - bias;                /* smallest normal exponent */
  if (a == 0.0) return 0;
  if (isnan(a)) return ((uint32_t)((1 << ebits) - 1) << mbits) | (1u << (mbits - 1));
  int E;
  frexp(a, &E); /* a = f * 2^E, f in [0.5, 1) */
  int e = E - 1; /* a in [2^e, 2^(e+1)) */
  if (e < emin) {
    /* subnormal: integer count of 2^(emin - mbits) */
    double q = nearbyint(ldexp(a, mbits - emin)); /* ties to even */
    return (uint32_t)q; /* q == 2^mbits becomes the smallest normal */
  }
  double frac = ldexp(a, -e) - 1.0;              /* exact, in [0, 1) */
  double q = nearbyint(ldexp(frac, mbits));       /* ties to even */
  if (q == ldexp(1.0, mbits)) { q = 0; e += 1; }
  if (e > emax) return (uint32_t)((1 << ebits) - 1) << mbits; /* inf */
  return ((uint32_t)(e + bias) << mbits) | (uint32_t)q;
}

uint16_t oracle_f64_to_f16(double x) {
  uint16_t s = signbit(x) ? 0x8000 : 0;
  return s | (uint16_t)round_to_format(fabs(x), 10, 15, 5);
}

uint16_t oracle_f64_to_bf16(double x) {
  uint16_t s = signbit(x) ? 0x8000 : 0;
  return s | (uint16_t)round_to_format(fabs(x), 7, 127, 8);
}

/* ------------------------------------------------------------------------- */
/* YaRN rotary table [YARN], [AUTO].                                          */

typedef struct {
  double rope_base;
  int32_t rot_dim;
  int32_t reserved;
  double factor;       /* s; 1 = no scaling */
  int64_t orig_max_pos;
  double beta_fast;    /* 32 */
  double beta_slow;    /* 1 */
  double ext_factor;   /* < 0: 1 when s > 1, else 0 */
  double attn_factor;  /* <= 0: 1 + 0.1 ln s when s > 1, else 1 */
} oracle_yarn_params;

/* The dimension-pair index at which a frequency completes `beta` full turns
 * over the original context: solves orig * base^(-2j/d) / (2 pi) = beta. */
static double corr_dim(int d, double base, double orig, double beta) {
  return d * log(orig / (beta * 2.0 * M_PI)) / (2.0 * log(base));
}

/* theta[j], j < rot_dim/2: per-position angle increment of pair j; returns
 * the table scale (mscale). low/high receive the ramp bounds. */
double oracle_yarn_theta(const oracle_yarn_params* p, double* theta, double* low_out,
                         double* high_out) {
  const int d = p->rot_dim;
  const double s = p->factor;
  const double ext = p->ext_factor < 0 ? (s > 1.0 ? 1.0 : 0.0) : p->ext_factor;
  const double mscale = p->attn_factor > 0 ? p->attn_factor : (s > 1.0 ? 1.0 + 0.1 * log(s) : 1.0);
  double low = floor(corr_dim(d, p->rope_base, (double)p->orig_max_pos, p->beta_fast));
  double high = ceil(corr_dim(d, p->rope_base, (double)p->orig_max_pos, p->beta_slow));
  if (low < 0) low = 0;
  if (high > d - 1) high = d - 1;
  for (int j = 0; j < d / 2; ++j) {
    const double omega = pow(p->rope_base, -2.0 * j / d);
    double y = (j - low) / fmax(0.001, high - low);
    if (y < 0) y = 0;
    if (y > 1) y = 1;
    const double ramp = (1.0 - y) * ext; /* 1: keep omega, 0: omega / s */
    theta[j] = (omega / s) * (1.0 - ramp) + omega * ramp;
  }
  if (low_out) *low_out = low;
  if (high_out) *high_out = high;
  return mscale;
}

/* cos/sin [n_pos][rot_dim/2] of positions pos0 .. pos0+n_pos-1, times mscale. */
void oracle_yarn_table(const oracle_yarn_params* p, int64_t pos0, int64_t n_pos, double* cos_out,
                       double* sin_out) {
  const int h = p->rot_dim / 2;
  double theta[512];
  const double ms = oracle_yarn_theta(p, theta, 0, 0);
  for (int64_t i = 0; i < n_pos; ++i)
    for (int j = 0; j < h; ++j) {
      const double a = (double)(pos0 + i) * theta[j];
      cos_out[i * h + j] = ms * cos(a);
      sin_out[i * h + j] = ms * sin(a);
    }
}

/* NEOX rotate-half on dims [0, rot_dim) of each head, in double:
 * (x_j, x_{j+h}) -> (x_j c - x_{j+h} s, x_{j+h} c + x_j s), c/s from the
 * table at the token's position; dims >= rot_dim pass through. */
void oracle_rope_apply_f64(const double* x, double* out, const int64_t* positions, int n_tok,
                           int n_heads, int head_dim, const oracle_yarn_params* p) {
  const int d = p->rot_dim, h = d / 2;
  double theta[512];
  const double ms = oracle_yarn_theta(p, theta, 0, 0);
  for (int t = 0; t < n_tok; ++t)
    for (int hh = 0; hh < n_heads; ++hh) {
      const double* xi = x + ((size_t)t * n_heads + hh) * head_dim;
      double* yo = out + ((size_t)t * n_heads + hh) * head_dim;
      for (int j = 0; j < h; ++j) {
        const double a = (double)positions[t] * theta[j];
        const double c = ms * cos(a), s = ms * sin(a);
        const double x0 = xi[j], x1 = xi[j + h];
        yo[j] = x0 * c - x1 * s;
        yo[j + h] = x1 * c + x0 * s;
      }
      for (int j = d; j < head_dim; ++j) yo[j] = xi[j];
    }
}

/* bf16 in, bf16 out (round to nearest even from the double result). */
void oracle_rope_apply_bf16(const uint16_t* x, uint16_t* out, const int64_t* positions, int n_tok,
                            int n_heads, int head_dim, const oracle_yarn_params* p) {
  const int d = p->rot_dim, h = d / 2;
  double theta[512];
  const double ms = oracle_yarn_theta(p, theta, 0, 0);
  for (int t = 0; t < n_tok; ++t)
    for (int hh = 0; hh < n_heads; ++hh) {
      const uint16_t* xi = x + ((size_t)t * n_heads + hh) * head_dim;
      uint16_t* yo = out + ((size_t)t * n_heads + hh) * head_dim;
      for (int j = 0; j < h; ++j) {
        const double a = (double)positions[t] * theta[j];
        const double c = ms * cos(a), s = ms * sin(a);
        const double x0 = oracle_bf16_to_f64(xi[j]), x1 = oracle_bf16_to_f64(xi[j + h]);
        yo[j] = oracle_f64_to_bf16(x0 * c - x1 * s);
        yo[j + h] = oracle_f64_to_bf16(x1 * c + x0 * s);
      }
      for (int j = d; j < head_dim; ++j) yo[j] = xi[j];
    }
}

/* ------------------------------------------------------------------------- */
/* F4 quantisation [F4].                                                     */

/* A group of n values (n even, <= 1024) sharing one scale: scale =
 * fp16(amax / 7) (saturating at 65504), code_i = clamp(rint(x_i / scale),
 * -8, 7) + 8, all codes 8 when scale is 0; byte b holds element 2b in bits
 * 0-3 and element 2b+1 in bits 4-7. The PR's K cells are groups of 32; its V
 * scale is "one scale per token per V head", a group of head_dim. */
void oracle_quantize_group(const uint16_t* x, int n, uint8_t* bytes, uint16_t* scale_out) {
  double amax = 0;
  for (int i = 0; i < n; ++i) amax = fmax(amax, fabs(oracle_bf16_to_f64(x[i])));
  uint16_t sc = oracle_f64_to_f16(amax / 7.0);
  if ((sc & 0x7FFF) == 0x7C00) sc = 0x7BFF; /* saturate to 65504 */
  const double s = oracle_f16_to_f64(sc);
  int code[1024];
  for (int i = 0; i < n; ++i) {
    if (s == 0) { code[i] = 8; continue; }
    double r = nearbyint(oracle_bf16_to_f64(x[i]) / s); /* ties to even */
    if (r < -8) r = -8;
    if (r > 7) r = 7;
    code[i] = (int)r + 8;
  }
  for (int b = 0; b < n / 2; ++b) bytes[b] = (uint8_t)(code[2 * b] | (code[2 * b + 1] << 4));
  *scale_out = sc;
}

/* One 32-value cell. */
void oracle_quantize_cell(const uint16_t* x, uint8_t* bytes, uint16_t* scale_out) {
  oracle_quantize_group(x, 32, bytes, scale_out);
}

/* Paged cache, per layer and for each of K and V:
 *   data  u8  [num_pages][kv_heads][block_size][head_dim/2]
 *   scale f16 [num_pages][kv_heads][block_size][head_dim/32] for K, and
 *             [num_pages][kv_heads][block_size][head_dim/v_group] for V
 *             (v_group 32: per cell; head_dim: one scale per token)
 * Token i of a sequence lives in page page_table[i / B] at offset i % B; a
 * write goes to slot = page * B + offset. Slots < 0 are skipped; slots past
 * the pool are skipped and counted. Returns the count of skipped bad slots. */
int oracle_kv_write_f4(const uint16_t* k, const uint16_t* v, const int64_t* slots, int64_t n_tok,
                       uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                       int kv_heads, int head_dim, int block_size, int64_t num_pages, int v_group) {
  int bad = 0;
  const int cells = head_dim / 32, vgroups = head_dim / v_group;
  for (int64_t t = 0; t < n_tok; ++t) {
    const int64_t slot = slots[t];
    if (slot < 0) continue;
    if (slot >= num_pages * block_size) { ++bad; continue; }
    const int64_t page = slot / block_size, off = slot % block_size;
    for (int h = 0; h < kv_heads; ++h) {
      const size_t row = ((size_t)page * kv_heads + h) * block_size + off;
      for (int c = 0; c < cells; ++c) {
        const size_t src = ((size_t)t * kv_heads + h) * head_dim + 32 * c;
        oracle_quantize_cell(k + src, k_data + row * (head_dim / 2) + 16 * c, k_scale + row * cells + c);
      }
      for (int c = 0; c < vgroups; ++c) {
        const size_t src = ((size_t)t * kv_heads + h) * head_dim + (size_t)v_group * c;
        oracle_quantize_group(v + src, v_group, v_data + row * (head_dim / 2) + (v_group / 2) * c,
                              v_scale + row * vgroups + c);
      }
    }
  }
  return bad;
}

/* Dequantised element d of the cache row: (code - 8) * scale, exact in
 * double; `group` values share a scale. */
static double deq(const uint8_t* data, const uint16_t* scale, size_t row, int head_dim, int group, int d) {
  const uint8_t byte = data[row * (head_dim / 2) + d / 2];
  const int code = (d & 1) ? (byte >> 4) : (byte & 15);
  return (code - 8) * oracle_f16_to_f64(scale[row * (head_dim / group) + d / group]);
}

/* ------------------------------------------------------------------------- */
/* Exact softmax attention over the paged cache [SPLIT].                     */

/* For each sequence s and query head h (KV head h / (Hq/Hkv)) over context
 * tokens [tok_begin[s], tok_end[s]):
 *   score_t = softmax_scale * sum_d q[d] * k^_t[d]
 *   out     = sum_t exp(score_t - m) v^_t / sum_t exp(score_t - m)
 *   lse2    = log2 sum_t exp(score_t)
 * An empty range gives out = 0 and lse2 = -inf. out [n_seq][Hq][D] and
 * lse2 [n_seq][Hq] are double. */
void oracle_paged_attention(const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
                            const uint8_t* v_data, const uint16_t* v_scale,
                            const int32_t* page_table, int max_pages_per_seq,
                            const int32_t* tok_begin, const int32_t* tok_end, int n_seq,
                            int q_heads, int kv_heads, int head_dim, int block_size,
                            double softmax_scale, double* out, double* lse2, int n_threads, int v_group) {
  const int group = q_heads / kv_heads;
  const long rows = (long)n_seq * q_heads;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long r = 0; r < rows; ++r) {
    const int s = (int)(r / q_heads), h = (int)(r % q_heads), kvh = h / group;
    const int t0 = tok_begin[s], t1 = tok_end[s];
    double* o = out + (size_t)r * head_dim;
    for (int d = 0; d < head_dim; ++d) o[d] = 0;
    if (t1 <= t0) { lse2[r] = -INFINITY; continue; }
    double qd[1024];
    for (int d = 0; d < head_dim; ++d) qd[d] = oracle_bf16_to_f64(q[(size_t)r * head_dim + d]);
    /* pass 1: scores and their maximum */
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
      const size_t row = ((size_t)page_table[(size_t)s * max_pages_per_seq + t / block_size] * kv_heads + kvh) * block_size + t % block_size;
      double dot = 0;
      for (int d = 0; d < head_dim; ++d) dot += qd[d] * deq(k_data, k_scale, row, head_dim, 32, d);
      const double sc = softmax_scale * dot;
      if (sc > m) m = sc;
    }
    /* pass 2: weights, normaliser, weighted values */
    double z = 0;
    for (int t = t0; t < t1; ++t) {
      const size_t row = ((size_t)page_table[(size_t)s * max_pages_per_seq + t / block_size] * kv_heads + kvh) * block_size + t % block_size;
      double dot = 0;
      for (int d = 0; d < head_dim; ++d) dot += qd[d] * deq(k_data, k_scale, row, head_dim, 32, d);
      const double w = exp(softmax_scale * dot - m);
      z += w;
      for (int d = 0; d < head_dim; ++d) o[d] += w * deq(v_data, v_scale, row, head_dim, v_group, d);
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= z;
    lse2[r] = (m + log(z)) / log(2.0);
  }
}

/* ------------------------------------------------------------------------- */
/* Paged -> contiguous gather of the F4 cache [GATHER].                      */

/* For each sequence s and each of its context tokens t < seq_lens[s], every
 * KV head h and element d:
 *   k_out[out_start[s] + t][h][d] = bf16((code - 8) * k_scale)
 *   v_out[...]                    = bf16((code - 8) * v_scale)
 * The product is exact in double; bf16 rounds to nearest even. A token whose
 * page-table entry lies outside [0, num_pages) gives zero rows; the return
 * value counts such tokens. */
int64_t oracle_gather_kv_f4(const uint8_t* k_data, const uint16_t* k_scale, const uint8_t* v_data,
                            const uint16_t* v_scale, const int32_t* page_table, int max_pages_per_seq,
                            const int32_t* seq_lens, const int64_t* out_start, int n_seq, int kv_heads,
                            int head_dim, int block_size, int64_t num_pages, int v_group, uint16_t* k_out,
                            uint16_t* v_out) {
  int64_t bad = 0;
  for (int s = 0; s < n_seq; ++s) {
    for (int t = 0; t < seq_lens[s]; ++t) {
      const int32_t page = page_table[(size_t)s * max_pages_per_seq + t / block_size];
      const int ok = page >= 0 && page < num_pages;
      bad += !ok;
      for (int h = 0; h < kv_heads; ++h) {
        const size_t dst = ((size_t)(out_start[s] + t) * kv_heads + h) * head_dim;
        const size_t row = ((size_t)(ok ? page : 0) * kv_heads + h) * block_size + t % block_size;
        for (int d = 0; d < head_dim; ++d) {
          k_out[dst + d] = ok ? oracle_f64_to_bf16(deq(k_data, k_scale, row, head_dim, 32, d)) : 0;
          v_out[dst + d] = ok ? oracle_f64_to_bf16(deq(v_data, v_scale, row, head_dim, v_group, d)) : 0;
        }
      }
    }
  }
  return bad;
}

/* ------------------------------------------------------------------------- */
/* log2-sum-exp fold of partials [SPLIT].                                     */

/* parts: o [n_parts][rows][D], lse2 [n_parts][rows]. Per row:
 *   M = max_i lse2_i, w_i = 2^(lse2_i - M), O = sum_i w_i o_i / sum_i w_i,
 *   lse2 = M + log2 sum_i w_i. Parts with lse2 = -inf carry no weight; a row
 * with no weighted part gives O = 0 and lse2 = -inf. */
void oracle_lse_merge(const double* o_parts, const double* lse2_parts, int n_parts, int rows,
                      int head_dim, double* out, double* lse2_out) {
  for (int r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int i = 0; i < n_parts; ++i) M = fmax(M, lse2_parts[(size_t)i * rows + r]);
    double* o = out + (size_t)r * head_dim;
    for (int d = 0; d < head_dim; ++d) o[d] = 0;
    if (M == -INFINITY) { lse2_out[r] = -INFINITY; continue; }
    double wsum = 0;
    for (int i = 0; i < n_parts; ++i) {
      const double l = lse2_parts[(size_t)i * rows + r];
      if (l == -INFINITY) continue;
      const double w = exp2(l - M);
      wsum += w;
      for (int d = 0; d < head_dim; ++d) o[d] += w * o_parts[((size_t)i * rows + r) * head_dim + d];
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= wsum;
    lse2_out[r] = M + log2(wsum);
  }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Array forms of the format conversions (used by the tests). */
void oracle_f64_to_f16_array(const double* x, uint16_t* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = oracle_f64_to_f16(x[i]);
}
void oracle_f16_to_f64_array(const uint16_t* x, double* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = oracle_f16_to_f64(x[i]);
}
void oracle_f64_to_bf16_array(const double* x, uint16_t* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = oracle_f64_to_bf16(x[i]);
}
void oracle_bf16_to_f64_array(const uint16_t* x, double* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = oracle_bf16_to_f64(x[i]);
}
