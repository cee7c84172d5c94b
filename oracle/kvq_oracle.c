/*
 * kvq_oracle.c -- plain single-threaded CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and the bench's CPU baseline may load
 * this code.  It is written straight from the pages, step by step in their
 * order, with no blocking, fusion or reordering:
 *   [P1] Strata PR #21 "Q4_0 KV cache + FWHT-256" (What, Why, How 1-3, and the
 *        maintainer's merge note).
 *   [P5] vLLM API page "vllm.v1.attention.ops.rocm_octave".
 * Where the pages leave a step open, the reading taken is stated at the step.
 * Build flags: -O2 -ffp-contract=off -fno-fast-math (no fused multiply-add,
 * IEEE round-to-nearest single precision on x86-64 SSE).
 */
#include "kvq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define Q4_DIM 256   /* head dimension of the Q4_0 path [P1 What: D=256] */
#define Q4_BLK 32    /* values per Q4_0 block [P1 How 2] */
#define OCT_HB 64    /* Octave HADAMARD_BLOCK (reading: 64-dim blocks) */
#define OCT_ROPE_BITS 4   /* [P5 module text: RoPE blocks get 4-bit codes] */
#define OCT_NOPE_BITS 3   /* [P5 module text: NoPE blocks get 3-bit codes] */
#define OCT_LUT_ONE 64.0f /* reading: any power of two; 64 keeps fp16 scales normal */

static int finite_f(float x) { return isfinite(x) != 0; }

/* ===================================================================== */
/* Scalar conversions                                                     */
/* ===================================================================== */

/* fp32 -> IEEE 754 binary16, round to nearest, ties to even, written from the
 * format definition (1 sign, 5 exponent bits with bias 15, 10 fraction bits,
 * subnormals m * 2^-24). */
uint16_t orc_f32_to_f16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  uint32_t sign = (x >> 16) & 0x8000u;
  uint32_t exp = (x >> 23) & 0xFFu;
  uint32_t man = x & 0x7FFFFFu;
  if (exp == 0xFFu) {                       /* inf / nan */
    if (man) return (uint16_t)(sign | 0x7E00u | (man >> 13));
    return (uint16_t)(sign | 0x7C00u);
  }
  int e = (int)exp - 127;
  if (e > 15) return (uint16_t)(sign | 0x7C00u);  /* |f| >= 2^16: overflow */
  if (e >= -14) {                                  /* normal binary16 */
    uint32_t h = ((uint32_t)(e + 15) << 10) | (man >> 13);
    uint32_t rem = man & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h++; /* carry may reach inf */
    return (uint16_t)(sign | h);
  }
  if (e < -25) return (uint16_t)sign;              /* below half the smallest subnormal */
  /* subnormal result: m = round(|f| / 2^-24) */
  uint32_t sig = 0x800000u | man;
  int shift = -e - 1;                              /* 14 .. 24 */
  uint32_t m = sig >> shift;
  uint32_t rem = sig & ((1u << shift) - 1u);
  uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (m & 1u))) m++;
  return (uint16_t)(sign | m);
}

float orc_f16_to_f32(uint16_t h) {
  uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
  uint32_t exp = (h >> 10) & 0x1Fu;
  uint32_t man = h & 0x3FFu;
  float out;
  if (exp == 0) {
    /* zero or subnormal: man * 2^-24, exact in fp32 */
    out = (float)man * 5.9604644775390625e-08f;
    if (sign) out = -out;
    return out;
  }
  uint32_t bits;
  if (exp == 0x1Fu) bits = sign | 0x7F800000u | (man << 13);
  else bits = sign | ((exp - 15u + 127u) << 23) | (man << 13);
  memcpy(&out, &bits, 4);
  return out;
}

float orc_bf16_to_f32(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float out;
  memcpy(&out, &bits, 4);
  return out;
}

void orc_f32_to_f16_array(const float *x, uint16_t *y, int64_t n) {
  for (int64_t i = 0; i < n; i++) y[i] = orc_f32_to_f16(x[i]);
}

static float load_elem(const void *p, int dtype, int64_t i) {
  if (dtype == 1) return orc_bf16_to_f32(((const uint16_t *)p)[i]);
  return ((const float *)p)[i];
}

/* ===================================================================== */
/* Rotation [P5 fwht_blocks; P1 How 1]                                    */
/* ===================================================================== */

static int is_pow2(int n) { return n > 0 && (n & (n - 1)) == 0; }

/* One block, fp32: stages h = 1, 2, 4, ...; within each stage every pair
 * (i, i+h) with i's h-bit clear becomes (a + b, a - b); the orthonormal scale
 * fp32(1/sqrt(block)) is applied once, after the last stage. */
static void fwht_block_f32(float *y, int block) {
  for (int h = 1; h < block; h *= 2) {
    for (int i = 0; i < block; i += 2 * h) {
      for (int j = i; j < i + h; j++) {
        float a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
    }
  }
  float s = (float)(1.0 / sqrt((double)block));
  for (int j = 0; j < block; j++) y[j] = y[j] * s;
}

static void fwht_block_f64(double *y, int block) {
  for (int h = 1; h < block; h *= 2) {
    for (int i = 0; i < block; i += 2 * h) {
      for (int j = i; j < i + h; j++) {
        double a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
    }
  }
  double s = 1.0 / sqrt((double)block);
  for (int j = 0; j < block; j++) y[j] = y[j] * s;
}

int orc_fwht_f32(float *x, int64_t n_vec, int dim, int block) {
  if (!x || n_vec < 0 || !is_pow2(block) || dim <= 0 || dim % block) return -1;
  for (int64_t v = 0; v < n_vec; v++)
    for (int b = 0; b < dim; b += block) fwht_block_f32(x + v * dim + b, block);
  return 0;
}

int orc_fwht_f64(double *x, int64_t n_vec, int dim, int block) {
  if (!x || n_vec < 0 || !is_pow2(block) || dim <= 0 || dim % block) return -1;
  for (int64_t v = 0; v < n_vec; v++)
    for (int b = 0; b < dim; b += block) fwht_block_f64(x + v * dim + b, block);
  return 0;
}

/* ===================================================================== */
/* Q4_0 [P1 How 2: 1 fp16 scale + 16 bytes for 32 nibbles; merge note:    */
/* the max-abs tie-break a > amax || (a == amax && v > mval)]             */
/* ===================================================================== */

/* Reading (the pages give only the block size, the storage and the tie-break;
 * the type name is GGML's, so its convention is taken):
 *   scan for the max-abs element with the tie-break, starting from
 *   amax = 0, mval = +0;  d = mval / -8;  id = d != 0 ? 1/d : 0;
 *   code_j = min(15, trunc(z_j * id + 8.5)) with the product and the sum
 *   rounded separately;  byte j = code_j | code_{j+16} << 4;
 *   stored scale = fp16(d); dequantized value = (code - 8) * fp16(d). */
int orc_q4_0_block(const float z[32], uint8_t qs[16], uint16_t *d_bits) {
  float amax = 0.0f, mval = 0.0f;
  for (int j = 0; j < Q4_BLK; j++) {
    if (!finite_f(z[j])) return -2;
    float a = fabsf(z[j]);
    if (a > amax || (a == amax && z[j] > mval)) {
      amax = a;
      mval = z[j];
    }
  }
  float d = mval / -8.0f;
  float id = (d != 0.0f) ? 1.0f / d : 0.0f;
  int code[Q4_BLK];
  for (int j = 0; j < Q4_BLK; j++) {
    float t = z[j] * id;
    t = t + 8.5f;
    int c = (int)t; /* t >= 0.5 for finite input, so truncation is floor */
    code[j] = c > 15 ? 15 : c;
  }
  for (int j = 0; j < 16; j++) qs[j] = (uint8_t)(code[j] | (code[j + 16] << 4));
  *d_bits = orc_f32_to_f16(d);
  return 0;
}

int orc_q4_0_dequant_block(const uint8_t qs[16], uint16_t d_bits, double out[32]) {
  double d = (double)orc_f16_to_f32(d_bits);
  for (int j = 0; j < 16; j++) {
    out[j] = (double)((int)(qs[j] & 15) - 8) * d;
    out[j + 16] = (double)((int)(qs[j] >> 4) - 8) * d;
  }
  return 0;
}

/* ---------------- Q8_0 ----------------
 * The 8-bit variant the pages compare Q4_0 against ("int8 KV", "Q8_0").
 * Reading (the pages name the type but not its steps; the name is GGML's, so
 * its convention is taken): amax = max |z_j|;  d = amax / 127;
 * id = d != 0 ? 1/d : 0;  code_j = roundf(z_j * id) (product rounded to fp32,
 * then rounded to the nearest integer, halves away from zero), stored as int8;
 * stored scale = fp16(d); dequantized value = code * fp16(d). */
int orc_q8_0_block(const float z[32], int8_t qs[32], uint16_t *d_bits) {
  float amax = 0.0f;
  for (int j = 0; j < Q4_BLK; j++) {
    if (!finite_f(z[j])) return -2;
    float a = fabsf(z[j]);
    if (a > amax) amax = a;
  }
  float d = amax / 127.0f;
  float id = (d != 0.0f) ? 1.0f / d : 0.0f;
  for (int j = 0; j < Q4_BLK; j++) {
    float t = z[j] * id;
    qs[j] = (int8_t)roundf(t);
  }
  *d_bits = orc_f32_to_f16(d);
  return 0;
}

int orc_q8_0_dequant_block(const int8_t qs[32], uint16_t d_bits, double out[32]) {
  double d = (double)orc_f16_to_f32(d_bits);
  for (int j = 0; j < Q4_BLK; j++) out[j] = (double)qs[j] * d;
  return 0;
}

/* FWHT-256 (fp32) then Q4_0 (bits 4) or Q8_0 (bits 8) over the 8
 * consecutive 32-value blocks of the rotated vector [P1 How 1-2: rotate
 * before quantization].  Code row: 128 (Q4_0) or 256 (Q8_0) bytes. */
static int kv_quantize_one(int bits, const void *x, int dtype, int64_t base, uint8_t *codes,
                           uint16_t *scales) {
  float y[Q4_DIM];
  for (int j = 0; j < Q4_DIM; j++) {
    y[j] = load_elem(x, dtype, base + j);
    if (!finite_f(y[j])) return -2;
  }
  fwht_block_f32(y, Q4_DIM);
  for (int b = 0; b < Q4_DIM / Q4_BLK; b++) {
    int r = bits == 8 ? orc_q8_0_block(y + b * Q4_BLK, (int8_t *)codes + b * 32, scales + b)
                      : orc_q4_0_block(y + b * Q4_BLK, codes + b * 16, scales + b);
    if (r) return r;
  }
  return 0;
}

static int row_bytes(int bits) { return bits == 8 ? 256 : 128; }

int orc_q4_quantize_vectors(const void *x, int dtype, int64_t n_vec, uint8_t *codes,
                            uint16_t *scales) {
  if (!x || !codes || !scales || n_vec < 0 || (dtype != 0 && dtype != 1)) return -1;
  for (int64_t v = 0; v < n_vec; v++) {
    int r = kv_quantize_one(4, x, dtype, v * Q4_DIM, codes + v * 128, scales + v * 8);
    if (r) return r;
  }
  return 0;
}

int orc_q8_quantize_vectors(const void *x, int dtype, int64_t n_vec, int8_t *codes,
                            uint16_t *scales) {
  if (!x || !codes || !scales || n_vec < 0 || (dtype != 0 && dtype != 1)) return -1;
  for (int64_t v = 0; v < n_vec; v++) {
    int r = kv_quantize_one(8, x, dtype, v * Q4_DIM, (uint8_t *)codes + v * 256, scales + v * 8);
    if (r) return r;
  }
  return 0;
}

static int64_t q4_row(int b, int h, int t, int n_kv_heads, int max_tokens,
                      const int32_t *block_table, int page_size, int max_pages) {
  if (!block_table) return ((int64_t)b * n_kv_heads + h) * max_tokens + t;
  int32_t page = block_table[(int64_t)b * max_pages + t / page_size];
  if (page < 0) return -1;
  return ((int64_t)page * n_kv_heads + h) * page_size + (t % page_size);
}

static int kv_append(int bits, uint8_t *k_codes, uint16_t *k_scales, uint8_t *v_codes,
                  uint16_t *v_scales, int n_kv_heads, int max_tokens,
                  const int32_t *block_table, int page_size, int max_pages,
                  const void *k, const void *v, int dtype, int batch, int t_new,
                  const int32_t *start_pos) {
  if (!k_codes || !k_scales || !v_codes || !v_scales || !k || !v || !start_pos)
    return -1;
  if (n_kv_heads <= 0 || batch < 0 || t_new < 0 || (dtype != 0 && dtype != 1)) return -1;
  if (block_table && (page_size <= 0 || max_pages <= 0)) return -1;
  for (int b = 0; b < batch; b++) {
    for (int i = 0; i < t_new; i++) {
      int t = start_pos[b] + i;
      if (t < 0) return -1;
      if (!block_table && t >= max_tokens) return -1;
      if (block_table && t / page_size >= max_pages) return -1;
      for (int h = 0; h < n_kv_heads; h++) {
        int64_t src = (((int64_t)b * t_new + i) * n_kv_heads + h) * Q4_DIM;
        int64_t row = q4_row(b, h, t, n_kv_heads, max_tokens, block_table,
                             page_size, max_pages);
        if (row < 0) return -1;
        const int rb = row_bytes(bits);
        int r = kv_quantize_one(bits, k, dtype, src, k_codes + row * rb, k_scales + row * 8);
        if (r) return r;
        r = kv_quantize_one(bits, v, dtype, src, v_codes + row * rb, v_scales + row * 8);
        if (r) return r;
      }
    }
  }
  return 0;
}

int orc_q4_append(uint8_t *k_codes, uint16_t *k_scales, uint8_t *v_codes,
                  uint16_t *v_scales, int n_kv_heads, int max_tokens,
                  const int32_t *block_table, int page_size, int max_pages,
                  const void *k, const void *v, int dtype, int batch, int t_new,
                  const int32_t *start_pos) {
  return kv_append(4, k_codes, k_scales, v_codes, v_scales, n_kv_heads, max_tokens, block_table,
                   page_size, max_pages, k, v, dtype, batch, t_new, start_pos);
}

int orc_q8_append(int8_t *k_codes, uint16_t *k_scales, int8_t *v_codes,
                  uint16_t *v_scales, int n_kv_heads, int max_tokens,
                  const int32_t *block_table, int page_size, int max_pages,
                  const void *k, const void *v, int dtype, int batch, int t_new,
                  const int32_t *start_pos) {
  return kv_append(8, (uint8_t *)k_codes, k_scales, (uint8_t *)v_codes, v_scales, n_kv_heads,
                   max_tokens, block_table, page_size, max_pages, k, v, dtype, batch, t_new,
                   start_pos);
}

/* Dequantize one cached row and rotate it back to the original basis in fp64
 * (H is symmetric and orthonormal, so H^-1 = H). */
static void kv_row_unrotated(int bits, const uint8_t *codes, const uint16_t *scales,
                             int64_t row, double *out) {
  for (int b = 0; b < Q4_DIM / Q4_BLK; b++) {
    if (bits == 8)
      orc_q8_0_dequant_block((const int8_t *)codes + row * 256 + b * 32, scales[row * 8 + b],
                             out + b * Q4_BLK);
    else
      orc_q4_0_dequant_block(codes + row * 128 + b * 16, scales[row * 8 + b], out + b * Q4_BLK);
  }
  fwht_block_f64(out, Q4_DIM);
}

/* Attention in the original basis: by the score invariance <Hq, Hk> = <q, k>
 * [P1 What] this is the quantity the rotated-space kernel computes. */
static int kv_decode_attn(int bits, const uint8_t *k_codes, const uint16_t *k_scales,
                       const uint8_t *v_codes, const uint16_t *v_scales,
                       int n_kv_heads, int max_tokens, const int32_t *block_table,
                       int page_size, int max_pages, const void *q, int dtype,
                       int batch, int n_q_heads, const int32_t *seq_lens,
                       double scale, double *out) {
  if (!k_codes || !k_scales || !v_codes || !v_scales || !q || !seq_lens || !out)
    return -1;
  if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads) return -1;
  if (dtype != 0 && dtype != 1) return -1;
  int group = n_q_heads / n_kv_heads;
  double kd[Q4_DIM];
  for (int b = 0; b < batch; b++) {
    int len = seq_lens[b];
    if (!block_table && len > max_tokens) return -1;
    if (block_table && len > 0 && (len - 1) / page_size >= max_pages) return -1;
    for (int h = 0; h < n_q_heads; h++) {
      double *o = out + ((int64_t)b * n_q_heads + h) * Q4_DIM;
      for (int j = 0; j < Q4_DIM; j++) o[j] = 0.0;
    }
    if (len <= 0) continue;
    double *sc = (double *)malloc(sizeof(double) * (size_t)len * group);
    double *qv = (double *)malloc(sizeof(double) * (size_t)group * Q4_DIM);
    if (!sc || !qv) { free(sc); free(qv); return -3; }
    for (int g = 0; g < n_kv_heads; g++) {
      for (int hh = 0; hh < group; hh++) {
        int h = g * group + hh;
        for (int j = 0; j < Q4_DIM; j++) {
          float f = load_elem(q, dtype, ((int64_t)b * n_q_heads + h) * Q4_DIM + j);
          if (!finite_f(f)) { free(sc); free(qv); return -2; }
          qv[hh * Q4_DIM + j] = (double)f;
        }
      }
      /* pass 1: scores */
      for (int t = 0; t < len; t++) {
        int64_t row = q4_row(b, g, t, n_kv_heads, max_tokens, block_table, page_size,
                             max_pages);
        if (row < 0) { free(sc); free(qv); return -1; }
        kv_row_unrotated(bits, k_codes, k_scales, row, kd);
        for (int hh = 0; hh < group; hh++) {
          double s = 0.0;
          for (int j = 0; j < Q4_DIM; j++) s += qv[hh * Q4_DIM + j] * kd[j];
          sc[(int64_t)t * group + hh] = s * scale;
        }
      }
      /* softmax per head, then pass 2: weighted values */
      for (int hh = 0; hh < group; hh++) {
        double m = -INFINITY;
        for (int t = 0; t < len; t++) m = fmax(m, sc[(int64_t)t * group + hh]);
        double l = 0.0;
        for (int t = 0; t < len; t++) {
          double p = exp(sc[(int64_t)t * group + hh] - m);
          sc[(int64_t)t * group + hh] = p;
          l += p;
        }
        for (int t = 0; t < len; t++) sc[(int64_t)t * group + hh] /= l;
      }
      for (int t = 0; t < len; t++) {
        int64_t row = q4_row(b, g, t, n_kv_heads, max_tokens, block_table, page_size,
                             max_pages);
        if (row < 0) { free(sc); free(qv); return -1; }
        kv_row_unrotated(bits, v_codes, v_scales, row, kd);
        for (int hh = 0; hh < group; hh++) {
          double p = sc[(int64_t)t * group + hh];
          double *o = out + ((int64_t)b * n_q_heads + g * group + hh) * Q4_DIM;
          for (int j = 0; j < Q4_DIM; j++) o[j] += p * kd[j];
        }
      }
    }
    free(sc);
    free(qv);
  }
  return 0;
}

int orc_q4_decode_attn(const uint8_t *k_codes, const uint16_t *k_scales,
                       const uint8_t *v_codes, const uint16_t *v_scales,
                       int n_kv_heads, int max_tokens, const int32_t *block_table,
                       int page_size, int max_pages, const void *q, int dtype,
                       int batch, int n_q_heads, const int32_t *seq_lens,
                       double scale, double *out) {
  return kv_decode_attn(4, k_codes, k_scales, v_codes, v_scales, n_kv_heads, max_tokens,
                        block_table, page_size, max_pages, q, dtype, batch, n_q_heads, seq_lens,
                        scale, out);
}

int orc_q8_decode_attn(const int8_t *k_codes, const uint16_t *k_scales,
                       const int8_t *v_codes, const uint16_t *v_scales,
                       int n_kv_heads, int max_tokens, const int32_t *block_table,
                       int page_size, int max_pages, const void *q, int dtype,
                       int batch, int n_q_heads, const int32_t *seq_lens,
                       double scale, double *out) {
  return kv_decode_attn(8, (const uint8_t *)k_codes, k_scales, (const uint8_t *)v_codes,
                        v_scales, n_kv_heads, max_tokens, block_table, page_size, max_pages, q,
                        dtype, batch, n_q_heads, seq_lens, scale, out);
}

/* ===================================================================== */
/* Octave [P5]                                                            */
/* ===================================================================== */

/* Standard normal density and tail, fp64. */
static double npdf(double x) { return isinf(x) ? 0.0 : exp(-0.5 * x * x) / sqrt(2.0 * M_PI); }
/* P(X > x) for X ~ N(0,1) */
static double ntail(double x) { return 0.5 * erfc(x / sqrt(2.0)); }
/* P(a < X < b), computed on the side that avoids cancellation */
static double nmass(double a, double b) {
  if (a >= 0.0) return ntail(a) - ntail(b);
  if (b <= 0.0) return ntail(-b) - ntail(-a);
  return 1.0 - ntail(b) - ntail(-a);
}

/* Lloyd-Max quantizer for N(0,1) (textbook: Lloyd's method I / Max 1960):
 * alternate "each centroid is the conditional mean of its cell" and "each
 * boundary is the midpoint of adjacent centroids" until nothing moves.
 * The pages name the codebook (Lloyd-Max for N(0,1), stored as int8) but do
 * not print it [P5 module text]. */
int orc_lloyd_max(int bits, double *centroids, double *boundaries) {
  if (bits < 1 || bits > 4 || !centroids) return -1;
  int L = 1 << bits;
  double c[16], bd[17];
  for (int i = 0; i < L; i++) c[i] = -3.0 + 6.0 * (i + 0.5) / L;
  for (int it = 0; it < 200000; it++) {
    bd[0] = -INFINITY;
    bd[L] = INFINITY;
    for (int i = 1; i < L; i++) bd[i] = 0.5 * (c[i - 1] + c[i]);
    double delta = 0.0;
    for (int i = 0; i < L; i++) {
      double m = (npdf(bd[i]) - npdf(bd[i + 1])) / nmass(bd[i], bd[i + 1]);
      delta = fmax(delta, fabs(m - c[i]));
      c[i] = m;
    }
    if (delta < 1e-16) break;
  }
  for (int i = 0; i < L; i++) centroids[i] = c[i];
  if (boundaries)
    for (int i = 1; i < L; i++) boundaries[i - 1] = 0.5 * (c[i - 1] + c[i]);
  return 0;
}

/* int8 codebook: LUT[i] = round(c_i * 127 / c_max) (half away from zero), so
 * the outer codes are +-127, and LUT_MULT = fp32(127 / c_max) maps an
 * RMS-normalised value into LUT units.  (Reading: the pages name LUT and
 * LUT_MULT per bit width but give neither.) */
int orc_octave_codebook(int bits, int8_t *lut, float *lut_mult) {
  /* computed once per bit width (the oracle is single-threaded) */
  static int ready[5];
  static int8_t lut_c[5][16];
  static float mult_c[5];
  if (bits != 3 && bits != 4) return -1;
  if (!ready[bits]) {
    double c[16];
    orc_lloyd_max(bits, c, NULL);
    int L = 1 << bits;
    double mult = 127.0 / c[L - 1];
    for (int i = 0; i < L; i++) lut_c[bits][i] = (int8_t)lround(c[i] * mult);
    mult_c[bits] = (float)mult;
    ready[bits] = 1;
  }
  if (lut) memcpy(lut, lut_c[bits], (size_t)(1 << bits));
  if (lut_mult) *lut_mult = mult_c[bits];
  return 0;
}

/* Derived offsets, exactly as the OctaveFormat properties define them. */
int orc_octave_format(int head_size, int rope_dim, int v_bits, int compact,
                      orc_octave_fmt *f) {
  if (!f) return -1;
  if (v_bits != 3 && v_bits != 4) return -1;
  if (compact && (head_size & (head_size - 1))) return -1;
  if (head_size <= 0 || rope_dim < 0 || rope_dim % OCT_HB || head_size % OCT_HB) return -1;
  if (rope_dim > head_size) return -1;
  f->head_size = head_size;
  f->rope_dim = rope_dim;
  f->v_bits = v_bits;
  f->compact = compact ? 1 : 0;
  f->k_rotation_block = compact ? head_size : OCT_HB;
  f->k_wide_dim = compact ? 0 : rope_dim;
  f->nope_dim = head_size - rope_dim;
  f->num_k_blocks = head_size / OCT_HB;
  f->num_rope_blocks = rope_dim / OCT_HB;
  f->off_k_nope = f->k_wide_dim * OCT_ROPE_BITS / 8;
  f->off_v = f->off_k_nope + (head_size - f->k_wide_dim) * OCT_NOPE_BITS / 8;
  f->off_scales = f->off_v + head_size * v_bits / 8;
  f->num_k_scales = compact ? 1 : f->num_k_blocks;
  f->num_scales = f->num_k_scales + 1;
  int raw = f->off_scales + 2 * f->num_scales;
  int align = compact ? 4 : 8;
  f->slot_bytes = (raw + align - 1) / align * align;
  f->kernel_code = v_bits + (compact ? 16 : 0);
  return 0;
}

/* Bit packing [P5 module text and _pack]:
 * 4-bit: each little-endian 32-bit word covers 8 dims; byte j holds dim j in
 *        its low nibble and dim j+4 in its high nibble.
 * 3-bit: a 2-bit plane (one word per 16 dims, byte j gathers dims 4i+j of the
 *        word in bits 2i..2i+1) followed by a 1-bit plane (one word per 32
 *        dims, byte j gathers dims 4i+j in bit i); code = lo + 4 * hi. */
int orc_octave_pack(const uint8_t *codes, int n, int bits, uint8_t *out) {
  if (!codes || !out) return -1;
  if (bits == 4) {
    if (n % 8) return -1;
    for (int w = 0; w < n / 8; w++)
      for (int j = 0; j < 4; j++)
        out[4 * w + j] = (uint8_t)((codes[8 * w + j] & 15) | ((codes[8 * w + 4 + j] & 15) << 4));
    return 0;
  }
  if (bits == 3) {
    if (n % 32) return -1;
    uint8_t *lo = out, *hi = out + n / 4;
    for (int w = 0; w < n / 16; w++)
      for (int j = 0; j < 4; j++) {
        int byte = 0;
        for (int i = 0; i < 4; i++) byte |= (codes[16 * w + 4 * i + j] & 3) << (2 * i);
        lo[4 * w + j] = (uint8_t)byte;
      }
    for (int w = 0; w < n / 32; w++)
      for (int j = 0; j < 4; j++) {
        int byte = 0;
        for (int i = 0; i < 8; i++) byte |= ((codes[32 * w + 4 * i + j] >> 2) & 1) << i;
        hi[4 * w + j] = (uint8_t)byte;
      }
    return 0;
  }
  return -1;
}

int orc_octave_unpack(const uint8_t *in, int n, int bits, uint8_t *codes) {
  if (!codes || !in) return -1;
  if (bits == 4) {
    if (n % 8) return -1;
    for (int w = 0; w < n / 8; w++)
      for (int j = 0; j < 4; j++) {
        codes[8 * w + j] = in[4 * w + j] & 15;
        codes[8 * w + 4 + j] = in[4 * w + j] >> 4;
      }
    return 0;
  }
  if (bits == 3) {
    if (n % 32) return -1;
    const uint8_t *lo = in, *hi = in + n / 4;
    for (int d = 0; d < n; d++) {
      int wl = d / 16, il = (d % 16) / 4, jl = d % 4;
      int wh = d / 32, ih = (d % 32) / 4;
      int l2 = (lo[4 * wl + jl] >> (2 * il)) & 3;
      int h1 = (hi[4 * wh + jl] >> ih) & 1;
      codes[d] = (uint8_t)(l2 + 4 * h1);
    }
    return 0;
  }
  return -1;
}

/* Fixed pairwise summation: v[i] += v[i + n/2], halving n until one value is
 * left.  (Reading: the page sums with torch, whose order is unspecified; a
 * fixed tree makes the scale reproducible bit for bit.)  Destroys v. */
static float tree_sum_f32(float *v, int n) {
  while (n > 1) {
    n >>= 1;
    for (int i = 0; i < n; i++) v[i] = v[i] + v[i + n];
  }
  return v[0];
}

/* [P5 _quantize_lut] nearest Lloyd-Max code on the block RMS; the scale keeps
 * x . x_hat = |x|^2 (x_hat = LUT[c] * scale / LUT_ONE). */
int orc_octave_quantize_lut(const float *x, int n, int bits, uint8_t *codes, float *scale) {
  if (!x || !codes || !scale || !is_pow2(n) || n > 512) return -1;
  int8_t lut[16];
  float mult;
  if (orc_octave_codebook(bits, lut, &mult)) return -1;
  int L = 1 << bits;
  float mid[15];
  for (int i = 0; i < L - 1; i++) mid[i] = ((float)lut[i + 1] + (float)lut[i]) / 2.0f;
  float tmp[512];
  for (int i = 0; i < n; i++) {
    if (!finite_f(x[i])) return -2;
    tmp[i] = x[i] * x[i];
  }
  float ss = tree_sum_f32(tmp, n);
  float rms = sqrtf(ss / (float)n);
  if (rms < 1e-12f) rms = 1e-12f;
  for (int i = 0; i < n; i++) {
    float y = x[i] / rms;
    y = y * mult;
    int c = 0;
    for (int k = 0; k < L - 1; k++)
      if (mid[k] < y) c++; /* bucketize, right=False: a tie goes to the lower code */
    codes[i] = (uint8_t)c;
  }
  for (int i = 0; i < n; i++) tmp[i] = x[i] * (float)lut[codes[i]];
  float dot = tree_sum_f32(tmp, n);
  float q = ss / (dot > 1e-30f ? dot : 1e-30f);
  float s = dot > 0.0f ? q : 0.0f;
  *scale = s * OCT_LUT_ONE;
  return 0;
}

/* rotate(x, s, b) = fwht_blocks(x * s, b): sign flips before the Hadamard
 * [P5 module text]. */
int orc_octave_rotate(float *x, const float *signs, int d, int block) {
  if (!x || !signs || !is_pow2(block) || d % block) return -1;
  for (int i = 0; i < d; i++) x[i] = x[i] * signs[i];
  for (int b = 0; b < d; b += block) fwht_block_f32(x + b, block);
  return 0;
}

/* unrotate(y, s, b) = fwht_blocks(y, b) * s: the inverse of rotate, since the
 * block transform is its own inverse and s * s = 1. */
int orc_octave_unrotate_f64(double *y, const float *signs, int d, int block) {
  if (!y || !signs || !is_pow2(block) || d % block) return -1;
  for (int b = 0; b < d; b += block) fwht_block_f64(y + b, block);
  for (int i = 0; i < d; i++) y[i] = y[i] * (double)signs[i];
  return 0;
}

/* [P5 v_block] V is one rotation block when head_size is a power of two. */
static int oct_v_block(int head_size) { return is_pow2(head_size) ? head_size : OCT_HB; }

/* [P5 reference_quantize] (T, H, D) K and V -> (T, H, slot_bytes) slots. */
int orc_octave_quantize(int head_size, int rope_dim, int v_bits, int compact,
                        const void *key, const void *value, int dtype, int T, int H,
                        const float *signs, uint8_t *out) {
  orc_octave_fmt f;
  if (orc_octave_format(head_size, rope_dim, v_bits, compact, &f)) return -1;
  if (!is_pow2(head_size) || head_size > 512) return -1; /* fixed-tree sums need 2^k */
  if (!key || !value || !signs || !out || T < 0 || H <= 0 || (dtype != 0 && dtype != 1))
    return -1;
  int d = head_size;
  float x[512];
  uint8_t codes[512];
  float scales[16];
  for (int t = 0; t < T; t++) {
    for (int h = 0; h < H; h++) {
      int64_t base = ((int64_t)t * H + h) * d;
      uint8_t *slot = out + ((int64_t)t * H + h) * f.slot_bytes;
      memset(slot, 0, (size_t)f.slot_bytes);
      /* K */
      for (int i = 0; i < d; i++) x[i] = load_elem(key, dtype, base + i);
      if (orc_octave_rotate(x, signs, d, f.k_rotation_block)) return -1;
      if (f.compact) {
        int r = orc_octave_quantize_lut(x, d, OCT_NOPE_BITS, codes, &scales[0]);
        if (r) return r;
        orc_octave_pack(codes, d, OCT_NOPE_BITS, slot);
      } else {
        for (int kb = 0; kb < f.num_k_blocks; kb++) {
          int bits = kb < f.num_rope_blocks ? OCT_ROPE_BITS : OCT_NOPE_BITS;
          int r = orc_octave_quantize_lut(x + kb * OCT_HB, OCT_HB, bits,
                                          codes + kb * OCT_HB, &scales[kb]);
          if (r) return r;
        }
        orc_octave_pack(codes, f.rope_dim, OCT_ROPE_BITS, slot);
        orc_octave_pack(codes + f.rope_dim, f.nope_dim, OCT_NOPE_BITS, slot + f.off_k_nope);
      }
      /* V */
      for (int i = 0; i < d; i++) x[i] = load_elem(value, dtype, base + i);
      if (orc_octave_rotate(x, signs, d, oct_v_block(d))) return -1;
      int r = orc_octave_quantize_lut(x, d, v_bits, codes, &scales[f.num_k_scales]);
      if (r) return r;
      orc_octave_pack(codes, d, v_bits, slot + f.off_v);
      /* fp16 scales, little-endian, K scales first then V */
      for (int s = 0; s < f.num_scales; s++) {
        uint16_t hb = orc_f32_to_f16(scales[s]);
        slot[f.off_scales + 2 * s] = (uint8_t)(hb & 0xFF);
        slot[f.off_scales + 2 * s + 1] = (uint8_t)(hb >> 8);
      }
    }
  }
  return 0;
}

static double lut_value(int bits, int code) {
  int8_t lut[16];
  orc_octave_codebook(bits, lut, NULL);
  return (double)lut[code];
}

/* [P5 reference_dequantize] slots -> K, V; a code c of a block with scale s
 * stands for LUT[c] * s / LUT_ONE. */
int orc_octave_dequantize(int head_size, int rope_dim, int v_bits, int compact,
                          const uint8_t *slots, int T, int H, const float *signs,
                          int rotated, double *k, double *v) {
  orc_octave_fmt f;
  if (orc_octave_format(head_size, rope_dim, v_bits, compact, &f)) return -1;
  if (!slots || !signs || !k || !v || T < 0 || H <= 0) return -1;
  int d = head_size;
  double lut3[16], lut4[16];
  for (int i = 0; i < 8; i++) lut3[i] = lut_value(3, i);
  for (int i = 0; i < 16; i++) lut4[i] = lut_value(4, i);
  uint8_t codes[512];
  for (int t = 0; t < T; t++) {
    for (int h = 0; h < H; h++) {
      const uint8_t *slot = slots + ((int64_t)t * H + h) * f.slot_bytes;
      double sc[16];
      for (int s = 0; s < f.num_scales; s++) {
        uint16_t hb = (uint16_t)(slot[f.off_scales + 2 * s] | (slot[f.off_scales + 2 * s + 1] << 8));
        sc[s] = (double)orc_f16_to_f32(hb) / (double)OCT_LUT_ONE;
      }
      double *kr = k + ((int64_t)t * H + h) * d;
      double *vr = v + ((int64_t)t * H + h) * d;
      if (f.compact) {
        orc_octave_unpack(slot, d, OCT_NOPE_BITS, codes);
        for (int i = 0; i < d; i++) kr[i] = lut3[codes[i]] * sc[0];
      } else {
        orc_octave_unpack(slot, f.rope_dim, OCT_ROPE_BITS, codes);
        orc_octave_unpack(slot + f.off_k_nope, f.nope_dim, OCT_NOPE_BITS, codes + f.rope_dim);
        for (int i = 0; i < d; i++) {
          double lv = i < f.rope_dim ? lut4[codes[i]] : lut3[codes[i]];
          kr[i] = lv * sc[i / OCT_HB];
        }
      }
      orc_octave_unpack(slot + f.off_v, d, v_bits, codes);
      for (int i = 0; i < d; i++) vr[i] = (v_bits == 4 ? lut4[codes[i]] : lut3[codes[i]]) * sc[f.num_scales - 1];
      if (!rotated) {
        orc_octave_unrotate_f64(kr, signs, d, f.k_rotation_block);
        orc_octave_unrotate_f64(vr, signs, d, oct_v_block(d));
      }
    }
  }
  return 0;
}

/* [P5 reference_attention] per query token i: attend to the first
 * q_to_klen[i] tokens of request q_to_req[i] through the block table; GQA by
 * repeat_interleave (query head h reads kv head h / group); softmax in fp64
 * here; klen <= 0 gives a zero row. */
int orc_octave_attention(int head_size, int rope_dim, int v_bits, int compact,
                         const void *query, int dtype, int n_q, int n_q_heads,
                         const uint8_t *cache, int64_t num_blocks, int n_kv_heads,
                         int block_size,
                         const int32_t *block_table, int max_blocks,
                         const int32_t *q_to_req, const int32_t *q_to_klen, double scale,
                         const float *signs, double *out) {
  orc_octave_fmt f;
  if (orc_octave_format(head_size, rope_dim, v_bits, compact, &f)) return -1;
  if (!query || !cache || !block_table || !q_to_req || !q_to_klen || !signs || !out)
    return -1;
  if (n_kv_heads <= 0 || n_q_heads % n_kv_heads || block_size <= 0) return -1;
  int d = head_size, group = n_q_heads / n_kv_heads;
  for (int i = 0; i < n_q; i++) {
    for (int h = 0; h < n_q_heads; h++)
      for (int j = 0; j < d; j++) out[((int64_t)i * n_q_heads + h) * d + j] = 0.0;
    int klen = q_to_klen[i];
    if (klen <= 0) continue;
    if ((klen - 1) / block_size >= max_blocks) return -1;
    int req = q_to_req[i];
    for (int t = 0; t < klen; t += block_size) {
      int32_t blk = block_table[(int64_t)req * max_blocks + t / block_size];
      if (blk < 0 || blk >= num_blocks) return -1;
    }
    double *k = (double *)malloc(sizeof(double) * (size_t)klen * n_kv_heads * d);
    double *v = (double *)malloc(sizeof(double) * (size_t)klen * n_kv_heads * d);
    uint8_t *slots = (uint8_t *)malloc((size_t)klen * n_kv_heads * f.slot_bytes);
    double *p = (double *)malloc(sizeof(double) * (size_t)klen);
    if (!k || !v || !slots || !p) { free(k); free(v); free(slots); free(p); return -3; }
    for (int t = 0; t < klen; t++) {
      int32_t blk = block_table[(int64_t)req * max_blocks + t / block_size];
      for (int g = 0; g < n_kv_heads; g++)
        memcpy(slots + ((int64_t)t * n_kv_heads + g) * f.slot_bytes,
               cache + (((int64_t)blk * n_kv_heads + g) * block_size + t % block_size) * f.slot_bytes,
               (size_t)f.slot_bytes);
    }
    orc_octave_dequantize(head_size, rope_dim, v_bits, compact, slots, klen, n_kv_heads,
                          signs, 0, k, v);
    for (int h = 0; h < n_q_heads; h++) {
      int g = h / group;
      double m = -INFINITY;
      for (int t = 0; t < klen; t++) {
        double s = 0.0;
        for (int j = 0; j < d; j++)
          s += (double)load_elem(query, dtype, ((int64_t)i * n_q_heads + h) * d + j) *
               k[((int64_t)t * n_kv_heads + g) * d + j];
        p[t] = s * scale;
        m = fmax(m, p[t]);
      }
      double l = 0.0;
      for (int t = 0; t < klen; t++) {
        p[t] = exp(p[t] - m);
        l += p[t];
      }
      double *o = out + ((int64_t)i * n_q_heads + h) * d;
      for (int t = 0; t < klen; t++) {
        double w = p[t] / l;
        for (int j = 0; j < d; j++) o[j] += w * v[((int64_t)t * n_kv_heads + g) * d + j];
      }
    }
    free(k); free(v); free(slots); free(p);
  }
  return 0;
}
