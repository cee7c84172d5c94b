/*
 * kvq_oracle.h -- plain single-threaded CPU oracle for the Hadamard-rotated
 * low-bit KV cache (FWHT-256 + Q4_0, its Q8_0 counterpart, and the Octave
 * block-Hadamard variant).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this library: only tests/, __graft_entry__.smoke() and the bench's
 * cpu_baseline / reference leg use it.  It shares no code, header, table or
 * constant generator with the CUDA library; the two meet only through the
 * seeded input generator and the documented byte layouts.
 *
 * Sources restated here (page title, then section):
 *   [P1] Strata PR #21 "Q4_0 KV cache + FWHT-256": What / Why / How 1-3,
 *        and the maintainer's merge note (deterministic quantization bullet,
 *        per-token path bullet).
 *   [P5] vLLM API page "vllm.v1.attention.ops.rocm_octave": module text
 *        (slot layout, 4-bit / 3-bit codes, scales), OctaveFormat, _pack,
 *        _quantize_lut, fwht_blocks, reference_quantize, reference_dequantize,
 *        reference_attention, v_block.
 *
 * Floating point: fp32 wherever the pages fix fp32 (the rotation and both
 * quantizers, which must be reproduced bit for bit), IEEE round-to-nearest,
 * compiled with -ffp-contract=off so no multiply-add is ever fused; fp64 for
 * the attention result, which the GPU must match only to a tolerance.
 *
 * Every function returns 0 on success and a negative value on a bad argument
 * or a non-finite input (non-finite inputs are outside the method's contract).
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------- scalar conversions ---------------- */
uint16_t orc_f32_to_f16(float f);          /* IEEE binary16, round to nearest even */
float    orc_f16_to_f32(uint16_t h);
float    orc_bf16_to_f32(uint16_t h);
void     orc_f32_to_f16_array(const float *x, uint16_t *y, int64_t n);

/* ---------------- rotation ----------------
 * Orthonormal Walsh-Hadamard transform over consecutive `block`-sized blocks
 * of each `dim`-long vector, in place.  Stage order h = 1, 2, 4, ..., block/2;
 * pair (i, i+h) -> (a+b, a-b); one multiply by fp32(1/sqrt(block)) at the end.
 * [P5 fwht_blocks; P1 How 1: normalisation 1/sqrt(256) = 1/16] */
int orc_fwht_f32(float *x, int64_t n_vec, int dim, int block);
int orc_fwht_f64(double *x, int64_t n_vec, int dim, int block);

/* ---------------- Q4_0 ----------------
 * One 32-value block -> 16 nibble bytes + fp16 scale bits.  [P1 How 2; merge
 * note, deterministic quantization] */
int orc_q4_0_block(const float z[32], uint8_t qs[16], uint16_t *d_bits);
int orc_q4_0_dequant_block(const uint8_t qs[16], uint16_t d_bits, double out[32]);

/* ---------------- Q8_0 ----------------
 * The 8-bit KV variant the pages compare Q4_0 against; GGML's Q8_0 steps:
 * d = amax / 127, id = d ? 1/d : 0, code = roundf(z * id) (int8), fp16(d). */
int orc_q8_0_block(const float z[32], int8_t qs[32], uint16_t *d_bits);
int orc_q8_0_dequant_block(const int8_t qs[32], uint16_t d_bits, double out[32]);
/* Rotate + Q8_0-quantize n_vec vectors: codes n_vec x 256 int8, scales
 * n_vec x 8 fp16 bit patterns. */
int orc_q8_quantize_vectors(const void *x, int dtype, int64_t n_vec, int8_t *codes,
                            uint16_t *scales);

/* Rotate (fp32 FWHT-256) + Q4_0-quantize n_vec vectors of 256 values.
 * dtype: 0 = fp32 input, 1 = bf16 input (raw uint16 bits).
 * codes: n_vec x 128 bytes; scales: n_vec x 8 fp16 bit patterns. */
int orc_q4_quantize_vectors(const void *x, int dtype, int64_t n_vec,
                            uint8_t *codes, uint16_t *scales);

/* Quantize-on-append into a Q4_0 cache.
 * Cache layout (structure of arrays): row(b, h, t) =
 *   contiguous (block_table == NULL): (b * n_kv_heads + h) * max_tokens + t
 *   paged: (block_table[b * max_pages + t / page_size] * n_kv_heads + h)
 *          * page_size + t % page_size
 * k_codes/v_codes hold 128 bytes per row, k_scales/v_scales 8 fp16 per row.
 * k, v: [batch][t_new][n_kv_heads][256]; token i of sequence b lands at
 * position start_pos[b] + i. */
int orc_q4_append(uint8_t *k_codes, uint16_t *k_scales, uint8_t *v_codes,
                  uint16_t *v_scales, int n_kv_heads, int max_tokens,
                  const int32_t *block_table, int page_size, int max_pages,
                  const void *k, const void *v, int dtype, int batch,
                  int t_new, const int32_t *start_pos);

/* Single-token decode attention over the Q4_0 cache, fp64.
 * q: [batch][n_q_heads][256] (dtype as above); out: [batch][n_q_heads][256].
 * Query head h reads kv head h / (n_q_heads / n_kv_heads).  Keys and values
 * are dequantized and rotated back to the original basis, then
 * out = softmax(scale * <q, k_t>) . v_t over t < seq_lens[b]; a sequence with
 * seq_len <= 0 gives a zero row.  [P1 What (score invariance), How 2; P5
 * reference_attention] */
int orc_q4_decode_attn(const uint8_t *k_codes, const uint16_t *k_scales,
                       const uint8_t *v_codes, const uint16_t *v_scales,
                       int n_kv_heads, int max_tokens,
                       const int32_t *block_table, int page_size,
                       int max_pages, const void *q, int dtype, int batch,
                       int n_q_heads, const int32_t *seq_lens, double scale,
                       double *out);

/* The same two calls over a Q8_0 cache (256 int8 code bytes per row). */
int orc_q8_append(int8_t *k_codes, uint16_t *k_scales, int8_t *v_codes,
                  uint16_t *v_scales, int n_kv_heads, int max_tokens,
                  const int32_t *block_table, int page_size, int max_pages,
                  const void *k, const void *v, int dtype, int batch,
                  int t_new, const int32_t *start_pos);
int orc_q8_decode_attn(const int8_t *k_codes, const uint16_t *k_scales,
                       const int8_t *v_codes, const uint16_t *v_scales,
                       int n_kv_heads, int max_tokens,
                       const int32_t *block_table, int page_size,
                       int max_pages, const void *q, int dtype, int batch,
                       int n_q_heads, const int32_t *seq_lens, double scale,
                       double *out);

/* ---------------- Octave ---------------- */
/* Lloyd-Max codebook for N(0,1) with 2^bits levels (bits = 3 or 4):
 * centroids (fp64, ascending), the int8 LUT round(c_i * mult) and
 * mult = fp32(127 / c_max). */
int orc_lloyd_max(int bits, double *centroids, double *boundaries);
int orc_octave_codebook(int bits, int8_t *lut, float *lut_mult);

/* Format derived quantities [P5 OctaveFormat]. */
typedef struct {
  int head_size, rope_dim, v_bits, compact;
  int k_rotation_block, k_wide_dim, nope_dim, num_k_blocks, num_rope_blocks;
  int off_k_nope, off_v, off_scales, num_k_scales, num_scales, slot_bytes;
  int kernel_code;
} orc_octave_fmt;
int orc_octave_format(int head_size, int rope_dim, int v_bits, int compact,
                      orc_octave_fmt *f);

int orc_octave_pack(const uint8_t *codes, int n, int bits, uint8_t *out);
int orc_octave_unpack(const uint8_t *in, int n, int bits, uint8_t *codes);

/* Nearest Lloyd-Max code on the block RMS, scale keeps x . x_hat = |x|^2.
 * n must be a power of two (fixed pairwise summation order). */
int orc_octave_quantize_lut(const float *x, int n, int bits, uint8_t *codes,
                            float *scale);

/* x <- fwht_blocks(x * signs, block) ; and its inverse. */
int orc_octave_rotate(float *x, const float *signs, int d, int block);
int orc_octave_unrotate_f64(double *y, const float *signs, int d, int block);

/* key, value: [T][H][d]; out: [T][H][slot_bytes]. */
int orc_octave_quantize(int head_size, int rope_dim, int v_bits, int compact,
                        const void *key, const void *value, int dtype,
                        int T, int H, const float *signs, uint8_t *out);
/* slots: [T][H][slot]; k, v: [T][H][d] fp64; rotated != 0 skips unrotate. */
int orc_octave_dequantize(int head_size, int rope_dim, int v_bits, int compact,
                          const uint8_t *slots, int T, int H,
                          const float *signs, int rotated, double *k,
                          double *v);
/* query: [Q][Hq][d]; cache: [num_blocks][Hkv][block_size][slot];
 * block_table: [num_reqs][max_blocks]; an entry a query reads must name one of
 * the num_blocks blocks, else -1 is returned.  out: [Q][Hq][d] fp64. */
int orc_octave_attention(int head_size, int rope_dim, int v_bits, int compact,
                         const void *query, int dtype, int n_q, int n_q_heads,
                         const uint8_t *cache, int64_t num_blocks, int n_kv_heads, int block_size,
                         const int32_t *block_table, int max_blocks,
                         const int32_t *q_to_req, const int32_t *q_to_klen,
                         double scale, const float *signs, double *out);

#ifdef __cplusplus
}
#endif
#endif
