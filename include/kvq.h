/*
 * kvq.h -- C ABI of the Hadamard-rotated low-bit KV cache for NVIDIA B200
 * (sm_100a).
 *
 * Method (page title, then section):
 *   Strata PR #21 "Q4_0 KV cache + FWHT-256": What / Why / How 1-2 and the
 *   maintainer's merge note -- each K/V head vector (D = 256) is rotated by the
 *   orthonormal Walsh-Hadamard transform (scale 1/16) and stored as Q4_0 blocks
 *   (32 values: one fp16 scale + 16 bytes of nibbles, deterministic max-abs
 *   tie-break); decode attention rotates the query the same way, dequantizes
 *   the nibbles in registers inside an online softmax, and rotates the output
 *   back once per query head.
 *   vLLM API page "vllm.v1.attention.ops.rocm_octave" -- the Octave variant:
 *   sign flips + 64-dim block Hadamard for K (4-bit RoPE / 3-bit NoPE codes),
 *   whole-head rotation for V, a Lloyd-Max N(0,1) int8 codebook and fp16 scales
 *   chosen so that x . x_hat = |x|^2, in 8-byte-padded per-(token, head) slots.
 *
 * Conventions for every call:
 *   - All buffers are owned by the caller.  "device" pointers must point to
 *     memory of the current CUDA device; "host" pointers to host memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream; the library never allocates, never
 *     frees and never synchronizes (the one exception is the diagnostic
 *     kvq_device_errors, which reads the device error word after the device
 *     has finished its work).
 *   - Argument checks happen on the host before any launch and return
 *     KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED / KVQ_ERR_WORKSPACE without
 *     touching the GPU.  A failed launch returns KVQ_ERR_CUDA.  Values that live
 *     in device memory (positions, lengths, page tables) cannot be checked on
 *     the host; the kernels clamp them so that no access leaves the buffers the
 *     caller described, and document what an out-of-range value does.
 *   - Kernels never trap or assert; what they cannot return as a status they
 *     record in the device error word (kvq_device_errors).
 *   - Inputs must be finite; the bit-exact contract for the quantizers covers
 *     finite inputs whose 32-value blocks have max |value| either 0 or at least
 *     2^-120 (below that the reciprocal of the block scale overflows).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, inconsistent shapes */
  KVQ_ERR_UNSUPPORTED = 2, /* a valid configuration this build does not implement */
  KVQ_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace size */
  KVQ_ERR_CUDA = 4         /* a kernel launch failed (see cudaGetLastError) */
} kvq_status;

typedef enum {
  KVQ_F32 = 0,  /* IEEE binary32 */
  KVQ_BF16 = 1  /* bfloat16, raw 16-bit patterns; widened to fp32 exactly */
} kvq_dtype;

/* Human-readable name of a status code (static string, never NULL). */
KVQ_API const char *kvq_status_string(kvq_status s);

/* Version of this library as major * 10000 + minor * 100 + patch. */
KVQ_API int kvq_version(void);

/* ------------------------------------------------------------------------ */
/* Q4_0 + FWHT-256 cache                                                      */
/* ------------------------------------------------------------------------ */

/* Q4_0 / Q8_0 cache descriptor (structure of arrays, all planes in device
 * memory).  A "row" is one (sequence, kv head, token) vector of 256 values,
 * rotated by FWHT-256 and cut into 8 blocks of 32:
 *   k_codes / v_codes   code_bits 0 or 4 (Q4_0): row * 128 bytes, block b at
 *                       bytes 16b..16b+15, byte j of a block
 *                       = code_j | code_{j+16} << 4 (Strata PR #21, How 2);
 *                       code_bits 8 (Q8_0, the 8-bit variant the same pages
 *                       measure Q4_0 against): row * 256 bytes, element j of
 *                       block b at byte 32b + j as a two's-complement int8;
 *   k_scales / v_scales row * 8 fp16 bit patterns, the scale of block b at b.
 * Row index of (sequence b, kv head h, token t):
 *   contiguous (block_table == NULL):
 *       (b * num_kv_heads + h) * max_tokens + t,       t < max_tokens
 *   paged (block_table != NULL, device, int32[batch][max_pages_per_seq]):
 *       (block_table[b][t / page_size] * num_kv_heads + h) * page_size
 *         + t % page_size,                              physical page < num_pages
 * The planes must hold num_rows() rows: batch_capacity * num_kv_heads *
 * max_tokens (contiguous) or num_pages * num_kv_heads * page_size (paged). */
typedef struct {
  uint8_t *k_codes;
  uint16_t *k_scales;
  uint8_t *v_codes;
  uint16_t *v_scales;
  int32_t num_kv_heads;        /* >= 1 */
  int32_t head_dim;            /* must be 256 */
  int32_t max_tokens;          /* contiguous: token capacity per (sequence, head) */
  int32_t batch_capacity;      /* contiguous: number of sequences the planes hold */
  const int32_t *block_table;  /* NULL => contiguous */
  int32_t page_size;           /* paged: tokens per page, a multiple of 64 */
  int32_t max_pages_per_seq;   /* paged: columns of block_table */
  int32_t num_pages;           /* paged: physical pages in the planes */
  int32_t code_bits;           /* 0 or 4: Q4_0 rows as above; 8: Q8_0 rows */
} kvq_cache;

/* kvq_rotate -- y = H x for n_vec vectors of `dim` values, H the orthonormal
 * Walsh-Hadamard matrix (Strata PR #21, How 1: normalisation 1/sqrt(256)).
 * The butterfly stages run in the order h = 1, 2, ..., 128 with one multiply
 * by 1/16 at the end (vLLM rocm_octave page, fwht_blocks), in fp32 with IEEE
 * round-to-nearest, so the result is bit-identical to that sequence of fp32
 * operations.
 *   x: device, [n_vec][dim] of `dtype`; y: device, [n_vec][dim] fp32 (may not
 *   alias x).  dim must be 256.  n_vec == 0 is a no-op. */
KVQ_API kvq_status kvq_rotate(const void *x, kvq_dtype dtype, float *y, int64_t n_vec,
                      int32_t dim, void *stream);

/* kvq_quantize_append -- rotate and Q4_0- (or Q8_0-) quantize t_new new tokens of K and V
 * per sequence and store them in the cache (Strata PR #21, How 1-2 and the
 * merge note's deterministic tie-break a > amax || (a == amax && v > mval)).
 *   k, v: device, [batch][t_new][num_kv_heads][256] of `dtype`.
 *   d_start_pos: device int32[batch]; token i of sequence b is stored at
 *   position start_pos[b] + i.  A token whose position falls outside the
 *   cache (negative, >= max_tokens, or a page outside the table or outside
 *   [0, num_pages)) is skipped.
 * Codes and scales are bit-identical to: fp32 FWHT-256 as in kvq_rotate, then
 * per 32-value block d = mval / -8, id = d ? 1/d : 0,
 * code = min(15, trunc(z * id + 8.5)) (product and sum rounded separately),
 * scale = fp16(d) (round to nearest even).  Q8_0 (code_bits 8): per block
 * amax = max |z|, d = amax / 127, id = d ? 1/d : 0, code = round(z * id)
 * (product rounded to fp32, halves away from zero), scale = fp16(d).
 * batch must be <= batch_capacity for a contiguous cache; one call handles
 * fewer than 2^30 vectors per tensor (batch * t_new * num_kv_heads),
 * KVQ_ERR_UNSUPPORTED otherwise. */
KVQ_API kvq_status kvq_quantize_append(const kvq_cache *cache, const void *k, const void *v,
                               kvq_dtype dtype, int32_t batch, int32_t t_new,
                               const int32_t *d_start_pos, void *stream);

/* Bytes of scratch kvq_decode_attn needs for this shape (split-K partials). */
KVQ_API size_t kvq_decode_attn_workspace(const kvq_cache *cache, int32_t batch,
                                 int32_t num_q_heads, int32_t max_seq_len);

/* kvq_decode_attn -- one query token per sequence over the Q4_0 or Q8_0
 * cache (Strata PR #21, How 2; merge note: the per-token path rotates Q and
 * the output).  For query head h (kv head h / (num_q_heads / num_kv_heads)):
 *   out[b][h] = H . sum_t softmax_t(scale * <H q[b][h], k_t>) v_t,
 *   t < seq_len[b], with k_t, v_t the dequantized cached rows.
 * Over a Q8_0 cache the rotated query of each head is rounded to integers at
 * a step of max|H q| / (127 * 2^14) (about 2^-21 of its largest element)
 * before the integer tensor-core products with the codes.
 * Split-K flash decoding: partial (max, sum, accumulator) per split in the
 * workspace, then a log-sum-exp combine that also applies the back-rotation.
 * Few rows: equal splits of each row.  Many rows (at least 37 (row, head
 * group) units): every SM's CTA takes an equal run of all rows' tiles, found
 * on the device from d_seq_lens, and writes one partial per row it touches.
 * Either way the result depends only on the inputs (run to run identical).
 * Both kernels are launched with programmatic stream serialization: they may
 * be scheduled while the previous kernel on the stream drains and wait for it
 * on the device before reading any input.
 *   q: device, [batch][num_q_heads][256] of `dtype`, 16-byte aligned.
 *   d_seq_lens: device int32[batch]; values are clamped to
 *   [0, min(max_seq_len, capacity)]; a sequence of length 0 gives a zero row.
 *   max_seq_len: host upper bound of the lengths (sizes the grid).
 *   out: device, [batch][num_q_heads][256] fp32, 16-byte aligned.
 *   workspace: device, >= kvq_decode_attn_workspace(...) bytes, 16-byte
 *   aligned; its contents are scratch.
 * num_q_heads must be a multiple of num_kv_heads with a group size of 1, 2,
 * 4, 8 or 16.  Accuracy: fp32 accumulation; within 2e-3 max-abs of an fp64
 * evaluation of the same dequantized cache for the documented workloads.
 * Pages referenced by a paged cache must lie in [0, num_pages); a token on a
 * page outside that range contributes nothing. */
KVQ_API kvq_status kvq_decode_attn(const kvq_cache *cache, const void *q, kvq_dtype dtype,
                           int32_t batch, int32_t num_q_heads,
                           const int32_t *d_seq_lens, int32_t max_seq_len, float scale,
                           float *out, void *workspace, size_t workspace_bytes,
                           void *stream);

/* kvq_decode_attn_multi -- several query tokens per sequence (speculative
 * verification, multi-token prediction): query i attends over the first
 * d_q_lens[i] tokens of sequence d_q_to_seq[i] of the Q4_0 cache (the causal
 * prefix of each drafted token is expressed through its length, as in the
 * q_to_req / q_to_klen arguments of the Octave page's reference_attention).
 * Otherwise as kvq_decode_attn with batch = n_q:
 *   q: device, [n_q][num_q_heads][256] of `dtype`, 16-byte aligned.
 *   d_q_to_seq: device int32[n_q]; a value outside [0, num_seqs) gives a zero
 *   row.  num_seqs: sequences in the cache (contiguous: <= batch_capacity;
 *   paged: rows of the block table).
 *   d_q_lens: device int32[n_q], clamped to [0, min(max_seq_len, capacity)].
 *   out: device, [n_q][num_q_heads][256] fp32, 16-byte aligned.
 *   workspace: >= kvq_decode_attn_workspace(cache, n_q, num_q_heads,
 *   max_seq_len) bytes.
 * Each query streams its sequence's cache on its own (no sharing of KV reads
 * between the queries of one sequence). */
KVQ_API kvq_status kvq_decode_attn_multi(const kvq_cache *cache, const void *q, kvq_dtype dtype,
                                         int32_t n_q, int32_t num_q_heads,
                                         const int32_t *d_q_to_seq, const int32_t *d_q_lens,
                                         int32_t num_seqs, int32_t max_seq_len, float scale,
                                         float *out, void *workspace, size_t workspace_bytes,
                                         void *stream);

/* kvq_decode_step -- one decode step of the per-token path in a single call:
 * quantize-on-append of each sequence's new token, then decode attention over
 * the sequence including it (Strata PR #21, merge note: the per-token path
 * rotates the new K/V and the query, attends, and rotates the output back).
 * Equivalent to kvq_quantize_append(cache, k_new, v_new, dtype, batch, 1,
 * d_pos) followed by kvq_decode_attn(cache, q, dtype, batch, num_q_heads,
 * seq_lens = d_pos + 1, max_seq_len, scale, out, ...): the cache bytes are
 * bit-identical to that pair of calls, and so is the output when the batch
 * has few rows (fewer than 37 (row, head group) units: one split per CTA).
 * Larger batches use the balanced schedule, in which the CTA appending a
 * token is given fewer tiles; the output then matches the pair of calls to
 * fp32 rounding.  The CTA whose tiles hold position d_pos[b] quantizes the
 * token in its prologue, so the append costs no launch of its own.
 *   k_new, v_new: device, [batch][num_kv_heads][256] of `dtype`, 16-byte
 *   aligned.  q: device, [batch][num_q_heads][256] of `dtype`, 16-byte aligned.
 *   d_pos: device int32[batch], position of the new token; a position outside
 *   the cache (negative, >= capacity) appends nothing; the attended length is
 *   d_pos[b] + 1 clamped to [0, min(max_seq_len, capacity)].
 *   max_seq_len: host upper bound of d_pos[b] + 1.
 *   out, workspace: as kvq_decode_attn (kvq_decode_attn_workspace sizes it).
 * Errors as kvq_decode_attn. */
KVQ_API kvq_status kvq_decode_step(const kvq_cache *cache, const void *k_new, const void *v_new,
                                   const void *q, kvq_dtype dtype, int32_t batch,
                                   int32_t num_q_heads, const int32_t *d_pos,
                                   int32_t max_seq_len, float scale, float *out, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* kvq_decode_attn_noalloc -- kvq_decode_attn without a caller-provided
 * workspace.  (The pages have no counterpart: this is an interface
 * convenience, not part of the method.)
 * Some callers cannot hand the library device scratch memory: a plugin
 * interface that passes only the input and output tensors, a C host program
 * without a device allocator, or a latency-critical decode loop that must
 * never call cudaMalloc (slow, and it can synchronize the device).  This call
 * allocates nothing: its split-K partials live in a fixed device array inside
 * the library, KVQ_DECODE_NOALLOC_SCRATCH_BYTES large, which every GPU that
 * loads the library holds until the process exits.
 *   Arguments, layouts and results are those of kvq_decode_attn, and so are
 *   the argument checks and their order: a bad argument returns the status
 *   kvq_decode_attn would return for it.  A valid shape whose workspace
 *   (kvq_decode_attn_workspace) exceeds KVQ_DECODE_NOALLOC_SCRATCH_BYTES
 *   returns KVQ_ERR_WORKSPACE before any launch; use kvq_decode_attn with a
 *   workspace for such shapes.
 *   The first call on a device looks up the array's device address with that
 *   device current (KVQ_ERR_CUDA if the lookup fails); make that first call
 *   before any stream capture.  The address is kept for the life of the
 *   process: after cudaDeviceReset on a device, do not call this entry point
 *   on that device again.
 *   All calls on a device share the one array: every call overwrites the
 *   records it reads, so nothing carries over from the previous call, but two
 *   calls whose kernels overlap on the GPU (different streams, no ordering
 *   between them) race on it and give undefined results. */
#define KVQ_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)
KVQ_API kvq_status kvq_decode_attn_noalloc(const kvq_cache *cache, const void *q,
                                           kvq_dtype dtype, int32_t batch, int32_t num_q_heads,
                                           const int32_t *d_seq_lens, int32_t max_seq_len,
                                           float scale, float *out, void *stream);

/* ------------------------------------------------------------------------ */
/* Conditions kernels cannot return as a status                               */
/* ------------------------------------------------------------------------ */

/* (The pages have no counterpart: these calls are diagnostics of this
 * library.)  A kernel that meets a condition it cannot report through a
 * kvq_status -- it runs after the call has returned -- ORs one of these flags
 * into a 32-bit error word the library keeps on each device:
 *   KVQ_DEVERR_WAIT_TIMEOUT  a decode kernel's bounded wait for a tile of the
 *                            cache gave up (the poll limit below); the
 *                            affected CTAs stop, their partial results are NaN
 *                            and so are the outputs that include them;
 *   KVQ_DEVERR_BOUNDS        a build compiled with KVQ_DEBUG_BOUNDS found a
 *                            computed address outside the buffer it should
 *                            lie in and skipped the access. */
#define KVQ_DEVERR_WAIT_TIMEOUT 1u
#define KVQ_DEVERR_BOUNDS 2u

/* kvq_device_errors -- the error word of the current device: *flags gets the
 * OR of the flags recorded since the previous call, and the word is cleared.
 * Unlike every other call this one synchronizes the device (it reads the word
 * after all work on the device has finished); KVQ_ERR_CUDA if that or the
 * copy fails.  flags: host pointer. */
KVQ_API kvq_status kvq_device_errors(uint32_t *flags);

/* kvq_set_wait_limit -- poll limit of the decode kernels' bounded waits on
 * their tile loads, for kernels launched after the call (process-wide).
 * Each poll waits up to about 1 us; the default (polls = -1) is 2^20, far
 * beyond any load that is merely slow.  polls = 0 makes each wait a single
 * non-blocking test, so that a wait on a tile still in flight gives up: a way
 * to exercise the timeout path (KVQ_DEVERR_WAIT_TIMEOUT, NaN outputs) without
 * a fault.  After giving up, a CTA still waits, with the default limit, for
 * the copies it has issued before it exits.  polls < -1: KVQ_ERR_INVALID_ARG. */
KVQ_API kvq_status kvq_set_wait_limit(int32_t polls);

/* ------------------------------------------------------------------------ */
/* Octave variant (vLLM API page "vllm.v1.attention.ops.rocm_octave")        */
/* ------------------------------------------------------------------------ */

/* Format, as OctaveFormat: head_size, rope_dim, v_bits (3 or 4), compact. */
typedef struct {
  int32_t head_size;
  int32_t rope_dim;
  int32_t v_bits;
  int32_t compact;
} kvq_octave_fmt;

/* Derived byte layout of one (token, kv head) slot:
 * [k_rope codes][k_nope codes][v codes][fp16 scales][pad to 8 (4 if compact)]
 * with the offsets of OctaveFormat (off_k_nope, off_v, off_scales,
 * num_scales, slot_bytes) and kernel_code = v_bits + 16 * compact. */
typedef struct {
  int32_t off_k_nope, off_v, off_scales, num_k_scales, num_scales, slot_bytes;
  int32_t kernel_code;
} kvq_octave_layout;

/* Host only: validate a format (the OctaveFormat checks: v_bits in {3, 4},
 * compact needs a power-of-two head, head and rope multiples of 64) and fill
 * its layout.  Returns KVQ_ERR_INVALID_ARG for an invalid format. */
KVQ_API kvq_status kvq_octave_layout_of(const kvq_octave_fmt *fmt, kvq_octave_layout *out);

/* Host only: the int8 Lloyd-Max codebook for N(0,1) with 2^bits levels
 * (bits = 3 or 4), ascending, LUT[i] = round(c_i * 127 / c_max), and
 * lut_mult = fp32(127 / c_max), the factor that maps an RMS-normalised value
 * into LUT units.  lut must hold 2^bits entries; lut_mult may be NULL. */
KVQ_API kvq_status kvq_octave_codebook(int32_t bits, int8_t *lut, float *lut_mult);

/* kvq_octave_quantize -- reference_quantize into a paged cache.
 *   key, value: device, [num_tokens][num_kv_heads][head_size] of `dtype`,
 *   16-byte aligned.
 *   d_slot_mapping: device int64[num_tokens]; token i goes to block
 *   slot / block_size, offset slot % block_size; a negative slot or a block
 *   outside [0, num_blocks) skips the token.
 *   cache: device, [num_blocks][num_kv_heads][block_size][slot_bytes] bytes.
 *   sign_bits: host, head_size / 32 int32 words, bit i set where the fixed
 *   sign pattern is -1 (vLLM rocm_octave page, sign_bits).
 * K: x * signs, FWHT over each 64-dim block, nearest Lloyd-Max code on each
 * block's RMS (4-bit for RoPE blocks, 3-bit for NoPE blocks); V: x * signs,
 * one FWHT over the head (power-of-two heads), v_bits codes.  Each scale is
 * fp16(|x|^2 / (x . LUT[c]) * LUT_ONE) (0 when that dot is not positive) with
 * LUT_ONE = 64; sums run in the fixed pairwise order v[i] + v[i + n/2],
 * halving n.  Bit-identical to that fp32 sequence.  Compact K (kernel code
 * 16 + v_bits): K x signs, one FWHT over the whole head, 3-bit codes and one
 * scale for the head.  This build implements head_size 128 with v_bits 3 or
 * 4, compact or not; other valid formats return KVQ_ERR_UNSUPPORTED. */
KVQ_API kvq_status kvq_octave_quantize(const kvq_octave_fmt *fmt, const void *key,
                               const void *value, kvq_dtype dtype, int32_t num_tokens,
                               int32_t num_kv_heads, const int64_t *d_slot_mapping,
                               uint8_t *cache, int32_t block_size, int64_t num_blocks,
                               const int32_t *sign_bits, void *stream);

/* Bytes of scratch kvq_octave_decode_attn needs for this shape. */
KVQ_API size_t kvq_octave_decode_attn_workspace(const kvq_octave_fmt *fmt, int32_t num_q,
                                        int32_t num_q_heads, int32_t max_klen);

/* kvq_octave_decode_attn -- reference_attention over the paged Octave cache:
 * query token i attends to the first q_to_klen[i] tokens of request
 * q_to_req[i] (block table indirection); query head h reads kv head
 * h / (num_q_heads / num_kv_heads); scores are computed in the rotated space
 * (the query is rotated like K) and the output is rotated back once per query
 * head; klen <= 0 gives a zero row.
 *   query: device, [num_q][num_q_heads][head_size] of `dtype`.
 *   cache: device, [num_blocks][num_kv_heads][block_size][slot_bytes].
 *   d_block_table: device int32[num_reqs][max_blocks_per_req].
 *   d_q_to_req, d_q_to_klen: device int32[num_q]; a request outside
 *   [0, num_reqs) gives a zero row; klen is clamped to
 *   [0, min(max_klen, max_blocks_per_req * block_size)]; a block outside
 *   [0, num_blocks) contributes nothing.
 *   max_klen: host upper bound of q_to_klen (sizes the grid).
 *   sign_bits: host, as for kvq_octave_quantize.
 *   out: device, [num_q][num_q_heads][head_size] fp32.
 * Same implemented formats as kvq_octave_quantize; group size 1, 2, 4 or 8.
 * On the k3v4 tensor-core path the split kernel and the combine are launched
 * as programmatic dependents of the work before them on `stream`; each
 * waits for that work to finish before it reads any input, so stream order
 * holds as for plain launches. */
KVQ_API kvq_status kvq_octave_decode_attn(const kvq_octave_fmt *fmt, const void *query,
                                  kvq_dtype dtype, int32_t num_q, int32_t num_q_heads,
                                  const uint8_t *cache, int32_t num_kv_heads,
                                  int32_t block_size, int64_t num_blocks,
                                  const int32_t *d_block_table, int32_t num_reqs,
                                  int32_t max_blocks_per_req, const int32_t *d_q_to_req,
                                  const int32_t *d_q_to_klen, int32_t max_klen,
                                  float scale, const int32_t *sign_bits, float *out,
                                  void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
