// kvq_internal.cuh -- device helpers and launcher declarations shared by the
// kernels of the KV-cache library.  Nothing here is part of the C ABI.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kDim = 256;       // Q4_0 path head dimension
constexpr int kQBlock = 32;     // values per Q4_0 block
constexpr int kRowCodeBytes = 128;
constexpr int kRowScales = 8;
constexpr int kNumSMs = 148;    // B200

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ldg_stream_u4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, 65536, 0;" : "=r"(r) : "r"(w));
  return __uint_as_float(r);
}
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// maximum that returns NaN if either input is NaN (split-K combines: a record
// left NaN by a split that gave up must reach the output)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// ---------------------------------------------------------------- packed fp32
// Packed fp32x2 arithmetic.  Used only where no multiply feeds an add
// (butterflies, end scaling, the round-toward-zero add): a packed multiply
// followed by a packed add has been observed to be fused into one rounding
// even with an explicit .rn, so that pattern uses scalar __fmul_rn / __fadd_rn.
__device__ __forceinline__ uint64_t pk(float2 a) {
  return (uint64_t)__float_as_uint(a.x) | ((uint64_t)__float_as_uint(a.y) << 32);
}
__device__ __forceinline__ float2 upk(uint64_t v) {
  return make_float2(__uint_as_float((uint32_t)v), __uint_as_float((uint32_t)(v >> 32)));
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __fadd2_rn(a, make_float2(-b.x, -b.y));
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// a * b + 0, rounded once: the same value as RN(a * b) except that a -0
// product comes out +0.  Unlike a plain multiply, ptxas cannot rewrite it into
// a multiply and contract that with a following add.
__device__ __forceinline__ float2 mul2_rn_p0(float2 a, float2 b) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)), "l"(0ull));
  return upk(r);
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}
__device__ __forceinline__ float2 add2_rz(float2 a, float2 b) {
  uint64_t r;
  asm("add.rz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}

// ---------------------------------------------------------------- row index
// Row of (sequence b, kv head h, token t) in the structure-of-arrays Q4_0
// cache; -1 when the position lies outside the cache.
__device__ __forceinline__ int64_t q4_row(const kvq_cache &c, int b, int h, int t) {
  if (t < 0) return -1;
  if (c.block_table == nullptr) {
    if (t >= c.max_tokens) return -1;
    return ((int64_t)b * c.num_kv_heads + h) * c.max_tokens + t;
  }
  int pi = t / c.page_size;
  if (pi >= c.max_pages_per_seq) return -1;
  int page = __ldg(c.block_table + (int64_t)b * c.max_pages_per_seq + pi);
  if (page < 0 || page >= c.num_pages) return -1;
  return ((int64_t)page * c.num_kv_heads + h) * c.page_size + (t - pi * c.page_size);
}

// ---------------------------------------------------------------- bounds
// Rows of the cache planes (contiguous or paged).
__device__ __forceinline__ int64_t cache_rows(const kvq_cache &c) {
  return c.block_table ? (int64_t)c.num_pages * c.num_kv_heads * c.page_size
                       : (int64_t)c.batch_capacity * c.num_kv_heads * c.max_tokens;
}
// Debug builds (compiled with KVQ_DEBUG_BOUNDS): true if [lo, hi) lies
// inside [0, n); otherwise KVQ_DEVERR_BOUNDS goes into the error word and the
// caller skips or redirects the access.  Release builds: always true (the
// index arithmetic keeps every access inside the buffers the call describes).
__device__ __forceinline__ bool in_bounds(int64_t lo, int64_t hi, int64_t n, uint32_t *err) {
#ifdef KVQ_DEBUG_BOUNDS
  if (lo >= 0 && lo <= hi && hi <= n) return true;
  if (err != nullptr) atomicOr(err, KVQ_DEVERR_BOUNDS);
  return false;
#else
  (void)lo, (void)hi, (void)n, (void)err;
  return true;
#endif
}

// ---------------------------------------------------------------- errors
// Device address of the library's error word on the current device (nullptr
// if the lookup fails), and the mbarrier poll limit of the decode kernels'
// bounded waits (kvq_set_wait_limit; 1 << 20 by default).
uint32_t *device_error_word();
int wait_poll_limit();

// ---------------------------------------------------------------- launchers
cudaError_t launch_rotate(const void *x, int bf16, float *y, int64_t n_vec, cudaStream_t s);
// code_bits 4: Q4_0 (128-byte code rows), 8: Q8_0 (256-byte code rows)
cudaError_t launch_q4_append(const kvq_cache &c, const void *k, const void *v, int bf16,
                             int batch, int t_new, const int32_t *start_pos, cudaStream_t s,
                             int code_bits = 4);

struct DecodePlan {
  int splits;       // split mode: splits per (query row, head group)
  int split_tokens; // split mode: tokens per split (multiple of 64)
  int stream;       // 1: balanced stream schedule over all units (see decode_common.cuh)
  int ctas;         // stream mode: CTAs of the split kernel
  int n_units;      // query rows x head groups
  int tile;         // stream mode: tokens per tile of the split kernel
};
// split-K plan over `units` independent problems with `slots` resident CTAs
DecodePlan plan_split_k(int units, int max_len, int slots, int max_splits, int granule = 64,
                        int overhead_tokens = 0);
// n_head_groups: q heads / min(group, 8); tile: 128 (Q4_0) or 64 (Q8_0)
DecodePlan plan_decode(int batch, int n_head_groups, int max_seq_len, int tile = 128);
int q4_decode_ctas_per_sm();
int q4_decode_tile_tokens();
// k_new, v_new, pos: fused decode step (append one token per sequence at
// pos[b], then attend over pos[b] + 1 tokens); all nullptr for plain decode.
// q_to_seq: several queries per sequence (batch = number of queries, query b
// reads sequence q_to_seq[b] < num_seqs with length seq_lens[b]); nullptr: b.
cudaError_t launch_q4_decode_mma(const kvq_cache &c, const void *q, int bf16, int batch,
                                 int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                                 float scale, float *ws, const DecodePlan &p, cudaStream_t s,
                                 const void *k_new = nullptr, const void *v_new = nullptr,
                                 const int32_t *pos = nullptr, const int32_t *q_to_seq = nullptr,
                                 int num_seqs = 0);
// the same over a Q8_0 cache (c.code_bits == 8); p.split_tokens a multiple of 64
cudaError_t launch_q8_decode_mma(const kvq_cache &c, const void *q, int bf16, int batch,
                                 int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                                 float scale, float *ws, const DecodePlan &p, cudaStream_t s,
                                 const void *k_new = nullptr, const void *v_new = nullptr,
                                 const int32_t *pos = nullptr, const int32_t *q_to_seq = nullptr,
                                 int num_seqs = 0);
size_t decode_workspace_bytes(int batch, int n_q_heads, const DecodePlan &p);
// host: the argument checks of kvq_decode_attn that precede its workspace checks
kvq_status check_decode_args(const kvq_cache *cache, const void *q, kvq_dtype dtype,
                             int32_t batch, int32_t num_q_heads, const int32_t *d_seq_lens,
                             int32_t max_seq_len, float scale, const float *out);
cudaError_t launch_q4_decode(const kvq_cache &c, const void *q, int bf16, int batch,
                             int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                             float scale, float *out, float *ws, const DecodePlan &p,
                             cudaStream_t s, const void *k_new = nullptr,
                             const void *v_new = nullptr, const int32_t *pos = nullptr,
                             const int32_t *q_to_seq = nullptr, int num_seqs = 0);

struct OctaveParams {
  // rope_dim here is the K dims coded with 4 bits (0 for compact K, whose
  // codes are all 3-bit over one whole-head rotation with one scale)
  int head_size, rope_dim, v_bits, compact;
  int off_k_nope, off_v, off_scales, slot_bytes;
  uint32_t sign_words[16];  // up to 512 dims
  int8_t lut3[8];
  int8_t lut4[16];
  float mult3, mult4;
};
cudaError_t launch_octave_quantize(const OctaveParams &p, const void *key, const void *value,
                                   int bf16, int num_tokens, int n_kv_heads,
                                   const int64_t *slot_mapping, uint8_t *cache,
                                   int block_size, int64_t num_blocks, cudaStream_t s);
DecodePlan plan_octave_decode(int num_q, int n_head_groups, int max_klen);
bool octave_mma_supported(const OctaveParams &p);
cudaError_t launch_octave_decode_mma(const OctaveParams &P, const void *query, int bf16, int num_q,
                                     int n_q_heads, const uint8_t *cache, int n_kv_heads,
                                     int block_size, int64_t num_blocks,
                                     const int32_t *block_table, int num_reqs, int max_blocks,
                                     const int32_t *q_to_req, const int32_t *q_to_klen,
                                     int max_klen, float scale, float *ws,
                                     const DecodePlan &plan, cudaStream_t s);
size_t octave_workspace_bytes(int num_q, int n_q_heads, int head_size, const DecodePlan &p);
cudaError_t launch_octave_decode(const OctaveParams &p, const void *query, int bf16, int num_q,
                                 int n_q_heads, const uint8_t *cache, int n_kv_heads,
                                 int block_size, int64_t num_blocks, const int32_t *block_table,
                                 int num_reqs, int max_blocks, const int32_t *q_to_req,
                                 const int32_t *q_to_klen, int max_klen, float scale,
                                 float *out, float *ws, const DecodePlan &plan, cudaStream_t s);

}  // namespace kvq
