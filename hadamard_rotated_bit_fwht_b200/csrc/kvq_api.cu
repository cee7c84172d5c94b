// kvq_api.cu -- the extern "C" entry points declared in include/kvq.h: host-side
// argument validation, the Octave codebook, and dispatch to the kernels.
#include <math.h>
#include <string.h>

#include <mutex>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kvq_status check_cache(const kvq_cache *c) {
  if (!c || !c->k_codes || !c->k_scales || !c->v_codes || !c->v_scales) return KVQ_ERR_INVALID_ARG;
  if (c->num_kv_heads < 1 || c->head_dim <= 0) return KVQ_ERR_INVALID_ARG;
  if (c->head_dim != kDim) return KVQ_ERR_UNSUPPORTED;
  if (c->code_bits != 0 && c->code_bits != 4 && c->code_bits != 8) return KVQ_ERR_INVALID_ARG;
  if (!aligned(c->k_codes, 16) || !aligned(c->v_codes, 16) || !aligned(c->k_scales, 16) ||
      !aligned(c->v_scales, 16))
    return KVQ_ERR_INVALID_ARG;
  if (c->block_table) {
    if (c->page_size <= 0 || c->page_size % 64 || c->max_pages_per_seq <= 0 || c->num_pages <= 0)
      return KVQ_ERR_INVALID_ARG;
  } else {
    if (c->max_tokens <= 0 || c->batch_capacity <= 0) return KVQ_ERR_INVALID_ARG;
  }
  return KVQ_OK;
}

// ---- Lloyd-Max codebook for N(0,1), computed once per bit width on the host.
// Lloyd's method: each level is the mean of N(0,1) over its cell, each cell
// edge is the midpoint of its two levels; iterate to a fixed point (fp64).
struct Codebook {
  int8_t lut[16];
  float mult;
};

double phi(double x) { return isinf(x) ? 0.0 : exp(-0.5 * x * x) * 0.3989422804014327; }
double upper_tail(double x) { return 0.5 * erfc(x * 0.7071067811865476); }

void lloyd_levels(int levels, double *c) {
  for (int i = 0; i < levels; i++) c[i] = 6.0 * ((i + 0.5) / levels - 0.5);
  double edge[17];
  for (int iter = 0; iter < 200000; iter++) {
    edge[0] = -INFINITY;
    edge[levels] = INFINITY;
    for (int i = 1; i < levels; i++) edge[i] = 0.5 * (c[i - 1] + c[i]);
    double moved = 0.0;
    for (int i = 0; i < levels; i++) {
      const double lo = edge[i], hi = edge[i + 1];
      double mass;
      if (lo >= 0.0) mass = upper_tail(lo) - upper_tail(hi);
      else if (hi <= 0.0) mass = upper_tail(-hi) - upper_tail(-lo);
      else mass = 1.0 - upper_tail(hi) - upper_tail(-lo);
      const double mean = (phi(lo) - phi(hi)) / mass;
      moved = fmax(moved, fabs(mean - c[i]));
      c[i] = mean;
    }
    if (moved < 1e-16) break;
  }
}

const Codebook &codebook(int bits) {
  static Codebook cb[5];
  static std::once_flag once[5];
  std::call_once(once[bits], [bits] {
    const int levels = 1 << bits;
    double c[16];
    lloyd_levels(levels, c);
    const double mult = 127.0 / c[levels - 1];
    for (int i = 0; i < levels; i++) cb[bits].lut[i] = (int8_t)lround(c[i] * mult);
    cb[bits].mult = (float)mult;
  });
  return cb[bits];
}

bool is_pow2(int n) { return n > 0 && (n & (n - 1)) == 0; }

kvq_status octave_layout(const kvq_octave_fmt *f, kvq_octave_layout *o) {
  if (!f || !o) return KVQ_ERR_INVALID_ARG;
  const int d = f->head_size, r = f->rope_dim;
  if (f->v_bits != 3 && f->v_bits != 4) return KVQ_ERR_INVALID_ARG;
  if (f->compact && !is_pow2(d)) return KVQ_ERR_INVALID_ARG;
  if (d <= 0 || r < 0 || r > d || r % 64 || d % 64) return KVQ_ERR_INVALID_ARG;
  const int k_wide = f->compact ? 0 : r;
  o->off_k_nope = k_wide * 4 / 8;
  o->off_v = o->off_k_nope + (d - k_wide) * 3 / 8;
  o->off_scales = o->off_v + d * f->v_bits / 8;
  o->num_k_scales = f->compact ? 1 : d / 64;
  o->num_scales = o->num_k_scales + 1;
  const int raw = o->off_scales + 2 * o->num_scales;
  const int align = f->compact ? 4 : 8;
  o->slot_bytes = (raw + align - 1) / align * align;
  o->kernel_code = f->v_bits + (f->compact ? 16 : 0);
  return KVQ_OK;
}

kvq_status octave_params(const kvq_octave_fmt *f, const int32_t *sign_bits, OctaveParams &p) {
  kvq_octave_layout lay;
  kvq_status st = octave_layout(f, &lay);
  if (st != KVQ_OK) return st;
  if (!sign_bits) return KVQ_ERR_INVALID_ARG;
  if (f->head_size != 128 || f->rope_dim > 128) return KVQ_ERR_UNSUPPORTED;
  memset(&p, 0, sizeof(p));
  p.head_size = f->head_size;
  p.rope_dim = f->compact ? 0 : f->rope_dim;
  p.compact = f->compact ? 1 : 0;
  p.v_bits = f->v_bits;
  p.off_k_nope = lay.off_k_nope;
  p.off_v = lay.off_v;
  p.off_scales = lay.off_scales;
  p.slot_bytes = lay.slot_bytes;
  for (int w = 0; w < f->head_size / 32; w++) p.sign_words[w] = (uint32_t)sign_bits[w];
  const Codebook &c3 = codebook(3), &c4 = codebook(4);
  memcpy(p.lut3, c3.lut, 8);
  memcpy(p.lut4, c4.lut, 16);
  p.mult3 = c3.mult;
  p.mult4 = c4.mult;
  return KVQ_OK;
}

}  // namespace

extern "C" {

const char *kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

int kvq_version(void) { return 100; }

kvq_status kvq_rotate(const void *x, kvq_dtype dtype, float *y, int64_t n_vec, int32_t dim,
                      void *stream) {
  if (n_vec < 0 || (dtype != KVQ_F32 && dtype != KVQ_BF16)) return KVQ_ERR_INVALID_ARG;
  if (dim != kDim) return dim > 0 ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_INVALID_ARG;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_rotate(x, dtype == KVQ_BF16, y, n_vec, as_stream(stream)));
}

kvq_status kvq_quantize_append(const kvq_cache *cache, const void *k, const void *v,
                               kvq_dtype dtype, int32_t batch, int32_t t_new,
                               const int32_t *d_start_pos, void *stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (batch < 0 || t_new < 0 || (dtype != KVQ_F32 && dtype != KVQ_BF16)) return KVQ_ERR_INVALID_ARG;
  if (!cache->block_table && batch > cache->batch_capacity) return KVQ_ERR_INVALID_ARG;
  if (batch == 0 || t_new == 0) return KVQ_OK;
  if (!k || !v || !d_start_pos || !aligned(k, 16) || !aligned(v, 16)) return KVQ_ERR_INVALID_ARG;
  // the kernel indexes the 2 * batch * t_new * heads vectors with 31-bit counts
  if (2LL * batch * t_new * cache->num_kv_heads >= (1LL << 31)) return KVQ_ERR_UNSUPPORTED;
  return from_cuda(launch_q4_append(*cache, k, v, dtype == KVQ_BF16, batch, t_new, d_start_pos,
                                    as_stream(stream), cache->code_bits == 8 ? 8 : 4));
}

// CTAs per (sequence, split): q heads in groups of at most 8 per kv head
// tokens per tile of the split kernel (the stream schedule's granule)
static int decode_tile(const kvq_cache *c) { return c->code_bits == 8 ? 64 : 128; }

static int head_groups(int num_q_heads, int num_kv_heads) {
  const int group = num_q_heads / num_kv_heads;
  return num_q_heads / (group < 8 ? (group > 0 ? group : 1) : 8);
}

size_t kvq_decode_attn_workspace(const kvq_cache *cache, int32_t batch, int32_t num_q_heads,
                                 int32_t max_seq_len) {
  if (!cache || batch <= 0 || num_q_heads <= 0 || cache->num_kv_heads <= 0) return 0;
  DecodePlan p = plan_decode(batch, head_groups(num_q_heads, cache->num_kv_heads), max_seq_len,
                             decode_tile(cache));
  return decode_workspace_bytes(batch, num_q_heads, p);
}

}  // extern "C"

// Every argument check of kvq_decode_attn except the workspace ones, in the
// same order; shared with the allocation-free variant so both report the same
// status for the same bad argument.
kvq_status kvq::check_decode_args(const kvq_cache *cache, const void *q, kvq_dtype dtype,
                                  int32_t batch, int32_t num_q_heads, const int32_t *d_seq_lens,
                                  int32_t max_seq_len, float scale, const float *out) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads <= 0 || max_seq_len < 0 || (dtype != KVQ_F32 && dtype != KVQ_BF16))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return KVQ_ERR_INVALID_ARG;
  const int group = num_q_heads / cache->num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return KVQ_ERR_UNSUPPORTED;
  if (!cache->block_table && batch > cache->batch_capacity) return KVQ_ERR_INVALID_ARG;
  if (!isfinite(scale)) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!q || !d_seq_lens || !out || !aligned(q, 16) || !aligned(out, 16)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

extern "C" {

kvq_status kvq_decode_attn(const kvq_cache *cache, const void *q, kvq_dtype dtype, int32_t batch,
                           int32_t num_q_heads, const int32_t *d_seq_lens, int32_t max_seq_len,
                           float scale, float *out, void *workspace, size_t workspace_bytes,
                           void *stream) {
  kvq_status st = check_decode_args(cache, q, dtype, batch, num_q_heads, d_seq_lens, max_seq_len,
                                    scale, out);
  if (st != KVQ_OK || batch == 0) return st;
  DecodePlan p = plan_decode(batch, head_groups(num_q_heads, cache->num_kv_heads), max_seq_len,
                             decode_tile(cache));
  const size_t need = decode_workspace_bytes(batch, num_q_heads, p);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return KVQ_ERR_WORKSPACE;
  return from_cuda(launch_q4_decode(*cache, q, dtype == KVQ_BF16, batch, num_q_heads, d_seq_lens,
                                    max_seq_len, scale, out, static_cast<float *>(workspace), p,
                                    as_stream(stream)));
}

kvq_status kvq_decode_attn_multi(const kvq_cache *cache, const void *q, kvq_dtype dtype,
                                 int32_t n_q, int32_t num_q_heads, const int32_t *d_q_to_seq,
                                 const int32_t *d_q_lens, int32_t num_seqs, int32_t max_seq_len,
                                 float scale, float *out, void *workspace, size_t workspace_bytes,
                                 void *stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (n_q < 0 || num_q_heads <= 0 || max_seq_len < 0 || num_seqs < 0 ||
      (dtype != KVQ_F32 && dtype != KVQ_BF16))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return KVQ_ERR_INVALID_ARG;
  const int group = num_q_heads / cache->num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return KVQ_ERR_UNSUPPORTED;
  if (!cache->block_table && num_seqs > cache->batch_capacity) return KVQ_ERR_INVALID_ARG;
  if (!isfinite(scale)) return KVQ_ERR_INVALID_ARG;
  if (n_q == 0) return KVQ_OK;
  if (!q || !d_q_to_seq || !d_q_lens || !out || !aligned(q, 16) || !aligned(out, 16))
    return KVQ_ERR_INVALID_ARG;
  DecodePlan p = plan_decode(n_q, head_groups(num_q_heads, cache->num_kv_heads), max_seq_len,
                             decode_tile(cache));
  const size_t need = decode_workspace_bytes(n_q, num_q_heads, p);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return KVQ_ERR_WORKSPACE;
  return from_cuda(launch_q4_decode(*cache, q, dtype == KVQ_BF16, n_q, num_q_heads, d_q_lens,
                                    max_seq_len, scale, out, static_cast<float *>(workspace), p,
                                    as_stream(stream), nullptr, nullptr, nullptr, d_q_to_seq,
                                    num_seqs));
}

kvq_status kvq_decode_step(const kvq_cache *cache, const void *k_new, const void *v_new,
                           const void *q, kvq_dtype dtype, int32_t batch, int32_t num_q_heads,
                           const int32_t *d_pos, int32_t max_seq_len, float scale, float *out,
                           void *workspace, size_t workspace_bytes, void *stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads <= 0 || max_seq_len < 0 || (dtype != KVQ_F32 && dtype != KVQ_BF16))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return KVQ_ERR_INVALID_ARG;
  const int group = num_q_heads / cache->num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return KVQ_ERR_UNSUPPORTED;
  if (!cache->block_table && batch > cache->batch_capacity) return KVQ_ERR_INVALID_ARG;
  if (!isfinite(scale)) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!q || !k_new || !v_new || !d_pos || !out || !aligned(q, 16) || !aligned(k_new, 16) ||
      !aligned(v_new, 16) || !aligned(out, 16))
    return KVQ_ERR_INVALID_ARG;
  DecodePlan p = plan_decode(batch, head_groups(num_q_heads, cache->num_kv_heads), max_seq_len,
                             decode_tile(cache));
  const size_t need = decode_workspace_bytes(batch, num_q_heads, p);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return KVQ_ERR_WORKSPACE;
  return from_cuda(launch_q4_decode(*cache, q, dtype == KVQ_BF16, batch, num_q_heads, nullptr,
                                    max_seq_len, scale, out, static_cast<float *>(workspace), p,
                                    as_stream(stream), k_new, v_new, d_pos));
}

kvq_status kvq_octave_layout_of(const kvq_octave_fmt *fmt, kvq_octave_layout *out) {
  return octave_layout(fmt, out);
}

kvq_status kvq_octave_codebook(int32_t bits, int8_t *lut, float *lut_mult) {
  if ((bits != 3 && bits != 4) || !lut) return KVQ_ERR_INVALID_ARG;
  const Codebook &c = codebook(bits);
  memcpy(lut, c.lut, (size_t)1 << bits);
  if (lut_mult) *lut_mult = c.mult;
  return KVQ_OK;
}

kvq_status kvq_octave_quantize(const kvq_octave_fmt *fmt, const void *key, const void *value,
                               kvq_dtype dtype, int32_t num_tokens, int32_t num_kv_heads,
                               const int64_t *d_slot_mapping, uint8_t *cache, int32_t block_size,
                               int64_t num_blocks, const int32_t *sign_bits, void *stream) {
  OctaveParams p;
  kvq_status st = octave_params(fmt, sign_bits, p);
  if (st != KVQ_OK) return st;
  if (num_tokens < 0 || num_kv_heads <= 0 || block_size <= 0 || num_blocks <= 0 ||
      (dtype != KVQ_F32 && dtype != KVQ_BF16))
    return KVQ_ERR_INVALID_ARG;
  if (num_tokens == 0) return KVQ_OK;
  if (!key || !value || !d_slot_mapping || !cache || !aligned(cache, 4) || !aligned(key, 16) ||
      !aligned(value, 16))
    return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_octave_quantize(p, key, value, dtype == KVQ_BF16, num_tokens,
                                          num_kv_heads, d_slot_mapping, cache, block_size,
                                          num_blocks, as_stream(stream)));
}

size_t kvq_octave_decode_attn_workspace(const kvq_octave_fmt *fmt, int32_t num_q,
                                        int32_t num_q_heads, int32_t max_klen) {
  if (!fmt || num_q <= 0 || num_q_heads <= 0) return 0;
  // the split plan depends on the kv head count, unknown here: size for the
  // most splits any plan makes (256-token splits)
  DecodePlan p;
  p.splits = (max(max_klen, 1) + 255) / 256;
  p.split_tokens = 256;
  return octave_workspace_bytes(num_q, num_q_heads, fmt->head_size, p);
}

kvq_status kvq_octave_decode_attn(const kvq_octave_fmt *fmt, const void *query, kvq_dtype dtype,
                                  int32_t num_q, int32_t num_q_heads, const uint8_t *cache,
                                  int32_t num_kv_heads, int32_t block_size, int64_t num_blocks,
                                  const int32_t *d_block_table, int32_t num_reqs,
                                  int32_t max_blocks_per_req, const int32_t *d_q_to_req,
                                  const int32_t *d_q_to_klen, int32_t max_klen, float scale,
                                  const int32_t *sign_bits, float *out, void *workspace,
                                  size_t workspace_bytes, void *stream) {
  OctaveParams p;
  kvq_status st = octave_params(fmt, sign_bits, p);
  if (st != KVQ_OK) return st;
  if (num_q < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || block_size <= 0 || num_blocks <= 0 ||
      num_reqs < 0 || max_blocks_per_req <= 0 || max_klen < 0 ||
      (dtype != KVQ_F32 && dtype != KVQ_BF16) || !isfinite(scale))
    return KVQ_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads) return KVQ_ERR_INVALID_ARG;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return KVQ_ERR_UNSUPPORTED;
  if (num_q == 0) return KVQ_OK;
  if (!query || !cache || !d_block_table || !d_q_to_req || !d_q_to_klen || !out ||
      !aligned(cache, 4))
    return KVQ_ERR_INVALID_ARG;
  DecodePlan plan = plan_octave_decode(num_q, head_groups(num_q_heads, num_kv_heads), max_klen);
  const size_t need = octave_workspace_bytes(num_q, num_q_heads, fmt->head_size, plan);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return KVQ_ERR_WORKSPACE;
  return from_cuda(launch_octave_decode(p, query, dtype == KVQ_BF16, num_q, num_q_heads, cache,
                                        num_kv_heads, block_size, num_blocks, d_block_table,
                                        num_reqs, max_blocks_per_req, d_q_to_req, d_q_to_klen,
                                        max_klen, scale, out, static_cast<float *>(workspace),
                                        plan, as_stream(stream)));
}

}  // extern "C"
