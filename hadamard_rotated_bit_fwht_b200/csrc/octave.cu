// octave.cu -- the Octave KV-cache variant (vLLM API page
// "vllm.v1.attention.ops.rocm_octave"): quantize into per-(token, head) byte
// slots, and decode attention over the paged slot cache.
//
// Quantize (reference_quantize): one warp per (token, kv head); lane l holds
// dims l, l+32, l+64, l+96 of the 128-dim head.
//   K: x * signs, FWHT over each 64-dim block (stages h = 1..16 across lanes
//      with xor-shuffles, h = 32 in registers, then x 1/8), then per block
//      _quantize_lut with 4-bit codes for RoPE blocks and 3-bit codes for NoPE
//      blocks.
//   V: x * signs, FWHT-128 over the head (h = 32, 64 in registers), x
//      fp32(1/sqrt(128)), _quantize_lut with v_bits codes.
//   _quantize_lut: ss = sum x^2 and dot = sum x * LUT[c] in the fixed pairwise
//      order (v[i] + v[i + n/2], halving n: in-register levels first, then
//      xor-shuffles 16, 8, 4, 2, 1, which add exactly the same pairs);
//      rms = max(sqrt(ss / n), 1e-12); y = x / rms * LUT_MULT; code = number
//      of LUT midpoints below y (ties go to the lower code);
//      scale = (dot > 0 ? ss / max(dot, 1e-30) : 0) * LUT_ONE, LUT_ONE = 64,
//      stored as fp16.
//   The slot is assembled in shared memory (bit packing of the page's module
//   text / _pack) and written with one 128-byte warp store.
// Decode (reference_attention, computed in the rotated space): one CTA per
//   (split, q-head group, query token); the query is rotated like K (signs +
//   64-dim blocks), each warp streams slots (one 32-bit word per lane,
//   shuffles to fetch its nibbles), dequantizes LUT[c] * s / 64, keeps an
//   online softmax, and the combine kernel merges the splits and rotates the
//   output back (FWHT-128 x fp32(1/sqrt(128)), then signs).
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kHead = 128;
constexpr int kORec = 132;  // m, l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLutOne = 64.f;

__device__ __forceinline__ float load_in(const void *p, int bf16, int64_t idx) {
  return bf16 ? __uint_as_float((uint32_t)static_cast<const uint16_t *>(p)[idx] << 16)
              : static_cast<const float *>(p)[idx];
}

__device__ __forceinline__ float sign_of(const OctaveParams &P, int d) {
  return ((P.sign_words[d >> 5] >> (d & 31)) & 1u) ? -1.f : 1.f;
}

// one cross-lane butterfly stage on lane-index bit h: v + o on the lower lane,
// o - v on the upper one, as one FMA with sg = +-1 (sg * v is exact, so the
// FMA rounds the same sum once)
__device__ __forceinline__ float xstage(float v, float sg, int h) {
  const float o = __shfl_xor_sync(kFull, v, h);
  return __fmaf_rn(sg, v, o);
}

// sum over the 32 lanes of one value per lane, pairs (i, i + 16), (i, i + 8), ...
__device__ __forceinline__ float xsum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, off));
  return v;
}

struct LutSmem {
  float lut[2][16];  // [0]: 3-bit (8 entries), [1]: 4-bit
  float mid[2][15];
};

// Number of the 2^BITS - 1 sorted LUT midpoints below y (bucketize with
// right=False: a tie goes to the lower code), by binary search.
template <int BITS>
__device__ __forceinline__ int bucket(float y, const float *mid) {
  int c = 0;
#pragma unroll
  for (int step = 1 << (BITS - 1); step >= 1; step >>= 1)
    if (mid[c + step - 1] < y) c += step;
  return c;
}

// _quantize_lut over n = 64 (two values per lane: dims l, l + 32 of the block)
// or n = 128 (four values per lane); codes out per value, returns the scale.
template <int NV, int BITS>
__device__ __forceinline__ float quantize_lut(const float (&x)[NV], float mult, const LutSmem &L,
                                              int (&code)[NV]) {
  constexpr int tb = BITS == 4 ? 1 : 0;
  float sq[NV];
#pragma unroll
  for (int k = 0; k < NV; k++) sq[k] = __fmul_rn(x[k], x[k]);
  // in-register levels: NV = 4 holds (l, l+32, l+64, l+96): first (l, l+64),
  // (l+32, l+96) [n = 128 -> 64], then their sum [64 -> 32]; NV = 2: (l, l+32).
  float ss;
  if (NV == 4) ss = __fadd_rn(__fadd_rn(sq[0], sq[2]), __fadd_rn(sq[1], sq[3]));
  else ss = __fadd_rn(sq[0], sq[1]);
  ss = xsum(ss);
  // ss / n for n = 64, 128: the product with the exact 1 / n is the same
  // real number, so it rounds the same
  float rms = __fsqrt_rn(__fmul_rn(ss, 1.f / (float)(NV * 32)));
  rms = rms < 1e-12f ? 1e-12f : rms;
  float pr[NV];
#pragma unroll
  for (int k = 0; k < NV; k++) {
    const float y = __fmul_rn(__fdiv_rn(x[k], rms), mult);
    const int c = bucket<BITS>(y, L.mid[tb]);
    code[k] = c;
    pr[k] = __fmul_rn(x[k], L.lut[tb][c]);
  }
  float dot;
  if (NV == 4) dot = __fadd_rn(__fadd_rn(pr[0], pr[2]), __fadd_rn(pr[1], pr[3]));
  else dot = __fadd_rn(pr[0], pr[1]);
  dot = xsum(dot);
  const float q = __fdiv_rn(ss, dot > 1e-30f ? dot : 1e-30f);
  return __fmul_rn(dot > 0.f ? q : 0.f, kLutOne);
}

// Word w (bytes 4w .. 4w+3) of the packed codes of a region of n dims whose
// codes (one per byte) start at c32 (layout of the page's module text):
//   4-bit: byte j of a word holds dim 8w + j (low nibble) and 8w + 4 + j;
//   3-bit: a 2-bit plane (byte j of word w gathers dims 16w + 4i + j in bits
//          2i..2i+1) followed by a 1-bit plane (byte j of word w gathers dims
//          32w + 4i + j in bit i); code = lo + 4 * hi.
__device__ __forceinline__ uint32_t pack_word(const uint32_t *c32, int n, int bits, int w) {
  if (bits == 4)
    return (c32[2 * w] & 0x0F0F0F0Fu) | ((c32[2 * w + 1] & 0x0F0F0F0Fu) << 4);
  if (w < n / 16) {
    const uint4 v = *reinterpret_cast<const uint4 *>(c32 + 4 * w);
    return (v.x & 0x03030303u) | ((v.y & 0x03030303u) << 2) | ((v.z & 0x03030303u) << 4) |
           ((v.w & 0x03030303u) << 6);
  }
  const int r = w - n / 16;
  const uint4 u = *reinterpret_cast<const uint4 *>(c32 + 8 * r);
  const uint4 v = *reinterpret_cast<const uint4 *>(c32 + 8 * r + 4);
  return ((u.x >> 2) & 0x01010101u) | (((u.y >> 2) & 0x01010101u) << 1) |
         (((u.z >> 2) & 0x01010101u) << 2) | (((u.w >> 2) & 0x01010101u) << 3) |
         (((v.x >> 2) & 0x01010101u) << 4) | (((v.y >> 2) & 0x01010101u) << 5) |
         (((v.z >> 2) & 0x01010101u) << 6) | (((v.w >> 2) & 0x01010101u) << 7);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
    octave_quantize_kernel(OctaveParams P, const void *__restrict__ key,
                           const void *__restrict__ value, int num_tokens,
                           int n_kv_heads, const int64_t *__restrict__ slot_mapping,
                           uint8_t *__restrict__ cache, int block_size, int64_t num_blocks) {
  __shared__ LutSmem L;
  __shared__ __align__(16) uint8_t kcodes[kWarps][kHead];
  __shared__ __align__(16) uint8_t vcodes[kWarps][kHead];
  for (int i = threadIdx.x; i < 16; i += blockDim.x) {
    L.lut[0][i] = i < 8 ? (float)P.lut3[i] : 0.f;
    L.lut[1][i] = (float)P.lut4[i];
    if (i < 7) L.mid[0][i] = ((float)P.lut3[i + 1] + (float)P.lut3[i]) / 2.0f;
    if (i < 15) L.mid[1][i] = ((float)P.lut4[i + 1] + (float)P.lut4[i]) / 2.0f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t items = (int64_t)num_tokens * n_kv_heads;
  const float vscale = 0.08838834764831845f;  // fp32(1 / sqrt(128))
  const int slot_words = P.slot_bytes / 4;
  const int w_kn = P.off_k_nope / 4, w_v = P.off_v / 4, w_sc = P.off_scales / 4;
  const uint32_t *kc32 = reinterpret_cast<const uint32_t *>(kcodes[warp]);
  const uint32_t *vc32 = reinterpret_cast<const uint32_t *>(vcodes[warp]);
  float sg[4];  // signs of dims lane + 32k (K and V share them)
#pragma unroll
  for (int k = 0; k < 4; k++) sg[k] = sign_of(P, lane + 32 * k);
  float bsg[5];  // butterfly signs of stages h = 1 .. 16
#pragma unroll
  for (int i = 0; i < 5; i++) bsg[i] = (lane >> i) & 1 ? -1.f : 1.f;
  const bool idx32 = items <= 0x7fffffff;  // 32-bit index arithmetic suffices
  for (int64_t it = (int64_t)blockIdx.x * kWarps + warp; it < items;
       it += (int64_t)gridDim.x * kWarps) {
    int tok, h;
    if (idx32) {
      tok = (int)it / n_kv_heads;
      h = (int)it - tok * n_kv_heads;
    } else {
      tok = (int)(it / n_kv_heads);
      h = (int)(it - (int64_t)tok * n_kv_heads);
    }
    const int64_t base = it * kHead;
    // ---- K: 64-dim blocks (4-bit RoPE dims, 3-bit others) or, compact, one
    // whole-head rotation with 3-bit codes and one scale
    float x[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const int d = lane + 32 * k;
      x[k] = __fmul_rn(load_in(key, BF16, base + d), sg[k]);
    }
#pragma unroll
    for (int i = 0; i < 5; i++)
#pragma unroll
      for (int k = 0; k < 4; k++) x[k] = xstage(x[k], bsg[i], 1 << i);
    {  // h = 32 inside each 64-block: (l, l+32), (l+64, l+96)
      float a = x[0], b = x[1];
      x[0] = __fadd_rn(a, b);
      x[1] = __fsub_rn(a, b);
      a = x[2];
      b = x[3];
      x[2] = __fadd_rn(a, b);
      x[3] = __fsub_rn(a, b);
    }
    float ks[2];
    if (P.compact) {
      float a = x[0], b = x[2];  // h = 64
      x[0] = __fadd_rn(a, b);
      x[2] = __fsub_rn(a, b);
      a = x[1];
      b = x[3];
      x[1] = __fadd_rn(a, b);
      x[3] = __fsub_rn(a, b);
#pragma unroll
      for (int k = 0; k < 4; k++) x[k] = __fmul_rn(x[k], vscale);
      int ck[4];
      ks[0] = quantize_lut<4, 3>(x, P.mult3, L, ck);
      ks[1] = 0.f;
#pragma unroll
      for (int k = 0; k < 4; k++) kcodes[warp][lane + 32 * k] = (uint8_t)ck[k];
    } else {
#pragma unroll
      for (int k = 0; k < 4; k++) x[k] = __fmul_rn(x[k], 0.125f);
#pragma unroll
      for (int kb = 0; kb < 2; kb++) {
        float xb[2] = {x[2 * kb], x[2 * kb + 1]};
        int cb[2];
        if (kb * 64 < P.rope_dim) ks[kb] = quantize_lut<2, 4>(xb, P.mult4, L, cb);
        else ks[kb] = quantize_lut<2, 3>(xb, P.mult3, L, cb);
        kcodes[warp][64 * kb + lane] = (uint8_t)cb[0];
        kcodes[warp][64 * kb + lane + 32] = (uint8_t)cb[1];
      }
    }
    // ---- V
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const int d = lane + 32 * k;
      x[k] = __fmul_rn(load_in(value, BF16, base + d), sg[k]);
    }
#pragma unroll
    for (int i = 0; i < 5; i++)
#pragma unroll
      for (int k = 0; k < 4; k++) x[k] = xstage(x[k], bsg[i], 1 << i);
    {
      float a = x[0], b = x[1];  // h = 32
      x[0] = __fadd_rn(a, b);
      x[1] = __fsub_rn(a, b);
      a = x[2];
      b = x[3];
      x[2] = __fadd_rn(a, b);
      x[3] = __fsub_rn(a, b);
      a = x[0];                  // h = 64
      b = x[2];
      x[0] = __fadd_rn(a, b);
      x[2] = __fsub_rn(a, b);
      a = x[1];
      b = x[3];
      x[1] = __fadd_rn(a, b);
      x[3] = __fsub_rn(a, b);
    }
#pragma unroll
    for (int k = 0; k < 4; k++) x[k] = __fmul_rn(x[k], vscale);
    int cv[4];
    const float vs = P.v_bits == 4 ? quantize_lut<4, 4>(x, P.mult4, L, cv)
                                   : quantize_lut<4, 3>(x, P.mult3, L, cv);
#pragma unroll
    for (int k = 0; k < 4; k++) vcodes[warp][lane + 32 * k] = (uint8_t)cv[k];
    __syncwarp();
    // ---- slot words: lane w builds word w (and w + 32) of the slot
    const int64_t sm = __ldg(slot_mapping + tok);
    uint32_t *dst = nullptr;
    if (sm >= 0) {
      int64_t blk, off;
      if (sm <= 0x7fffffff) {
        blk = (int)sm / block_size;
        off = (int)sm - (int)blk * block_size;
      } else {
        blk = sm / block_size;
        off = sm - blk * block_size;
      }
      if (blk < num_blocks)
        dst = reinterpret_cast<uint32_t *>(cache +
                                           ((blk * n_kv_heads + h) * block_size + off) * P.slot_bytes);
    }
    for (int w = lane; w < slot_words; w += 32) {
      uint32_t word = 0;
      // the 4-bit regions (K RoPE dims, 4-bit V) share one path, as do the
      // 3-bit ones, so that the warp runs each packing once
      const bool kr = w < w_kn, vr = w >= w_v && w < w_sc;
      if (kr || (vr && P.v_bits == 4)) word = pack_word(kr ? kc32 : vc32, 0, 4, kr ? w : w - w_v);
      else if (w < w_sc)
        word = vr ? pack_word(vc32, kHead, 3, w - w_v)
                  : pack_word(kc32 + P.rope_dim / 4, kHead - P.rope_dim, 3, w - w_kn);
      else if (w == w_sc)  // fp16 scales, K first then V
        word = (uint32_t)__half_as_ushort(__float2half_rn(ks[0])) |
               ((uint32_t)__half_as_ushort(__float2half_rn(P.compact ? vs : ks[1])) << 16);
      else if (w == w_sc + 1 && !P.compact)
        word = (uint32_t)__half_as_ushort(__float2half_rn(vs));
      if (dst) dst[w] = word;
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ decode
__device__ __forceinline__ uint32_t slot_byte(uint32_t myword, int p) {
  const uint32_t w = __shfl_sync(kFull, myword, p >> 2);
  return (w >> (8 * (p & 3))) & 0xFFu;
}

template <int GC, bool BF16>
__global__ void __launch_bounds__(kThreads)
    octave_decode_split_kernel(OctaveParams P, const void *__restrict__ query, int n_q_heads,
                               int group, const uint8_t *__restrict__ cache, int n_kv_heads,
                               int block_size, int64_t num_blocks,
                               const int32_t *__restrict__ block_table, int num_reqs,
                               int max_blocks, const int32_t *__restrict__ q_to_req,
                               const int32_t *__restrict__ q_to_klen, int max_klen,
                               float scale_log2, int split_tokens, int splits,
                               float *__restrict__ ws) {
  __shared__ float qs[GC][kHead];
  __shared__ float lut[2][16];
  __shared__ float red_m[kWarps][GC], red_l[kWarps][GC];
  __shared__ float red_o[kWarps][GC][kHead];
  const int s = blockIdx.x, hg = blockIdx.y, qi = blockIdx.z;
  const int h0 = hg * GC, kvh = h0 / group;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 16; i += blockDim.x) {
    lut[0][i] = i < 8 ? (float)P.lut3[i] : 0.f;
    lut[1][i] = (float)P.lut4[i];
  }
  const int req = __ldg(q_to_req + qi);
  int klen = min(max(__ldg(q_to_klen + qi), 0), min(max_klen, max_blocks * block_size));
  if (req < 0 || req >= num_reqs) klen = 0;
  const int t0 = s * split_tokens, t1 = min(klen, t0 + split_tokens);

  // query: signs, FWHT over the K rotation blocks (64 dims, or the whole
  // head for compact K), x fp32(1 / sqrt(block)), x scale*log2(e)
  const int kb_size = P.compact ? kHead : 64;
  for (int p = threadIdx.x; p < GC * kHead; p += blockDim.x) {
    const int hh = p / kHead, d = p % kHead;
    qs[hh][d] = load_in(query, BF16, ((int64_t)qi * n_q_heads + h0 + hh) * kHead + d) * sign_of(P, d);
  }
  for (int h = 1; h < kb_size; h <<= 1) {
    __syncthreads();
    for (int p = threadIdx.x; p < GC * 64; p += blockDim.x) {
      const int vv = p / 64, pi = p % 64;  // 64 pairs per head
      const int blk = pi / (kb_size / 2), pj = pi % (kb_size / 2);
      const int i0 = blk * kb_size + (pj / h) * 2 * h + (pj % h);
      const float a = qs[vv][i0], b = qs[vv][i0 + h];
      qs[vv][i0] = a + b;
      qs[vv][i0 + h] = a - b;
    }
  }
  __syncthreads();
  const float qscale = (P.compact ? 0.08838834764831845f : 0.125f) * scale_log2;
  float qr[GC][4];
#pragma unroll
  for (int hh = 0; hh < GC; hh++)
#pragma unroll
    for (int k = 0; k < 4; k++) qr[hh][k] = qs[hh][lane + 32 * k] * qscale;

  float m[GC], l[GC], o[GC][4];
#pragma unroll
  for (int hh = 0; hh < GC; hh++) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; k++) o[hh][k] = 0.f;
  }
  const int rope = P.rope_dim;
  for (int t = t0 + warp; t < t1; t += kWarps) {
    const int blk = __ldg(block_table + (int64_t)req * max_blocks + t / block_size);
    if (blk < 0 || blk >= num_blocks) continue;
    const uint8_t *sp = cache + (((int64_t)blk * n_kv_heads + kvh) * block_size + (t % block_size)) * P.slot_bytes;
    const uint32_t myword = lane < P.slot_bytes / 4 ? __ldg(reinterpret_cast<const uint32_t *>(sp) + lane) : 0u;
    // scales
    const uint32_t s01 = slot_byte(myword, P.off_scales) | (slot_byte(myword, P.off_scales + 1) << 8);
    const uint32_t s23 = slot_byte(myword, P.off_scales + 2) | (slot_byte(myword, P.off_scales + 3) << 8);
    const uint32_t s45 = slot_byte(myword, P.off_scales + 4) | (slot_byte(myword, P.off_scales + 5) << 8);
    // scales: K per 64-block then V, or (compact) one K scale then V
    const float sk0 = __half2float(__ushort_as_half((uint16_t)s01)) / kLutOne;
    const float sk1 = P.compact ? sk0 : __half2float(__ushort_as_half((uint16_t)s23)) / kLutOne;
    const float sv = __half2float(__ushort_as_half((uint16_t)(P.compact ? s23 : s45))) / kLutOne;
    float kd[4], vd[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const int d = lane + 32 * k;
      int code;
      if (d < rope) {  // 4-bit rope dims
        const uint32_t byte = slot_byte(myword, 4 * (d >> 3) + (d & 3));
        code = (byte >> (4 * ((d >> 2) & 1))) & 15;
        kd[k] = lut[1][code] * (d < 64 ? sk0 : sk1);
      } else {         // 3-bit nope dims
        const int n = d - rope;
        const uint32_t lo = slot_byte(myword, P.off_k_nope + 4 * (n >> 4) + (n & 3));
        const uint32_t hi = slot_byte(myword, P.off_k_nope + (kHead - rope) / 4 + 4 * (n >> 5) + (n & 3));
        code = ((lo >> (2 * ((n >> 2) & 3))) & 3) + 4 * ((hi >> ((n >> 2) & 7)) & 1);
        kd[k] = lut[0][code] * (d < 64 ? sk0 : sk1);
      }
      if (P.v_bits == 4) {
        const uint32_t byte = slot_byte(myword, P.off_v + 4 * (d >> 3) + (d & 3));
        vd[k] = lut[1][(byte >> (4 * ((d >> 2) & 1))) & 15] * sv;
      } else {
        const uint32_t lo = slot_byte(myword, P.off_v + 4 * (d >> 4) + (d & 3));
        const uint32_t hi = slot_byte(myword, P.off_v + kHead / 4 + 4 * (d >> 5) + (d & 3));
        vd[k] = lut[0][((lo >> (2 * ((d >> 2) & 3))) & 3) + 4 * ((hi >> ((d >> 2) & 7)) & 1)] * sv;
      }
    }
    float sc[GC];
#pragma unroll
    for (int hh = 0; hh < GC; hh++) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < 4; k++) a = fmaf(qr[hh][k], kd[k], a);
      sc[hh] = a;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int hh = 0; hh < GC; hh++) sc[hh] += __shfl_xor_sync(kFull, sc[hh], off);
#pragma unroll
    for (int hh = 0; hh < GC; hh++) {
      const float mn = fmaxf(m[hh], sc[hh]);
      const float alpha = exp2f(m[hh] - mn);
      const float p = exp2f(sc[hh] - mn);
      m[hh] = mn;
      l[hh] = l[hh] * alpha + p;
#pragma unroll
      for (int k = 0; k < 4; k++) o[hh][k] = fmaf(p, vd[k], o[hh][k] * alpha);
    }
  }
  if (lane == 0)
#pragma unroll
    for (int hh = 0; hh < GC; hh++) {
      red_m[warp][hh] = m[hh];
      red_l[warp][hh] = l[hh];
    }
#pragma unroll
  for (int hh = 0; hh < GC; hh++)
#pragma unroll
    for (int k = 0; k < 4; k++) red_o[warp][hh][lane + 32 * k] = o[hh][k];
  __syncthreads();
  for (int p = threadIdx.x; p < GC * kHead; p += blockDim.x) {
    const int hh = p / kHead, j = p % kHead;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, red_m[w][hh]);
    float Ls = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = exp2f(red_m[w][hh] - M);
        Ls += red_l[w][hh] * f;
        O += red_o[w][hh][j] * f;
      }
    }
    float *rec = ws + (((int64_t)qi * n_q_heads + h0 + hh) * splits + s) * kORec;
    rec[4 + j] = O;
    if (j == 0) {
      rec[0] = M;
      rec[1] = Ls;
    }
  }
}

__global__ void __launch_bounds__(kHead)
    octave_combine_kernel(OctaveParams P, const float *__restrict__ ws,
                          const int32_t *__restrict__ q_to_req,
                          const int32_t *__restrict__ q_to_klen, int num_reqs, int n_q_heads,
                          int splits, int max_klen, int cap, float *__restrict__ out) {
  __shared__ float ob[kHead];
  const int qh = blockIdx.x, j = threadIdx.x;
  const int qi = qh / n_q_heads;
  const int req = __ldg(q_to_req + qi);
  int klen = min(max(__ldg(q_to_klen + qi), 0), min(max_klen, cap));
  if (req < 0 || req >= num_reqs) klen = 0;
  const float *rec = ws + (int64_t)qh * splits * kORec;
  float M = -INFINITY;
  for (int s = 0; s < splits && klen > 0; s++) M = fmaxf(M, rec[s * kORec]);
  float L = 0.f, O = 0.f;
  if (klen > 0 && M != -INFINITY) {
    for (int s = 0; s < splits; s++) {
      const float ms = rec[s * kORec];
      if (ms == -INFINITY) continue;
      const float f = exp2f(ms - M);
      L += rec[s * kORec + 1] * f;
      O += rec[s * kORec + 4 + j] * f;
    }
  }
  ob[j] = L > 0.f ? O / L : 0.f;
  for (int h = 1; h < kHead; h <<= 1) {
    __syncthreads();
    if (j < 64) {
      const int i0 = (j / h) * 2 * h + (j % h);
      const float a = ob[i0], b = ob[i0 + h];
      ob[i0] = a + b;
      ob[i0 + h] = a - b;
    }
  }
  __syncthreads();
  out[(int64_t)qh * kHead + j] = ob[j] * 0.08838834764831845f * sign_of(P, j);
}

}  // namespace

cudaError_t launch_octave_quantize(const OctaveParams &p, const void *key, const void *value,
                                   int bf16, int num_tokens, int n_kv_heads,
                                   const int64_t *slot_mapping, uint8_t *cache,
                                   int block_size, int64_t num_blocks, cudaStream_t s) {
  const int64_t items = (int64_t)num_tokens * n_kv_heads;
  if (items == 0) return cudaSuccess;
  // one wave of resident CTAs, each warp striding over the (token, head) items
  static int resident[2] = {0, 0};
  int &per_sm = resident[bf16 ? 1 : 0];
  if (per_sm == 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &n, bf16 ? octave_quantize_kernel<true> : octave_quantize_kernel<false>, kThreads, 0);
    if (e != cudaSuccess) return e;
    per_sm = n > 0 ? n : 1;
  }
  const int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t wave = (int64_t)kNumSMs * per_sm;
  const int grid = (int)(blocks < wave ? blocks : wave);
  if (bf16)
    octave_quantize_kernel<true><<<grid, kThreads, 0, s>>>(p, key, value, num_tokens, n_kv_heads,
                                                          slot_mapping, cache, block_size, num_blocks);
  else
    octave_quantize_kernel<false><<<grid, kThreads, 0, s>>>(p, key, value, num_tokens, n_kv_heads,
                                                           slot_mapping, cache, block_size, num_blocks);
  return cudaGetLastError();
}

DecodePlan plan_octave_decode(int num_q, int n_head_groups, int max_klen) {
  return plan_split_k(num_q * n_head_groups, max_klen, kNumSMs * 4, 1 << 20);
}

size_t octave_workspace_bytes(int num_q, int n_q_heads, int head_size, const DecodePlan &p) {
  (void)head_size;
  return (size_t)num_q * n_q_heads * p.splits * kORec * sizeof(float);
}

cudaError_t launch_octave_decode(const OctaveParams &P, const void *query, int bf16, int num_q,
                                 int n_q_heads, const uint8_t *cache, int n_kv_heads,
                                 int block_size, int64_t num_blocks, const int32_t *block_table,
                                 int num_reqs, int max_blocks, const int32_t *q_to_req,
                                 const int32_t *q_to_klen, int max_klen, float scale,
                                 float *out, float *ws, const DecodePlan &plan, cudaStream_t s) {
  if (num_q == 0) return cudaSuccess;
  const int group = n_q_heads / n_kv_heads;
  const int gc = group < 8 ? group : 8;
  dim3 grid(plan.splits, n_q_heads / gc, num_q);
  const float sl2 = scale * kLog2e;
  if (octave_mma_supported(P)) {  // k3v4, head 128, rope 64: tensor-core split kernel
    cudaError_t e = launch_octave_decode_mma(P, query, bf16, num_q, n_q_heads, cache, n_kv_heads,
                                             block_size, num_blocks, block_table, num_reqs,
                                             max_blocks, q_to_req, q_to_klen, max_klen, scale, ws,
                                             plan, s);
    if (e != cudaSuccess) return e;
    octave_combine_kernel<<<num_q * n_q_heads, kHead, 0, s>>>(P, ws, q_to_req, q_to_klen,
                                                             num_reqs, n_q_heads, plan.splits,
                                                             max_klen, max_blocks * block_size,
                                                             out);
    return cudaGetLastError();
  }
#define KVQ_LAUNCH(G)                                                                         \
  do {                                                                                        \
    if (bf16)                                                                                 \
      octave_decode_split_kernel<G, true><<<grid, kThreads, 0, s>>>(                         \
          P, query, n_q_heads, group, cache, n_kv_heads, block_size, num_blocks, block_table, \
          num_reqs, max_blocks, q_to_req, q_to_klen, max_klen, sl2, plan.split_tokens,        \
          plan.splits, ws);                                                                   \
    else                                                                                      \
      octave_decode_split_kernel<G, false><<<grid, kThreads, 0, s>>>(                        \
          P, query, n_q_heads, group, cache, n_kv_heads, block_size, num_blocks, block_table, \
          num_reqs, max_blocks, q_to_req, q_to_klen, max_klen, sl2, plan.split_tokens,        \
          plan.splits, ws);                                                                   \
  } while (0)
  switch (gc) {
    case 1: KVQ_LAUNCH(1); break;
    case 2: KVQ_LAUNCH(2); break;
    case 4: KVQ_LAUNCH(4); break;
    default: KVQ_LAUNCH(8); break;
  }
#undef KVQ_LAUNCH
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  octave_combine_kernel<<<num_q * n_q_heads, kHead, 0, s>>>(P, ws, q_to_req, q_to_klen, num_reqs,
                                                           n_q_heads, plan.splits, max_klen,
                                                           max_blocks * block_size, out);
  return cudaGetLastError();
}

}  // namespace kvq
