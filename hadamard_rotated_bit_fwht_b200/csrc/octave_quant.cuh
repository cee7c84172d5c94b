// octave_quant.cuh -- quantize-on-append into the Octave slot cache (vLLM API
// page "vllm.v1.attention.ops.rocm_octave": reference_quantize, _quantize_lut,
// _pack, fwht_blocks, and the slot layout of the module text / OctaveFormat).
//
// One thread per (token, kv head) item, head 128.  The thread holds a vector
// in registers as pairs P[p] = (x[p], x[p + n/2]) (n = 64 for a K block, 128
// for V or a compact K), so that
//   * every FWHT stage h < n/2 is a packed f32x2 add and subtract of two pairs
//     and the last stage (h = n/2) adds and subtracts the two lanes of a pair;
//   * the fixed pairwise sums of _quantize_lut (v[i] + v[i + n/2], halving n)
//     start with the two lanes of each pair, then add pairs packed;
// both in exactly the page's operation order, so every value is bit-identical
// to the plain fp32 sequence.
//
// Codes.  _quantize_lut computes y = RN(RN(x / rms) * LUT_MULT) and counts
// the LUT midpoints strictly below it.  Every midpoint is (LUT[i] + LUT[i+1])
// / 2 of integer LUT entries, so 2 * midpoint is an integer.  The thread
// forms y2 = RN(x * RN(2 LUT_MULT / rms)), which differs from 2y by at most
// |2y| * 4 * 2^-24 <= 2^-14 for |2y| < 256 (four roundings of relative size
// <= 2^-24 against two).  When the fractional part of |y2| is farther than
// 2^-13 from 0 and 1, 2y lies strictly inside the same unit interval
// (n, n + 1), n = floor(|y2|), which holds no doubled midpoint, so the code
// and LUT value depend only on (n, sign of y): a 512-entry table per code
// width gives them (|y2| is clamped to 255.5, beyond every midpoint).  The
// other elements (about 2.4e-4 of them, and every element near zero) take the
// exact path: y by IEEE division and multiply, then the comparisons.  The
// result is the code of the exact sequence in every case.
//
// Work of a thread per item: K (two 64-dim blocks, or one 128-dim compact
// rotation), then V.  Each vector is rotated in registers, then parked in the
// thread's column of a shared-memory buffer, so that the per-element work
// runs as a short loop over groups of 8 pairs (a fully unrolled version of it
// overflowed the instruction cache); each finished 32-bit code word (bit
// packing of _pack) is stored to the slot as soon as it is complete.
#pragma once

#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace octq {

constexpr int kHead = 128;
constexpr int kThreads = 128;
constexpr float kNearEps = 1.f / 8192.f;  // 2^-13, twice the bound on |y2 - 2y|

struct QTables {
  uint2 e[2][512];        // [bits - 3][neg * 256 + floor|2y|] = {code, fp32 bits of LUT[code]}
  float lut[2][16];       // exact path: LUT values
  float mid[2][16];       // exact path: midpoints
  uint32_t sgn[kHead];    // sign flips: bf16 word j -> bits 15 / 31; fp32 dim d -> bit 31
};

__device__ __forceinline__ uint32_t bit(const OctaveParams &P, int d) {
  return (P.sign_words[d >> 5] >> (d & 31)) & 1u;
}

// Exact path for one element: y = RN(RN(x / rms) * mult), code = number of
// midpoints below y; returns {code, fp32 bits of x * LUT[code]}.  Out of line:
// it runs for about 2.4e-4 of the elements.
static __device__ __noinline__ uint2 exact_code(float x, float rms, float mult, int tb,
                                         const QTables *T) {
  const float y = __fmul_rn(__fdiv_rn(x, rms), mult);
  uint32_t c = 0;
  const int n = tb ? 15 : 7;
  for (int i = 0; i < n; i++) c += T->mid[tb][i] < y ? 1u : 0u;
  return make_uint2(c, __float_as_uint(__fmul_rn(x, T->lut[tb][c])));
}

// {code, fp32 bits of x * LUT[code]} of one element from the floor table,
// given y2 ~ 2y (see the file comment); near is set when |y2| lies within
// 2^-13 of an integer, where only the exact path decides.  No branch, so
// that the elements of a group overlap.
template <int BITS>
__device__ __forceinline__ uint2 code_fast(float x, float y2, const QTables &T, bool &near) {
  constexpr int tb = BITS - 3;
  const uint32_t yb = __float_as_uint(y2);
  const float a = fminf(__uint_as_float(yb & 0x7fffffffu), 255.5f);
  const float f = __fadd_rz(a, 8388608.f);  // 2^23 + floor(a)
  const float frac = __fsub_rn(a, __fsub_rn(f, 8388608.f));
  near = fabsf(__fsub_rn(frac, 0.5f)) > 0.5f - kNearEps;
  uint2 e = T.e[tb][(__float_as_uint(f) & 0xffu) | ((yb >> 23) & 0x100u)];
  e.y = __float_as_uint(__fmul_rn(x, __uint_as_float(e.y)));
  return e;
}

// Tree sum (v[i] + v[i + n/2], halving n) of the 2H values whose level-1
// nodes v[i] + v[i + H] are held as pairs Q[j] = (node[2j], node[2j + 1]).
template <int H>
__device__ __forceinline__ float tree_from_level1(float2 (&Q)[H / 2]) {
#pragma unroll
  for (int n = H / 2; n > 1; n >>= 1)
#pragma unroll
    for (int j = 0; j < n / 2; j++) Q[j] = add2_rn(Q[j], Q[j + n / 2]);
  return __fadd_rn(Q[0].x, Q[0].y);
}

// _quantize_lut over n = 2H values held as pairs P[p] = (x[p], x[p + H]).
// The pairs go to the thread's column of xs (xs[p * kThreads]); a loop over
// groups of 8 pairs then forms the codes, writes each finished 32-bit code
// word of the region to dst (when dst is not null), and leaves the level-1
// nodes of the dot-product tree in xs.  Region: 4-bit at slot word W, or
// 3-bit of ND dims at slot word W with this vector at dim D0 of it (the bit
// packing of _pack: 4-bit -- byte j of word w holds dims 8w + j and
// 8w + 4 + j; 3-bit -- a 2-bit plane, byte j of word w gathering dims
// 16w + 4i + j in bits 2i..2i+1, then a 1-bit plane, byte j of word w
// gathering dims 32w + 4i + j in bit i).  Returns scale * LUT_ONE in fp32.
template <int H, int BITS, int W, int ND, int D0>
__device__ __forceinline__ float quantize_pairs(float2 (&P)[H], float mult, const QTables &T,
                                                float2 *xs, uint32_t *dst) {
  float2 Q[H / 2];
#pragma unroll
  for (int j = 0; j < H / 2; j++) {
    const float2 a = mul2_rn_p0(P[2 * j], P[2 * j]);
    const float2 b = mul2_rn_p0(P[2 * j + 1], P[2 * j + 1]);
    Q[j] = make_float2(__fadd_rn(a.x, a.y), __fadd_rn(b.x, b.y));
  }
  const float ss = tree_from_level1<H>(Q);
  // ss / n with the exact power-of-two reciprocal: the same rounding
  float rms = __fsqrt_rn(__fmul_rn(ss, 1.f / (float)(2 * H)));
  rms = rms < 1e-12f ? 1e-12f : rms;
  const float c2 = __fdiv_rn(2.f * mult, rms);
#pragma unroll
  for (int p = 0; p < H; p++) xs[p * kThreads] = P[p];
  uint32_t lo_x = 0, lo_y = 0, hi_x = 0, hi_y = 0;  // 3-bit words being filled
#pragma unroll 1
  for (int g = 0; g < H / 8; g++) {
    float2 v[8];
    uint2 ex[8], ey[8];
    uint32_t near = 0;  // bit r: element 8g + r, bit 8 + r: element H + 8g + r
#pragma unroll
    for (int r = 0; r < 8; r++) {
      v[r] = xs[(8 * g + r) * kThreads];
      const float2 y2 = mul2_rn_p0(v[r], make_float2(c2, c2));
      bool nx, ny;
      ex[r] = code_fast<BITS>(v[r].x, y2.x, T, nx);
      ey[r] = code_fast<BITS>(v[r].y, y2.y, T, ny);
      near |= (nx ? 1u << r : 0u) | (ny ? 1u << (8 + r) : 0u);
    }
    if (near) {  // about 0.4% of the groups: the exact path for the flagged elements
#pragma unroll
      for (int r = 0; r < 8; r++) {
        if (near & (1u << r)) ex[r] = exact_code(v[r].x, rms, mult, BITS - 3, &T);
        if (near & (1u << (8 + r))) ey[r] = exact_code(v[r].y, rms, mult, BITS - 3, &T);
      }
    }
    uint32_t wx = 0, wy = 0;
#pragma unroll
    for (int r = 0; r < 8; r++) {
      // level-1 node of the dot tree: x[p] LUT + x[p + H] LUT
      reinterpret_cast<float *>(xs + (8 * g + r) * kThreads)[0] =
          __fadd_rn(__uint_as_float(ex[r].y), __uint_as_float(ey[r].y));
      if constexpr (BITS == 4) {
        wx |= ex[r].x << (8 * (r % 4) + 4 * (r / 4));
        wy |= ey[r].x << (8 * (r % 4) + 4 * (r / 4));
      } else {
        // dim d = D0 (+ H) + 8g + r: d % 4 = r % 4; (d % 16) / 4 = 2 (g % 2) + r / 4;
        // (d % 32) / 4 = 2 (g % 4) + r / 4
        wx |= (ex[r].x & 3u) << (8 * (r % 4) + 2 * (r / 4));
        wy |= (ey[r].x & 3u) << (8 * (r % 4) + 2 * (r / 4));
        hi_x |= (ex[r].x >> 2) << (8 * (r % 4) + r / 4 + 2 * (g % 4));
        hi_y |= (ey[r].x >> 2) << (8 * (r % 4) + r / 4 + 2 * (g % 4));
      }
    }
    if constexpr (BITS == 4) {
      if (dst) {
        dst[W + g] = wx;
        dst[W + H / 8 + g] = wy;
      }
    } else {
      lo_x |= wx << (4 * (g % 2));
      lo_y |= wy << (4 * (g % 2));
      if (g % 2 == 1) {
        if (dst) {
          dst[W + D0 / 16 + g / 2] = lo_x;
          dst[W + (D0 + H) / 16 + g / 2] = lo_y;
        }
        lo_x = lo_y = 0;
      }
      if (g % 4 == 3) {
        if (dst) {
          dst[W + ND / 16 + D0 / 32 + g / 4] = hi_x;
          dst[W + ND / 16 + (D0 + H) / 32 + g / 4] = hi_y;
        }
        hi_x = hi_y = 0;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < H / 2; j++)
    Q[j] = make_float2(reinterpret_cast<const float *>(xs + 2 * j * kThreads)[0],
                       reinterpret_cast<const float *>(xs + (2 * j + 1) * kThreads)[0]);
  const float dot = tree_from_level1<H>(Q);
  const float q = __fdiv_rn(ss, dot > 1e-30f ? dot : 1e-30f);
  return __fmul_rn(dot > 0.f ? q : 0.f, 64.f);  // LUT_ONE = 64
}

// FWHT over n = 2H values held as pairs, stages h = 1 .. H, then * scale.
template <int H>
__device__ __forceinline__ void fwht_pairs(float2 (&P)[H], float scale) {
#pragma unroll
  for (int h = 1; h < H; h <<= 1)
#pragma unroll
    for (int p = 0; p < H; p++)
      if ((p & h) == 0) {
        const float2 a = P[p], b = P[p + h];
        P[p] = add2_rn(a, b);
        P[p + h] = add2_rn(a, make_float2(-b.x, -b.y));
      }
#pragma unroll
  for (int p = 0; p < H; p++) {
    const float a = P[p].x, b = P[p].y;
    P[p] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
#pragma unroll
  for (int p = 0; p < H; p++) P[p] = mul2(P[p], make_float2(scale, scale));
}

// Load dims d0 .. d0 + 2H - 1 of a row into pairs (x[p], x[p + H]), sign flips applied.
template <bool BF16, int H>
__device__ __forceinline__ void load_pairs(const void *row, int d0, const QTables &T,
                                           float2 (&P)[H]) {
  if constexpr (BF16) {
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(row) + d0);
    uint32_t w[H];  // 2H bf16 values
#pragma unroll
    for (int i = 0; i < H / 4; i++) {
      const uint4 v = __ldg(src + i);
      w[4 * i] = v.x, w[4 * i + 1] = v.y, w[4 * i + 2] = v.z, w[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < H; j++) w[j] ^= T.sgn[d0 / 2 + j];
#pragma unroll
    for (int p = 0; p < H; p++) {
      const uint32_t lo = w[p / 2], hi = w[(p + H) / 2];
      P[p].x = (p & 1) ? __uint_as_float(lo & 0xffff0000u) : __uint_as_float(lo << 16);
      P[p].y = (p & 1) ? __uint_as_float(hi & 0xffff0000u) : __uint_as_float(hi << 16);
    }
  } else {
    const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(row) + d0);
#pragma unroll
    for (int i = 0; i < H / 4; i++) {
      const float4 a = __ldg(src + i), b = __ldg(src + H / 4 + i);
      const float xa[4] = {a.x, a.y, a.z, a.w}, xb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const int p = 4 * i + k;
        P[p].x = __uint_as_float(__float_as_uint(xa[k]) ^ T.sgn[d0 + p]);
        P[p].y = __uint_as_float(__float_as_uint(xb[k]) ^ T.sgn[d0 + p + H]);
      }
    }
  }
}

// K block KB (dims 64 KB .. 64 KB + 63): signs, FWHT-64, x 1/8, then 4-bit
// codes for the RB RoPE blocks, 3-bit codes (NoPE region after them) else.
template <bool BF16, int KB, int RB>
__device__ __forceinline__ float k_block(const void *krow, const OctaveParams &P,
                                         const QTables &T, float2 *xs, uint32_t *dst) {
  float2 X[32];
  load_pairs<BF16, 32>(krow, 64 * KB, T, X);
  fwht_pairs<32>(X, 0.125f);
  if constexpr (KB < RB) return quantize_pairs<32, 4, 8 * KB, 0, 0>(X, P.mult4, T, xs, dst);
  else return quantize_pairs<32, 3, 8 * RB, 64 * (2 - RB), 64 * (KB - RB)>(X, P.mult3, T, xs, dst);
}

// RB: K blocks with 4-bit codes (rope_dim / 64; unused when COMPACT)
template <bool BF16, bool COMPACT, int VBITS, int RB>
__global__ void __launch_bounds__(kThreads, 3)
    octave_quant_kernel(const __grid_constant__ OctaveParams P, const void *__restrict__ key,
                        const void *__restrict__ value, int64_t items, int n_kv_heads,
                        const int64_t *__restrict__ slot_mapping, uint8_t *__restrict__ cache,
                        int block_size, int64_t num_blocks, uint32_t *__restrict__ err) {
  __shared__ QTables T;
  extern __shared__ float2 xs_all[];  // [64 pairs][kThreads]
  for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
    const int tb = t >> 9, neg = (t >> 8) & 1, n = t & 255, L = tb ? 16 : 8;
    const int8_t *lut = tb ? P.lut4 : P.lut3;
    // any y2 with |y2| in (n, n + 1) and this sign: compare with doubled midpoints
    const float y2 = neg ? -(n + 0.5f) : (n + 0.5f);
    uint32_t c = 0;
    for (int i = 0; i < L - 1; i++) c += (float)(lut[i] + lut[i + 1]) < y2 ? 1u : 0u;
    T.e[tb][t & 511] = make_uint2(c, __float_as_uint((float)lut[c]));
  }
  for (int t = threadIdx.x; t < 32; t += blockDim.x) {
    const int tb = t >> 4, i = t & 15, L = tb ? 16 : 8;
    const int8_t *lut = tb ? P.lut4 : P.lut3;
    T.lut[tb][i] = i < L ? (float)lut[i] : 0.f;
    T.mid[tb][i] = i < L - 1 ? ((float)lut[i + 1] + (float)lut[i]) / 2.0f : 0.f;
  }
  for (int d = threadIdx.x; d < kHead; d += blockDim.x)
    T.sgn[d] = BF16 ? (d < kHead / 2 ? (bit(P, 2 * d) << 15) | (bit(P, 2 * d + 1) << 31) : 0u)
                    : bit(P, d) << 31;
  __syncthreads();

  constexpr int kKWords = COMPACT ? 12 : 8 * RB + 6 * (2 - RB);  // K code words
  constexpr int kVWords = VBITS == 4 ? 16 : 12;
  constexpr int kSc = kKWords + kVWords;                        // first scale word
  constexpr int kSlotBytes = COMPACT ? 4 * (kSc + 1) : 4 * (kSc + 2);
  const float vscale = 0.08838834764831845f;  // fp32(1 / sqrt(128))
  float2 *xs = xs_all + threadIdx.x;

  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items; it += stride) {
    const int tok = (int)(it / n_kv_heads);
    const int h = (int)(it - (int64_t)tok * n_kv_heads);
    const int64_t sm = __ldg(slot_mapping + tok);
    uint32_t *dst = nullptr;  // the slot, or null for a skipped token
    if (sm >= 0) {
      const int64_t blk = sm / block_size, off = sm - blk * block_size;
      const int64_t si = (blk * n_kv_heads + h) * block_size + off;
      if (blk < num_blocks && in_bounds(si, si + 1, num_blocks * n_kv_heads * block_size, err))
        dst = reinterpret_cast<uint32_t *>(cache + si * (int64_t)kSlotBytes);
    }
    const void *krow = static_cast<const char *>(key) + it * kHead * (BF16 ? 2 : 4);
    const void *vrow = static_cast<const char *>(value) + it * kHead * (BF16 ? 2 : 4);
    float ks0, ks1 = 0.f;
    if constexpr (COMPACT) {
      float2 X[64];
      load_pairs<BF16, 64>(krow, 0, T, X);
      fwht_pairs<64>(X, vscale);
      ks0 = quantize_pairs<64, 3, 0, kHead, 0>(X, P.mult3, T, xs, dst);
    } else {
      ks0 = k_block<BF16, 0, RB>(krow, P, T, xs, dst);
      ks1 = k_block<BF16, 1, RB>(krow, P, T, xs, dst);
    }
    float vs;
    {
      float2 X[64];
      load_pairs<BF16, 64>(vrow, 0, T, X);
      fwht_pairs<64>(X, vscale);
      if constexpr (VBITS == 4) vs = quantize_pairs<64, 4, kKWords, 0, 0>(X, P.mult4, T, xs, dst);
      else vs = quantize_pairs<64, 3, kKWords, kHead, 0>(X, P.mult3, T, xs, dst);
    }
    // fp16 scales, K first then V, little-endian; the pad bytes are zero
    if (dst) {
      const uint32_t hk0 = __half_as_ushort(__float2half_rn(ks0));
      const uint32_t hv = __half_as_ushort(__float2half_rn(vs));
      if constexpr (COMPACT) {
        dst[kSc] = hk0 | hv << 16;
      } else {
        dst[kSc] = hk0 | (uint32_t)__half_as_ushort(__float2half_rn(ks1)) << 16;
        dst[kSc + 1] = hv;
      }
    }
  }
}

constexpr int kXsBytes = 64 * kThreads * (int)sizeof(float2);

template <bool BF16, bool COMPACT, int VBITS, int RB>
cudaError_t launch_one(const OctaveParams &p, const void *key, const void *value, int64_t items,
                       int n_kv_heads, const int64_t *slot_mapping, uint8_t *cache,
                       int block_size, int64_t num_blocks, cudaStream_t s) {
  // one wave of resident CTAs; every thread strides over the items
  static std::mutex mu;
  static int resident = 0;
  static unsigned configured = 0u;  // devices with the shared-memory carve-out set
  auto kern = octave_quant_kernel<BF16, COMPACT, VBITS, RB>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!(configured & (1u << (dev & 31)))) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kXsBytes);
      if (e != cudaSuccess) return e;
      configured |= 1u << (dev & 31);
    }
    if (resident == 0) {
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, kXsBytes);
      if (e != cudaSuccess) return e;
      resident = n > 0 ? n : 1;
    }
  }
  const int64_t blocks = (items + kThreads - 1) / kThreads;
  const int64_t wave = (int64_t)kNumSMs * resident;
  const int grid = (int)(blocks < wave ? blocks : wave);
  kern<<<grid, kThreads, kXsBytes, s>>>(p, key, value, items, n_kv_heads, slot_mapping, cache,
                                        block_size, num_blocks, device_error_word());
  return cudaGetLastError();
}

}  // namespace octq

// launchers of the format instances, one translation unit per (input type,
// V code width) so that they compile in parallel
#define KVQ_OCTQ_DECL(NAME) \
  cudaError_t NAME(const OctaveParams &p, const void *key, const void *value, int64_t items, \
                   int n_kv_heads, const int64_t *slot_mapping, uint8_t *cache, int block_size, \
                   int64_t num_blocks, cudaStream_t s)
KVQ_OCTQ_DECL(octave_quant_bf16_v4);
KVQ_OCTQ_DECL(octave_quant_bf16_v3);
KVQ_OCTQ_DECL(octave_quant_f32_v4);
KVQ_OCTQ_DECL(octave_quant_f32_v3);

}  // namespace kvq
