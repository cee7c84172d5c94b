// octave_quant.cuh -- quantize-on-append into the Octave slot cache (vLLM API
// page "vllm.v1.attention.ops.rocm_octave": reference_quantize, _quantize_lut,
// _pack, fwht_blocks, and the slot layout of the module text / OctaveFormat).
//
// Eight threads per (token, kv head) item, head 128.  A vector of n = 16 T
// values (T = 8 threads for V or a compact K, T = 4 threads per 64-dim K
// block, the two K blocks side by side in one octet) is held 16 values per
// thread in two layouts:
//   * contiguous: thread t holds elements 16 t + m (m = 0..15), the row as
//     loaded; the FWHT stages h = 1, 2, 4, 8 pair elements of one thread;
//   * strided: thread t holds elements t + T k (k = 0..15), reached through
//     one shared-memory transpose; the stages h = 16 .. n/2 pair k with
//     k ^ (h / T), again inside a thread.
// The fixed pairwise sums of _quantize_lut (v[i] + v[i + n/2], halving n)
// pair k with k + 8, 4, 2, 1 inside a thread, then threads t ^ T/2 .. t ^ 1
// by shuffles.  Every butterfly and every sum takes the page's operands in
// the page's order (a sum a + b computed by the partner as b + a is the same
// rounded value), so every value is bit-identical to the plain fp32 sequence.
//
// Codes.  _quantize_lut computes y = RN(RN(x / rms) * LUT_MULT) and counts
// the LUT midpoints strictly below it.  Every midpoint is (LUT[i] + LUT[i+1])
// / 2 of integer LUT entries, so 2 * midpoint is an integer.  A thread forms
// y2 = RN(x * RN(2 LUT_MULT / rms)), which differs from 2y by at most
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
// Packing.  The codes go to a 128-byte shared row in element order; each
// thread then builds whole 32-bit words of _pack's bit layout from it and
// stores them to the slot, so an octet writes its slot in a few coalesced
// rounds.  Per item: K (two 64-dim blocks, or one 128-dim compact rotation),
// then V, then the fp16 scales.
#pragma once

#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace octq {

constexpr int kHead = 128;
constexpr int kThreads = 128;
constexpr int kOct = kThreads / 8;        // items in flight per CTA
constexpr int kXb = 168;                  // floats per octet transpose row (8 x 20, + 8)
constexpr float kNearEps = 1.f / 8192.f;  // 2^-13, twice the bound on |y2 - 2y|
constexpr unsigned kFull = 0xffffffffu;

struct QTables {
  // [bits - 3][neg * 256 + floor|2y|]: fp32 bits of LUT[code] with the code
  // in the low byte (an int8 LUT value leaves the low 16 bits of its fp32 zero)
  uint32_t e[2][512];
  float lut[2][16];  // exact path: LUT values
  float mid[2][16];  // exact path: midpoints
};

struct Smem {
  QTables T;
  float xb[kOct][kXb];     // transpose rows: element 16 q + m of thread q at 20 q + m
  uint32_t cb[kOct][34];   // code bytes in element order (rows 34 words apart: the
                           // byte stores of the four octets of a warp meet no bank twice)
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

// {code, fp32 bits of x * LUT[code]} of one element from the floor table of
// code width tb + 3, given y2 ~ 2y (see the file comment); near is set when
// |y2| lies within 2^-13 of an integer, where only the exact path decides.
__device__ __forceinline__ bool near_int(float a, float f) {  // a = min(|y2|, 255.5)
  const float frac = __fsub_rn(a, __fsub_rn(f, 8388608.f));
  return fabsf(__fsub_rn(frac, 0.5f)) > 0.5f - kNearEps;
}
// The same for two elements at once, the floating-point steps as packed
// fp32x2 operations (each lane rounds as the scalar form): table words (the
// code in the low byte) in w0, w1, the products x * LUT[code] in prod (a zero
// product comes out +0, which no sum or scale below can tell from -0), and
// near when either element is near an integer.
__device__ __forceinline__ void code_fast2(float2 x, float2 y2, const uint32_t *tab, uint32_t &w0,
                                          uint32_t &w1, float2 &prod, bool &near) {
  const uint32_t b0 = __float_as_uint(y2.x), b1 = __float_as_uint(y2.y);
  const float2 a = make_float2(fminf(__uint_as_float(b0 & 0x7fffffffu), 255.5f),
                               fminf(__uint_as_float(b1 & 0x7fffffffu), 255.5f));
  const float2 f = add2_rz(a, make_float2(8388608.f, 8388608.f));  // 2^23 + floor(a)
  const float2 fl = add2_rn(f, make_float2(-8388608.f, -8388608.f));
  const float2 frac = add2_rn(a, make_float2(-fl.x, -fl.y));
  const float2 g = add2_rn(frac, make_float2(-0.5f, -0.5f));
  near = fabsf(g.x) > 0.5f - kNearEps || fabsf(g.y) > 0.5f - kNearEps;
  w0 = tab[(__float_as_uint(f.x) & 0xffu) | ((b0 >> 23) & 0x100u)];
  w1 = tab[(__float_as_uint(f.y) & 0xffu) | ((b1 >> 23) & 0x100u)];
  prod = mul2_rn_p0(x, make_float2(__uint_as_float(w0 & 0xffffff00u),
                                   __uint_as_float(w1 & 0xffffff00u)));
}

// One vector of n = 16 T values over T threads (t = this thread's index in
// its group, x = its 16 contiguous elements 16 t .. 16 t + 15, sign flips
// applied): FWHT (stages h = 1 .. n/2, then * scale), _quantize_lut with code
// width 3 + tb, codes to cb (element order, bytes), returns scale * LUT_ONE.
// xr: the group's transpose row; cbb: the group's code bytes.
template <int T>
__device__ __forceinline__ float quantize_vec(float (&x)[16], int t, float scale, float mult,
                                              int tb, const QTables &Q, float *xr,
                                              uint8_t *cbb) {
  constexpr int N = 16 * T;
  // stages h = 1, 2, 4, 8 on the contiguous elements
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int m = 0; m < 16; m++)
      if ((m & h) == 0) {
        const float a = x[m], b = x[m + h];
        x[m] = __fadd_rn(a, b);
        x[m + h] = __fsub_rn(a, b);
      }
  // to the strided layout: element 16 u + m at 20 u + m (u = the holding thread)
#pragma unroll
  for (int m = 0; m < 16; m += 4)
    *reinterpret_cast<float4 *>(xr + 20 * t + m) = make_float4(x[m], x[m + 1], x[m + 2], x[m + 3]);
  __syncwarp();
  float y[16];
#pragma unroll
  for (int k = 0; k < 16; k++) {
    const int e = t + T * k;
    y[k] = xr[20 * (e >> 4) + (e & 15)];
  }
  __syncwarp();  // the row is free again
  // stages h = 16 .. n/2: element t + T k pairs k with k + h / T
#pragma unroll
  for (int kk = 16 / T; kk < 16; kk <<= 1)
#pragma unroll
    for (int k = 0; k < 16; k++)
      if ((k & kk) == 0) {
        const float a = y[k], b = y[k + kk];
        y[k] = __fadd_rn(a, b);
        y[k + kk] = __fsub_rn(a, b);
      }
#pragma unroll
  for (int k = 0; k < 16; k++) y[k] = __fmul_rn(y[k], scale);

  // tree sum of v[i] (i = t + T k): k + 8, 4, 2, 1 in the thread, then t ^ T/2 .. t ^ 1
  auto tree = [&](float (&v)[16]) {
#pragma unroll
    for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
      for (int k = 0; k < n; k++) v[k] = __fadd_rn(v[k], v[k + n]);
    float s = v[0];
#pragma unroll
    for (int o = T / 2; o >= 1; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, o));
    return s;
  };
  float v[16];
#pragma unroll
  for (int k = 0; k < 16; k++) v[k] = __fmul_rn(y[k], y[k]);
  const float ss = tree(v);
  // ss / n with the exact power-of-two reciprocal: the same rounding
  float rms = __fsqrt_rn(__fmul_rn(ss, 1.f / (float)N));
  rms = rms < 1e-12f ? 1e-12f : rms;
  const float c2 = __fdiv_rn(2.f * mult, rms);
  const uint32_t *tab = Q.e[tb];
  bool any_near = false;
#pragma unroll
  for (int k = 0; k < 8; k++) {  // elements k and k + 8
    bool nk;
    uint32_t w0, w1;
    float2 pr;
    const float2 yy = make_float2(y[k], y[k + 8]);
    code_fast2(yy, mul2_rn_p0(yy, make_float2(c2, c2)), tab, w0, w1, pr, nk);
    cbb[t + T * k] = (uint8_t)w0;
    cbb[t + T * (k + 8)] = (uint8_t)w1;
    v[k] = pr.x;
    v[k + 8] = pr.y;
    any_near = any_near || nk;
  }
  if (any_near) {
    // the exact path for the flagged elements (the flags recomputed here, off
    // the common path), as a rolled loop over this thread's segment of the
    // (free) transpose row, so that y and v stay in registers: y in, x *
    // LUT[code] back
    float *seg = xr + 20 * t;
    uint32_t near = 0;
#pragma unroll
    for (int k = 0; k < 16; k++) {
      const float a = fminf(fabsf(__fmul_rn(y[k], c2)), 255.5f);
      if (near_int(a, __fadd_rz(a, 8388608.f))) {
        near |= 1u << k;
        seg[k] = y[k];
      }
    }
#pragma unroll 1
    for (int k = 0; k < 16; k++)
      if (near & (1u << k)) {
        const uint2 e = exact_code(seg[k], rms, mult, tb, &Q);
        cbb[t + T * k] = (uint8_t)e.x;
        seg[k] = __uint_as_float(e.y);
      }
#pragma unroll
    for (int k = 0; k < 16; k++)
      if (near & (1u << k)) v[k] = seg[k];
  }
  const float dot = tree(v);
  const float q = __fdiv_rn(ss, dot > 1e-30f ? dot : 1e-30f);
  return __fmul_rn(dot > 0.f ? q : 0.f, 64.f);  // LUT_ONE = 64
}

// _pack of n = 16 T codes (bytes in element order at cbb) by the T threads of
// a group: 4-bit at slot word W (byte j of word w = dims 8w + j | 8w + 4 + j
// << 4), or 3-bit into a region of ND dims at word W with this vector at dim
// D0 (a 2-bit plane, byte j of word w gathering dims 16w + 4i + j in bits
// 2i..2i+1, then a 1-bit plane, byte j of word w gathering dims 32w + 4i + j
// in bit i).
template <int T>
__device__ __forceinline__ void pack_4(const uint8_t *cbb, int t, int W, uint32_t *dst) {
  const uint32_t *c = reinterpret_cast<const uint32_t *>(cbb);
#pragma unroll
  for (int r = 0; r < 2; r++) {
    const int w = t + T * r;
    dst[W + w] = c[2 * w] | c[2 * w + 1] << 4;
  }
}
template <int T>
__device__ __forceinline__ void pack_3(const uint8_t *cbb, int t, int W, int ND, int D0,
                                       uint32_t *dst) {
  const uint32_t *c = reinterpret_cast<const uint32_t *>(cbb);
  {  // 2-bit plane: T words, one per thread
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) w |= (c[4 * t + i] & 0x03030303u) << (2 * i);
    dst[W + D0 / 16 + t] = w;
  }
  if (t < T / 2) {  // 1-bit plane: T / 2 words
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) w |= ((c[8 * t + i] >> 2) & 0x01010101u) << i;
    dst[W + ND / 16 + D0 / 32 + t] = w;
  }
}

// this thread's 16 contiguous dims 16 q .. 16 q + 15 of a row: fetched raw
// (so that the load of the next vector overlaps the work on this one), then
// widened with the sign flips applied (sm: for bf16 the XOR masks of the 8
// words, bits 15 and 31; for fp32 bit m of sm[0] is the sign of dim 16 q + m)
template <bool BF16>
struct Raw16 {
  uint4 w[BF16 ? 2 : 4];
};
template <bool BF16>
__device__ __forceinline__ void fetch16(const void *row, int q, bool valid, Raw16<BF16> &r) {
  const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const char *>(row) +
                                                     16 * q * (BF16 ? 2 : 4));
#pragma unroll
  for (int j = 0; j < (BF16 ? 2 : 4); j++)
    r.w[j] = valid ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
}
template <bool BF16>
__device__ __forceinline__ void unpack16(const Raw16<BF16> &r, const uint32_t (&sm)[8],
                                         float (&x)[16]) {
  if constexpr (BF16) {
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint4 u = r.w[j / 4];
      const uint32_t w = (j % 4 == 0 ? u.x : j % 4 == 1 ? u.y : j % 4 == 2 ? u.z : u.w) ^ sm[j];
      x[2 * j] = __uint_as_float(w << 16);
      x[2 * j + 1] = __uint_as_float(w & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const uint32_t f[4] = {r.w[j].x, r.w[j].y, r.w[j].z, r.w[j].w};
#pragma unroll
      for (int i = 0; i < 4; i++)
        x[4 * j + i] = __uint_as_float(f[i] ^ (((sm[0] >> (4 * j + i)) & 1u) << 31));
    }
  }
}

// RB: K blocks with 4-bit codes (rope_dim / 64; unused when COMPACT)
template <bool BF16, bool COMPACT, int VBITS, int RB>
__global__ void __launch_bounds__(kThreads)
    octave_quant_kernel(const __grid_constant__ OctaveParams P, const void *__restrict__ key,
                        const void *__restrict__ value, int64_t items, int n_kv_heads,
                        const int64_t *__restrict__ slot_mapping, uint8_t *__restrict__ cache,
                        int block_size, int64_t num_blocks, uint32_t *__restrict__ err) {
  __shared__ Smem S;
  for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
    const int tb = t >> 9, neg = (t >> 8) & 1, n = t & 255, L = tb ? 16 : 8;
    const int8_t *lut = tb ? P.lut4 : P.lut3;
    // any y2 with |y2| in (n, n + 1) and this sign: compare with doubled midpoints
    const float y2 = neg ? -(n + 0.5f) : (n + 0.5f);
    uint32_t c = 0;
    for (int i = 0; i < L - 1; i++) c += (float)(lut[i] + lut[i + 1]) < y2 ? 1u : 0u;
    S.T.e[tb][t & 511] = __float_as_uint((float)lut[c]) | c;
  }
  for (int t = threadIdx.x; t < 32; t += blockDim.x) {
    const int tb = t >> 4, i = t & 15, L = tb ? 16 : 8;
    const int8_t *lut = tb ? P.lut4 : P.lut3;
    S.T.lut[tb][i] = i < L ? (float)lut[i] : 0.f;
    S.T.mid[tb][i] = i < L - 1 ? ((float)lut[i + 1] + (float)lut[i]) / 2.0f : 0.f;
  }
  __syncthreads();

  constexpr int kKWords = COMPACT ? 12 : 8 * RB + 6 * (2 - RB);  // K code words
  constexpr int kVWords = VBITS == 4 ? 16 : 12;
  constexpr int kSc = kKWords + kVWords;                        // first scale word
  constexpr int kSlotBytes = COMPACT ? 4 * (kSc + 1) : 4 * (kSc + 2);
  const float vscale = 0.08838834764831845f;  // fp32(1 / sqrt(128))
  const int lane = threadIdx.x & 31, q = lane & 7;
  const int o = threadIdx.x >> 3;  // octet of the CTA
  float *xr = S.xb[o];
  uint8_t *cbb = reinterpret_cast<uint8_t *>(S.cb[o]);
  // sign bits of dims 16 q .. 16 q + 15, as XOR masks
  const uint32_t sg = (P.sign_words[q >> 1] >> (16 * (q & 1))) & 0xffffu;
  uint32_t sm[8];
#pragma unroll
  for (int j = 0; j < 8; j++)
    sm[j] = BF16 ? (((sg >> (2 * j)) & 1u) << 15) | (((sg >> (2 * j + 1)) & 1u) << 31)
                 : (j == 0 ? sg : 0u);

  // whole warps step through the items together (the shuffles), four octets each
  const int64_t wbase0 = ((int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31)) / 8;
  const int64_t wstride = (int64_t)gridDim.x * kOct;
  auto row_of = [&](const void *base, int64_t item) {
    return static_cast<const char *>(base) + item * kHead * (BF16 ? 2 : 4);
  };
  Raw16<BF16> kraw, vraw;
  {
    const int64_t it0 = wbase0 + (lane >> 3);
    fetch16<BF16>(row_of(key, it0 < items ? it0 : 0), q, it0 < items, kraw);
  }
  for (int64_t wb = wbase0; wb < items; wb += wstride) {
    const int64_t it = wb + (lane >> 3);
    const bool valid = it < items;
    fetch16<BF16>(row_of(value, valid ? it : 0), q, valid, vraw);
    uint32_t *dst = nullptr;  // the slot, or null for a skipped token
    if (valid) {
      const int tok = (int)(it / n_kv_heads);
      const int h = (int)(it - (int64_t)tok * n_kv_heads);
      const int64_t sm_ = __ldg(slot_mapping + tok);
      if (sm_ >= 0) {
        const int64_t blk = sm_ / block_size, off = sm_ - blk * block_size;
        const int64_t si = (blk * n_kv_heads + h) * block_size + off;
        if (blk < num_blocks && in_bounds(si, si + 1, num_blocks * n_kv_heads * block_size, err))
          dst = reinterpret_cast<uint32_t *>(cache + si * (int64_t)kSlotBytes);
      }
    }
    float x[16];
    float ks0, ks1 = 0.f;
    unpack16<BF16>(kraw, sm, x);
    if constexpr (COMPACT) {
      ks0 = quantize_vec<8>(x, q, vscale, P.mult3, 0, S.T, xr, cbb);
      __syncwarp();
      if (dst) pack_3<8>(cbb, q, 0, kHead, 0, dst);
    } else {
      // K block b = q / 4 on threads 4 b .. 4 b + 3: 4-bit if b < RB, else 3-bit
      const int b = q >> 2, t = q & 3;
      const bool four = b < RB;
      const float ks = quantize_vec<4>(x, t, 0.125f, four ? P.mult4 : P.mult3, four ? 1 : 0,
                                       S.T, xr + 80 * b, cbb + 64 * b);
      __syncwarp();
      if (dst) {
        if (four) pack_4<4>(cbb + 64 * b, t, 8 * b, dst);
        else pack_3<4>(cbb + 64 * b, t, 8 * RB, 64 * (2 - RB), 64 * (b - RB), dst);
      }
      ks0 = __shfl_sync(kFull, ks, lane & ~7);
      ks1 = __shfl_sync(kFull, ks, (lane & ~7) | 4);
    }
    __syncwarp();  // the code row is free again
    {  // the next item's K row, while this one's V is worked on
      const int64_t itn = it + wstride;
      fetch16<BF16>(row_of(key, itn < items ? itn : 0), q, itn < items, kraw);
    }
    float vs;
    unpack16<BF16>(vraw, sm, x);
    vs = quantize_vec<8>(x, q, vscale, VBITS == 4 ? P.mult4 : P.mult3, VBITS == 4 ? 1 : 0, S.T,
                         xr, cbb);
    __syncwarp();
    if (dst) {
      if constexpr (VBITS == 4) pack_4<8>(cbb, q, kKWords, dst);
      else pack_3<8>(cbb, q, kKWords, kHead, 0, dst);
      // fp16 scales, K first then V, little-endian; the pad bytes are zero
      if (q == 0) {
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
    __syncwarp();  // the code row is free again
  }
}

template <bool BF16, bool COMPACT, int VBITS, int RB>
cudaError_t launch_one(const OctaveParams &p, const void *key, const void *value, int64_t items,
                       int n_kv_heads, const int64_t *slot_mapping, uint8_t *cache,
                       int block_size, int64_t num_blocks, cudaStream_t s) {
  // one wave of resident CTAs; every octet strides over the items
  static std::mutex mu;
  static int resident = 0;
  auto kern = octave_quant_kernel<BF16, COMPACT, VBITS, RB>;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (resident == 0) {
      int n = 0;
      cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, 0);
      if (e != cudaSuccess) return e;
      resident = n > 0 ? n : 1;
    }
  }
  const int64_t blocks = (items + kOct - 1) / kOct;
  const int64_t wave = (int64_t)kNumSMs * resident;
  const int grid = (int)(blocks < wave ? blocks : wave);
  kern<<<grid, kThreads, 0, s>>>(p, key, value, items, n_kv_heads, slot_mapping, cache,
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
