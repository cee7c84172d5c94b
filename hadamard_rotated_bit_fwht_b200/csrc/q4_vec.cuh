// q4_vec.cuh -- warp-level FWHT-256 + Q4_0 quantization of head vectors,
// shared by the append kernel (q4_quant.cu) and the fused decode step
// (q4_decode_mma.cu).  Nothing here is part of the C ABI.
//
// Method: Strata PR #21 "Q4_0 KV cache + FWHT-256", How 1 (orthonormal
// Walsh-Hadamard transform of each D = 256 head vector, scale 1/16) and How 2
// (Q4_0 blocks: 32 values, one fp16 scale, 16 bytes of nibbles), with the
// maintainer's deterministic tie-break a > amax || (a == amax && v > mval).
// Stage order and end scaling: vLLM rocm_octave page, fwht_blocks.
//
// Work decomposition (one warp = 4 vectors, 8 lanes per vector, 32 values
// per lane; no shared-memory barrier, only __syncwarp):
//   L0 (after the load): lane i holds x[u + 8i + 64j] in r[u + 8j] -- each
//       lane reads four 16-byte chunks, so a warp instruction reads 512
//       contiguous bytes of bf16 input.  Stages h = 1, 2, 4 run in registers.
//   One register transpose through 1 KB of shared memory per vector
//   (128-bit stores and loads, XOR swizzle, no bank conflicts) gives
//   L1: lane i holds x[i + 8u + 64j] in r[u + 8j]; stages h = 8 ... 128 run in
//       registers.  The two halves of each packed fp32x2 operation are
//       r[k] and r[k + 16], so every stage but h = 128 uses add/sub.f32x2.
//   Quantization in L1: a 32-value block is (8 lanes) x (4 registers); its
//   max-abs key is reduced with three xor-shuffles; lane i computes the scale
//   of block i and broadcasts 1/d; codes are formed with the fp32 magic
//   number 2^23 (round-toward-zero add) instead of a float-to-int conversion;
//   the 16 nibble bytes of block i are regrouped through shared memory so
//   each lane stores one 16-byte chunk.
// Every fp32 operation is the IEEE round-to-nearest operation of the stated
// sequence (explicit-rounding PTX for the packed butterflies, scalar _rn
// intrinsics where a product is followed by a sum), so codes and scales are
// bit-identical to that sequence.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {
namespace q4v {

constexpr unsigned kVFull = 0xffffffffu;

// ------------------------------------------------------------------ load (L0)
// 16-byte chunks per lane: bf16 -> 4 chunks (8 values each), fp32 -> 8 chunks.
template <bool BF16>
struct Raw {
  uint4 w[BF16 ? 4 : 8];
};

template <bool BF16>
__device__ __forceinline__ void fetch_raw(const void *vec, int i, bool valid, Raw<BF16> &raw) {
  if (!valid) {
#pragma unroll
    for (int j = 0; j < (BF16 ? 4 : 8); j++) raw.w[j] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  if (BF16) {
    const uint16_t *p = static_cast<const uint16_t *>(vec);
#pragma unroll
    for (int j = 0; j < 4; j++) raw.w[j] = ldg_stream_u4(p + 8 * (i + 8 * j));
  } else {
    const float *p = static_cast<const float *>(vec);
#pragma unroll
    for (int j = 0; j < 4; j++) {
      raw.w[2 * j] = ldg_stream_u4(p + 8 * (i + 8 * j));
      raw.w[2 * j + 1] = ldg_stream_u4(p + 8 * (i + 8 * j) + 4);
    }
  }
}

// L0: lane i holds x[u + 8i + 64j] in r[u + 8j]
template <bool BF16>
__device__ __forceinline__ void unpack_l0(const Raw<BF16> &raw, float r[32]) {
#pragma unroll
  for (int j = 0; j < 4; j++) {
    if (BF16) {
      const uint4 w = raw.w[j];
      r[8 * j + 0] = bf16lo(w.x);
      r[8 * j + 1] = bf16hi(w.x);
      r[8 * j + 2] = bf16lo(w.y);
      r[8 * j + 3] = bf16hi(w.y);
      r[8 * j + 4] = bf16lo(w.z);
      r[8 * j + 5] = bf16hi(w.z);
      r[8 * j + 6] = bf16lo(w.w);
      r[8 * j + 7] = bf16hi(w.w);
    } else {
      const uint4 a = raw.w[2 * j], b = raw.w[2 * j + 1];
      r[8 * j + 0] = __uint_as_float(a.x);
      r[8 * j + 1] = __uint_as_float(a.y);
      r[8 * j + 2] = __uint_as_float(a.z);
      r[8 * j + 3] = __uint_as_float(a.w);
      r[8 * j + 4] = __uint_as_float(b.x);
      r[8 * j + 5] = __uint_as_float(b.y);
      r[8 * j + 6] = __uint_as_float(b.z);
      r[8 * j + 7] = __uint_as_float(b.w);
    }
  }
}

// Butterfly on register-index bit M (M in {1,2,4,8}): pairs (k, k+M) become
// (a+b, a-b); r[k] and r[k+16] travel together in one fp32x2 operation.
template <int M>
__device__ __forceinline__ void bfly_packed(float r[32]) {
#pragma unroll
  for (int k = 0; k < 16; k++) {
    if (k & M) continue;
    float2 a = make_float2(r[k], r[k + 16]);
    float2 b = make_float2(r[k + M], r[k + M + 16]);
    float2 s = add2(a, b), d = sub2(a, b);
    r[k] = s.x;
    r[k + 16] = s.y;
    r[k + M] = d.x;
    r[k + M + 16] = d.y;
  }
}

// Butterfly on register-index bit 16 (the packed pair itself): scalar.
__device__ __forceinline__ void bfly16(float r[32]) {
#pragma unroll
  for (int k = 0; k < 16; k++) {
    float a = r[k], b = r[k + 16];
    r[k] = __fadd_rn(a, b);
    r[k + 16] = __fsub_rn(a, b);
  }
}

// L0 -> L1 through shared memory.  Slot of element e (low 6 bits): float4 at
// index ((e & 7) ^ ((e >> 3) & 7)) + 8 * ((e >> 3) & 7), holding e + 64j for
// j = 0..3.  Both the stores (L0) and the loads (L1) of 8 lanes of a vector
// touch 8 distinct bank quads.
__device__ __forceinline__ void transpose_l0_l1(float r[32], float4 *buf, int i) {
#pragma unroll
  for (int u = 0; u < 8; u++)
    buf[(u ^ i) + 8 * i] = make_float4(r[u], r[u + 8], r[u + 16], r[u + 24]);
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 8; u++) {
    float4 w = buf[(i ^ u) + 8 * u];
    r[u] = w.x;
    r[u + 8] = w.y;
    r[u + 16] = w.z;
    r[u + 24] = w.w;
  }
  __syncwarp();
}

// Full FWHT-256 of the 4 vectors of this warp from layout L0: stages,
// transpose, stages, end scaling.  Leaves layout L1.
// SCALE = false leaves the stages' output unscaled (16x the rotation); the
// quantizer folds the 1/16 into its per-block scale instead.
template <bool SCALE = true>
__device__ __forceinline__ void fwht256_warp(int i, float4 *buf, float r[32]) {
  bfly_packed<1>(r);  // h = 1
  bfly_packed<2>(r);  // h = 2
  bfly_packed<4>(r);  // h = 4
  transpose_l0_l1(r, buf, i);
  bfly_packed<1>(r);  // h = 8
  bfly_packed<2>(r);  // h = 16
  bfly_packed<4>(r);  // h = 32
  bfly_packed<8>(r);  // h = 64
  bfly16(r);          // h = 128
  if (SCALE) {
    const float2 s = make_float2(0.0625f, 0.0625f);
#pragma unroll
    for (int k = 0; k < 16; k++) {
      float2 v = mul2(make_float2(r[k], r[k + 16]), s);
      r[k] = v.x;
      r[k + 16] = v.y;
    }
  }
}

// ------------------------------------------------------------------ quantize
// The tie-break scan (start (amax, mval) = (0, +0); take z when |z| > amax, or
// |z| == amax and z > mval) ends on the lexicographic maximum of (|z|, z).
// Each lane reduces its 4 values of a block to amax_t = max |z| and a flag
// "+amax_t occurs"; the key (bits(amax_t) << 1) | flag orders exactly like
// (|z|, z), so the maximum key over the 8 lanes identifies mval.  An all-zero
// block gives key 1, i.e. mval = +0, like the scan.
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key >> 1) | ((~key & 1u) << 31));
}

// three-input maximum (one instruction on sm_100); exact, like fmaxf
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

struct QuantOut {
  uint32_t items[8];  // block B: byte i | byte (i + 8) << 8 of the block's 16 code bytes
  uint16_t scale;     // fp16 bits of this lane's block (block index = lane i)
};

// Quantize the 8 blocks of one vector held in layout L1 (this lane: i).  r
// holds the unscaled stage output w = 16 z.  Scaling by 2^-4 is exact (the
// bit-exact contract excludes blocks whose max-abs value is below 2^-120), so
// with w the tie-break order is the same, d = (w_mval / -8) / 16 exactly, and
// z * RN(1/d) = w * RN(1/(16 d)) is the same real product, rounded once.
__device__ __forceinline__ void q4_quantize_l1(const float r[32], int lane, int i, QuantOut &o) {
  // register of block B, in-block row m: 4 * (B & 1) + m + 8 * (B >> 1)
  uint32_t key[8];
#pragma unroll
  for (int B = 0; B < 8; B++) {
    const int r0 = 4 * (B & 1) + 8 * (B >> 1);
    const float z0 = r[r0], z1 = r[r0 + 1], z2 = r[r0 + 2], z3 = r[r0 + 3];
    const float am = fmaxf(max3f(fabsf(z0), fabsf(z1), fabsf(z2)), fabsf(z3));
    const float mz = fmaxf(max3f(z0, z1, z2), z3);
    uint32_t k;
    asm("mad.lo.u32 %0, %1, 2, %2;" : "=r"(k) : "r"(__float_as_uint(am)), "r"(mz == am ? 1u : 0u));
    key[B] = k;
  }
  // transposed max-reduction over the 8 lanes of the vector: each xor level
  // halves the blocks a lane keeps, so lane i ends with the key of block i
#pragma unroll
  for (int j = 0; j < 4; j++) {  // lanes with bit 2 set keep blocks 4..7
    const bool up = i & 4;
    const uint32_t send = up ? key[j] : key[j + 4];
    const uint32_t keep = up ? key[j + 4] : key[j];
    key[j] = max(keep, __shfl_xor_sync(kVFull, send, 4));
  }
#pragma unroll
  for (int j = 0; j < 2; j++) {  // bit 1: upper two of the four
    const bool up = i & 2;
    const uint32_t send = up ? key[j] : key[j + 2];
    const uint32_t keep = up ? key[j + 2] : key[j];
    key[j] = max(keep, __shfl_xor_sync(kVFull, send, 2));
  }
  uint32_t kmine;
  {
    const bool up = i & 1;
    const uint32_t send = up ? key[0] : key[1];
    const uint32_t keep = up ? key[1] : key[0];
    kmine = max(keep, __shfl_xor_sync(kVFull, send, 1));
  }
  const float wval = key_value(kmine);
  const float dw = __fmul_rn(wval, -0.125f);    // 16 d (exact)
  const float id = (dw != 0.f) ? __frcp_rn(dw) : 0.f;  // RN(1 / (16 d))
  o.scale = __half_as_ushort(__float2half_rn(__fmul_rn(dw, 0.0625f)));
  float idb[8];
#pragma unroll
  for (int B = 0; B < 8; B++) idb[B] = __shfl_sync(kVFull, id, (lane & ~7) | B);

  const float2 magic = make_float2(8388608.f, 8388608.f);
  const uint32_t fifteen = 0x000F000Fu;
#pragma unroll
  for (int B = 0; B < 8; B++) {
    const int r0 = 4 * (B & 1) + 8 * (B >> 1);
    // z * id and + 8.5 round separately.  A packed multiply followed by a
    // packed add was observed to be merged into one multiply-add (which moves
    // a value sitting on a rounding tie); the product is therefore a packed
    // fma with a +0 addend, which has the product's rounding and cannot be
    // merged.
    const float2 idv = make_float2(idb[B], idb[B]), half8 = make_float2(8.5f, 8.5f);
    const float2 t02 = add2_rn(mul2_rn_p0(make_float2(r[r0], r[r0 + 2]), idv), half8);
    const float2 t13 = add2_rn(mul2_rn_p0(make_float2(r[r0 + 1], r[r0 + 3]), idv), half8);
    // 2^23 + floor(t) for t >= 0; the low 16 bits are floor(t) in 0..16
    const float2 f02 = add2_rz(t02, magic);
    const float2 f13 = add2_rz(t13, magic);
    // element-in-block i + 8m: byte i = c0 | c2 << 4, byte i + 8 = c1 | c3 << 4
    const uint32_t x02 = min_u16x2(__byte_perm(__float_as_uint(f02.x), __float_as_uint(f02.y), 0x5410), fifteen);
    const uint32_t x13 = min_u16x2(__byte_perm(__float_as_uint(f13.x), __float_as_uint(f13.y), 0x5410), fifteen);
    // y = x + (x >> 12) = x | (x >> 12) (no overlapping bits), as a high
    // multiply-add; item = y02 + 256 y13 in the low 16 bits
    uint32_t y02, y13, it;
    asm("mad.hi.u32 %0, %1, 1048576, %1;" : "=r"(y02) : "r"(x02));
    asm("mad.hi.u32 %0, %1, 1048576, %1;" : "=r"(y13) : "r"(x13));
    asm("mad.lo.u32 %0, %1, 256, %2;" : "=r"(it) : "r"(y13), "r"(y02));
    o.items[B] = it;  // (byte i, byte i + 8) in the low 16 bits
  }
}

// Regroup the per-lane items so lane i holds the 16 code bytes of block i.
__device__ __forceinline__ uint4 gather_block_bytes(const QuantOut &o, uint8_t *stage, int i) {
  uint16_t *s16 = reinterpret_cast<uint16_t *>(stage);
#pragma unroll
  for (int B = 0; B < 8; B++) s16[B * 8 + i] = (uint16_t)o.items[B];
  __syncwarp();
  uint4 w = *reinterpret_cast<const uint4 *>(stage + 16 * i);  // (b0,b8,b1,b9 | b2,b10,b3,b11 | ...)
  __syncwarp();
  uint4 out;
  out.x = __byte_perm(w.x, w.y, 0x6420);
  out.y = __byte_perm(w.z, w.w, 0x6420);
  out.z = __byte_perm(w.x, w.y, 0x7531);
  out.w = __byte_perm(w.z, w.w, 0x7531);
  return out;
}


// ------------------------------------------------------------------ Q8_0
// Q8_0 of the 8 blocks of one vector in layout L1 (unscaled stage output
// w = 16 z, this lane: i): amax = max |z|, d = amax / 127, id = d ? 1/d : 0,
// code = roundf(z * id) (product rounded to fp32, halves away from zero),
// stored as int8 with fp16(d).  As for Q4_0, the 1/16 folds exactly:
// RN(16a / 127) = 16 RN(a / 127), RN(1 / (16 d)) = RN(1/d) / 16, and
// w * RN(1/(16 d)) is the same real product as z * RN(1/d).
// Lane i returns the 32 code bytes of block i (elements 0..31 in order) and
// the fp16 bits of its scale; stage: 256 bytes of shared memory per vector.
__device__ __forceinline__ void q8_quantize_l1(const float r[32], int lane, int i,
                                               uint32_t *stage, uint4 (&bytes)[2],
                                               uint16_t &scale) {
  uint32_t key[8];  // |.| bits: non-negative floats order like unsigned ints
#pragma unroll
  for (int B = 0; B < 8; B++) {
    const int r0 = 4 * (B & 1) + 8 * (B >> 1);
    const float am = fmaxf(max3f(fabsf(r[r0]), fabsf(r[r0 + 1]), fabsf(r[r0 + 2])), fabsf(r[r0 + 3]));
    key[B] = __float_as_uint(am);
  }
#pragma unroll
  for (int j = 0; j < 4; j++) {
    const bool up = i & 4;
    const uint32_t send = up ? key[j] : key[j + 4];
    const uint32_t keep = up ? key[j + 4] : key[j];
    key[j] = max(keep, __shfl_xor_sync(kVFull, send, 4));
  }
#pragma unroll
  for (int j = 0; j < 2; j++) {
    const bool up = i & 2;
    const uint32_t send = up ? key[j] : key[j + 2];
    const uint32_t keep = up ? key[j + 2] : key[j];
    key[j] = max(keep, __shfl_xor_sync(kVFull, send, 2));
  }
  uint32_t kmine;
  {
    const bool up = i & 1;
    const uint32_t send = up ? key[0] : key[1];
    const uint32_t keep = up ? key[1] : key[0];
    kmine = max(keep, __shfl_xor_sync(kVFull, send, 1));
  }
  const float dw = __fdiv_rn(__uint_as_float(kmine), 127.f);  // 16 d
  const float id = (dw != 0.f) ? __frcp_rn(dw) : 0.f;         // RN(1 / (16 d))
  scale = __half_as_ushort(__float2half_rn(__fmul_rn(dw, 0.0625f)));
  float idb[8];
#pragma unroll
  for (int B = 0; B < 8; B++) idb[B] = __shfl_sync(kVFull, id, (lane & ~7) | B);
  // lane i holds elements i, i + 8, i + 16, i + 24 of each block: one word each
#pragma unroll
  for (int B = 0; B < 8; B++) {
    const int r0 = 4 * (B & 1) + 8 * (B >> 1);
    // products rounded once each (packed, as in q4_quantize_l1)
    const float2 idv = make_float2(idb[B], idb[B]);
    const float2 p01 = mul2_rn_p0(make_float2(r[r0], r[r0 + 1]), idv);
    const float2 p23 = mul2_rn_p0(make_float2(r[r0 + 2], r[r0 + 3]), idv);
    const float p[4] = {p01.x, p01.y, p23.x, p23.y};
    uint32_t w = 0;
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const int c = (int)roundf(p[m]);
      w |= (uint32_t)(c & 0xFF) << (8 * m);
    }
    stage[B * 8 + i] = w;
  }
  __syncwarp();
  // block i: word u (from lane u) holds elements u, u + 8, u + 16, u + 24
  uint32_t wv[8];
#pragma unroll
  for (int u = 0; u < 8; u++) wv[u] = stage[i * 8 + u];
  __syncwarp();
  uint32_t ow[8];  // output word k: elements 4k .. 4k + 3
#pragma unroll
  for (int k = 0; k < 8; k++) {
    const int u0 = (4 * k) & 7, m = (4 * k) >> 3;  // elements 4k + j: word u0 + j, byte m
    // selector: result byte 0 <- byte m of the first word, byte 1 <- byte m of the second
    const uint32_t lo = __byte_perm(wv[u0], wv[u0 + 1], 0x40 + 0x11 * m);
    const uint32_t hi = __byte_perm(wv[u0 + 2], wv[u0 + 3], 0x40 + 0x11 * m);
    ow[k] = __byte_perm(lo, hi, 0x5410);
  }
  bytes[0] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  bytes[1] = make_uint4(ow[4], ow[5], ow[6], ow[7]);
}

// One warp Q8_0-quantizes up to 4 vectors (as quantize_vector); lane i % 8
// returns the 32 code bytes of block i and its fp16 scale.  buf: 64 float4 of
// shared memory per vector.
template <bool BF16>
__device__ __forceinline__ void quantize_vector_q8(const void *src, bool valid, int lane,
                                                   float4 *buf, uint4 (&bytes)[2],
                                                   uint16_t &scale) {
  const int i = lane & 7;
  Raw<BF16> raw;
  fetch_raw<BF16>(src, i, valid, raw);
  float r[32];
  unpack_l0<BF16>(raw, r);
  fwht256_warp<false>(i, buf, r);
  q8_quantize_l1(r, lane, i, reinterpret_cast<uint32_t *>(buf), bytes, scale);
}

// One warp quantizes up to 4 vectors (vector vg = lane / 8): FWHT-256 of the
// input vector `src` (bf16 or fp32, 256 values; ignored when !valid), Q4_0 of
// its 8 blocks.  Lane i = lane % 8 returns the 16 code bytes of block i and its
// fp16 scale.  buf: 64 float4 of shared memory per vector (vectors of a warp
// need distinct buffers).
template <bool BF16>
__device__ __forceinline__ void quantize_vector(const void *src, bool valid, int lane,
                                                float4 *buf, uint4 &bytes, uint16_t &scale) {
  const int vg = lane >> 3, i = lane & 7;
  Raw<BF16> raw;
  fetch_raw<BF16>(src, i, valid, raw);
  float r[32];
  unpack_l0<BF16>(raw, r);
  fwht256_warp<false>(i, buf, r);
  QuantOut o;
  q4_quantize_l1(r, lane, i, o);
  bytes = gather_block_bytes(o, reinterpret_cast<uint8_t *>(buf) + 16 * vg, i);
  scale = o.scale;
}

}  // namespace q4v
}  // namespace kvq
