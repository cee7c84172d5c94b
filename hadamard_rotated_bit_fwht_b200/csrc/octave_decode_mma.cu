// octave_decode_mma.cu -- tensor-core split-K decode over the Octave cache
// (vLLM API page "vllm.v1.attention.ops.rocm_octave": module text -- scores in
// the rotated space, output rotated back once per query head -- and
// reference_attention), for the k3v4 format with head 128 and rope 64:
//   slot bytes  0..31  K RoPE block, 4-bit codes (word w: byte j = dims 8w+j | 8w+j+4 << 4)
//              32..55  K NoPE block, 3-bit codes (2-bit plane 32..47, 1-bit plane 48..55)
//              56..119 V, 4-bit codes over 128 dims
//             120..125 fp16 scales: K RoPE, K NoPE, V.
// A code c of a block with scale s stands for LUT[c] * s / 64.
//   * QK on the integer tensor path (mma.sync m16n8k32, s8 x s8 -> s32).  The
//     signed int8 codebook sits in registers; prmt selects four table bytes at
//     a time from nibble-packed codes (two 8-entry halves plus a
//     sign-replicated mask for 4-bit codes, one prmt for 3-bit codes), and
//     those bytes are B-fragment registers as they stand.  The rotated query
//     of each head is scaled by S = 127 * 2^14 / max|q|, rounded to an
//     integer and split exactly into three int8 digits
//     (S q = 2^14 H + 2^7 M + L, |M|, |L| <= 64).  Up to 4 heads per CTA, one
//     A tile holds all three: H in rows 0-3, L in rows 4-7, M in rows 8-11,
//     and the L dot products come from the lanes 16 apart by one shuffle; with
//     more heads one A tile holds H (rows 0-7) and M (rows 8-15), a second
//     one L.  The columns are stored in the order the codes arrive in.  Per
//     (block, 8 tokens) the digit dot products are combined in fp32
//     (2^14 d_H + (2^7 d_M + d_L))
//     and multiplied by the block scale; 1 / S joins the softmax scale.  The
//     query is thereby carried to 2.4e-7 of its largest element.  (Two
//     digits, 14 bits, left up to 2.3e-3 of error in the outputs of the
//     16 x 16384-token workload, whose keys carry x16 outlier channels.)
//   * PV on the fp16 path (m16n8k16, fp32 accumulation): A = V^T codes through
//     the biased table (each byte u becomes the exact fp16 1024 + u = LUT[c] +
//     1152 by pairing it with 0x64, and one half2 subtract of 1152 leaves the
//     exact LUT[c]), read by ldmatrix.trans from the swizzled tile; B = p *
//     s_v / 64 split hi + lo.  The subtract stays ahead of the MMA: folding
//     the 1152 out of the fp32 accumulators after the sum instead (an
//     all-ones MMA for sum_t p) carried the accumulation error of 1152 * l,
//     2e-3 in the outputs at 16k-256k tokens, against 5e-5 this way.  Up to
//     4 heads per CTA, the hi parts sit in B columns 0-3 and the lo parts in
//     columns 4-7 (one MMA per tile instead of two); the merge adds the two
//     halves.
//     The V region starts 8 bytes into a 16-byte chunk: the used halves of
//     chunks 3 and 7 are joined by one lane shuffle, so the 64 V bytes make
//     exactly 8 M-tiles.
// Tiles of 64 slots (one 128-byte row per token) are staged by cp.async with
// the 128-byte XOR swizzle through a 3-stage ring; each row is addressed
// through the block table by one lookup, so any block size works, and a
// token whose block entry names no block contributes nothing.  (Block sizes
// that are multiples of 64 take one 64-row TMA box per tile instead.)
// The kernel and the combine after it are programmatic dependent launches:
// each is scheduled while the grid before it drains and waits for that grid
// (griddepcontrol.wait) before its first global read.
#include <cstring>

#include "decode_common.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 64;
constexpr int kStages = 3;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kHead = 128;
constexpr int kORec = 132;  // m, l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQRange = 2080768.f;  // 127 * 2^14
constexpr int kStageBytes = kTile * 128;
constexpr int kOffF = kStages * kStageBytes;  // fp32 scales [3][64] of the current tile
constexpr int kOffV = kOffF + 3 * kTile * 4;  // per stage, per token: 1 if its block is mapped
constexpr int kQStride = 144;                 // int8 query row: 128 B + 16 B pad
constexpr int kOffQ = kOffV + kStages * kTile;  // int8 query rows: 0-7 H, 8-15 M, 16-23 L, 24-31 zero
constexpr int kOffBar = kOffQ + 32 * kQStride;  // TMA staging: full barriers [kStages]
constexpr int kOffTok = kOffBar + 8 * kStages;  // TMA staging: 1 if the tile's block is mapped [kStages]
constexpr int kOffAbort = kOffTok + 8;          // TMA staging: a wait gave up
constexpr int kSmemUsed = kOffAbort + 8;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kStageBytes % 1024 == 0, "stages keep the 128-byte swizzle atoms aligned");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d += A(s8, 16 x 32) * B(s8, 32 x 8)
__device__ __forceinline__ void imma16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(s));
  return r;
}
// a * 2^k + b and (a >> (32 - k)) + b as integer multiply-adds, which issue
// to the FMA pipe (this kernel's ALU pipe is its busiest)
template <int K>
__device__ __forceinline__ uint32_t shl_add(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "n"(1u << K), "r"(b));
  return r;
}
template <int K>
__device__ __forceinline__ uint32_t shr_add(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "n"(1u << (32 - K)), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t lop3_sel(uint32_t lo, uint32_t hi, uint32_t m) {
  uint32_t r;  // m ? hi : lo, bitwise
  asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(r) : "r"(lo), "r"(hi), "r"(m));
  return r;
}

// Table bytes T[c] for four nibble-packed 4-bit codes (sel bits 0-15; the
// higher bits are ignored): two 8-entry lookups on the low three bits, then a
// per-byte choice by the fourth bit (sign-replicated into a mask by prmt).
struct Lut4 {
  uint32_t lo0, lo1, hi0, hi1;
};
__device__ __forceinline__ uint32_t lut4_bytes(uint32_t sel, const Lut4 &T) {
  const uint32_t s = sel & 0x7777u;
  const uint32_t plo = prmt(T.lo0, T.lo1, s);
  const uint32_t phi = prmt(T.hi0, T.hi1, s);
  const uint32_t m = prmt(shl_add<4>(sel, 0u), sel, 0xD9C8u);
  return lop3_sel(plo, phi, m);
}
// biased bytes (a, b) of R, U = LUT + 128 -> half2 (LUT_a, LUT_b) exactly: the
// pairing with 0x64 makes the fp16 1024 + U, and 1024 + U - 1152 is exact
__device__ __forceinline__ uint32_t lut_half2(uint32_t R, uint32_t selector) {
  const uint32_t biased = prmt(R, 0x64646464u, selector);
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(biased), "r"(0x64806480u));  // 1152, 1152
  return r;
}

__device__ __forceinline__ void split_hilo(float2 w, uint32_t &hi, uint32_t &lo) {
  __half2 h = __float22half2_rn(w);
  float2 hf = __half22float2(h);
  __half2 l = __float22half2_rn(make_float2(w.x - hf.x, w.y - hf.y));
  hi = *reinterpret_cast<uint32_t *>(&h);
  lo = *reinterpret_cast<uint32_t *>(&l);
}

// Head dim of column k (0..31) of the query's virtual chunk vc: chunks 0, 1
// follow the RoPE codes as lut4_bytes returns them (word of lane tg = dims
// 32 vc + 8 tg + 0..7, bytes in the order 0 4 1 5 | 2 6 3 7); chunks 2, 3 the
// NoPE codes as the NoPE lookup returns them: lane tg holds dims
// 64 + 16 tg + 4 f + j (2-bit field f of plane byte j), chunk 2 fields 0 and
// 2, chunk 3 fields 1 and 3, byte order (f, j) = (a, 0) (a + 2, 0) (a, 1)
// (a + 2, 1) | the same for j = 2, 3.
__device__ __forceinline__ int qcol_dim(int vc, int k) {
  const int tg = (k & 15) >> 2, jp = k & 3, hi = k >> 4;
  if (vc < 2) return 32 * vc + 8 * tg + 2 * hi + (jp >> 1) + 4 * (jp & 1);
  const int f = (vc - 2) + 2 * (jp & 1), j = 2 * hi + (jp >> 1);
  return 64 + 16 * tg + 4 * f + j;
}

// PACK: gc <= 4, the three query digits in one A tile.  TMA: the tiles come
// by one 64-row tensor copy each (block sizes that are multiples of 64: a
// tile lies in one block), staged through mbarriers; otherwise by cp.async,
// row by row through the block table.
template <bool BF16, bool PACK, bool TMA>
__global__ void __launch_bounds__(kThreads, 4)
    octave_decode_mma_kernel(const __grid_constant__ CUtensorMap slots, int wait_polls,
                             OctaveParams P, const void *__restrict__ query, int n_q_heads,
                             int group, int gc, const uint8_t *__restrict__ cache, int n_kv_heads,
                             int block_size, int64_t num_blocks,
                             const int32_t *__restrict__ block_table, int num_reqs,
                             int max_blocks, const int32_t *__restrict__ q_to_req,
                             const int32_t *__restrict__ q_to_klen, int max_klen,
                             float scale_log2, int split_tokens, int splits,
                             float *__restrict__ ws, uint32_t *__restrict__ err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int s = blockIdx.x, hg = blockIdx.y, qi = blockIdx.z;
  const int h0 = hg * gc, kvh = h0 / group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  // launched as a programmatic dependent of the kernel before it (which may
  // write the slots or the inputs): wait for that grid before the first global
  // read, then let the combine grid be scheduled behind this one
  dec::grid_dependency_wait();
  dec::launch_dependents();
  const int req = __ldg(q_to_req + qi);
  int klen = min(max(__ldg(q_to_klen + qi), 0), min(max_klen, max_blocks * block_size));
  if (req < 0 || req >= num_reqs) klen = 0;
  const int t0 = s * split_tokens, t1 = min(klen, t0 + split_tokens);
  const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;

  // codebook tables: signed bytes for QK, biased (+128) bytes for PV
  Lut4 T4, U4;
  uint32_t T3lo, T3hi;
  {
    uint32_t b[16], u[16];
#pragma unroll
    for (int i = 0; i < 16; i++) {
      b[i] = (uint32_t)P.lut4[i] & 0xFFu;
      u[i] = (uint32_t)(P.lut4[i] + 128) & 0xFFu;
    }
    T4.lo0 = b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24;
    T4.lo1 = b[4] | b[5] << 8 | b[6] << 16 | b[7] << 24;
    T4.hi0 = b[8] | b[9] << 8 | b[10] << 16 | b[11] << 24;
    T4.hi1 = b[12] | b[13] << 8 | b[14] << 16 | b[15] << 24;
    U4.lo0 = u[0] | u[1] << 8 | u[2] << 16 | u[3] << 24;
    U4.lo1 = u[4] | u[5] << 8 | u[6] << 16 | u[7] << 24;
    U4.hi0 = u[8] | u[9] << 8 | u[10] << 16 | u[11] << 24;
    U4.hi1 = u[12] | u[13] << 8 | u[14] << 16 | u[15] << 24;
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; i++) c[i] = (uint32_t)P.lut3[i] & 0xFFu;
    T3lo = c[0] | c[1] << 8 | c[2] << 16 | c[3] << 24;
    T3hi = c[4] | c[5] << 8 | c[6] << 16 | c[7] << 24;
  }

  // ---- query: signs, FWHT over the two 64-dim blocks; int8 H / M / L rows
  float *qs = reinterpret_cast<float *>(smem);  // [8][128]
  {
    // thread tid always holds dim tid: sign bit (tid & 31) of word tid / 32
    // (constant indices only, so the parameter block stays in constant memory)
    const uint32_t sw = warp == 0 ? P.sign_words[0]
                        : warp == 1 ? P.sign_words[1]
                        : warp == 2 ? P.sign_words[2]
                                    : P.sign_words[3];
    const float sgn = ((sw >> lane) & 1u) ? -1.f : 1.f;
    for (int hh = 0; hh < 8; hh++) {
      float v = 0.f;
      if (hh < gc) {
        const int64_t off = ((int64_t)qi * n_q_heads + h0 + hh) * kHead + tid;
        v = (BF16 ? __uint_as_float((uint32_t)static_cast<const uint16_t *>(query)[off] << 16)
                  : static_cast<const float *>(query)[off]) *
            sgn;
      }
      qs[hh * kHead + tid] = v;
    }
  }
  for (int h = 1; h < 64; h <<= 1) {
    __syncthreads();
    for (int p = tid; p < 8 * 64; p += kThreads) {
      const int vv = p >> 6, pi = p & 63, blk = pi >> 5, pj = pi & 31;
      const int i0 = blk * 64 + (pj / h) * 2 * h + (pj % h);
      float *y = qs + vv * kHead;
      const float a = y[i0], bb = y[i0 + h];
      y[i0] = a + bb;
      y[i0 + h] = a - bb;
    }
  }
  __syncthreads();
  float *qmax = reinterpret_cast<float *>(smem + kOffF);  // [8]
#pragma unroll
  for (int i = 0; i < 2; i++) {  // warp w: heads 2w, 2w + 1
    const int hh = 2 * warp + i;
    float m = fmaxf(fmaxf(fabsf(qs[hh * kHead + lane]), fabsf(qs[hh * kHead + lane + 32])),
                    fmaxf(fabsf(qs[hh * kHead + lane + 64]), fabsf(qs[hh * kHead + lane + 96])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    if (lane == 0) qmax[hh] = m;
  }
  __syncthreads();
  uint8_t *qrow = smem + kOffQ;
  for (int p = tid; p < 8 * kHead; p += kThreads) {
    const int hh = p >> 7, col = p & 127;
    const float m = qmax[hh];
    const int dim = qcol_dim(col >> 5, col & 31);
    // |x| <= 127 * 2^14 < 2^21, so x is a multiple of 2^-3 at worst and every
    // difference below is exact; the digits sum to rint(x)
    const float x = m > 0.f ? qs[hh * kHead + dim] * (kQRange / m) : 0.f;
    const float hi = rintf(x * (1.f / 16384.f));
    const float r1 = x - 16384.f * hi;  // |r1| <= 2^13
    const float mid = rintf(r1 * 0.0078125f);
    const float lo = rintf(r1 - 128.f * mid);  // |lo| <= 64
    if (PACK) {  // H rows 0-3, L rows 4-7, M rows 8-11, zero rows 12-15
      if (hh < 4) {
        qrow[hh * kQStride + col] = (uint8_t)(int8_t)(int)hi;
        qrow[(4 + hh) * kQStride + col] = (uint8_t)(int8_t)(int)lo;
        qrow[(8 + hh) * kQStride + col] = (uint8_t)(int8_t)(int)mid;
        qrow[(12 + hh) * kQStride + col] = 0;
      }
    } else {
      qrow[hh * kQStride + col] = (uint8_t)(int8_t)(int)hi;
      qrow[(8 + hh) * kQStride + col] = (uint8_t)(int8_t)(int)mid;
      qrow[(16 + hh) * kQStride + col] = (uint8_t)(int8_t)(int)lo;
      qrow[(24 + hh) * kQStride + col] = 0;
    }
  }
  __syncthreads();
  uint32_t qa[4][4], qb[4][4];  // A fragments of the virtual chunks: (H, M) and (L, 0)
  {
    const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
    const uint32_t qaddr = smem_u32(qrow) + row * kQStride + 16 * (lane >> 4);
#pragma unroll
    for (int vc = 0; vc < 4; vc++) {
      ldsm_x4(qaddr + 32 * vc, qa[vc]);
      if (!PACK) ldsm_x4(qaddr + 16 * kQStride + 32 * vc, qb[vc]);
    }
  }
  // FWHT-64 blocks carry 1 / 8; the query ints carry S
  const float sl = scale_log2 * (qmax[g] * (0.125f / kQRange));
  __syncthreads();

  // ---- loader: thread tid copies chunks 4 (tid & 1) .. + 3 of row tid / 2
  const int lr = tid >> 1, lc0 = 4 * (tid & 1);
  // block index of a token: a shift for power-of-two block sizes
  const int bs_shift = (block_size & (block_size - 1)) == 0 ? __ffs(block_size) - 1 : -1;
  auto issue = [&](int it) {  // cp.async staging (all threads)
    uint8_t *st = smem + (it % kStages) * kStageBytes;
    const int t = t0 + it * kTile + lr;
    bool ok = t < t1;
    const uint8_t *src = cache;
    if (ok) {
      const int bi = bs_shift >= 0 ? t >> bs_shift : t / block_size;
      const int blk = __ldg(block_table + (int64_t)req * max_blocks + bi);
      ok = blk >= 0 && blk < num_blocks;
      const int64_t si = ((int64_t)blk * n_kv_heads + kvh) * block_size + (t - bi * block_size);
      ok = ok && in_bounds(si, si + 1, num_blocks * n_kv_heads * block_size, err);
      if (ok) src = cache + si * P.slot_bytes;
    }
    if (lc0 == 0) smem[kOffV + (it % kStages) * kTile + lr] = ok ? 1 : 0;
    const uint32_t rowa = smem_u32(st) + lr * 128;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int ch = lc0 + i;
      cp_async16(rowa + ((ch ^ (lr & 7)) << 4), ok ? src + ch * 16 : cache, ok);
    }
  };

  // TMA staging: thread 0 issues each tile as one 64 x 128-byte box of the
  // slot rows (the map's 128-byte swizzle is the XOR pattern used above) and
  // records whether its block is mapped
  const uint32_t full0 = smem_u32(smem + kOffBar);
  volatile uint8_t *tok = smem + kOffTok;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);
  int issued = 0;  // thread 0: tiles issued so far
  auto issue_tma = [&](int it) {
    const int st = it % kStages;
    const int t = t0 + it * kTile;  // a multiple of 64, inside one block
    const int bi = bs_shift >= 0 ? t >> bs_shift : t / block_size;
    const int blk = __ldg(block_table + (int64_t)req * max_blocks + bi);
    bool ok = blk >= 0 && blk < num_blocks;
    const int64_t row = ((int64_t)blk * n_kv_heads + kvh) * block_size + (t - bi * block_size);
    ok = ok && in_bounds(row, row + kTile, num_blocks * n_kv_heads * block_size, err);
    tok[st] = ok ? 1 : 0;
    const uint32_t bar = full0 + 8 * st;
    if (ok) {
      dec::mbar_arrive_tx(bar, kStageBytes);
      dec::tma_load_2d(smem_u32(smem + st * kStageBytes), &slots, 0, (int)row, bar);
    } else {
      dec::mbar_arrive(bar);
    }
    issued = it + 1;
  };
  if (TMA) {
    if (tid == 0) {
      dec::prefetch_map(&slots);
#pragma unroll
      for (int i = 0; i < kStages; i++) dec::mbar_init(full0 + 8 * i, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      // the query set-up above wrote stage 0 through the generic proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
  }

  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; mt++) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  float *fsc = reinterpret_cast<float *>(smem + kOffF);

  if (TMA) {
    if (tid == 0)
      for (int i = 0; i < kStages - 1 && i < ntiles; i++) issue_tma(i);
  } else {
#pragma unroll
    for (int i = 0; i < kStages - 1; i++) {
      if (i < ntiles) issue(i);
      cp_async_commit();
    }
  }
  bool aborted = false;
  for (int it = 0; it < ntiles; it++) {
    if (TMA) {
      if (!dec::mbar_wait(full0 + 8 * (it % kStages), (it / kStages) & 1, abort_flag, wait_polls))
        *abort_flag = 1;
      __syncthreads();
      if (*abort_flag) {  // read by every thread after the barrier: a uniform exit
        aborted = true;
        break;
      }
    } else {
      cp_async_wait<kStages - 2>();
      __syncthreads();
    }
    uint8_t *st = smem + (it % kStages) * kStageBytes;
    if (tid < kTile) {  // scales at bytes 120..125 (chunk 7, offset 8): fp16 -> fp32 / 64
      const int r = tid;
      const uint8_t *row = st + r * 128 + ((7 ^ (r & 7)) << 4) + 8;
      const uint32_t w01 = *reinterpret_cast<const uint32_t *>(row);
      const uint32_t w2 = *reinterpret_cast<const uint16_t *>(row + 4);
      const float2 f01 = __half22float2(*reinterpret_cast<const __half2 *>(&w01));
      fsc[r] = f01.x * 0.015625f;
      fsc[kTile + r] = f01.y * 0.015625f;
      fsc[2 * kTile + r] = __half2float(__ushort_as_half((uint16_t)w2)) * 0.015625f;
    }
    if (TMA) {
      // every thread is past the barrier above, so the stage of tile it - 1
      // is free; its generic reads precede the async-proxy write
      if (tid == 0 && it + kStages - 1 < ntiles) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_tma(it + kStages - 1);
      }
    } else {
      if (it + kStages - 1 < ntiles) issue(it + kStages - 1);
      cp_async_commit();
    }
    __syncthreads();

    // bit k: token k of this warp's 16 is in range and on a mapped block
    const unsigned okmask =
        TMA ? __ballot_sync(kFull, (lane < 16) && tok[it % kStages] != 0 &&
                                       t0 + it * kTile + 16 * warp + (lane & 15) < t1) &
                  0xFFFFu
            : __ballot_sync(kFull,
                            (lane < 16) &&
                                smem[kOffV + (it % kStages) * kTile + 16 * warp + (lane & 15)] != 0) &
                  0xFFFFu;
    if (okmask != 0) {
      const bool partial = okmask != 0xFFFFu;
      const uint32_t base = smem_u32(st);
      // ldmatrix lane address: matrix m = lane / 8 (x4: T = m & 1, chunk +m >> 1)
      const int mr = 16 * warp + 8 * ((lane >> 3) & 1) + (lane & 7);
      const int mc = lane >> 4;
      auto chunk_addr = [&](int ch) -> uint32_t {
        return base + mr * 128 + ((ch ^ (mr & 7)) << 4);
      };
      // ---- QK: integer MMAs, accumulators per (block, 8 tokens): (H, M) rows
      // and L rows
      int accr[2][4] = {}, accn[2][4] = {}, accrl[2][4] = {}, accnl[2][4] = {};
      {  // RoPE: chunks 0, 1 (4-bit)
        uint32_t kr[4];
        ldsm_x4(chunk_addr(mc), kr);  // (T0, c0), (T1, c0), (T0, c1), (T1, c1)
#pragma unroll
        for (int m = 0; m < 4; m++) {
          const int T = m & 1, c = m >> 1;
          const uint32_t w = kr[m];
          // lut4_bytes reads selector bits 0..15 only
          const uint32_t b0 = lut4_bytes(w, T4), b1 = lut4_bytes(shr_add<16>(w, 0u), T4);
          imma16832(accr[T], qa[c], b0, b1);
          if (!PACK) imma16832(accrl[T], qb[c], b0, b1);
        }
      }
      {  // NoPE: 2-bit plane chunk 2, 1-bit plane in chunk 3 (words 0, 1)
        uint32_t lo[2], hi[2];
        {
          uint32_t r4[4];
          ldsm_x4(chunk_addr(2 + mc), r4);  // (T0, c2), (T1, c2), (T0, c3), (T1, c3)
          lo[0] = r4[0];
          lo[1] = r4[1];
          // the 1-bit plane word this lane needs (tg >> 1) sits in lane 4g + (tg >> 1),
          // its 4 bits per byte at 4 (tg & 1)
          hi[0] = __shfl_sync(kFull, r4[2], (lane & ~3) | (tg >> 1)) >> (4 * (tg & 1));
          hi[1] = __shfl_sync(kFull, r4[3], (lane & ~3) | (tg >> 1)) >> (4 * (tg & 1));
        }
#pragma unroll
        for (int T = 0; T < 2; T++) {
          // code of dim 16tg + 4f + j: 2-bit field f of lo byte j, bit f of hi
          // byte j on top.  Fields f and f + 2 go to the low and high nibble of
          // byte j (disjoint bits, so the multiply-adds only place them), and
          // each 16-bit half is then a selector of four codes.
          const uint32_t h = hi[T];
          uint32_t x02 = lo[T] & 0x33333333u;                 // fields 0, 2
          x02 = shl_add<2>(h & 0x01010101u, x02);             // bit 0 -> 2
          x02 = shl_add<4>(h & 0x04040404u, x02);             // bit 2 -> 6
          uint32_t x13 = shr_add<2>(lo[T] & 0xCCCCCCCCu, 0u);  // fields 1, 3
          x13 = shl_add<1>(h & 0x02020202u, x13);             // bit 1 -> 2
          x13 = shl_add<3>(h & 0x08080808u, x13);             // bit 3 -> 6
          uint32_t R[4];
          R[0] = prmt(T3lo, T3hi, x02);
          R[1] = prmt(T3lo, T3hi, shr_add<16>(x02, 0u));
          R[2] = prmt(T3lo, T3hi, x13);
          R[3] = prmt(T3lo, T3hi, shr_add<16>(x13, 0u));
          imma16832(accn[T], qa[2], R[0], R[1]);
          imma16832(accn[T], qa[3], R[2], R[3]);
          if (!PACK) {
            imma16832(accnl[T], qb[2], R[0], R[1]);
            imma16832(accnl[T], qb[3], R[2], R[3]);
          }
        }
      }
      float2 sacc[2];
#pragma unroll
      for (int T = 0; T < 2; T++) {
        const float2 dr = *reinterpret_cast<const float2 *>(fsc + 16 * warp + 8 * T + 2 * tg);
        const float2 dn =
            *reinterpret_cast<const float2 *>(fsc + kTile + 16 * warp + 8 * T + 2 * tg);
        if (PACK) {  // L sits in rows 4-7: the [0..1] of the lanes 16 apart
#pragma unroll
          for (int e = 0; e < 2; e++) {
            accrl[T][e] = __shfl_xor_sync(kFull, accr[T][e], 16);
            accnl[T][e] = __shfl_xor_sync(kFull, accn[T][e], 16);
          }
        }
        // digit dots: H in [0..1], M in [2..3] (rows g + 8), L in accrl / accnl [0..1]
        const float r0 = fmaf((float)accr[T][0], 16384.f, (float)(accr[T][2] * 128 + accrl[T][0]));
        const float r1 = fmaf((float)accr[T][1], 16384.f, (float)(accr[T][3] * 128 + accrl[T][1]));
        const float n0 = fmaf((float)accn[T][0], 16384.f, (float)(accn[T][2] * 128 + accnl[T][0]));
        const float n1 = fmaf((float)accn[T][1], 16384.f, (float)(accn[T][3] * 128 + accnl[T][1]));
        sacc[T].x = fmaf(dr.x, r0, dn.x * n0);
        sacc[T].y = fmaf(dr.y, r1, dn.y * n1);
      }
      // ---- online softmax (base 2), head g, this warp's 16 tokens
      float sc[4] = {sacc[0].x * sl, sacc[0].y * sl, sacc[1].x * sl, sacc[1].y * sl};
      if (partial) {
#pragma unroll
        for (int e = 0; e < 4; e++)
          if (!((okmask >> (8 * (e >> 1) + 2 * tg + (e & 1))) & 1u)) sc[e] = -INFINITY;
      }
      float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      if (__any_sync(kFull, mx > m_run + 8.f)) {
        const float mn = fmaxf(m_run, mx);
        const float alpha = exp2f(m_run - mn);
        m_run = mn;
        l_run *= alpha;
        // columns 2tg, 2tg + 1 belong to heads 2tg, 2tg + 1 (PACK: to heads
        // (2tg) & 3, (2tg + 1) & 3, hi in columns 0-3 and lo in 4-7)
        const int src = PACK ? 8 * (tg & 1) : 8 * tg;
        const float a0 = __shfl_sync(kFull, alpha, src);
        const float a1 = __shfl_sync(kFull, alpha, src + 4);
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
          o[mt][0] *= a0;
          o[mt][1] *= a1;
          o[mt][2] *= a0;
          o[mt][3] *= a1;
        }
      }
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        p[e] = exp2f(sc[e] - m_run);
        l_run += p[e];
      }
      // ---- PV: B = p * s_v / 64 (hi / lo), A = V^T codes through the LUT
      const float2 dv0 = *reinterpret_cast<const float2 *>(fsc + 2 * kTile + 16 * warp + 2 * tg);
      const float2 dv1 =
          *reinterpret_cast<const float2 *>(fsc + 2 * kTile + 16 * warp + 8 + 2 * tg);
      float2 w0 = make_float2(p[0] * dv0.x, p[1] * dv0.y);
      float2 w1 = make_float2(p[2] * dv1.x, p[3] * dv1.y);
      if (partial) {  // a zero-filled or unmapped row: keep its weight out exactly
        if (!((okmask >> (2 * tg)) & 1u)) w0.x = 0.f;
        if (!((okmask >> (2 * tg + 1)) & 1u)) w0.y = 0.f;
        if (!((okmask >> (8 + 2 * tg)) & 1u)) w1.x = 0.f;
        if (!((okmask >> (9 + 2 * tg)) & 1u)) w1.y = 0.f;
      }
      uint32_t bh0, bl0, bh1, bl1;
      split_hilo(w0, bh0, bl0);
      split_hilo(w1, bh1, bl1);
      if (PACK) {  // columns 4-7: the lo parts of heads 0-3 (lanes 16 apart)
        const uint32_t xl0 = __shfl_xor_sync(kFull, bl0, 16);
        const uint32_t xl1 = __shfl_xor_sync(kFull, bl1, 16);
        if (g >= 4) {
          bh0 = xl0;
          bh1 = xl1;
        }
      }
      // x2.trans: matrices (T0, chunk), (T1, chunk); lanes 0..15 give the rows
      const int vrow = 16 * warp + (lane & 15);
      const uint32_t vaddr = base + vrow * 128;
#pragma unroll
      for (int vc = 0; vc < 4; vc++) {
        uint32_t vr[2];
        if (vc == 0) {
          // joined chunk: row g < 4 <- chunk 3 element g + 4 (V bytes 2g, 2g + 1),
          // row g >= 4 <- chunk 7 element g - 4 (V bytes 48 + 2g, 49 + 2g)
          uint32_t c3[2], c7[2];
          ldsm_x2_t(vaddr + ((3 ^ (vrow & 7)) << 4), c3);
          ldsm_x2_t(vaddr + ((7 ^ (vrow & 7)) << 4), c7);
          vr[0] = __shfl_xor_sync(kFull, lane < 16 ? c7[0] : c3[0], 16);
          vr[1] = __shfl_xor_sync(kFull, lane < 16 ? c7[1] : c3[1], 16);
        } else {  // chunks 4, 5, 6: V bytes 16 vc - 8 + element
          ldsm_x2_t(vaddr + (((3 + vc) ^ (vrow & 7)) << 4), vr);
        }
#pragma unroll
        for (int par = 0; par < 2; par++) {
          // byte 2g + par of tokens (2tg, 2tg+1) [vr[0]] and (2tg+8, 2tg+9) [vr[1]]
          const uint32_t s0 = prmt(vr[0], 0u, par ? 0x0031u : 0x0020u);
          const uint32_t s1 = prmt(vr[1], 0u, par ? 0x0031u : 0x0020u);
          const uint32_t R0 = lut4_bytes(s0, U4);  // (tok a lo, tok a hi, tok b lo, tok b hi)
          const uint32_t R1 = lut4_bytes(s1, U4);
          const uint32_t a[4] = {lut_half2(R0, 0x4240u), lut_half2(R0, 0x4341u),
                                 lut_half2(R1, 0x4240u), lut_half2(R1, 0x4341u)};
          float(&acc)[4] = o[2 * vc + par];
          mma16816(acc, a, bh0, bh1);
          if (!PACK) mma16816(acc, a, bl0, bl1);
        }
      }
    }
  }
  if (TMA) {
    if (aborted) {
      // a tile never arrived: let the copies still in flight land (bounded,
      // ignoring the flag) before shared memory is reused, then write NaN
      // records, which the combine turns into NaN outputs
      if (tid == 0) {
        dec::report(err, KVQ_DEVERR_WAIT_TIMEOUT);
        for (int j = issued > kStages ? issued - kStages : 0; j < issued; j++)
          for (int i = 0; i < dec::kWaitPolls && !dec::mbar_try(full0 + 8 * (j % kStages), (j / kStages) & 1); i++) {
          }
      }
      __syncthreads();
      const float nan = __int_as_float(0x7fc00000);
      for (int p = tid; p < gc * kHead; p += kThreads) {
        const int hh = p >> 7, j = p & 127;
        float *rec = ws + (((int64_t)qi * n_q_heads + h0 + hh) * splits + s) * kORec;
        rec[4 + j] = nan;
        if (j == 0) rec[0] = rec[1] = nan;
      }
      return;
    }
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();

  // ---- merge the warps and write the partial records
  float *red_o = reinterpret_cast<float *>(smem);  // [warp][8][128]
  float *red_m = red_o + kWarps * 8 * kHead;
  float *red_l = red_m + kWarps * 8;
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  if (tg == 0) {
    red_m[warp * 8 + g] = m_run;
    red_l[warp * 8 + g] = l_run;
  }
#pragma unroll
  for (int vc = 0; vc < 4; vc++)
#pragma unroll
    for (int par = 0; par < 2; par++) {
      // V byte of row g: joined chunk -> 2g (+48 for g >= 4); chunk 3 + vc -> 16 vc - 8 + 2g
      const int vb = (vc == 0 ? (g < 4 ? 2 * g : 48 + 2 * g) : 16 * vc - 8 + 2 * g) + par;
      const int d = 8 * (vb >> 2) + (vb & 3);  // low nibble; high nibble is d + 4
      float acc[4];
#pragma unroll
      for (int e = 0; e < 4; e++) acc[e] = o[2 * vc + par][e];
      if (PACK) {  // hi (columns 0-3, tg < 2) + lo (columns 4-7, tg + 2)
#pragma unroll
        for (int e = 0; e < 4; e++) acc[e] += __shfl_xor_sync(kFull, acc[e], 2);
        if (tg >= 2) continue;
      }
      float *w = red_o + warp * 8 * kHead;
      w[(2 * tg) * kHead + d] = acc[0];
      w[(2 * tg + 1) * kHead + d] = acc[1];
      w[(2 * tg) * kHead + d + 4] = acc[2];
      w[(2 * tg + 1) * kHead + d + 4] = acc[3];
    }
  __syncthreads();
  for (int p = tid; p < gc * kHead; p += kThreads) {
    const int hh = p >> 7, j = p & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, red_m[w * 8 + hh]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = exp2f(red_m[w * 8 + hh] - M);
        L += red_l[w * 8 + hh] * f;
        O += red_o[(w * 8 + hh) * kHead + j] * f;
      }
    }
    float *rec = ws + (((int64_t)qi * n_q_heads + h0 + hh) * splits + s) * kORec;
    rec[4 + j] = O;
    if (j == 0) {
      rec[0] = M;
      rec[1] = L;
    }
  }
}

}  // namespace

bool octave_mma_supported(const OctaveParams &P) {
  return P.head_size == kHead && !P.compact && P.rope_dim == 64 && P.v_bits == 4 &&
         P.slot_bytes == 128;
}

cudaError_t launch_octave_decode_mma(const OctaveParams &P, const void *query, int bf16, int num_q,
                                     int n_q_heads, const uint8_t *cache, int n_kv_heads,
                                     int block_size, int64_t num_blocks,
                                     const int32_t *block_table, int num_reqs, int max_blocks,
                                     const int32_t *q_to_req, const int32_t *q_to_klen,
                                     int max_klen, float scale, float *ws,
                                     const DecodePlan &plan, cudaStream_t s) {
  const int group = n_q_heads / n_kv_heads;
  const int gc = group < 8 ? group : 8;
  dim3 grid(plan.splits, n_q_heads / gc, num_q);
  const float sl2 = scale * kLog2e;
  // one 64-row tensor copy per tile when every tile lies in one block (block
  // sizes that are multiples of 64; the splits are whole 64-token tiles) and
  // the slot rows fit the map's 32-bit coordinate
  const int64_t rows = num_blocks * n_kv_heads * block_size;
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  const bool tma = block_size % kTile == 0 && plan.split_tokens % kTile == 0 && rows > 0 &&
                   rows < (int64_t{1} << 31) &&
                   dec::make_map(&map, cache, (uint64_t)rows, 128, 128, kTile, true);
  const int idx = (bf16 ? 4 : 0) + (gc <= 4 ? 2 : 0) + (tma ? 1 : 0);
  auto fn = octave_decode_mma_kernel<false, false, false>;
  switch (idx) {
    case 1: fn = octave_decode_mma_kernel<false, false, true>; break;
    case 2: fn = octave_decode_mma_kernel<false, true, false>; break;
    case 3: fn = octave_decode_mma_kernel<false, true, true>; break;
    case 4: fn = octave_decode_mma_kernel<true, false, false>; break;
    case 5: fn = octave_decode_mma_kernel<true, false, true>; break;
    case 6: fn = octave_decode_mma_kernel<true, true, false>; break;
    case 7: fn = octave_decode_mma_kernel<true, true, true>; break;
    default: break;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, fn, map, wait_poll_limit(), P, query, n_q_heads, group, gc, cache, n_kv_heads,
      block_size, num_blocks, block_table, num_reqs, max_blocks, q_to_req, q_to_klen, max_klen,
      sl2, plan.split_tokens, plan.splits, ws, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvq
