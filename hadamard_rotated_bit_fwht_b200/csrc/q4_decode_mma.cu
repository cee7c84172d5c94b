// q4_decode_mma.cu -- tensor-core split-K decode attention over the Q4_0 +
// FWHT-256 cache (Strata PR #21 "Q4_0 KV cache + FWHT-256": What, How 2 and the
// merge note's per-token path that rotates Q and the output).
//
// With GQA the decode step is a small dense contraction per kv head:
// S = Q_rot K^T (G x T) and O = P V (G x 256).  At G = 8 fp32 FMAs alone would
// cap the kernel near a third of HBM bandwidth, so both products run on the
// tensor cores (warp-level mma.sync m16n8k16, fp16 inputs, fp32 accumulation)
// while keeping fp32-level accuracy:
//   * The nibble codes enter the MMA as exact fp16 values 64 + c: a nibble
//     sitting in bits 4..7 of a 16-bit lane, OR-ed with the bits of 64.0
//     (0x5400), is that value -- one LOP3 per pair, no conversion
//     instruction.  The bias 64 + 8 = 72 is removed in fp32: for scores,
//     72 * sum(q) per (head, block); for outputs, 72 * sum_t(p d_v) per
//     (head, block), accumulated alongside and subtracted once at the end.
//   * The query is split into fp16 hi + lo parts that fill the 16 M-rows of
//     the QK MMA (rows 0-7 hi, rows 8-15 lo of the 8 heads), so a head's score
//     is c0 + c2 of the accumulator and carries ~22 mantissa bits.  The query
//     fragments live in shared memory in ldmatrix order.
//   * The per-block Q4_0 scale depends on (token, block), so each 32-dim
//     block has its own fresh QK accumulator, scaled by the block's scale in
//     fp32 and added to the score.
//   * PV: A = V^T codes (dims x tokens, exact), B = p * d_v (token x head)
//     split hi + lo; the 16 dims of one M-tile lie in one block, so the V
//     scale rides in B.
//   * The QK accumulator layout (head g = lane / 4, tokens 2(lane % 4) + {0,1})
//     is exactly the PV B-fragment layout for tokens {0..7} and {8..15}, so no
//     data moves between the two products.
// Memory path: 64-token tiles of codes (rows of 128 bytes) and scales are
// staged by cp.async into a 3-stage shared-memory ring; code rows are stored
// with the 128-byte XOR swizzle (16-byte chunk c of row r at c ^ (r & 7)) so
// ldmatrix (K) and ldmatrix.trans (V) are conflict-free; the scales of the
// current tile are widened to fp32 once.  Three CTAs of four warps per SM.
// Online softmax in base 2 with a lazily updated reference maximum (rescale
// only when a score exceeds it by 8), split-K partials (m, l, o[256]) per
// (sequence, q head, split), and the combine + back-rotation kernel.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 64;          // tokens per pipeline stage (16 per warp)
constexpr int kStages = 3;
constexpr int kCtasPerSm = 3;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kRec = 260;          // partial record: m, l, pad, pad, o[256]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kBias = 72.f;      // 64 (magic) + 8 (Q4_0 zero point)

// shared memory layout (bytes)
constexpr int kOffKC = 0;                       // K codes: 64 rows x 128 B, swizzled
constexpr int kOffVC = kOffKC + kTile * 128;    // V codes
constexpr int kOffKS = kOffVC + kTile * 128;    // K scales: 64 rows x 8 fp16
constexpr int kOffVS = kOffKS + kTile * 16;     // V scales
constexpr int kStageBytes = kOffVS + kTile * 16;
constexpr int kOffF = kStages * kStageBytes;    // fp32 scales of the current tile [kv][block][token]
constexpr int kOffQ = kOffF + 2 * 8 * kTile * 4;  // query fragments: 16 tiles of 16x16 fp16
constexpr int kSmemBytes = kOffQ + 16 * 512;

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
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// nibbles at bits 4..7 and 20..23 of x -> half2 (64 + c) exactly
__device__ __forceinline__ uint32_t nib64(uint32_t x) {
  uint32_t h;
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(h) : "r"(x));  // (x & m) | c
  return h;
}

// fp32 pair -> fp16 hi + lo pairs (w ~= hi + lo to ~22 bits)
__device__ __forceinline__ void split_hilo(float2 w, uint32_t &hi, uint32_t &lo) {
  __half2 h = __float22half2_rn(w);
  float2 hf = __half22float2(h);
  __half2 l = __float22half2_rn(make_float2(w.x - hf.x, w.y - hf.y));
  hi = *reinterpret_cast<uint32_t *>(&h);
  lo = *reinterpret_cast<uint32_t *>(&l);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  return __ffma2_rn(a, b, c);
}

// byte offset of element (row, col) of one 16x16 fp16 query-fragment tile;
// the 16-byte halves are XOR-swizzled with bit 2 of the row so the eight rows
// read by one ldmatrix phase fall in distinct banks
__device__ __forceinline__ int qfrag_off(int row, int col) {
  return row * 32 + (((col >> 3) ^ ((row >> 2) & 1)) << 4) + (col & 7) * 2;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    q4_decode_mma_kernel(kvq_cache c, const void *__restrict__ q,
                         const int32_t *__restrict__ seq_lens, int max_seq_len, int n_q_heads,
                         int group, int gc, float scale_log2, int split_tokens, int splits,
                         float *__restrict__ ws) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int s = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int h0 = hg * gc, kvh = h0 / group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  const int cap = c.block_table ? c.max_pages_per_seq * c.page_size : c.max_tokens;
  const int len = min(max(__ldg(seq_lens + b), 0), min(max_seq_len, cap));
  const int t0 = s * split_tokens;
  const int t1 = min(len, t0 + split_tokens);
  const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;

  // ---- query: rotate (FWHT-256 in shared memory), split hi/lo into fragments
  float *qs = reinterpret_cast<float *>(smem);  // [8][256] in the ring, before it is used
  for (int p = tid; p < 8 * kDim; p += kThreads) {
    const int hh = p >> 8, j = p & 255;
    float v = 0.f;
    if (hh < gc) {
      const int64_t off = ((int64_t)b * n_q_heads + h0 + hh) * kDim + j;
      v = BF16 ? __uint_as_float((uint32_t)static_cast<const uint16_t *>(q)[off] << 16)
               : static_cast<const float *>(q)[off];
    }
    qs[p] = v;
  }
  for (int h = 1; h < kDim; h <<= 1) {
    __syncthreads();
    for (int p = tid; p < 8 * 128; p += kThreads) {
      const int vv = p >> 7, pi = p & 127;
      const int i0 = ((pi / h) * 2 * h) + (pi % h);
      float *y = qs + vv * kDim;
      const float a = y[i0], bb = y[i0 + h];
      y[i0] = a + bb;
      y[i0 + h] = a - bb;
    }
  }
  __syncthreads();
  // Fragment tile (bb, kk) row r: hi (r < 8) or lo (r >= 8) of head r & 7;
  // column k <-> dim 32bb + 16kk + 4((k & 7) >> 1) + (k >> 3) + 2(k & 1).
  // q_rot = FWHT / 16 is of order one, so its split stays in the normal fp16
  // range; scale * log2(e) is applied to the scores.
  uint8_t *qf = smem + kOffQ;
  for (int p = tid; p < 16 * 8 * 16; p += kThreads) {  // (tile, head, col) for hi and lo
    const int tile = p >> 7, hh = (p >> 4) & 7, k = p & 15;
    const int bb = tile >> 1, kk = tile & 1;
    const int dim = 32 * bb + 16 * kk + 4 * ((k & 7) >> 1) + (k >> 3) + 2 * (k & 1);
    const float x = qs[hh * kDim + dim] * 0.0625f;
    const __half hi = __float2half_rn(x);
    const __half lo = __float2half_rn(x - __half2float(hi));
    *reinterpret_cast<__half *>(qf + tile * 512 + qfrag_off(hh, k)) = hi;
    *reinterpret_cast<__half *>(qf + tile * 512 + qfrag_off(hh + 8, k)) = lo;
  }
  // bias correction of the scores: 72 * sum over each block of (hi + lo), one
  // thread per (head, block), into shared memory
  float *sqs = reinterpret_cast<float *>(smem + kOffF);  // reused by the scale widening later
  if (tid < 64) {
    const int hh = tid >> 3, bb = tid & 7;
    const float *qr = qs + hh * kDim + 32 * bb;
    float a = 0.f;
    for (int j = 0; j < 32; j++) {
      const float x = qr[(j + tid) & 31] * 0.0625f;  // rotated start: spreads the banks
      const __half hi = __float2half_rn(x);
      const __half lo = __float2half_rn(x - __half2float(hi));
      a += __half2float(hi) + __half2float(lo);
    }
    sqs[tid] = kBias * a;
  }
  __syncthreads();
  float sqb[8];
#pragma unroll
  for (int bb = 0; bb < 8; bb++) sqb[bb] = sqs[g * 8 + bb];
  __syncthreads();  // qs (ring area) is overwritten by the loads below

  // ---- tile loader
  auto tile_row0 = [&](int tstart) -> int64_t {  // first cache row of the tile, -1 if unmapped
    if (c.block_table == nullptr) return ((int64_t)b * c.num_kv_heads + kvh) * c.max_tokens + tstart;
    const int pi = tstart / c.page_size;
    const int page = __ldg(c.block_table + (int64_t)b * c.max_pages_per_seq + pi);
    if (page < 0 || page >= c.num_pages) return -1;
    return ((int64_t)page * c.num_kv_heads + kvh) * c.page_size + (tstart - pi * c.page_size);
  };
  auto issue = [&](int it) {
    uint8_t *st = smem + (it % kStages) * kStageBytes;
    const int tstart = t0 + it * kTile;
    const int64_t row0 = tile_row0(tstart);
    const int nvalid = row0 < 0 ? 0 : min(kTile, t1 - tstart);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int idx = tid + kThreads * i;  // 0..511
      const int r = idx >> 3, ch = idx & 7;
      const bool ok = r < nvalid;
      const int64_t row = ok ? row0 + r : 0;
      const uint32_t so = r * 128 + ((ch ^ (r & 7)) << 4);
      cp_async16(smem_u32(st + kOffKC + so), c.k_codes + row * 128 + ch * 16, ok);
      cp_async16(smem_u32(st + kOffVC + so), c.v_codes + row * 128 + ch * 16, ok);
    }
    {
      const int r = tid & 63;
      const bool ok = r < nvalid;
      const int64_t row = ok ? row0 + r : 0;
      if (tid < 64) cp_async16(smem_u32(st + kOffKS + r * 16), c.k_scales + row * 8, ok);
      else cp_async16(smem_u32(st + kOffVS + r * 16), c.v_scales + row * 8, ok);
    }
  };

  float o[16][4];
#pragma unroll
  for (int mt = 0; mt < 16; mt++) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float swb[8];  // sum over tokens of p * d_v, per block, for head g
#pragma unroll
  for (int bb = 0; bb < 8; bb++) swb[bb] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  const uint32_t qbase = smem_u32(qf);
  // ldmatrix.x4 lane address inside a query tile: matrix m = lane / 8 gives
  // (rows 8 * (m & 1) + lane % 8, 16-byte half m >> 1)
  const int qrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const uint32_t qlane = qrow * 32 + ((((lane >> 4) & 1) ^ ((qrow >> 2) & 1)) << 4);
  float *fsc = reinterpret_cast<float *>(smem + kOffF);

#pragma unroll
  for (int i = 0; i < kStages - 1; i++) {
    if (i < ntiles) issue(i);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; it++) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    uint8_t *st = smem + (it % kStages) * kStageBytes;
    {  // widen the scales of this tile to fp32: [kv][block][token]
      const int r = tid & 63, kv = tid >> 6;
      const uint4 w = *reinterpret_cast<const uint4 *>(st + (kv ? kOffVS : kOffKS) + r * 16);
      float *f = fsc + kv * 8 * kTile;
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k2 = 0; k2 < 4; k2++) {
        const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&ww[k2]));
        f[(2 * k2) * kTile + r] = p.x;
        f[(2 * k2 + 1) * kTile + r] = p.y;
      }
    }
    if (it + kStages - 1 < ntiles) issue(it + kStages - 1);
    cp_async_commit();
    __syncthreads();

    const int tstart = t0 + it * kTile;
    // tokens of this warp's 16; a tile on an unmapped page contributes nothing
    const int live = tile_row0(tstart) < 0 ? 0 : min(kTile, t1 - tstart) - 16 * warp;
    if (live > 0) {
      const uint32_t kbase = smem_u32(st + kOffKC), vbase = smem_u32(st + kOffVC);
      const float *fk = fsc + 16 * warp + 2 * tg;
      const float *fv = fk + 8 * kTile;
      // ldmatrix row address of this lane in a code tile: matrix m = lane / 8
      // -> (token group T = m & 1, block offset m >> 1), row = lane % 8
      const int mr = 16 * warp + 8 * ((lane >> 3) & 1) + (lane & 7);
      const int mb = lane >> 4;
      // ---- QK
      float2 sacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int bp = 0; bp < 4; bp++) {
        uint32_t kr[4];
        const int blk = 2 * bp + mb;
        ldsm_x4(kbase + mr * 128 + ((blk ^ (mr & 7)) << 4), kr);
#pragma unroll
        for (int half = 0; half < 2; half++) {
          const int bb = 2 * bp + half;
          uint32_t qa0[4], qa1[4];
          ldsm_x4(qbase + (2 * bb) * 512 + qlane, qa0);
          ldsm_x4(qbase + (2 * bb + 1) * 512 + qlane, qa1);
#pragma unroll
          for (int T = 0; T < 2; T++) {
            const uint32_t w = kr[2 * half + T];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            // chunk 0: low nibbles of bytes (0, 2) and (1, 3); chunk 1: high nibbles
            mma16816(acc, qa0, nib64(w << 4), nib64(w >> 4));
            mma16816(acc, qa1, nib64(w), nib64(w >> 8));
            const float2 d = *reinterpret_cast<const float2 *>(fk + bb * kTile + 8 * T);
            const float2 hl = make_float2(acc[0] + acc[2] - sqb[bb], acc[1] + acc[3] - sqb[bb]);
            sacc[T] = ffma2(d, hl, sacc[T]);
          }
        }
      }
      // ---- online softmax (base 2) for head g over this warp's 16 tokens
      const float2 sl2 = make_float2(scale_log2, scale_log2);
      const float2 s0 = __fmul2_rn(sacc[0], sl2), s1 = __fmul2_rn(sacc[1], sl2);
      float sc[4] = {s0.x, s0.y, s1.x, s1.y};
      if (live < 16) {
#pragma unroll
        for (int e = 0; e < 4; e++)
          if (8 * (e >> 1) + 2 * tg + (e & 1) >= live) sc[e] = -INFINITY;
      }
      float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      if (__any_sync(kFull, mx > m_run + 8.f)) {
        const float mn = fmaxf(m_run, mx);
        const float alpha = exp2f(m_run - mn);  // 0 while m_run is -inf
        m_run = mn;
        l_run *= alpha;
#pragma unroll
        for (int bb = 0; bb < 8; bb++) swb[bb] *= alpha;
        const float a0 = __shfl_sync(kFull, alpha, 8 * tg);      // head 2tg
        const float a1 = __shfl_sync(kFull, alpha, 8 * tg + 4);  // head 2tg + 1
#pragma unroll
        for (int mt = 0; mt < 16; mt++) {
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
      const float2 p01 = make_float2(p[0], p[1]), p23 = make_float2(p[2], p[3]);
      // ---- PV: per block, B = p * d_v (hi / lo), A = V^T codes
#pragma unroll
      for (int bp = 0; bp < 4; bp++) {
        uint32_t vr[4];
        const int blk = 2 * bp + mb;
        ldsm_x4_t(vbase + mr * 128 + ((blk ^ (mr & 7)) << 4), vr);
#pragma unroll
        for (int half = 0; half < 2; half++) {
          const int bb = 2 * bp + half;
          float2 w0 = __fmul2_rn(p01, *reinterpret_cast<const float2 *>(fv + bb * kTile));
          float2 w1 = __fmul2_rn(p23, *reinterpret_cast<const float2 *>(fv + bb * kTile + 8));
          if (live < 16) {  // tokens past the end: p is 0, keep a stale scale out too
            if (2 * tg >= live) w0.x = 0.f;
            if (2 * tg + 1 >= live) w0.y = 0.f;
            if (8 + 2 * tg >= live) w1.x = 0.f;
            if (9 + 2 * tg >= live) w1.y = 0.f;
          }
          swb[bb] += (w0.x + w0.y) + (w1.x + w1.y);
          uint32_t bh0, bl0, bh1, bl1;
          split_hilo(w0, bh0, bl0);
          split_hilo(w1, bh1, bl1);
          const uint32_t r0 = vr[2 * half], r1 = vr[2 * half + 1];  // tokens 0-7, 8-15
          {  // even M-tile: rows g <-> low nibble of byte 2g, rows g + 8 <-> its high nibble
            const uint32_t a[4] = {nib64(r0 << 4), nib64(r0), nib64(r1 << 4), nib64(r1)};
            float(&acc)[4] = o[2 * bb];
            mma16816(acc, a, bh0, bh1);
            mma16816(acc, a, bl0, bl1);
          }
          {  // odd M-tile: byte 2g + 1
            const uint32_t a[4] = {nib64(r0 >> 4), nib64(r0 >> 8), nib64(r1 >> 4),
                                   nib64(r1 >> 8)};
            float(&acc)[4] = o[2 * bb + 1];
            mma16816(acc, a, bh0, bh1);
            mma16816(acc, a, bl0, bl1);
          }
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- remove the 72 * sum(p d_v) bias, merge the four warps, write partials
#pragma unroll
  for (int bb = 0; bb < 8; bb++) {
    swb[bb] += __shfl_xor_sync(kFull, swb[bb], 1);
    swb[bb] += __shfl_xor_sync(kFull, swb[bb], 2);
  }
  float *red_o = reinterpret_cast<float *>(smem);            // [warp][8 heads][256]
  float *red_m = red_o + kWarps * 8 * kDim;                 // [warp][8]
  float *red_l = red_m + kWarps * 8;
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  if (tg == 0) {
    red_m[warp * 8 + g] = m_run;
    red_l[warp * 8 + g] = l_run;
  }
#pragma unroll
  for (int bb = 0; bb < 8; bb++) {
    const float c0 = kBias * __shfl_sync(kFull, swb[bb], 8 * tg);      // head 2tg
    const float c1 = kBias * __shfl_sync(kFull, swb[bb], 8 * tg + 4);  // head 2tg + 1
#pragma unroll
    for (int par = 0; par < 2; par++) {
      const float(&acc)[4] = o[2 * bb + par];
      const int d0 = 32 * bb + 2 * g + par;  // dim of row g; row g + 8 is d0 + 16
      float *w = red_o + warp * 8 * kDim;
      w[(2 * tg) * kDim + d0] = acc[0] - c0;
      w[(2 * tg + 1) * kDim + d0] = acc[1] - c1;
      w[(2 * tg) * kDim + d0 + 16] = acc[2] - c0;
      w[(2 * tg + 1) * kDim + d0 + 16] = acc[3] - c1;
    }
  }
  __syncthreads();
  for (int p = tid; p < gc * kDim; p += kThreads) {
    const int hh = p >> 8, j = p & 255;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, red_m[w * 8 + hh]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float f = exp2f(red_m[w * 8 + hh] - M);
        L += red_l[w * 8 + hh] * f;
        O += red_o[(w * 8 + hh) * kDim + j] * f;
      }
    }
    float *rec = ws + (((int64_t)b * n_q_heads + h0 + hh) * splits + s) * kRec;
    rec[4 + j] = O;
    if (j == 0) {
      rec[0] = M;
      rec[1] = L;
    }
  }
}

}  // namespace

int q4_decode_ctas_per_sm() { return kCtasPerSm; }

cudaError_t launch_q4_decode_mma(const kvq_cache &c, const void *q, int bf16, int batch,
                                 int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                                 float scale, float *ws, const DecodePlan &p, cudaStream_t s) {
  const int group = n_q_heads / c.num_kv_heads;
  const int gc = group < 8 ? group : 8;
  dim3 grid(p.splits, n_q_heads / gc, batch);
  const float sl2 = scale * kLog2e;
  // opt in to the large dynamic shared-memory carve-out once per device
  static unsigned configured[2] = {0u, 0u};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned bit = 1u << (dev & 31);
  if (!(configured[bf16] & bit)) {
    e = bf16 ? cudaFuncSetAttribute(q4_decode_mma_kernel<true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)
             : cudaFuncSetAttribute(q4_decode_mma_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[bf16] |= bit;
  }
  if (bf16)
    q4_decode_mma_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(
        c, q, seq_lens, max_seq_len, n_q_heads, group, gc, sl2, p.split_tokens, p.splits, ws);
  else
    q4_decode_mma_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(
        c, q, seq_lens, max_seq_len, n_q_heads, group, gc, sl2, p.split_tokens, p.splits, ws);
  return cudaGetLastError();
}

}  // namespace kvq
