// q4_decode_mma.cu -- tensor-core split-K decode attention over the Q4_0 +
// FWHT-256 cache (Strata PR #21 "Q4_0 KV cache + FWHT-256": What, How 2 and the
// merge note's per-token path that rotates Q and the output).
//
// With GQA the decode step is a small dense contraction per kv head:
// S = Q_rot K^T (G x T) and O = P V (G x 256), G <= 8 heads per CTA.  Both
// products run on the tensor cores (warp-level mma.sync) at fp32-level
// accuracy; a CTA of four warps walks its split in 64-token tiles:
//   * Tiles arrive by TMA (cp.async.bulk.tensor, 2-D maps over the cache's
//     128-byte code rows and 16-byte scale rows, hardware 128-byte swizzle)
//     into a ring of shared-memory stages guarded by mbarriers; one thread
//     issues, every wait is bounded.
//   * QK: warp w scores tokens 16w..16w+15 of the tile for all 8 heads on the
//     integer tensor path (m16n8k32, s8 x u8 -> s32).  A Q4_0 block is 32
//     dims, one MMA K-step; its codes enter as bytes with three logic ops per
//     8 codes (low nibbles = dims 0..15, high nibbles = dims 16..31 of the
//     block, the B-fragment rows).  The rotated query of each head is scaled
//     by S = 127 * 2^14 / max|q| and split exactly into int8 levels H, M, L
//     with S q = 2^14 H + 2^7 M + L (|M|, |L| <= 64); one MMA takes H and M
//     (rows 0-7, 8-15), a second takes L.  Their accumulators start at the
//     bits of 1.5 * 2^23 minus the zero-point term 8 * sum(level), so each
//     exact integer sum over the block becomes an fp32 by one subtraction;
//     2^7 F_HM + F_L times the block's scale is added to the score.  The
//     query is carried to about 2^-22 of its largest element.
//   * Softmax: the tile maximum per head is shared through shared memory, so
//     every warp keeps the same running maximum (rescaling lazily, only when
//     a score passes it by 8); p goes to shared memory.
//   * PV: warp w owns output dims 64w..64w+63 (Q4_0 blocks 2w, 2w+1) for all
//     64 tokens of the tile: A = V^T codes as the exact fp16 values 64 + c (a
//     nibble in bits 4..7 of a 16-bit lane OR-ed with the bits of 64.0, one
//     LOP3 per pair, read by ldmatrix.trans), B = p * d_v split into fp16
//     hi + lo (the 16 dims of an M-tile lie in one block, so the V scale rides
//     in B).  The bias 64 + 8 = 72 is removed at the end with
//     72 * sum_t(p d_v) per (head, block).
//   * The QK accumulator layout (head g = lane / 4, tokens 2(lane % 4) + {0,1})
//     is the PV B-fragment layout for tokens {0..7} and {8..15}.
// Split-K partials (m, l, o[256]) per (sequence, q head, split) go to the
// combine + back-rotation kernel.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 64;          // tokens per stage (16 per warp for QK)
constexpr int kStages = 2;
constexpr int kCtasPerSm = 4;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kRec = 260;          // partial record: m, l, pad, pad, o[256]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kBias = 72.f;      // 64 (magic) + 8 (Q4_0 zero point)
constexpr float kQRange = 2080768.f;         // 127 * 2^14
constexpr uint32_t kTileBytes = 2 * kTile * 128 + 2 * kTile * 16;  // one TMA transaction

// shared memory layout (bytes from a 1024-aligned base: 128-byte swizzle atoms)
constexpr int kOffKC = 0;                       // K codes: 64 rows x 128 B (TMA-swizzled)
constexpr int kOffVC = kOffKC + kTile * 128;    // V codes
constexpr int kOffKS = kOffVC + kTile * 128;    // K scales: 64 rows x 8 fp16
constexpr int kOffVS = kOffKS + kTile * 16;     // V scales
constexpr int kStageBytes = kOffVS + kTile * 16;  // 18432 = 18 KiB
constexpr int kOffF = kStages * kStageBytes;    // fp32 scales, 2 buffers x [kv][block][token]
constexpr int kFBuf = 2 * 8 * kTile;            // floats per buffer
constexpr int kPStride = 72;                    // p rows: 64 tokens + pad (conflict-free)
constexpr int kOffP = kOffF + 2 * kFBuf * 4;    // p [8 heads][kPStride] fp32
constexpr int kOffRed = kOffP + 8 * kPStride * 4;  // tile maxima [warp][8], then l [warp][8]
constexpr int kQStride = 272;                   // int8 query row: 256 B + 16 B pad
constexpr int kOffQ = kOffRed + 2 * kWarps * 8 * 4;  // rows 0-7 H, 8-15 M, 16-23 L
constexpr int kOffZ = kOffQ + 24 * kQStride;    // 16 zero bytes (ldmatrix rows of zeros)
constexpr int kOffBar = kOffZ + 16;             // mbarriers, 8 B each
constexpr int kSmemUsed = kOffBar + kStages * 8;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kStageBytes % 1024 == 0, "stages must keep the swizzle atoms aligned");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

// bounded waits: ~2^20 polls of up to ~1 us each
constexpr int kWaitPolls = 1 << 20;

struct TmaMaps {
  CUtensorMap kc, vc, ks, vs;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// true once the phase with this parity has completed; false after the poll limit
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (int i = 0; i < kWaitPolls; i++) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    if (done) return true;
  }
  return false;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
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
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d = A(s8, 16 x 32) * B(u8, 32 x 8), accumulating from zero
__device__ __forceinline__ void imma16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "n"(0));
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

template <bool BF16>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    q4_decode_mma_kernel(const __grid_constant__ TmaMaps maps, kvq_cache c,
                         const void *__restrict__ q, const int32_t *__restrict__ seq_lens,
                         int max_seq_len, int n_q_heads, int group, int gc, float scale_log2,
                         int split_tokens, int splits, float *__restrict__ ws) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int s = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int h0 = hg * gc, kvh = h0 / group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  const int cap = c.block_table ? c.max_pages_per_seq * c.page_size : c.max_tokens;
  const int len = min(max(__ldg(seq_lens + b), 0), min(max_seq_len, cap));
  const int t0 = s * split_tokens;
  const int t1 = min(len, t0 + split_tokens);
  const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
  const uint32_t bar0 = smem_u32(smem + kOffBar);

  // first cache row of a tile, -1 if its page is unmapped
  auto tile_row0 = [&](int tstart) -> int64_t {
    if (c.block_table == nullptr) return ((int64_t)b * c.num_kv_heads + kvh) * c.max_tokens + tstart;
    const int pi = tstart / c.page_size;
    const int page = __ldg(c.block_table + (int64_t)b * c.max_pages_per_seq + pi);
    if (page < 0 || page >= c.num_pages) return -1;
    return ((int64_t)page * c.num_kv_heads + kvh) * c.page_size + (tstart - pi * c.page_size);
  };
  // one thread: a whole tile (codes + scales of K and V) onto the stage's barrier
  auto issue = [&](int it) {
    const int st = it % kStages;
    const uint32_t bar = bar0 + 8 * st;
    const int64_t row0 = tile_row0(t0 + it * kTile);
    if (row0 < 0) {  // nothing to load: complete the phase without bytes
      mbar_arrive(bar);
      return;
    }
    const uint32_t dst = smem_u32(smem + st * kStageBytes);
    mbar_arrive_tx(bar, kTileBytes);
    tma_load_2d(dst + kOffKC, &maps.kc, 0, (int)row0, bar);
    tma_load_2d(dst + kOffVC, &maps.vc, 0, (int)row0, bar);
    tma_load_2d(dst + kOffKS, &maps.ks, 0, (int)row0, bar);
    tma_load_2d(dst + kOffVS, &maps.vs, 0, (int)row0, bar);
  };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kStages; i++) mbar_init(bar0 + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }

  // ---- query: rotate (FWHT-256 in shared memory), then int8 H / M / L rows
  float *qs = reinterpret_cast<float *>(smem);  // [8][256] in the stages, before any load
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
  float *red = reinterpret_cast<float *>(smem + kOffRed);
#pragma unroll
  for (int i = 0; i < 2; i++) {  // warp w: max |FWHT(q)| of heads 2w, 2w + 1
    const int hh = 2 * warp + i;
    float m = 0.f;
    for (int j = lane; j < kDim; j += 32) m = fmaxf(m, fabsf(qs[hh * kDim + j]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    if (lane == 0) red[hh] = m;
  }
  __syncthreads();
  uint8_t *qi = smem + kOffQ;
  for (int p = tid; p < 8 * kDim; p += kThreads) {
    const int hh = p >> 8, j = p & 255;
    const float m = red[hh];
    const float x = m > 0.f ? qs[p] * (kQRange / m) : 0.f;  // |x| <= 127 * 2^14 (+ rounding)
    const float hi = rintf(x * (1.f / 16384.f));
    const float r = x - 16384.f * hi;          // exact, |r| <= 2^13
    const float mid = rintf(r * (1.f / 128.f));
    const float lo = rintf(r - 128.f * mid);   // exact difference, |lo| <= 64
    qi[hh * kQStride + j] = (uint8_t)(int8_t)(int)hi;
    qi[(8 + hh) * kQStride + j] = (uint8_t)(int8_t)(int)mid;
    qi[(16 + hh) * kQStride + j] = (uint8_t)(int8_t)(int)lo;
  }
  if (tid < 4) reinterpret_cast<uint32_t *>(smem + kOffZ)[tid] = 0u;
  __syncthreads();
  // zero-point term of head g, block bb: 8 * sum over the block of 2^14 H + 2^7 M + L
  int bq[8];
#pragma unroll
  for (int bb = 0; bb < 8; bb++) {
    // lane (g, tg) sums dims 32 bb + 8 tg .. + 7, then the 4 lanes of head g combine
    int acc = 0;
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const int d = 32 * bb + 8 * tg + j;
      acc += 16384 * (int)(int8_t)qi[g * kQStride + d] + 128 * (int)(int8_t)qi[(8 + g) * kQStride + d] +
             (int)(int8_t)qi[(16 + g) * kQStride + d];
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    bq[bb] = 8 * acc;
  }
  // A fragments of block bb: rows 0-15 (H, M) by ldmatrix.x4; L rows with a
  // zero row in place of rows 8-15, also by ldmatrix.x4 (bytes 32 bb + 0..15,
  // + 16..31)
  uint32_t qhm[8][4];
  const uint32_t zrow = smem_u32(smem + kOffZ);
  const uint32_t qla = ((lane >> 3) & 1) ? zrow : smem_u32(qi) + (16 + (lane & 7)) * kQStride + 16 * (lane >> 4);
  const uint32_t qlstep = ((lane >> 3) & 1) ? 0u : 32u;
  {
    const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
    const uint32_t a4 = smem_u32(qi) + row * kQStride + 16 * (lane >> 4);
#pragma unroll
    for (int bb = 0; bb < 8; bb++) ldsm_x4(a4 + 32 * bb, qhm[bb]);
  }
  // score scale for head g: max / (16 * 127 * 2^14) undoes S and the FWHT's 1 / 16
  const float sl2 = scale_log2 * (red[g] * (0.0625f / kQRange));
  __syncthreads();  // qs, red are reused below; the barriers are initialised

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kStages - 1; i++)
      if (i < ntiles) issue(i);
  }

  float o[4][4];  // M-tiles: block 2w + (mt >> 1), parity mt & 1
#pragma unroll
  for (int mt = 0; mt < 4; mt++) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float swb[2] = {0.f, 0.f};  // sum over this lane's tokens of p * d_v, head g, blocks 2w, 2w+1
  float m_run = -INFINITY, l_run = 0.f;  // head g; m_run is the same in every warp
  float *pbuf = reinterpret_cast<float *>(smem + kOffP);
  bool failed = false;

  for (int it = 0; it < ntiles; it++) {
    const int st = it % kStages;
    uint8_t *stage = smem + st * kStageBytes;
    const int tstart = t0 + it * kTile;
    const bool tile_ok = tile_row0(tstart) >= 0;
    const int nvalid = min(kTile, t1 - tstart);
    if (!mbar_wait(bar0 + 8 * st, (it / kStages) & 1)) failed = true;
    float *fsc = reinterpret_cast<float *>(smem + kOffF) + (it & 1) * kFBuf;
    {  // widen this tile's scales to fp32 [kv][block][token]; rows past the end are 0
      const int r = tid & 63, kv = tid >> 6;
      const uint4 w = *reinterpret_cast<const uint4 *>(stage + (kv ? kOffVS : kOffKS) + r * 16);
      const bool ok = r < nvalid;
      float *f = fsc + kv * 8 * kTile;
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k2 = 0; k2 < 4; k2++) {
        const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&ww[k2]));
        f[(2 * k2) * kTile + r] = ok ? p.x : 0.f;
        f[(2 * k2 + 1) * kTile + r] = ok ? p.y : 0.f;
      }
    }
    // (1) scales widened; every warp is done with tile it - 1; a failed wait
    // anywhere stops the whole CTA
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    if (tid == 0 && it + kStages - 1 < ntiles) issue(it + kStages - 1);
    if (!tile_ok) continue;  // uniform across the CTA

    // ---- QK: warp w, tokens 16w .. 16w + 15
    const uint32_t kbase = smem_u32(stage + kOffKC), vbase = smem_u32(stage + kOffVC);
    const int live = nvalid - 16 * warp;  // tokens of this warp's 16 inside the split
    float2 sacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    {
      const float *fk = fsc + 16 * warp + 2 * tg;
      // ldmatrix: matrix m = lane / 8 -> (token group T = m & 1, block offset m >> 1)
      const int mr = 16 * warp + 8 * ((lane >> 3) & 1) + (lane & 7);
      const int mb = lane >> 4;
#pragma unroll
      for (int bp = 0; bp < 4; bp++) {
        uint32_t kr[4];
        ldsm_x4(kbase + mr * 128 + (((2 * bp + mb) ^ (mr & 7)) << 4), kr);
#pragma unroll
        for (int half = 0; half < 2; half++) {
          const int bb = 2 * bp + half;
          uint32_t ql[4];
          ldsm_x4(qla + qlstep * bb, ql);
#pragma unroll
          for (int T = 0; T < 2; T++) {
            const uint32_t w = kr[2 * half + T];
            const uint32_t b0 = w & 0x0F0F0F0Fu, b1 = (w >> 4) & 0x0F0F0F0Fu;
            int dhm[4], dl[4];
            imma16832(dhm, qhm[bb], b0, b1);
            imma16832(dl, ql, b0, b1);
            // sum over the block of (2^14 H + 2^7 M + L)(c - 8), exact in int32
            const int t0 = (dhm[0] << 14) + ((dhm[2] << 7) + dl[0]) - bq[bb];
            const int t1 = (dhm[1] << 14) + ((dhm[3] << 7) + dl[1]) - bq[bb];
            const float2 d = *reinterpret_cast<const float2 *>(fk + bb * kTile + 8 * T);
            sacc[T] = __ffma2_rn(d, make_float2((float)t0, (float)t1), sacc[T]);
          }
        }
      }
    }
    // ---- softmax: tile maximum per head across the four warps
    float sc[4] = {sacc[0].x * sl2, sacc[0].y * sl2, sacc[1].x * sl2, sacc[1].y * sl2};
    if (live < 16) {
#pragma unroll
      for (int e = 0; e < 4; e++)
        if (8 * (e >> 1) + 2 * tg + (e & 1) >= live) sc[e] = -INFINITY;
    }
    float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    if (tg == 0) red[warp * 8 + g] = mx;
    __syncthreads();  // (2)
    const float mt_ = fmaxf(fmaxf(red[g], red[8 + g]), fmaxf(red[16 + g], red[24 + g]));
    if (__any_sync(kFull, mt_ > m_run + 8.f)) {
      const float mn = fmaxf(m_run, mt_);
      const float alpha = exp2f(m_run - mn);  // 0 while m_run is -inf
      m_run = mn;
      l_run *= alpha;
      swb[0] *= alpha;
      swb[1] *= alpha;
      const float a0 = __shfl_sync(kFull, alpha, 8 * tg);      // head 2tg
      const float a1 = __shfl_sync(kFull, alpha, 8 * tg + 4);  // head 2tg + 1
#pragma unroll
      for (int mt = 0; mt < 4; mt++) {
        o[mt][0] *= a0;
        o[mt][1] *= a1;
        o[mt][2] *= a0;
        o[mt][3] *= a1;
      }
    }
    {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        p[e] = exp2f(sc[e] - m_run);
        l_run += p[e];
      }
      float *pr = pbuf + g * kPStride + 16 * warp + 2 * tg;
      *reinterpret_cast<float2 *>(pr) = make_float2(p[0], p[1]);
      *reinterpret_cast<float2 *>(pr + 8) = make_float2(p[2], p[3]);
    }
    __syncthreads();  // (3) p of all 64 tokens
    // ---- PV: warp w, blocks 2w, 2w + 1, all 64 tokens in 4 steps of 16
    {
      const float *fv = fsc + 8 * kTile + (2 * warp) * kTile + 2 * tg;
      const float *pp = pbuf + g * kPStride + 2 * tg;
      const int blk = 2 * warp + (lane >> 4);  // ldmatrix block of this lane's matrices
#pragma unroll
      for (int ks = 0; ks < 4; ks++) {
        const int mr = 16 * ks + 8 * ((lane >> 3) & 1) + (lane & 7);
        uint32_t vr[4];  // (T0, blk 2w), (T1, blk 2w), (T0, blk 2w+1), (T1, blk 2w+1)
        ldsm_x4_t(vbase + mr * 128 + ((blk ^ (mr & 7)) << 4), vr);
        const float2 p01 = *reinterpret_cast<const float2 *>(pp + 16 * ks);
        const float2 p23 = *reinterpret_cast<const float2 *>(pp + 16 * ks + 8);
#pragma unroll
        for (int half = 0; half < 2; half++) {
          const float2 w0 =
              __fmul2_rn(p01, *reinterpret_cast<const float2 *>(fv + half * kTile + 16 * ks));
          const float2 w1 =
              __fmul2_rn(p23, *reinterpret_cast<const float2 *>(fv + half * kTile + 16 * ks + 8));
          swb[half] += (w0.x + w0.y) + (w1.x + w1.y);
          uint32_t bh0, bl0, bh1, bl1;
          split_hilo(w0, bh0, bl0);
          split_hilo(w1, bh1, bl1);
          const uint32_t r0 = vr[2 * half], r1 = vr[2 * half + 1];  // tokens 0-7, 8-15
          {  // even M-tile: rows g <-> low nibble of byte 2g, rows g + 8 <-> its high nibble
            const uint32_t a[4] = {nib64(r0 << 4), nib64(r0), nib64(r1 << 4), nib64(r1)};
            mma16816(o[2 * half], a, bh0, bh1);
            mma16816(o[2 * half], a, bl0, bl1);
          }
          {  // odd M-tile: byte 2g + 1
            const uint32_t a[4] = {nib64(r0 >> 4), nib64(r0 >> 8), nib64(r1 >> 4),
                                   nib64(r1 >> 8)};
            mma16816(o[2 * half + 1], a, bh0, bh1);
            mma16816(o[2 * half + 1], a, bl0, bl1);
          }
        }
      }
    }
  }

  // ---- partial records: m (same in every warp), l summed over warps, o per warp
  if (failed) {
    // a load never arrived: let what was issued land (bounded), then mark the
    // records of this split invalid with NaN so the output shows it
    __syncthreads();
    if (tid == 0)
      for (int i = 0; i < kStages; i++) (void)mbar_wait(bar0 + 8 * i, 0), (void)mbar_wait(bar0 + 8 * i, 1);
    __syncthreads();
    for (int p = tid; p < gc * kRec; p += kThreads) {
      const int hh = p / kRec, j = p % kRec;
      ws[(((int64_t)b * n_q_heads + h0 + hh) * splits + s) * kRec + j] = __int_as_float(0x7fc00000);
    }
    return;
  }
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  __syncthreads();  // red is reused
  if (tg == 0) red[kWarps * 8 + warp * 8 + g] = l_run;
#pragma unroll
  for (int half = 0; half < 2; half++) {
    swb[half] += __shfl_xor_sync(kFull, swb[half], 1);
    swb[half] += __shfl_xor_sync(kFull, swb[half], 2);
  }
  __syncthreads();
  const int hA = 2 * tg, hB = 2 * tg + 1;  // heads of this lane's O columns
#pragma unroll
  for (int half = 0; half < 2; half++) {
    const float cA = kBias * __shfl_sync(kFull, swb[half], 4 * hA);
    const float cB = kBias * __shfl_sync(kFull, swb[half], 4 * hB);
#pragma unroll
    for (int par = 0; par < 2; par++) {
      const float(&acc)[4] = o[2 * half + par];
      const int d0 = 64 * warp + 32 * half + 2 * g + par;  // row g; row g + 8 is d0 + 16
      if (hA < gc) {
        float *rec = ws + (((int64_t)b * n_q_heads + h0 + hA) * splits + s) * kRec + 4;
        rec[d0] = acc[0] - cA;
        rec[d0 + 16] = acc[2] - cA;
      }
      if (hB < gc) {
        float *rec = ws + (((int64_t)b * n_q_heads + h0 + hB) * splits + s) * kRec + 4;
        rec[d0] = acc[1] - cB;
        rec[d0 + 16] = acc[3] - cB;
      }
    }
  }
  if (warp == 0 && tg == 0 && g < gc) {
    float *rec = ws + (((int64_t)b * n_q_heads + h0 + g) * splits + s) * kRec;
    rec[0] = m_run;
    rec[1] = red[kWarps * 8 + g] + red[kWarps * 8 + 8 + g] + red[kWarps * 8 + 16 + g] +
             red[kWarps * 8 + 24 + g];
  }
}

// ---- host: 2-D tensor maps over the cache planes (cached per plane)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// rows x row_bytes uint8 plane, boxes of 64 rows x row_bytes
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t row_bytes, bool swizzle) {
  struct Entry {
    const void *base;
    uint64_t rows;
    uint32_t row_bytes;
    CUtensorMap map;
  };
  static Entry cache[16];
  static int next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : cache)
    if (e.base == base && e.rows == rows && e.row_bytes == row_bytes) {
      *m = e.map;
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {row_bytes, (cuuint32_t)kTile};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cache[next] = Entry{base, rows, row_bytes, *m};
  next = (next + 1) % 16;
  return true;
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
  const uint64_t rows = c.block_table
                            ? (uint64_t)c.num_pages * c.num_kv_heads * c.page_size
                            : (uint64_t)c.batch_capacity * c.num_kv_heads * c.max_tokens;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;  // TMA row coordinates are 32-bit
  TmaMaps maps;
  if (!make_map(&maps.kc, c.k_codes, rows, 128, true) ||
      !make_map(&maps.vc, c.v_codes, rows, 128, true) ||
      !make_map(&maps.ks, c.k_scales, rows, 16, false) ||
      !make_map(&maps.vs, c.v_scales, rows, 16, false))
    return cudaErrorInvalidValue;
  // opt in to the large dynamic shared-memory carve-out once per device
  static std::mutex mu;
  static unsigned configured[2] = {0u, 0u};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    const unsigned bit = 1u << (dev & 31);
    if (!(configured[bf16] & bit)) {
      e = bf16 ? cudaFuncSetAttribute(q4_decode_mma_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)
               : cudaFuncSetAttribute(q4_decode_mma_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[bf16] |= bit;
    }
  }
  if (bf16)
    q4_decode_mma_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(
        maps, c, q, seq_lens, max_seq_len, n_q_heads, group, gc, sl2, p.split_tokens, p.splits,
        ws);
  else
    q4_decode_mma_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(
        maps, c, q, seq_lens, max_seq_len, n_q_heads, group, gc, sl2, p.split_tokens, p.splits,
        ws);
  return cudaGetLastError();
}

}  // namespace kvq
