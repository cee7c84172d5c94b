// q8_decode_mma.cu -- split-K decode attention over the Q8_0 + FWHT-256 cache
// (the 8-bit KV variant the Strata PR #21 pages compare Q4_0 against; rotation
// and per-token path as in "Q4_0 KV cache + FWHT-256", What, How 2 and the
// merge note).  A Q8_0 row holds 8 blocks of 32 int8 codes (256 bytes) and 8
// fp16 scales; code c of a block with scale d stands for c * d.
//
// One CTA per SM, 8 warps in two groups; group gq takes the 64-token tiles
// it with it % 2 == gq (6-stage TMA ring, an even count so that every stage
// serves one group), warp wi = warp % 4 tokens 16 wi .. 16 wi + 15, with its
// own online softmax; the 8 states are merged once per split.
//   * QK on the integer tensor path (mma.sync m16n8k32, s8 x s8 -> s32): the
//     K codes are the B fragments exactly as ldmatrix delivers them (no
//     conversion).  The rotated query of each head is scaled by
//     S = 127 * 2^14 / max|q|, rounded to integers n and split exactly into
//     int8 digits n = 2^14 H + 2^7 M + L (|M|, |L| <= 64); one MMA takes H and
//     M (rows 0-7, 8-15), a second one L.  Both accumulators start at the bits
//     of 1.5 * 2^23, so each exact integer block dot becomes an fp32 by one
//     subtraction; the three are combined with their weights and the block's
//     scale, read straight from the staged fp16 scale rows.  1 / (16 S) joins
//     the softmax scale.
//   * PV on the fp16 path (m16n8k16, fp32 accumulation): A = V^T codes
//     (ldmatrix.trans) as exact fp16 values: sign bit flipped, each byte paired
//     with the exponent byte of 1024 (1152 + c), 1152 subtracted; B = p * d_v
//     as fp16 hi + lo (fp16 TwoProduct).  With scales of amax / 127 the low
//     part of small weights falls into fp16's subnormal range and is rounded;
//     a zero-point bias carried through the accumulator and removed with
//     exactly computed weight sums would turn that rounding into an error
//     shared by all 32 dims of a block, which the back-rotation collects into
//     single output dims, so the codes enter without bias.
// The work schedule (one split per CTA, or the balanced stream schedule over
// all units) is the Q4_0 kernel's; the partial records (m, l, o[256]) go to
// the same combine and back-rotation kernel.
#include "decode_common.cuh"
#include "q4_vec.cuh"

namespace kvq {
namespace {

using namespace dec;

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 64;             // tokens per stage, 16 per warp of the group
constexpr int kStages = 6;            // even: stage it % 6 always serves group it % 2
constexpr unsigned kFull = 0xffffffffu;
constexpr int kRec = 260;             // partial record: m, l, pad, pad, o[256]
constexpr int kCodeRow = 256;         // Q8_0 code bytes per row
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQRange = 2080768.f;  // 127 * 2^14
constexpr uint32_t kMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.f;
// stage: K codes as two 64-row x 128-byte planes (dims 0-127, 128-255; 128B
// swizzle) brought by one 3-D box, V codes likewise, then K and V scale rows
// (64 x 16 bytes, 1-D bulk copies)
constexpr int kBox = kTile * 128;
constexpr int kOffKC = 0;
constexpr int kOffVC = kOffKC + 2 * kBox;
constexpr int kOffKS = kOffVC + 2 * kBox;
constexpr int kOffVS = kOffKS + kTile * 16;
constexpr int kStageBytes = kOffVS + kTile * 16;  // 34 KB
// after the ring
constexpr int kOffQ = kStages * kStageBytes;       // query digits int8 [level][head][256]
constexpr int kOffQS = kOffQ + 3 * 8 * 256;        // per-head 1 / (16 S), fp32 [8]
constexpr int kOffQT = kOffQS + 128;               // query fragment table [8][32] x 32 B
constexpr int kOffBar = kOffQT + 8 * 32 * 32;      // full[kStages]
constexpr int kOffRel = kOffBar + kStages * 8;     // release counters [kStages]
constexpr int kOffAbort = kOffRel + kStages * 4;   // abort flag, tiles issued
constexpr int kSmemUsed = kOffAbort + 8;
constexpr int kSmemBytes = kSmemUsed + 1024;
// end-of-split merge, reusing the ring (as the Q4_0 kernel)
constexpr int kMergeHead = 264;
constexpr int kMergeWarpFloats = 16 + 8 * kMergeHead;
constexpr int kOffMergeF = kWarps * kMergeWarpFloats * 4;
static_assert(kStages % 2 == 0, "each stage must serve one warp group");
static_assert(kStageBytes % 1024 == 0, "stages must keep the swizzle atoms aligned");
static_assert(kOffMergeF + (kWarps + 2) * 8 * 4 <= kStages * kStageBytes, "merge fits the ring");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");
static_assert(kOffQT % 16 == 0, "fragment table alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

// d = A(s8, 16 x 32, row) * B(s8, 32 x 8, col) + the bits of 1.5 * 2^23
__device__ __forceinline__ void imma16832(uint32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(kMagicBits));
}

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ __half2 as_h2(uint32_t x) { return *reinterpret_cast<const __half2 *>(&x); }

__device__ __forceinline__ float2 as_f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}

// bytes (sel & 0xf, (sel >> 8) & 0xf) of a sign-flipped code word -> half2 of
// the two codes' exact values: (1024 + c + 128) - 1152
__device__ __forceinline__ uint32_t s8pair(uint32_t xflip, uint32_t sel) {
  const uint32_t h = __byte_perm(xflip, 0x64646464u, sel);
  const __half2 r = __hsub2(*reinterpret_cast<const __half2 *>(&h), __float2half2_rn(1152.f));
  return *reinterpret_cast<const uint32_t *>(&r);
}

// 4 int8 in a word -> packed bytes of 4 digits
__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (uint32_t)(a & 255) | ((uint32_t)(b & 255) << 8) | ((uint32_t)(c & 255) << 16) |
         ((uint32_t)(d & 255) << 24);
}

// STREAM: the balanced schedule over all units (gridDim.x CTAs) instead of
// one split per CTA (a separate instance, so the split path keeps its code)
template <bool BF16, bool STREAM>
__global__ void __launch_bounds__(kThreads, 1)
    q8_decode_mma_kernel(const __grid_constant__ TmaMaps maps, kvq_cache c,
                         const void *__restrict__ q, const int32_t *__restrict__ seq_lens,
                         int max_seq_len, int n_q_heads, int group, int gc, float sl2,
                         int split_tokens, int splits, int n_hg, int n_units,
                         int append_tiles, float *__restrict__ ws,
                         const void *__restrict__ k_new, const void *__restrict__ v_new,
                         const int32_t *__restrict__ pos, const int32_t *__restrict__ q_to_seq,
                         int num_seqs, uint32_t *__restrict__ err, int wait_polls) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  const uint32_t full0 = smem_u32(smem + kOffBar);
  int *rel = reinterpret_cast<int *>(smem + kOffRel);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffAbort);
  volatile int *issued = abort_flag + 1;

  if (tid == 0) {
    prefetch_map(&maps.kc);
    prefetch_map(&maps.vc);
  }
  grid_dependency_wait();
  launch_dependents();
  const int cap = c.block_table ? c.max_pages_per_seq * c.page_size : c.max_tokens;
  auto row_len = [&](int row) {
    return decode_len(row, seq_lens, pos, q_to_seq, num_seqs, max_seq_len, cap);
  };
  // a unit's tiles, plus append_tiles that stand for the fused append of the
  // new token (the schedule gives the CTA holding it correspondingly fewer
  // real tiles; tiles past the length hold no work)
  auto unit_tiles = [&](int u) {
    const int l = row_len(u / n_hg);
    return l > 0 ? (l + kTile - 1) / kTile + append_tiles : 0;
  };
  // this CTA's segments, as in the Q4_0 kernel: stream mode walks the units its
  // share of the concatenated tiles crosses, split mode has one split
  int seg_unit = -1, seg_start = 0, t_cur = 0, t_end = 0;
  if constexpr (STREAM) {
    // min(CTAs, T) CTAs share the tiles, so every one of them owns at least one
    auto share = [&](int c, int total) {
      return (int)((int64_t)c * total / min((int)gridDim.x, total));
    };
    const StreamLoc L = stream_locate<kThreads>(
        n_units, unit_tiles,
        [&](int total) { return (int)blockIdx.x < min((int)gridDim.x, total) ? share(blockIdx.x, total) : -1; },
        -1, reinterpret_cast<int *>(smem));
    if ((int)blockIdx.x < min((int)gridDim.x, L.total)) {
      t_cur = share(blockIdx.x, L.total);
      t_end = share(blockIdx.x + 1, L.total);
      seg_unit = L.unit;
      seg_start = L.start;
    }
  }
  const float nan = __int_as_float(0x7fc00000);
  bool dead = false;  // a load never arrived: the remaining segments write NaN
  for (int seg = 0; STREAM || seg < 1; seg++) {
    int b, hg, t0, t1;
    int64_t rec_base, rec_hstride;  // record of head h0 + hh: ws + (rec_base + hh * rec_hstride) * kRec
    if constexpr (STREAM) {
      if (seg_unit < 0 || seg_unit >= n_units || t_cur >= t_end) break;
      int n = unit_tiles(seg_unit);
      while (n == 0 && seg_unit + 1 < n_units) n = unit_tiles(++seg_unit);  // units without tiles hold none of the range
      if (n == 0) break;
      b = seg_unit / n_hg;
      hg = seg_unit % n_hg;
      const int hi = min(t_end, seg_start + n) - seg_start;
      t0 = (t_cur - seg_start) * kTile;
      t1 = min(row_len(b), hi * kTile);
      rec_base = ((int64_t)seg_unit + blockIdx.x) * gc;
      rec_hstride = 1;
      t_cur = seg_start + hi;
      seg_start += n;
      seg_unit++;
    } else {
      b = blockIdx.z;
      hg = blockIdx.y;
      t0 = blockIdx.x * split_tokens;
      t1 = min(row_len(b), t0 + split_tokens);
      rec_base = ((int64_t)b * n_q_heads + hg * gc) * splits + blockIdx.x;
      rec_hstride = splits;
    }
    const int h0 = hg * gc, kvh = h0 / group;
    // this segment's global inputs first: their latency overlaps the sizing
    // and the barrier set-up below
    const int p_new = pos ? __ldg(pos + b) : -1;
    const int bs = q_to_seq ? __ldg(q_to_seq + b) : b;
    float x[8];  // warp w: query head h0 + w, dims 8 lane .. 8 lane + 7
    if (warp < gc) {
      const int64_t off = ((int64_t)b * n_q_heads + h0 + warp) * kDim + 8 * lane;
      if (BF16) {
        const uint4 r = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(q) + off));
        const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
        #pragma unroll
        for (int i = 0; i < 4; i++) {
          x[2 * i] = bf16lo(rr[i]);
          x[2 * i + 1] = bf16hi(rr[i]);
        }
      } else {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(q) + off);
        const float4 u = __ldg(p), v = __ldg(p + 1);
        x[0] = u.x, x[1] = u.y, x[2] = u.z, x[3] = u.w;
        x[4] = v.x, x[5] = v.y, x[6] = v.z, x[7] = v.w;
      }
    } else {
      #pragma unroll
      for (int i = 0; i < 8; i++) x[i] = 0.f;
    }
    // the barriers are set up before the length is needed, so that this
    // overlaps the length load; the previous segment is done with shared
    // memory and its generic writes (the merge) precede the copies that
    // will overwrite the ring (a dead CTA may still have copies in flight
    // and leaves its barriers alone)
    if (!dead) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (tid == 0) {
        #pragma unroll
        for (int i = 0; i < kStages; i++) {
          if (seg > 0) asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(full0 + 8 * i) : "memory");
          mbar_init(full0 + 8 * i, 1);
          rel[i] = 0;
        }
        *abort_flag = 0;
        *issued = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncthreads();
    }
    const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
    if (ntiles == 0) continue;  // a split past the length writes no record
    if (dead) {
      for (int hh = 0; hh < gc; hh++) {
        float *rec = ws + (rec_base + hh * rec_hstride) * kRec;
        rec[4 + tid] = nan;
        if (tid == 0) rec[0] = rec[1] = nan;
      }
      continue;
    }
    const bool appender = p_new >= t0 && p_new < t1;

    // first cache row of the 64-token tile starting at token t, -1 if unmapped
    auto tile_row = [&](int t) -> int {
      if (c.block_table == nullptr) return (int)(((int64_t)bs * c.num_kv_heads + kvh) * c.max_tokens + t);
      const int pi = t / c.page_size;
      const int page = __ldg(c.block_table + (int64_t)bs * c.max_pages_per_seq + pi);
      if (page < 0 || page >= c.num_pages) return -1;
      return (int)(((int64_t)page * c.num_kv_heads + kvh) * c.page_size + (t - pi * c.page_size));
    };
    // first row of a run of scale rows, inside the planes (debug builds check
    // and report; release builds use it as is)
    auto scale_src = [&](int64_t r, int n) -> int64_t {
      return in_bounds(r, r + n, cache_rows(c), err) ? r : 0;
    };
    auto issue = [&](int it) {
      const int st = it % kStages;
      const int r = tile_row(t0 + it * kTile);
      const uint32_t bar = full0 + 8 * st;
      if (r < 0) {
        mbar_arrive(bar);
      } else {
        // scale rows of this (sequence, head) only: contiguous caches end each
        // head's rows at max_tokens, pages hold whole 64-token tiles
        const int nrows = c.block_table ? kTile : min(kTile, c.max_tokens - (t0 + it * kTile));
        mbar_arrive_tx(bar, 4 * kBox + 2 * nrows * 16);
        const uint32_t dst = smem_u32(smem + st * kStageBytes);
        tma_load_3d(dst + kOffKC, &maps.kc, 0, r, 0, bar);
        tma_load_3d(dst + kOffVC, &maps.vc, 0, r, 0, bar);
        bulk_load(dst + kOffKS, c.k_scales + scale_src(r, nrows) * kRowScales, nrows * 16, bar);
        bulk_load(dst + kOffVS, c.v_scales + scale_src(r, nrows) * kRowScales, nrows * 16, bar);
      }
      atomicMax(const_cast<int *>(issued), it + 1);
    };
    // initial tiles: warp w issues tile w, except the tile holding the new
    // token of a fused step, which the appending warp issues once the token's
    // rows are in the cache (a later tile holding it is refilled inside the
    // loop, after the barrier that follows the append)
    const int it_new = appender ? (p_new - t0) / kTile : -1;
    if (lane == 0 && warp < kStages && warp < ntiles && warp != it_new) issue(warp);
    if (appender && warp == 0) {
      // scratch outside the ring (the fragment table is written after the
      // query digits, which this warp reaches after the append)
      float4 *scratch = reinterpret_cast<float4 *>(smem + kOffQT);
      {
        const int vg = lane >> 3, i = lane & 7;
        const bool valid = vg < 2;  // lanes 0-7: K, 8-15: V
        const void *src =
            static_cast<const char *>(vg == 1 ? v_new : k_new) +
            ((int64_t)b * c.num_kv_heads + kvh) * kDim * (BF16 ? 2 : 4);
        uint4 bytes[2];
        uint16_t sc;
        q4v::quantize_vector_q8<BF16>(valid ? src : k_new, valid, lane, scratch + 64 * vg, bytes, sc);
        const int64_t row = q4_row(c, bs, kvh, p_new);
        if (valid && row >= 0 && in_bounds(row, row + 1, cache_rows(c), err)) {
          uint8_t *dst = (vg ? c.v_codes : c.k_codes) + row * kCodeRow + 32 * i;
          *reinterpret_cast<uint4 *>(dst) = bytes[0];
          *reinterpret_cast<uint4 *>(dst + 16) = bytes[1];
          (vg ? c.v_scales : c.k_scales)[row * kRowScales + i] = sc;
        }
      }
      // the rows are read back by TMA (async proxy)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0 && it_new < kStages) issue(it_new);
    }

    // (1) query: warp w rotates head h0 + w (zeros past gc), scales it to the
    // int8 digit range and writes its digits and 1 / (16 S)
    {
      warp_fwht256(x, lane);
      float m = 0.f;
      #pragma unroll
      for (int i = 0; i < 8; i++) m = fmaxf(m, fabsf(x[i]));
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      const float S = m > 0.f ? __fdiv_rn(kQRange, m) : 0.f;
      int H[8], M[8], L[8];
      #pragma unroll
      for (int i = 0; i < 8; i++) {
        const int n = __float2int_rn(x[i] * S);
        L[i] = ((n + 64) & 127) - 64;
        const int n1 = (n - L[i]) >> 7;
        M[i] = ((n1 + 64) & 127) - 64;
        H[i] = (n1 - M[i]) >> 7;
      }
      // levels H, M, L 2048 bytes (256 uint2) apart
      uint2 *qd = reinterpret_cast<uint2 *>(smem + kOffQ + warp * 256 + 8 * lane);
      qd[0] = make_uint2(pack_s8x4(H[0], H[1], H[2], H[3]), pack_s8x4(H[4], H[5], H[6], H[7]));
      qd[256] = make_uint2(pack_s8x4(M[0], M[1], M[2], M[3]), pack_s8x4(M[4], M[5], M[6], M[7]));
      qd[512] =
          make_uint2(pack_s8x4(L[0], L[1], L[2], L[3]), pack_s8x4(L[4], L[5], L[6], L[7]));
      if (lane == 0)
        reinterpret_cast<float *>(smem + kOffQS)[warp] = S > 0.f ? __frcp_rn(S) * 0.0625f : 0.f;
    }
    __syncthreads();
    // fragment table in shared memory (registers hold the accumulators):
    // entry (bb, lane) = the H, M, H, M, L, L words of head lane / 4, block bb
    float sf;  // log2-domain factor of head g: sl2 / (16 S)
    const uint4 *qtab = reinterpret_cast<const uint4 *>(smem + kOffQT);
    {
      const int bb = warp;
      const uint32_t *qw = reinterpret_cast<const uint32_t *>(smem + kOffQ) + g * 64 + tg;
      uint4 *dst = reinterpret_cast<uint4 *>(smem + kOffQT) + 2 * (bb * 32 + lane);
      // level stride 2048 bytes = 512 words; dims 32bb + 4tg and 32bb + 16 + 4tg
      dst[0] = make_uint4(qw[8 * bb], qw[512 + 8 * bb], qw[8 * bb + 4], qw[512 + 8 * bb + 4]);
      dst[1] = make_uint4(qw[1024 + 8 * bb], qw[1024 + 8 * bb + 4], 0u, 0u);
      sf = sl2 * reinterpret_cast<const float *>(smem + kOffQS)[g];
    }
    __syncthreads();
    uint4 qhm_r[8];
    #pragma unroll
    for (int bb = 0; bb < 8; bb++) qhm_r[bb] = qtab[2 * (bb * 32 + lane)];

    // (2) the split: warp group gq = warp / 4 takes the tiles it with it % 2 == gq,
    // warp wi = warp % 4 tokens 16wi .. 16wi + 15 of each of them
    const int gq = warp >> 2, wi = warp & 3;
    float o[8][2][4];  // [block][M-tile: dims 32bb + 16m + (2g, 2g + 1)][reg]
    #pragma unroll
    for (int bb = 0; bb < 8; bb++)
      #pragma unroll
      for (int m = 0; m < 2; m++) o[bb][m][0] = o[bb][m][1] = o[bb][m][2] = o[bb][m][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // head g
    // ldmatrix rows: lanes 8j .. 8j + 7 address matrix j = (token half j & 1,
    // 16-byte chunk 2bb + (j >> 1)); the chunk is swizzled by the row (128B mode)
    const int tr = 16 * wi + (lane & 7) + 8 * ((lane >> 3) & 1);
    const uint32_t lrow = tr * 128, lz = ((lane >> 4) ^ (tr & 7)) << 4;

    for (int it = gq; it < ntiles; it += 2) {
      const int st = it % kStages;
      if (!mbar_wait(full0 + 8 * st, (it / kStages) & 1, abort_flag, wait_polls)) {
        *abort_flag = 1;
        report(err, KVQ_DEVERR_WAIT_TIMEOUT);
        break;
      }
      const uint8_t *stage = smem + st * kStageBytes;
      const int ttile = t0 + it * kTile;
      const int tw = ttile + 16 * wi;  // first token of this warp
      const int nvalid = min(16, t1 - tw);
      bool live = nvalid > 0;
      if (live && c.block_table != nullptr) live = tile_row(ttile) >= 0;
      if (live) {
        // scale rows of tokens 2tg, 2tg + 1, 8 + 2tg, 9 + 2tg of this warp: 8 fp16
        // each, the scale of block bb in half bb
        const uint8_t *ksr = stage + kOffKS + (16 * wi + 2 * tg) * 16;
        const uint4 kq0 = *reinterpret_cast<const uint4 *>(ksr);
        const uint4 kq1 = *reinterpret_cast<const uint4 *>(ksr + 16);
        const uint4 kq8 = *reinterpret_cast<const uint4 *>(ksr + 128);
        const uint4 kq9 = *reinterpret_cast<const uint4 *>(ksr + 144);
        const uint32_t kbase = smem_u32(stage + kOffKC) + lrow, vbase = smem_u32(stage + kOffVC) + lrow;

        // ---- QK: head g, tokens 8T + 2tg + {0, 1}, T = 0, 1
        float2 sacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        #pragma unroll
        for (int bb = 0; bb < 8; bb++) {
          const uint4 qhm = qhm_r[bb];
          const uint2 ql = *reinterpret_cast<const uint2 *>(qtab + 2 * (bb * 32 + lane) + 1);
          uint32_t kr[4];  // (tokens 0-7, dims 0-15 of block bb), (8-15, 0-15), (0-7, 16-31), (8-15, 16-31)
          ldsm_x4(kbase + (bb >> 2) * kBox + ((((2 * bb) & 7) << 4) ^ lz), kr);
          const uint32_t sel = (bb & 1) ? 0x7632u : 0x5410u;
          const float2 dk0 = __half22float2(as_h2(__byte_perm(word(kq0, bb >> 1), word(kq1, bb >> 1), sel)));
          const float2 dk1 = __half22float2(as_h2(__byte_perm(word(kq8, bb >> 1), word(kq9, bb >> 1), sel)));
          #pragma unroll
          for (int T = 0; T < 2; T++) {
            uint32_t a1[4], a2[4];
            imma16832(a1, qhm.x, qhm.y, qhm.z, qhm.w, kr[T], kr[2 + T]);
            imma16832(a2, ql.x, 0u, ql.y, 0u, kr[T], kr[2 + T]);
            const float2 mg = make_float2(-kMagic, -kMagic);
            const float2 hH = __fadd2_rn(as_f2(a1[0], a1[1]), mg);   // 2^14-digit dot, exact
            const float2 hM = __fadd2_rn(as_f2(a1[2], a1[3]), mg);   // 2^7-digit dot, exact
            const float2 hL = __fadd2_rn(as_f2(a2[0], a2[1]), mg);   // 1-digit dot, exact
            const float2 t = __ffma2_rn(hM, make_float2(128.f, 128.f), hL);
            const float2 v = __ffma2_rn(hH, make_float2(16384.f, 16384.f), t);
            const float2 d = T ? dk1 : dk0;
            sacc[T] = __ffma2_rn(d, v, sacc[T]);
          }
        }
        // ---- online softmax of head g over this warp's 16 tokens
        float xs[4] = {sacc[0].x * sf, sacc[0].y * sf, sacc[1].x * sf, sacc[1].y * sf};
        if (nvalid < 16) {
          #pragma unroll
          for (int e2 = 0; e2 < 4; e2++)
            if (8 * (e2 >> 1) + 2 * tg + (e2 & 1) >= nvalid) xs[e2] = -INFINITY;
        }
        float mx = fmaxf(fmaxf(xs[0], xs[1]), fmaxf(xs[2], xs[3]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        if (__any_sync(kFull, mx > m_run)) {
          const float mn = fmaxf(m_run, mx);
          const float alpha = mn == m_run ? 1.f : ex2(m_run - mn);
          m_run = mn;
          l_run *= alpha;
          const float a0 = __shfl_sync(kFull, alpha, 8 * tg);
          const float a1 = __shfl_sync(kFull, alpha, 8 * tg + 4);
          #pragma unroll
          for (int bb = 0; bb < 8; bb++)
            #pragma unroll
            for (int m = 0; m < 2; m++) {
              o[bb][m][0] *= a0;
              o[bb][m][1] *= a1;
              o[bb][m][2] *= a0;
              o[bb][m][3] *= a1;
            }
        }
        uint32_t ph[2], pl[2];  // p of head g as fp16 hi + lo pairs, token groups T
        #pragma unroll
        for (int T = 0; T < 2; T++) {
          const float p0 = ex2(xs[2 * T] - m_run), p1 = ex2(xs[2 * T + 1] - m_run);
          l_run += p0 + p1;
          split_hilo(make_float2(p0, p1), ph[T], pl[T]);
        }
        // ---- PV over the 16 tokens (one k-step)
        const uint8_t *vsr = stage + kOffVS + (16 * wi + 2 * tg) * 16;
        uint4 vq0 = *reinterpret_cast<const uint4 *>(vsr);
        uint4 vq1 = *reinterpret_cast<const uint4 *>(vsr + 16);
        uint4 vq8 = *reinterpret_cast<const uint4 *>(vsr + 128);
        uint4 vq9 = *reinterpret_cast<const uint4 *>(vsr + 144);
        if (nvalid < 16) {  // tokens past the end: zero scales (their rows may hold anything)
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          if (2 * tg >= nvalid) vq0 = z;
          if (2 * tg + 1 >= nvalid) vq1 = z;
          if (8 + 2 * tg >= nvalid) vq8 = z;
          if (9 + 2 * tg >= nvalid) vq9 = z;
        }
        const __half2 ph0 = *reinterpret_cast<const __half2 *>(&ph[0]);
        const __half2 ph1 = *reinterpret_cast<const __half2 *>(&ph[1]);
        const __half2 pl0 = *reinterpret_cast<const __half2 *>(&pl[0]);
        const __half2 pl1 = *reinterpret_cast<const __half2 *>(&pl[1]);
        #pragma unroll
        for (int bb = 0; bb < 8; bb++) {
          uint32_t vr[4];  // (tokens 0-7, dims 0-15), (8-15, 0-15), (0-7, 16-31), (8-15, 16-31)
          ldsm_x4_t(vbase + (bb >> 2) * kBox + ((((2 * bb) & 7) << 4) ^ lz), vr);
          const uint32_t vsel = (bb & 1) ? 0x7632u : 0x5410u;
          const __half2 d01 = as_h2(__byte_perm(word(vq0, bb >> 1), word(vq1, bb >> 1), vsel));
          const __half2 d89 = as_h2(__byte_perm(word(vq8, bb >> 1), word(vq9, bb >> 1), vsel));
          // w = p d_v exactly as hi + lo (TwoProduct with fp16 FMA)
          const __half2 wh0 = __hmul2_rn(ph0, d01), wh1 = __hmul2_rn(ph1, d89);
          const __half2 wl0 = __hfma2(pl0, d01, __hfma2(ph0, d01, __hneg2(wh0)));
          const __half2 wl1 = __hfma2(pl1, d89, __hfma2(ph1, d89, __hneg2(wh1)));
          const uint32_t bh0 = *reinterpret_cast<const uint32_t *>(&wh0);
          const uint32_t bh1 = *reinterpret_cast<const uint32_t *>(&wh1);
          const uint32_t bl0 = *reinterpret_cast<const uint32_t *>(&wl0);
          const uint32_t bl1 = *reinterpret_cast<const uint32_t *>(&wl1);
          #pragma unroll
          for (int m = 0; m < 2; m++) {
            // byte j of a transposed word: token 2tg + (j >> 1), dim 2g + (j & 1)
            const uint32_t x0 = vr[2 * m] ^ 0x80808080u, x1 = vr[2 * m + 1] ^ 0x80808080u;
            const uint32_t a[4] = {s8pair(x0, 0x4240), s8pair(x0, 0x4341), s8pair(x1, 0x4240),
                                   s8pair(x1, 0x4341)};
            mma16816(o[bb][m], a, bh0, bh1);
            mma16816(o[bb][m], a, bl0, bl1);
          }
        }
      }
      // release the stage; the last of its 4 warps refills it with tile it + kStages
      __syncwarp();
      if (lane == 0) {
        int old;
        asm volatile("atom.release.cta.shared::cta.add.s32 %0, [%1], 1;"
                     : "=r"(old)
                     : "r"(smem_u32(rel + st))
                     : "memory");
        if (old == 3) {
          asm volatile("fence.acq_rel.cta;" ::: "memory");
          rel[st] = 0;
          if (it + kStages < ntiles && !*abort_flag) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(it + kStages);
          }
        }
      }
    }

    // (3) merge the 8 warps' states into this split's records
    l_run += __shfl_xor_sync(kFull, l_run, 1);
    l_run += __shfl_xor_sync(kFull, l_run, 2);
    __syncthreads();  // every warp is done with the ring
    const bool abort_all = *abort_flag != 0;
    if (abort_all) {
      // a load never arrived: let every load still in flight land (bounded,
      // ignoring the flag) before the CTA's shared memory goes away
      if (tid == 0) {
        const int n = *issued;
        for (int it = n > kStages ? n - kStages : 0; it < n; it++)
          for (int i = 0; i < kWaitPolls && !mbar_try(full0 + 8 * (it % kStages), (it / kStages) & 1); i++) {
          }
      }
      __syncthreads();
    }
    float *mw = reinterpret_cast<float *>(smem) + warp * kMergeWarpFloats;
    if (!abort_all) {
      if (tg == 0) {
        mw[g] = m_run;
        mw[8 + g] = l_run;
      }
      #pragma unroll
      for (int bb = 0; bb < 8; bb++)
        #pragma unroll
        for (int m = 0; m < 2; m++) {
          const int d0 = 32 * bb + 16 * m + 2 * g;  // row g; row g + 8 is d0 + 1
          float *oa = mw + 16 + (2 * tg) * kMergeHead + d0;
          float *ob = oa + kMergeHead;
          oa[0] = o[bb][m][0];
          ob[0] = o[bb][m][1];
          oa[1] = o[bb][m][2];
          ob[1] = o[bb][m][3];
        }
    }
    __syncthreads();
    float *fac = reinterpret_cast<float *>(smem + kOffMergeF);  // [warp][head] exp2 factors
    float *mh = fac + kWarps * 8;                                // M, L per head
    if (!abort_all && tid < 8) {
      const float *m0 = reinterpret_cast<const float *>(smem);
      float M = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kWarps; w++) M = fmaxf(M, m0[w * kMergeWarpFloats + tid]);
      float L = 0.f;
      #pragma unroll
      for (int w = 0; w < kWarps; w++) {
        const float mwv = m0[w * kMergeWarpFloats + tid];
        const float f = mwv == -INFINITY ? 0.f : ex2(mwv - M);
        fac[w * 8 + tid] = f;
        L += f * m0[w * kMergeWarpFloats + 8 + tid];
      }
      mh[tid] = M;
      mh[8 + tid] = L;
    }
    __syncthreads();
    for (int hh = 0; hh < gc; hh++) {
      float *rec = ws + (rec_base + hh * rec_hstride) * kRec;
      float acc = 0.f;
      if (!abort_all) {
        #pragma unroll
        for (int w = 0; w < kWarps; w++)
          acc += fac[w * 8 + hh] *
                 reinterpret_cast<const float *>(smem)[w * kMergeWarpFloats + 16 + hh * kMergeHead + tid];
      }
      rec[4 + tid] = abort_all ? nan : acc;
      if (tid == 0) {
        rec[0] = abort_all ? nan : mh[hh];
        rec[1] = abort_all ? nan : mh[8 + hh];
      }
    }
    if (abort_all) dead = true;
  }  // segments
}
}  // namespace

cudaError_t launch_q8_decode_mma(const kvq_cache &c, const void *q, int bf16, int batch,
                                 int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                                 float scale, float *ws, const DecodePlan &p, cudaStream_t s,
                                 const void *k_new, const void *v_new, const int32_t *pos,
                                 const int32_t *q_to_seq, int num_seqs) {
  const int group = n_q_heads / c.num_kv_heads;
  const int gc = group < 8 ? group : 8;
  if (p.stream ? p.tile != kTile : p.split_tokens % kTile) return cudaErrorInvalidValue;
  const int n_hg = n_q_heads / gc;
  const int append_tiles = p.stream && pos ? kAppendTokens / kTile : 0;
  const float sl2 = scale * kLog2e;
  const uint64_t rows = c.block_table
                            ? (uint64_t)c.num_pages * c.num_kv_heads * c.page_size
                            : (uint64_t)c.batch_capacity * c.num_kv_heads * c.max_tokens;
  if (rows >= (1ull << 31)) return cudaErrorInvalidValue;  // TMA row coordinates are 32-bit
  TmaMaps maps;
  if (!make_map(&maps.kc, c.k_codes, rows, kCodeRow, 128, kTile, true, 2) ||
      !make_map(&maps.vc, c.v_codes, rows, kCodeRow, 128, kTile, true, 2))
    return cudaErrorInvalidValue;
  maps.kc2 = maps.kc;  // a 64-token tile is one box already
  maps.vc2 = maps.vc;
  static std::mutex mu;
  static unsigned configured[4] = {0u, 0u, 0u, 0u};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int variant = bf16 + 2 * p.stream;
  {
    std::lock_guard<std::mutex> lock(mu);
    const unsigned bit = 1u << (dev & 31);
    if (!(configured[variant] & bit)) {
      const void *fn = variant == 0   ? (const void *)q8_decode_mma_kernel<false, false>
                       : variant == 1 ? (const void *)q8_decode_mma_kernel<true, false>
                       : variant == 2 ? (const void *)q8_decode_mma_kernel<false, true>
                                      : (const void *)q8_decode_mma_kernel<true, true>;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[variant] |= bit;
    }
  }
  uint32_t *err = device_error_word();
  const int polls = wait_poll_limit();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = p.stream ? dim3(p.ctas) : dim3(p.splits, n_q_heads / gc, batch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (variant) {
    case 0:
      e = cudaLaunchKernelEx(&cfg, q8_decode_mma_kernel<false, false>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    case 1:
      e = cudaLaunchKernelEx(&cfg, q8_decode_mma_kernel<true, false>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    case 2:
      e = cudaLaunchKernelEx(&cfg, q8_decode_mma_kernel<false, true>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    default:
      e = cudaLaunchKernelEx(&cfg, q8_decode_mma_kernel<true, true>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvq
