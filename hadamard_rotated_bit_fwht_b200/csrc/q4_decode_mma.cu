// q4_decode_mma.cu -- split-K decode attention over the Q4_0 + FWHT-256 cache on
// the tensor cores (Strata PR #21 "Q4_0 KV cache + FWHT-256": What, How 2 and the
// merge note's per-token path that rotates Q and the output).
//
// With GQA the decode step is a small dense contraction per kv head:
// S = Q_rot K^T (G x T) and O = P V (G x 256), G <= 8 heads per CTA.  One CTA
// per SM (8 warps, ~170 KB of shared memory):
//   * 128-token tiles of the split (codes and fp16 scales of K and V, 36 KB)
//     stream into a ring of 4 stages, each guarded by a full mbarrier: code
//     rows by TMA (2-D maps over the 128-byte rows, hardware 128-byte
//     swizzle), scale rows by 1-D bulk copies.  The first 4 tiles are issued
//     before the query is prepared; afterwards the last warp to release a
//     stage (a shared-memory counter per stage) issues its refill, so no warp
//     is spent on producing and every warp keeps the full register budget.
//     Every wait is bounded.
//   * warp group gq = warp / 4 takes the tiles it with it % 2 == gq, warp
//     wi = warp % 4 tokens 32 wi .. 32 wi + 31 of each, with its own online
//     softmax (no CTA-wide barrier per tile).  The 8 running states are
//     merged once at the end of the split.
//   * QK on mma.sync m16n8k16 (f16 x f16 -> f32): A = the rotated query of the
//     8 heads split exactly into fp16 hi (rows 0-7) and lo (rows 8-15), held in
//     registers for the whole split; B = K codes of 8 tokens as the exact fp16
//     values 64 + c (a nibble in bits 4..7 of a 16-bit lane OR-ed with the bits
//     of 64.0, one LOP3 per pair).  One Q4_0 block (32 dims) is two k-steps; the
//     dims of a k-step are permuted (the same way in A and B) so that each
//     thread's code word feeds both k-steps without a byte shuffle.  The
//     accumulator starts at -72 * sum(q over the block) (zero point 8 plus the
//     magic 64), and hi + lo times the block's scale is added to the score.
//   * PV on mma.sync: A = V^T codes (64 + c, via ldmatrix.trans), B = p * d_v
//     split into fp16 hi + lo (the 32 dims of a block share the token's scale,
//     so the scale rides in B); O = 16 dims x 8 heads per M-tile, 64 fp32
//     registers per thread.  The bias 72 * sum_t(p d_v) per (head, block) is
//     removed at the end.
//   * The QK accumulator layout (head g = lane / 4, tokens 2(lane % 4) + {0,1},
//     + 8) is the PV B-fragment layout, so p never leaves registers.
// Split-K partials (m, l, o[256]) per (query row, q head, split) -- or, under
// the balanced stream schedule, per (unit, CTA) segment -- go to the combine +
// back-rotation kernel (q4_decode.cu).
#include "decode_common.cuh"
#include "q4_vec.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 8;           // 2 groups of 4; group gq takes the tiles it with it % 2 == gq
constexpr int kThreads = 32 * kWarps;
constexpr int kTile = 128;          // tokens per stage, 32 per warp of the group
constexpr int kSub = 64;            // rows per TMA box (the page-size granule)
constexpr int kStages = 4;          // even: stage it % 4 always serves group it % 2
constexpr unsigned kFull = 0xffffffffu;
constexpr int kRec = 260;           // partial record: m, l, pad, pad, o[256]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kBias = 72.f;       // 64 (magic) + 8 (Q4_0 zero point)
constexpr uint32_t kSubBytes = 2 * kSub * 128 + 2 * kSub * 16;  // one sub-tile, K + V

// stage layout (bytes from a 1024-aligned stage base)
constexpr int kOffKC = 0;                      // K codes: 128 rows x 128 B (TMA 128B swizzle)
constexpr int kOffVC = kOffKC + kTile * 128;   // V codes
constexpr int kOffKS = kOffVC + kTile * 128;   // K scales: 128 rows x 8 fp16
constexpr int kOffVS = kOffKS + kTile * 16;    // V scales
constexpr int kStageBytes = kOffVS + kTile * 16;  // 36 KB
// after the ring
constexpr int kFsK = 8 * 32 * 4;               // per-warp K scales fp32 [block][32 pos]
constexpr int kFsV = 8 * 32 * 2;               // per-warp V scales fp16 [block][32 pos]
constexpr int kOffFs = kStages * kStageBytes;
constexpr int kOffQF = kOffFs + kWarps * (kFsK + kFsV);  // query fragments [h][b][ks][tg] x 16 B
constexpr int kOffQB = kOffQF + 8 * 8 * 2 * 4 * 16;      // accumulator starts [h][b]
constexpr int kOffBar = kOffQB + 8 * 8 * 4;              // full[kStages]
constexpr int kOffRel = kOffBar + kStages * 8;           // release counters [kStages]
constexpr int kOffAbort = kOffRel + kStages * 4;         // abort flag, tiles issued
constexpr int kSmemUsed = kOffAbort + 8;
constexpr int kSmemBytes = kSmemUsed + 1024;   // slack for the 1024-byte alignment
// end-of-split merge, reusing the ring: per warp m[8], l[8], o[8][264]
// (head stride 264 floats spreads the 4 heads a warp writes at once over banks)
constexpr int kMergeHead = 264;
constexpr int kMergeWarpFloats = 16 + 8 * kMergeHead;
constexpr int kOffMergeF = kWarps * kMergeWarpFloats * 4;  // per-warp m, l [warp][8], then M, L
static_assert(kStages % 2 == 0, "each stage must serve one warp group");
static_assert(kStageBytes % 1024 == 0, "stages must keep the swizzle atoms aligned");
static_assert(kOffMergeF + (2 * kWarps + 2) * 8 * 4 <= kStages * kStageBytes, "merge fits the ring");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

using namespace dec;

// STREAM: the balanced schedule over all units (gridDim.x CTAs) instead of
// one split per CTA (a separate instance, so the split path keeps its code)
template <bool BF16, bool STREAM>
__global__ void __launch_bounds__(kThreads, 1)
    q4_decode_mma_kernel(const __grid_constant__ TmaMaps maps, kvq_cache c,
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
  volatile int *issued = abort_flag + 1;  // tiles issued so far (in order)

  if (tid == 0) {
    prefetch_map(&maps.kc);
    prefetch_map(&maps.vc);
    if (c.block_table) {
      prefetch_map(&maps.kc2);
      prefetch_map(&maps.vc2);
    }
  }
  // inputs may come from the kernel launched just before this one
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
  // this CTA's segments: stream mode walks the (query row, head group) units
  // its share of the concatenated tiles crosses; split mode has the one split
  // (blockIdx.x of row blockIdx.z, head group blockIdx.y)
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
    // fused decode step (pos != nullptr): the new token goes to position pos[b]
    // and the sequence then has pos[b] + 1 tokens
    const int p_new = pos ? __ldg(pos + b) : -1;
    // several queries per sequence (q_to_seq != nullptr): query b reads the cache
    // of sequence bs
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
    // fused step: every CTA whose split holds the new token quantizes the
    // token's K and V rows of its kv head into the cache before it issues a tile
    // load (CTAs of the same kv head write identical bytes)
    const bool appender = p_new >= t0 && p_new < t1;

    // first cache row of the 64-token sub-tile starting at token t, -1 if unmapped
    auto sub_row = [&](int t) -> int {
      if (c.block_table == nullptr) return (int)(((int64_t)bs * c.num_kv_heads + kvh) * c.max_tokens + t);
      const int pi = t / c.page_size;
      const int page = __ldg(c.block_table + (int64_t)bs * c.max_pages_per_seq + pi);
      if (page < 0 || page >= c.num_pages) return -1;
      return (int)(((int64_t)page * c.num_kv_heads + kvh) * c.page_size + (t - pi * c.page_size));
    };
    // one thread: tile `it` onto its stage's full barrier.  Contiguous cache:
    // the tile's rows are consecutive, one 128-row box per code plane and one
    // bulk copy of the scale rows of this (sequence, head) per scale plane.
    // Paged: the same when the tile's two 64-token halves are consecutive rows
    // of one page, else each half that holds tokens of the split on its own.
    // (A tile of 8 copies with 16-byte scale boxes kept the issuing thread busy
    // about twice as long.)
    // first row of a run of scale rows, inside the planes (debug builds check
    // and report; release builds use it as is)
    auto scale_src = [&](int64_t r, int n) -> int64_t {
      return in_bounds(r, r + n, cache_rows(c), err) ? r : 0;
    };
    auto issue = [&](int it) {
      const int st = it % kStages;
      const int tstart = t0 + it * kTile;
      const uint32_t bar = full0 + 8 * st;
      const uint32_t dst = smem_u32(smem + st * kStageBytes);
      if (c.block_table == nullptr) {
        const int r = sub_row(tstart);
        const int nrows = min(kTile, c.max_tokens - tstart);
        mbar_arrive_tx(bar, 2 * kTile * 128 + 2 * nrows * 16);
        tma_load_2d(dst + kOffKC, &maps.kc, 0, r, bar);
        tma_load_2d(dst + kOffVC, &maps.vc, 0, r, bar);
        bulk_load(dst + kOffKS, c.k_scales + scale_src(r, nrows) * kRowScales, nrows * 16, bar);
        bulk_load(dst + kOffVS, c.v_scales + scale_src(r, nrows) * kRowScales, nrows * 16, bar);
      } else {
        const int r0 = sub_row(tstart);
        const int r1 = tstart + kSub < t1 ? sub_row(tstart + kSub) : -1;
        const int n = (r0 >= 0) + (r1 >= 0);
        if (n == 0) {
          mbar_arrive(bar);
        } else if (r0 >= 0 && r1 == r0 + kSub) {
          // both halves on one page, consecutive rows: copies as for a contiguous cache
          mbar_arrive_tx(bar, 2 * kSubBytes);
          tma_load_2d(dst + kOffKC, &maps.kc2, 0, r0, bar);
          tma_load_2d(dst + kOffVC, &maps.vc2, 0, r0, bar);
          bulk_load(dst + kOffKS, c.k_scales + scale_src(r0, kTile) * kRowScales, kTile * 16, bar);
          bulk_load(dst + kOffVS, c.v_scales + scale_src(r0, kTile) * kRowScales, kTile * 16, bar);
        } else {
          mbar_arrive_tx(bar, n * kSubBytes);
          #pragma unroll
          for (int j = 0; j < 2; j++) {
            const int r = j ? r1 : r0;
            if (r < 0) continue;
            tma_load_2d(dst + kOffKC + j * kSub * 128, &maps.kc, 0, r, bar);
            tma_load_2d(dst + kOffVC + j * kSub * 128, &maps.vc, 0, r, bar);
            bulk_load(dst + kOffKS + j * kSub * 16, c.k_scales + scale_src(r, kSub) * kRowScales, kSub * 16, bar);
            bulk_load(dst + kOffVS + j * kSub * 16, c.v_scales + scale_src(r, kSub) * kRowScales, kSub * 16, bar);
          }
        }
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
      // scratch outside the ring (the per-warp scale areas of warps 0 and 1,
      // used only inside the tile loop)
      float4 *scratch = reinterpret_cast<float4 *>(smem + kOffFs);
      {
        const int vg = lane >> 3, i = lane & 7;
        const bool valid = vg < 2;  // lanes 0-7: K, 8-15: V
        const void *src =
            static_cast<const char *>(vg == 1 ? v_new : k_new) +
            ((int64_t)b * c.num_kv_heads + kvh) * kDim * (BF16 ? 2 : 4);
          uint4 bytes;
        uint16_t sc;
        q4v::quantize_vector<BF16>(valid ? src : k_new, valid, lane, scratch + 64 * vg, bytes, sc);
        const int64_t row = q4_row(c, bs, kvh, p_new);
        if (valid && row >= 0 && in_bounds(row, row + 1, cache_rows(c), err)) {
          *reinterpret_cast<uint4 *>((vg ? c.v_codes : c.k_codes) + row * kRowCodeBytes + 16 * i) =
              bytes;
          (vg ? c.v_scales : c.k_scales)[row * kRowScales + i] = sc;
        }
      }
      // the rows are read back by TMA (async proxy)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0 && it_new < kStages) issue(it_new);
    }

    // (1) query: warp w rotates head h0 + w (zeros past gc), splits it into
    // fp16 hi + lo and writes the MMA fragments of its 8 blocks x 2 k-steps
    {
      warp_fwht256(x, lane);
      float hi[8], lo[8], sq = 0.f;
      #pragma unroll
      for (int i = 0; i < 8; i++) {
        const float v = x[i] * 0.0625f;  // the FWHT's 1/16 (exact)
        hi[i] = __half2float(__float2half_rn(v));
        lo[i] = __half2float(__float2half_rn(v - hi[i]));
        sq += hi[i] + lo[i];
      }
      // lane L holds dims 8L..8L+7 = block L/4, k-step (L/2)&1, tg 2(L&1) and 2(L&1)+1
      uint4 *qf = reinterpret_cast<uint4 *>(smem + kOffQF) + (warp * 8 + (lane >> 2)) * 8 +
                  ((lane >> 1) & 1) * 4 + 2 * (lane & 1);
      #pragma unroll
      for (int e = 0; e < 2; e++) {
        const int i = 4 * e;
        qf[e] = make_uint4(pack_f16x2(hi[i], hi[i + 2]), pack_f16x2(lo[i], lo[i + 2]),
                           pack_f16x2(hi[i + 1], hi[i + 3]), pack_f16x2(lo[i + 1], lo[i + 3]));
      }
      sq += __shfl_xor_sync(kFull, sq, 1);
      sq += __shfl_xor_sync(kFull, sq, 2);
      if ((lane & 3) == 0)
        reinterpret_cast<float *>(smem + kOffQB)[warp * 8 + (lane >> 2)] = -kBias * sq;
    }
    __syncthreads();
    uint4 qa[8][2];
    float cb[8];  // accumulator start of the hi rows: -72 * sum over the block of (hi + lo)
    {
      const uint4 *qf = reinterpret_cast<const uint4 *>(smem + kOffQF) + g * 64 + tg;
      #pragma unroll
      for (int bb = 0; bb < 8; bb++) {
        qa[bb][0] = qf[bb * 8];
        qa[bb][1] = qf[bb * 8 + 4];
        cb[bb] = reinterpret_cast<const float *>(smem + kOffQB)[g * 8 + bb];
      }
    }

    // (2) the split: warp group gq = warp / 4 takes the tiles it with it % 2 == gq,
    // warp wi = warp % 4 tokens 32wi .. 32wi + 31 of each of them
    const int gq = warp >> 2, wi = warp & 3;
    float o[8][2][4];  // [block][M-tile X (dims 2g, 2g+1) / Y (16 + 2g, 17 + 2g)][reg]
    #pragma unroll
    for (int bb = 0; bb < 8; bb++)
      #pragma unroll
      for (int m = 0; m < 2; m++) o[bb][m][0] = o[bb][m][1] = o[bb][m][2] = o[bb][m][3] = 0.f;
    float wacc[4] = {0.f, 0.f, 0.f, 0.f};  // sum_t p d_v: head g (hi, lo rows) x blocks 2tg, 2tg+1
    float m_run = -INFINITY, l_run = 0.f;  // head g
    float *fsk = reinterpret_cast<float *>(smem + kOffFs + warp * (kFsK + kFsV));
    __half *fsv = reinterpret_cast<__half *>(smem + kOffFs + warp * (kFsK + kFsV) + kFsK);
    const int row_l = 32 * wi + 8 * ((lane >> 3) & 1) + (lane & 7);  // ldmatrix row (T = 0/1)
    const int blk_l = lane >> 4;

    for (int it = gq; it < ntiles; it += 2) {
      const int st = it % kStages;
      if (!mbar_wait(full0 + 8 * st, (it / kStages) & 1, abort_flag, wait_polls)) {
        *abort_flag = 1;
        report(err, KVQ_DEVERR_WAIT_TIMEOUT);
        break;
      }
      const uint8_t *stage = smem + st * kStageBytes;
      const int tw = t0 + it * kTile + 32 * wi;  // first token of this warp
      const int nvalid = min(32, t1 - tw);
      bool live = nvalid > 0;
      if (live && c.block_table != nullptr) live = sub_row(tw & ~(kSub - 1)) >= 0;
      if (live) {
        {  // widen: lane = token; K scales -> fp32, V scales fp16, [block][pos]; invalid -> 0
          const int t = lane;
          const uint4 wk = *reinterpret_cast<const uint4 *>(stage + kOffKS + (32 * wi + t) * 16);
          const uint4 wv = *reinterpret_cast<const uint4 *>(stage + kOffVS + (32 * wi + t) * 16);
          // pos: 16 * (T >> 1) + 4 * tg + 2 * (T & 1) + e for t = 8T + 2tg + e
          const int T = t >> 3, tg2 = (t >> 1) & 3, e = t & 1;
          const int pos = 16 * (T >> 1) + 4 * tg2 + 2 * (T & 1) + e;
          const bool ok = t < nvalid;
          const uint32_t kk[4] = {wk.x, wk.y, wk.z, wk.w}, vv[4] = {wv.x, wv.y, wv.z, wv.w};
          #pragma unroll
          for (int k2 = 0; k2 < 4; k2++) {
            const float2 pk2 = __half22float2(*reinterpret_cast<const __half2 *>(&kk[k2]));
            fsk[(2 * k2) * 32 + pos] = ok ? pk2.x : 0.f;
            fsk[(2 * k2 + 1) * 32 + pos] = ok ? pk2.y : 0.f;
            const uint32_t v2 = ok ? vv[k2] : 0u;
            reinterpret_cast<uint16_t *>(fsv)[(2 * k2) * 32 + pos] = (uint16_t)(v2 & 0xffffu);
            reinterpret_cast<uint16_t *>(fsv)[(2 * k2 + 1) * 32 + pos] = (uint16_t)(v2 >> 16);
          }
        }
        __syncwarp();
        const uint32_t kbase = smem_u32(stage + kOffKC), vbase = smem_u32(stage + kOffVC);

        // ---- QK: head g, tokens 8T + 2tg + {0, 1}, T = 0..3
        float2 sacc[4];
        #pragma unroll
        for (int T = 0; T < 4; T++) sacc[T] = make_float2(0.f, 0.f);
        #pragma unroll
        for (int bp = 0; bp < 4; bp++) {
          #pragma unroll
          for (int tp = 0; tp < 2; tp++) {  // token groups 2tp, 2tp + 1
            uint32_t kr[4];  // (T0, block 2bp), (T1, 2bp), (T0, 2bp + 1), (T1, 2bp + 1)
            ldsm_x4(kbase + (row_l + 16 * tp) * 128 + (((2 * bp + blk_l) ^ (lane & 7)) << 4), kr);
            #pragma unroll
            for (int half = 0; half < 2; half++) {
              const int bb = 2 * bp + half;
              const float4 dk = *reinterpret_cast<const float4 *>(fsk + bb * 32 + 16 * tp + 4 * tg);
              #pragma unroll
              for (int T = 0; T < 2; T++) {
                const uint32_t w = kr[2 * half + T];
                float acc[4];
                mma16816c(acc, qa[bb][0], nib64(w << 4), nib64(w >> 4), cb[bb], 0.f);
                mma16816(acc, qa[bb][1], nib64(w), nib64(w >> 8));
                const float2 d = T ? make_float2(dk.z, dk.w) : make_float2(dk.x, dk.y);
                sacc[2 * tp + T] = __ffma2_rn(
                    d, __fadd2_rn(make_float2(acc[0], acc[1]), make_float2(acc[2], acc[3])), sacc[2 * tp + T]);
              }
            }
          }
        }
        // ---- online softmax of head g over this warp's 32 tokens
        float x[8];
        #pragma unroll
        for (int T = 0; T < 4; T++) {
          x[2 * T] = sacc[T].x * sl2;
          x[2 * T + 1] = sacc[T].y * sl2;
        }
        if (nvalid < 32) {
          #pragma unroll
          for (int e2 = 0; e2 < 8; e2++)
            if (8 * (e2 >> 1) + 2 * tg + (e2 & 1) >= nvalid) x[e2] = -INFINITY;
        }
        float mx = fmaxf(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])), fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7])));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        if (__any_sync(kFull, mx > m_run)) {
          const float mn = fmaxf(m_run, mx);
          const float alpha = mn == m_run ? 1.f : ex2(m_run - mn);
          m_run = mn;
          l_run *= alpha;
          #pragma unroll
          for (int k = 0; k < 4; k++) wacc[k] *= alpha;  // rows of head g
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
        uint32_t ph[4], pl[4];  // p of head g as fp16 hi + lo pairs, token groups T
        #pragma unroll
        for (int T = 0; T < 4; T++) {
          const float p0 = ex2(x[2 * T] - m_run), p1 = ex2(x[2 * T + 1] - m_run);
          l_run += p0 + p1;
          split_hilo(make_float2(p0, p1), ph[T], pl[T]);
        }
        // ---- PV: k-steps of 16 tokens (token groups 2ks, 2ks + 1)
        #pragma unroll
        for (int ks = 0; ks < 2; ks++) {
          {  // sum_t p d_v for blocks 2tg, 2tg+1 on the tensor cores (d_v exact in fp16)
            const uint2 dvb = *reinterpret_cast<const uint2 *>(fsv + g * 32 + 16 * ks + 4 * tg);
            const uint32_t a[4] = {ph[2 * ks], pl[2 * ks], ph[2 * ks + 1], pl[2 * ks + 1]};
            mma16816(wacc, a, dvb.x, dvb.y);
          }
          #pragma unroll
          for (int bp = 0; bp < 4; bp++) {
            uint32_t vr[4];  // (tokens 0-7, block 2bp), (8-15, 2bp), (0-7, 2bp + 1), (8-15, 2bp + 1)
            ldsm_x4_t(vbase + (row_l + 16 * ks) * 128 + (((2 * bp + blk_l) ^ (lane & 7)) << 4), vr);
            #pragma unroll
            for (int half = 0; half < 2; half++) {
              const int bb = 2 * bp + half;
              const uint2 dvp = *reinterpret_cast<const uint2 *>(fsv + bb * 32 + 16 * ks + 4 * tg);
              const __half2 d01 = *reinterpret_cast<const __half2 *>(&dvp.x);
              const __half2 d89 = *reinterpret_cast<const __half2 *>(&dvp.y);
              // w = p d_v exactly as hi + lo (TwoProduct with fp16 FMA)
              const __half2 ph0 = *reinterpret_cast<const __half2 *>(&ph[2 * ks]);
              const __half2 ph1 = *reinterpret_cast<const __half2 *>(&ph[2 * ks + 1]);
              const __half2 pl0 = *reinterpret_cast<const __half2 *>(&pl[2 * ks]);
              const __half2 pl1 = *reinterpret_cast<const __half2 *>(&pl[2 * ks + 1]);
              const __half2 wh0 = __hmul2_rn(ph0, d01), wh1 = __hmul2_rn(ph1, d89);
              const __half2 wl0 = __hfma2(pl0, d01, __hfma2(ph0, d01, __hneg2(wh0)));
              const __half2 wl1 = __hfma2(pl1, d89, __hfma2(ph1, d89, __hneg2(wh1)));
              const uint32_t bh0 = *reinterpret_cast<const uint32_t *>(&wh0);
              const uint32_t bh1 = *reinterpret_cast<const uint32_t *>(&wh1);
              const uint32_t bl0 = *reinterpret_cast<const uint32_t *>(&wl0);
              const uint32_t bl1 = *reinterpret_cast<const uint32_t *>(&wl1);
              const uint32_t r0 = vr[2 * half], r1 = vr[2 * half + 1];
              {
                const uint32_t a[4] = {nib64(r0 << 4), nib64(r0 >> 4), nib64(r1 << 4), nib64(r1 >> 4)};
                mma16816(o[bb][0], a, bh0, bh1);
                mma16816(o[bb][0], a, bl0, bl1);
              }
              {
                const uint32_t a[4] = {nib64(r0), nib64(r0 >> 8), nib64(r1), nib64(r1 >> 8)};
                mma16816(o[bb][1], a, bh0, bh1);
                mma16816(o[bb][1], a, bl0, bl1);
              }
            }
          }
        }
      }
      // release the stage; the last of its 4 warps refills it with tile it + kStages
      // (same warp group: kStages is even)
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
    // wacc: head g, blocks 2tg (hi + lo rows: [0] + [2]) and 2tg + 1 ([1] + [3])
    const float wA = wacc[0] + wacc[2], wB = wacc[1] + wacc[3];
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
    // per-warp (m, l) of each head, then every warp scales its accumulators to
    // the CTA maximum before storing them, so the final pass only adds
    float *ml = reinterpret_cast<float *>(smem + kOffMergeF);  // m [warp][head], l [warp][head]
    float *mh = ml + 2 * kWarps * 8;                            // M, L per head
    if (!abort_all && tg == 0) {
      ml[warp * 8 + g] = m_run;
      ml[kWarps * 8 + warp * 8 + g] = l_run;
    }
    __syncthreads();
    if (!abort_all) {
      // this thread's accumulator columns are heads 2tg and 2tg + 1
      const int ha = 2 * tg, hb = ha + 1;
      float Ma = -INFINITY, Mb = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kWarps; w++) {
        Ma = fmaxf(Ma, ml[w * 8 + ha]);
        Mb = fmaxf(Mb, ml[w * 8 + hb]);
      }
      const float ma = ml[warp * 8 + ha], mb = ml[warp * 8 + hb];
      const float fa = ma == -INFINITY ? 0.f : ex2(ma - Ma);
      const float fb = mb == -INFINITY ? 0.f : ex2(mb - Mb);
      float *mw = reinterpret_cast<float *>(smem) + warp * kMergeWarpFloats + 16;
        #pragma unroll
        for (int bb = 0; bb < 8; bb++) {
          // wsum of (head h, block bb) lives in lane 4h + bb/2, as wA (bb even) or wB (odd)
          const float sA = __shfl_sync(kFull, (bb & 1) ? wB : wA, 8 * tg + (bb >> 1));
          const float sB = __shfl_sync(kFull, (bb & 1) ? wB : wA, 8 * tg + 4 + (bb >> 1));
          const float cA = kBias * sA, cB = kBias * sB;
          #pragma unroll
          for (int m = 0; m < 2; m++) {
            const int d0 = 32 * bb + 16 * m + 2 * g;  // row g; row g + 8 is d0 + 1
            *reinterpret_cast<float2 *>(mw + ha * kMergeHead + d0) =
                make_float2((o[bb][m][0] - cA) * fa, (o[bb][m][2] - cA) * fa);
            *reinterpret_cast<float2 *>(mw + hb * kMergeHead + d0) =
                make_float2((o[bb][m][1] - cB) * fb, (o[bb][m][3] - cB) * fb);
          }
        }
      if (tid < 8) {
        float M = -INFINITY;
        #pragma unroll
        for (int w = 0; w < kWarps; w++) M = fmaxf(M, ml[w * 8 + tid]);
        float L = 0.f;
        #pragma unroll
        for (int w = 0; w < kWarps; w++) {
          const float mwv = ml[w * 8 + tid];
          L += (mwv == -INFINITY ? 0.f : ex2(mwv - M)) * ml[kWarps * 8 + w * 8 + tid];
        }
        mh[tid] = M;
        mh[8 + tid] = L;
      }
    }
    __syncthreads();
    for (int hh = 0; hh < gc; hh++) {
      float *rec = ws + (rec_base + hh * rec_hstride) * kRec;
      float acc = 0.f;
      if (!abort_all) {
        #pragma unroll
        for (int w = 0; w < kWarps; w++)
          acc += reinterpret_cast<const float *>(smem)[w * kMergeWarpFloats + 16 + hh * kMergeHead + tid];
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

int q4_decode_ctas_per_sm() { return 1; }
int q4_decode_tile_tokens() { return kTile; }

cudaError_t launch_q4_decode_mma(const kvq_cache &c, const void *q, int bf16, int batch,
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
  const uint32_t box = c.block_table ? kSub : kTile;  // rows per code box
  if (!make_map(&maps.kc, c.k_codes, rows, 128, 128, box, true) ||
      !make_map(&maps.vc, c.v_codes, rows, 128, 128, box, true))
    return cudaErrorInvalidValue;
  if (c.block_table) {
    if (!make_map(&maps.kc2, c.k_codes, rows, 128, 128, kTile, true) ||
        !make_map(&maps.vc2, c.v_codes, rows, 128, 128, kTile, true))
      return cudaErrorInvalidValue;
  } else {
    maps.kc2 = maps.kc;
    maps.vc2 = maps.vc;
  }
  // opt in to the large dynamic shared-memory carve-out once per device
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
      const void *fn = variant == 0   ? (const void *)q4_decode_mma_kernel<false, false>
                       : variant == 1 ? (const void *)q4_decode_mma_kernel<true, false>
                       : variant == 2 ? (const void *)q4_decode_mma_kernel<false, true>
                                      : (const void *)q4_decode_mma_kernel<true, true>;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[variant] |= bit;
    }
  }
  // programmatic dependent launch: this grid may be scheduled while the
  // previous kernel on the stream finishes; it waits for it (griddepcontrol)
  // before touching global memory
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
      e = cudaLaunchKernelEx(&cfg, q4_decode_mma_kernel<false, false>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    case 1:
      e = cudaLaunchKernelEx(&cfg, q4_decode_mma_kernel<true, false>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    case 2:
      e = cudaLaunchKernelEx(&cfg, q4_decode_mma_kernel<false, true>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
      break;
    default:
      e = cudaLaunchKernelEx(&cfg, q4_decode_mma_kernel<true, true>, maps, c, q, seq_lens, max_seq_len,
                           n_q_heads, group, gc, sl2, p.split_tokens, p.splits, n_hg,
                           p.n_units, append_tiles, ws, k_new, v_new,
                           pos, q_to_seq, q_to_seq ? num_seqs : batch, err, polls);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvq
