// q4_decode.cu -- single-token decode attention over the Q4_0 + FWHT-256 cache.
//
// Method: Strata PR #21 "Q4_0 KV cache + FWHT-256": What (score invariance
// <Hq, Hk> = <q, k>, so the query is rotated like K), How 2 (nibbles are
// dequantized in registers during the flash-attention score accumulation) and
// the merge note (the per-token path rotates Q and the output).
//
// Split-K flash decoding: the split kernel (tensor cores, q4_decode_mma.cu)
// writes one partial record (m, l, o[256]) per (sequence, q head, split); the
// combine kernel here merges the splits with a log-sum-exp and applies the
// back-rotation H o (FWHT-256) -- once per query head, after the combine.
#include "decode_common.cuh"

namespace kvq {
namespace {

constexpr int kRec = 260;  // floats per partial record: m, l, pad, pad, o[256]

// Log-sum-exp combine of the splits and back-rotation; one CTA of 256 threads
// per (sequence, q head).  Thread j owns dimension j and issues its loads of
// o_s[j] (up to kB splits at a time) first; meanwhile warp 0 reduces the
// split maxima and sums (lane-strided, shuffles) and publishes the weights, so
// a split count of up to kB costs one L2 round trip.  Warp 0 then applies
// the FWHT-256 (8 values per lane: strides 1, 2, 4 in registers, 8 .. 128
// across lanes) and the 1/16.
constexpr int kMaxSplitsSmem = 1024;
constexpr int kMaxStreamUnits = 4096;  // units scanned by every CTA of a stream schedule
// kB: records loaded per round trip.  48 for few heads with many splits; 16
// (4 CTAs per SM) for many heads with few records each
template <int kB>
__global__ void __launch_bounds__(256, kB <= 16 ? 4 : 1)
    q4_decode_combine_kernel(const float *__restrict__ ws, const int32_t *__restrict__ seq_lens,
                             const int32_t *__restrict__ pos, const int32_t *__restrict__ q_to_seq,
                             int num_seqs, int n_q_heads, int splits, int split_tokens,
                             int stream, int n_hg, int n_units, int ctas, int gc, int tile,
                             int append_tiles,
                             int max_seq_len, int cap, float *__restrict__ out) {
  __shared__ float ob[kDim];
  __shared__ float wgt[kMaxSplitsSmem];
  __shared__ float lsum;
  __shared__ int scan[2 * 8 + 4];
  const int bh = blockIdx.x, j = threadIdx.x, lane = j & 31, warp = j >> 5;
  const int b = bh / n_q_heads;
  // the lengths are inputs of the call: the split kernel releases this grid
  // only after its own dependency wait, so they are final here
  auto row_len = [&](int row) {
    return dec::decode_len(row, seq_lens, pos, q_to_seq, num_seqs, max_seq_len, cap);
  };
  const int len = row_len(b);
  // this head's partial records: rec + s * rstride, s < ns
  const float *rec = ws;
  int64_t rstride = kRec;
  int ns = 0;
  if (stream) {
    // the segments of unit u are the CTAs its tiles fall to (slots u + c)
    const int h = bh % n_q_heads, hg = h / gc, hh = h % gc, u = b * n_hg + hg;
    const dec::StreamLoc L = dec::stream_locate<256>(
        n_units,
        [&](int uu) {
          const int l = row_len(uu / n_hg);
          return l > 0 ? (l + tile - 1) / tile + append_tiles : 0;
        },
        [](int) { return -1; }, u, scan);
    const int n = (len + tile - 1) / tile;
    if (n > 0) {
      // the split kernel shares the T tiles over min(ctas, T) CTAs
      const int ge = min(ctas, L.total);
      const int c0 = dec::cta_of_tile(L.want, L.total, ge);
      const int c1 = dec::cta_of_tile(L.want + n - 1, L.total, ge);
      ns = c1 - c0 + 1;
      rec = ws + ((int64_t)(u + c0) * gc + hh) * kRec;
      rstride = (int64_t)gc * kRec;
    }
  } else {
    rec = ws + (int64_t)bh * splits * kRec;
    // splits past the length wrote no record
    ns = min(min(splits, (len + split_tokens - 1) / split_tokens), kMaxSplitsSmem);
  }
  // the partial records come from the split kernel launched just before
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float v[kB];
  auto fetch = [&](int s0) {
    // volatile asm keeps all kB loads ahead of the first use
#pragma unroll
    for (int k = 0; k < kB; k++) {
      const float *src = rec + min(s0 + k, ns - 1) * rstride + 4 + j;
      asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v[k]) : "l"(src));
    }
  };
  // warp 0 fetches the split maxima and sums (lane s: splits s and s + 32)
  // ahead of its record loads
  float2 r0 = make_float2(-INFINITY, 0.f), r1 = make_float2(-INFINITY, 0.f);
  if (warp == 0 && ns <= 64) {
    if (lane < ns) r0 = __ldg(reinterpret_cast<const float2 *>(rec + lane * rstride));
    if (lane + 32 < ns) r1 = __ldg(reinterpret_cast<const float2 *>(rec + (lane + 32) * rstride));
  }
  if (ns > 0) fetch(0);
  if (warp == 0 && ns <= 64) {
    float M = fmax_nan(r0.x, r1.x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmax_nan(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float f0 = (M == -INFINITY || r0.x == -INFINITY) ? 0.f : exp2f(r0.x - M);
    const float f1 = (M == -INFINITY || r1.x == -INFINITY) ? 0.f : exp2f(r1.x - M);
    if (lane < ns) wgt[lane] = f0;
    if (lane + 32 < ns) wgt[lane + 32] = f1;
    float L = f0 * r0.y + f1 * r1.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) lsum = L;
  } else if (warp == 0) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmax_nan(M, __ldg(rec + s * rstride));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmax_nan(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = __ldg(rec + s * rstride);
      const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : exp2f(ms - M);
      wgt[s] = f;
      L += f * __ldg(rec + s * rstride + 1);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) lsum = L;
  }
  __syncthreads();
  const float L = lsum;
  float O = 0.f;
  for (int s0 = 0; s0 < ns; s0 += kB) {
    if (s0 > 0) fetch(s0);
#pragma unroll
    for (int k = 0; k < kB; k++) {
      const float w = s0 + k < ns ? wgt[s0 + k] : 0.f;
      asm volatile("fma.rn.f32 %0, %1, %2, %0;" : "+f"(O) : "f"(w), "f"(v[k]));
    }
  }
  // L = 0: no token (zero row); L NaN: a split that gave up (its record is NaN)
  ob[j] = L > 0.f ? O / L : (L == 0.f ? 0.f : __int_as_float(0x7fc00000));
  __syncthreads();
  if (warp == 0) {
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; i++) x[i] = ob[8 * lane + i];
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
      for (int i = 0; i < 8; i++)
        if ((i & h) == 0) {
          const float a = x[i], c = x[i + h];
          x[i] = a + c;
          x[i + h] = a - c;
        }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = lane & m;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const float o2 = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = upper ? o2 - x[i] : x[i] + o2;
      }
    }
    float4 *dst = reinterpret_cast<float4 *>(out + (int64_t)bh * kDim + 8 * lane);
    dst[0] = make_float4(x[0] * 0.0625f, x[1] * 0.0625f, x[2] * 0.0625f, x[3] * 0.0625f);
    dst[1] = make_float4(x[4] * 0.0625f, x[5] * 0.0625f, x[6] * 0.0625f, x[7] * 0.0625f);
  }
}

}  // namespace

DecodePlan plan_split_k(int units, int max_len, int slots, int max_splits, int granule,
                        int overhead_tokens) {
  // Each of `units` independent problems (sequence, q-head group) is cut into
  // splits of whole `granule`-token tiles, at least 256 tokens each.  With
  // `slots` CTAs resident at once, the kernel takes about
  // waves x (tokens per split + a fixed per-CTA cost); the split count
  // minimising that (fewest splits on ties) wins.
  const int len = max(max_len, 1);
  const int tiles = (len + granule - 1) / granule;
  units = max(units, 1);
  DecodePlan best = {};
  const int min_tiles = max(256 / granule, 1);
  best.split_tokens = max(tiles, min_tiles) * granule;
  best.splits = 1;
  int64_t best_cost = -1;
  const int sp_max = min(tiles, 2 * ((slots + units - 1) / units) + 1);
  for (int sp = 1; sp <= sp_max; sp++) {
    const int per = max((tiles + sp - 1) / sp, min_tiles) * granule;
    const int splits = (len + per - 1) / per;
    if (splits > max_splits) continue;
    const int64_t waves = ((int64_t)units * splits + slots - 1) / slots;
    const int64_t cost = waves * (per + overhead_tokens);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best.split_tokens = per;
      best.splits = splits;
    }
  }
  while (best.splits > max_splits) {  // very long contexts: larger splits
    best.split_tokens *= 2;
    best.splits = (len + best.split_tokens - 1) / best.split_tokens;
  }
  return best;
}

DecodePlan plan_decode(int batch, int n_head_groups, int max_seq_len, int tile) {
  DecodePlan p = {};
  p.n_units = batch * n_head_groups;
  p.tile = tile;
  const int slots = kNumSMs * q4_decode_ctas_per_sm();
  if (p.n_units * 4 < slots) {
    // few long rows: one wave of equal splits (~3 tiles' worth of per-CTA work:
    // query rotation, ring fill, final merge); as even as the stream schedule
    // without its length scan
    DecodePlan q = plan_split_k(p.n_units, max_seq_len, slots, kMaxSplitsSmem, 128, 3 * 128);
    q.n_units = p.n_units;
    q.tile = tile;
    return q;
  }
  if (p.n_units <= kMaxStreamUnits) {
    // stream schedule: every CTA takes an equal share of all units' tiles,
    // whatever the (device-side) lengths; at most one CTA per tile
    const int64_t tiles_max = (int64_t)p.n_units * ((max(max_seq_len, 1) + tile - 1) / tile);
    p.stream = 1;
    p.ctas = tiles_max < slots ? (int)(tiles_max > 0 ? tiles_max : 1) : slots;
    p.splits = 0;
    p.split_tokens = tile;
    return p;
  }
  // very many rows: fixed chunks of 16 tiles, handed out by the block
  // scheduler in order, so short sequences leave room for long ones (chunks
  // past a length exit at once)
  p.split_tokens = 16 * 128;
  p.splits = max((max(max_seq_len, 1) + p.split_tokens - 1) / p.split_tokens, 1);
  while (p.splits > kMaxSplitsSmem) {
    p.split_tokens *= 2;
    p.splits = (max(max_seq_len, 1) + p.split_tokens - 1) / p.split_tokens;
  }
  return p;
}

size_t decode_workspace_bytes(int batch, int n_q_heads, const DecodePlan &p) {
  if (p.stream) {
    const int gc = n_q_heads / max(p.n_units / max(batch, 1), 1);
    return (size_t)(p.n_units + p.ctas) * gc * kRec * sizeof(float);
  }
  return (size_t)batch * n_q_heads * p.splits * kRec * sizeof(float);
}

cudaError_t launch_q4_decode(const kvq_cache &c, const void *q, int bf16, int batch,
                             int n_q_heads, const int32_t *seq_lens, int max_seq_len,
                             float scale, float *out, float *ws, const DecodePlan &p,
                             cudaStream_t s, const void *k_new, const void *v_new,
                             const int32_t *pos, const int32_t *q_to_seq, int num_seqs) {
  if (batch == 0) return cudaSuccess;
  cudaError_t e =
      c.code_bits == 8
          ? launch_q8_decode_mma(c, q, bf16, batch, n_q_heads, seq_lens, max_seq_len, scale, ws, p,
                                 s, k_new, v_new, pos, q_to_seq, num_seqs)
          : launch_q4_decode_mma(c, q, bf16, batch, n_q_heads, seq_lens, max_seq_len, scale, ws, p,
                                 s, k_new, v_new, pos, q_to_seq, num_seqs);
  if (e != cudaSuccess) return e;
  const int cap = c.block_table ? c.max_pages_per_seq * c.page_size : c.max_tokens;
  // programmatic dependent launch: scheduled while the split kernel drains,
  // waits for its records with griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch * n_q_heads);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int n_hg = p.n_units / batch;
  // records per head: the splits, or the CTAs one unit's tiles spread over
  const int per_head = p.stream ? p.ctas / max(p.n_units, 1) + 2 : p.splits;
  e = cudaLaunchKernelEx(&cfg,
                         per_head <= 16 ? q4_decode_combine_kernel<16> : q4_decode_combine_kernel<48>,
                         (const float *)ws, seq_lens, pos,
                         q_to_seq, q_to_seq ? num_seqs : batch, n_q_heads, p.splits,
                         p.split_tokens, p.stream, n_hg, p.n_units, p.ctas, n_q_heads / n_hg,
                         p.tile, p.stream && pos ? dec::kAppendTokens / p.tile : 0, max_seq_len, cap,
                         out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace kvq
