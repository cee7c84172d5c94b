// octave.cu -- the Octave KV-cache variant (vLLM API page
// "vllm.v1.attention.ops.rocm_octave"): decode attention over the paged slot
// cache (the SIMT split kernel for the formats the tensor-core kernel does not
// take, the split-K combine and the back-rotation).
//
// Quantize (reference_quantize) lives in octave_quant.cu.
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
                               float *__restrict__ ws, uint32_t *__restrict__ err) {
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
    const int64_t si = ((int64_t)blk * n_kv_heads + kvh) * block_size + (t % block_size);
    if (!in_bounds(si, si + 1, num_blocks * n_kv_heads * block_size, err)) continue;
    const uint8_t *sp = cache + si * P.slot_bytes;
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
  // after the tensor-core split kernel this grid is a programmatic dependent:
  // the records are read only once that grid has finished (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int qh = blockIdx.x, j = threadIdx.x;
  const int qi = qh / n_q_heads;
  const int req = __ldg(q_to_req + qi);
  int klen = min(max(__ldg(q_to_klen + qi), 0), min(max_klen, cap));
  if (req < 0 || req >= num_reqs) klen = 0;
  const float *rec = ws + (int64_t)qh * splits * kORec;
  float M = -INFINITY;
  for (int s = 0; s < splits && klen > 0; s++) M = fmax_nan(M, rec[s * kORec]);
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
  // L = 0: no token; L NaN: a split that gave up (its record is NaN)
  ob[j] = L > 0.f ? O / L : (L == 0.f ? 0.f : __int_as_float(0x7fc00000));
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
    // programmatic dependent launch: scheduled while the split kernel drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_q * n_q_heads);
    cfg.blockDim = dim3(kHead);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, octave_combine_kernel, P, (const float *)ws, q_to_req, q_to_klen,
                           num_reqs, n_q_heads, plan.splits, max_klen, max_blocks * block_size,
                           out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
#define KVQ_LAUNCH(G)                                                                         \
  do {                                                                                        \
    if (bf16)                                                                                 \
      octave_decode_split_kernel<G, true><<<grid, kThreads, 0, s>>>(                         \
          P, query, n_q_heads, group, cache, n_kv_heads, block_size, num_blocks, block_table, \
          num_reqs, max_blocks, q_to_req, q_to_klen, max_klen, sl2, plan.split_tokens,        \
          plan.splits, ws, err);                                                              \
    else                                                                                      \
      octave_decode_split_kernel<G, false><<<grid, kThreads, 0, s>>>(                        \
          P, query, n_q_heads, group, cache, n_kv_heads, block_size, num_blocks, block_table, \
          num_reqs, max_blocks, q_to_req, q_to_klen, max_klen, sl2, plan.split_tokens,        \
          plan.splits, ws, err);                                                              \
  } while (0)
  uint32_t *err = device_error_word();
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
