// q4_quant.cu -- FWHT-256 rotation (kvq_rotate) and Q4_0 quantize-on-append
// (kvq_quantize_append) kernels for B200; the warp-level vector code and its
// layout description are in q4_vec.cuh.
//
// Method: Strata PR #21 "Q4_0 KV cache + FWHT-256", How 1 and How 2, with the
// maintainer's tie-break; stage order and end scaling: vLLM rocm_octave page,
// fwht_blocks.
#include <mutex>

#include "q4_vec.cuh"

namespace kvq {
namespace {

using namespace q4v;

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kVecPerWarp = 4;
constexpr int kVecPerCta = kWarps * kVecPerWarp;

// ------------------------------------------------------------------ rotate
template <bool BF16>
__global__ void __launch_bounds__(kThreads, 4) rotate_kernel(const void *__restrict__ x,
                                                          float *__restrict__ y, int64_t n_vec) {
  __shared__ float4 smem[kWarps][kVecPerWarp][64];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vg = lane >> 3, i = lane & 7;
  float4 *buf = smem[warp][vg];
  const int64_t ngroups = (n_vec + kVecPerCta - 1) / kVecPerCta;
  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
    const int64_t v = g * kVecPerCta + warp * kVecPerWarp + vg;
    const bool valid = v < n_vec;
    const size_t esz = BF16 ? 2 : 4;
    const void *src = static_cast<const char *>(x) + (valid ? v : 0) * kDim * esz;
    Raw<BF16> raw;
    fetch_raw<BF16>(src, i, valid, raw);
    float r[32];
    unpack_l0<BF16>(raw, r);
    fwht256_warp(i, buf, r);
    if (valid) {
      float *dst = y + v * kDim;
#pragma unroll
      for (int j = 0; j < 4; j++)
#pragma unroll
        for (int u = 0; u < 8; u++) dst[i + 8 * u + 64 * j] = r[u + 8 * j];
    }
  }
}

// n / d for n < 2^31 by one 64-bit multiply: m = ceil(2^(31+p) / d) with
// 2^(p-1) < d <= 2^p gives floor(n * m / 2^(31+p)) = floor(n / d).
struct FastDiv {
  uint64_t m;
  uint32_t shift;
  uint32_t d;
};

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
  return (uint32_t)(((uint64_t)n * f.m) >> f.shift);
}

// Q8: Q8_0 codes (256-byte code rows) instead of Q4_0 (128-byte rows)
template <bool BF16, bool Q8>
__global__ void __launch_bounds__(kThreads, 5)
    q4_append_kernel(kvq_cache c, const void *__restrict__ k, const void *__restrict__ v,
                     int batch, int t_new, const int32_t *__restrict__ start_pos,
                     FastDiv div_heads, FastDiv div_tnew, uint32_t *__restrict__ err) {
  __shared__ float4 smem[kWarps][kVecPerWarp][64];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vg = lane >> 3, i = lane & 7;
  float4 *buf = smem[warp][vg];
  // code regrouping reuses 128 bytes of this vector's buffer, offset by 16
  // bytes per vector so the four vectors of a warp use different banks
  uint8_t *stage = reinterpret_cast<uint8_t *>(buf) + 16 * vg;
  // counts fit in 31 bits (checked on the host)
  const uint32_t per_tensor = (uint32_t)batch * (uint32_t)t_new * (uint32_t)c.num_kv_heads;
  const uint32_t n_vec = 2u * per_tensor;
  const uint32_t ngroups = (n_vec + kVecPerCta - 1) / kVecPerCta;
  constexpr size_t esz = BF16 ? 2 : 4;
  auto source = [&](uint32_t vid) -> const void * {
    const bool is_v = vid >= per_tensor;
    const uint32_t e = is_v ? vid - per_tensor : vid;
    return static_cast<const char *>(is_v ? v : k) + (size_t)e * kDim * esz;
  };
  // the next group's input is fetched before the current one is processed
  Raw<BF16> raw;
  uint32_t g = blockIdx.x;
  {
    const uint32_t vid = g * kVecPerCta + warp * kVecPerWarp + vg;
    const bool valid = g < ngroups && vid < n_vec;
    fetch_raw<BF16>(valid ? source(vid) : k, i, valid, raw);
  }
  for (; g < ngroups; g += gridDim.x) {
    const uint32_t vid = g * kVecPerCta + warp * kVecPerWarp + vg;
    const bool valid = vid < n_vec;
    float r[32];
    unpack_l0<BF16>(raw, r);
    {
      const uint32_t gn = g + gridDim.x;
      const uint32_t vn = gn * kVecPerCta + warp * kVecPerWarp + vg;
      const bool vnext = gn < ngroups && vn < n_vec;
      fetch_raw<BF16>(vnext ? source(vn) : k, i, vnext, raw);
    }
    fwht256_warp<false>(i, buf, r);
    uint4 bytes[2];
    uint16_t sc;
    if (Q8) {
      q8_quantize_l1(r, lane, i, reinterpret_cast<uint32_t *>(buf), bytes, sc);
    } else {
      QuantOut o;
      q4_quantize_l1(r, lane, i, o);
      bytes[0] = gather_block_bytes(o, stage, i);
      sc = o.scale;
    }
    if (valid) {
      const bool is_v = vid >= per_tensor;
      const uint32_t e = is_v ? vid - per_tensor : vid;
      const uint32_t bt = fdiv(e, div_heads);
      const int h = (int)(e - bt * div_heads.d);
      const uint32_t b = fdiv(bt, div_tnew);
      const int tok = (int)(bt - b * div_tnew.d);
      const int64_t row = q4_row(c, (int)b, h, __ldg(start_pos + b) + tok);
      if (row >= 0 && in_bounds(row, row + 1, cache_rows(c), err)) {
        uint16_t *scales = (is_v ? c.v_scales : c.k_scales) + row * kRowScales;
        if (Q8) {
          uint8_t *codes = (is_v ? c.v_codes : c.k_codes) + row * 256;
          *reinterpret_cast<uint4 *>(codes + 32 * i) = bytes[0];
          *reinterpret_cast<uint4 *>(codes + 32 * i + 16) = bytes[1];
        } else {
          uint8_t *codes = (is_v ? c.v_codes : c.k_codes) + row * kRowCodeBytes;
          *reinterpret_cast<uint4 *>(codes + 16 * i) = bytes[0];
        }
        scales[i] = sc;
      }
    }
  }
}

FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  uint32_t p = 0;
  while ((1u << p) < d) p++;
  f.shift = 31 + p;
  f.m = (((uint64_t)1 << f.shift) + d - 1) / d;
  f.d = d;
  return f;
}

// Grid of a grid-stride kernel: one wave of the CTAs that fit on the SMs at
// once (queried once per kernel), or fewer when there is less work.  A second,
// partial wave would leave most SMs idle while it runs.
template <auto Kernel>
int grid_for(int64_t groups) {
  static std::mutex mu;
  static int per_sm = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (per_sm == 0) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, kThreads, 0) != cudaSuccess ||
          n <= 0)
        n = 1;
      per_sm = n;
    }
  }
  const int64_t cap = (int64_t)kNumSMs * per_sm;
  return (int)(groups < cap ? (groups > 0 ? groups : 1) : cap);
}

}  // namespace

cudaError_t launch_rotate(const void *x, int bf16, float *y, int64_t n_vec, cudaStream_t s) {
  if (n_vec == 0) return cudaSuccess;
  const int64_t groups = (n_vec + kVecPerCta - 1) / kVecPerCta;
  if (bf16) rotate_kernel<true><<<grid_for<rotate_kernel<true>>(groups), kThreads, 0, s>>>(x, y, n_vec);
  else rotate_kernel<false><<<grid_for<rotate_kernel<false>>(groups), kThreads, 0, s>>>(x, y, n_vec);
  return cudaGetLastError();
}

cudaError_t launch_q4_append(const kvq_cache &c, const void *k, const void *v, int bf16,
                             int batch, int t_new, const int32_t *start_pos, cudaStream_t s,
                             int code_bits) {
  const int64_t n_vec = 2LL * batch * t_new * c.num_kv_heads;
  if (n_vec == 0) return cudaSuccess;
  const int64_t groups = (n_vec + kVecPerCta - 1) / kVecPerCta;
  const FastDiv dh = make_fastdiv((uint32_t)c.num_kv_heads), dt = make_fastdiv((uint32_t)t_new);
  uint32_t *err = device_error_word();
#define KVQ_APPEND(B, Q)                                                                     \
  q4_append_kernel<B, Q><<<grid_for<q4_append_kernel<B, Q>>(groups), kThreads, 0, s>>>(      \
      c, k, v, batch, t_new, start_pos, dh, dt, err)
  if (code_bits == 8) {
    if (bf16) KVQ_APPEND(true, true);
    else KVQ_APPEND(false, true);
  } else {
    if (bf16) KVQ_APPEND(true, false);
    else KVQ_APPEND(false, false);
  }
#undef KVQ_APPEND
  return cudaGetLastError();
}

}  // namespace kvq
