// decode_common.cuh -- device and host helpers shared by the split-K decode
// kernels (q4_decode_mma.cu, q8_decode_mma.cu): bounded mbarrier waits, TMA
// loads and tensor maps, ldmatrix / mma.sync wrappers, the fp16 hi/lo split,
// programmatic-dependent-launch controls and the in-register FWHT-256.
// Nothing here is part of the C ABI.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kvq_internal.cuh"

namespace kvq {
namespace dec {

constexpr unsigned kFullMask = 0xffffffffu;

// bounded waits: ~2^20 polls of up to ~1 us each, abandoned early once any
// thread of the CTA has given up
constexpr int kWaitPolls = 1 << 20;

// code planes; scale rows are contiguous and come by 1-D bulk copies.  kc2,
// vc2: the same planes with boxes of twice the rows (paged Q4_0 tiles whose
// two halves are consecutive rows of one page)
struct TmaMaps {
  CUtensorMap kc, vc, kc2, vc2;
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
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(1000u)
      : "memory");
  return done != 0;
}
// non-blocking test of the phase with this parity
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// true once the phase with this parity has completed; false after one
// non-blocking test and `polls` further polls (0: the test alone), or once
// *abort is set (by any thread of the CTA).  The common case, a tile that has
// already landed, is the one test and a branch.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          const volatile int *abort, int polls) {
  if (mbar_test(bar, parity)) return true;
  for (int i = 0; i < polls; i++) {
    if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
  }
  return false;
}
// record a condition in the library's device error word (see kvq_device_errors)
__device__ __forceinline__ void report(uint32_t *err, uint32_t flag) {
  if (err != nullptr) atomicOr(err, flag);
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// 1-D bulk copy of `bytes` bytes (a multiple of 16; both addresses 16-byte
// aligned) onto the barrier's transaction count
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// d += A(16 x 16, f16, row) * B(16 x 8, f16, col) in fp32
__device__ __forceinline__ void mma16816(float (&d)[4], const uint4 &a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d = A * B + c with the accumulator input c kept intact
__device__ __forceinline__ void mma16816c(float (&d)[4], const uint4 &a, uint32_t b0, uint32_t b1,
                                          float c0, float c1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%11,%11};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1), "f"(c0), "f"(c1));
}

// nibbles at bits 4..7 and 20..23 of x -> half2 (64 + c) exactly
__device__ __forceinline__ uint32_t nib64(uint32_t x) {
  uint32_t h;
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x54005400, 0xEA;" : "=r"(h) : "r"(x));  // (x & m) | c
  return h;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// fp32 pair -> fp16 hi + lo pairs (w ~= hi + lo to ~22 bits)
__device__ __forceinline__ void split_hilo(float2 w, uint32_t &hi, uint32_t &lo) {
  hi = pack_f16x2(w.x, w.y);
  const float2 hf = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
  lo = pack_f16x2(w.x - hf.x, w.y - hf.y);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// in-register FWHT-256 of one vector held as 8 consecutive values per lane
// (lane L: dims 8L .. 8L+7); stages h = 1, 2, ..., 128 in order, no scaling
__device__ __forceinline__ void warp_fwht256(float (&x)[8], int lane) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; i++)
      if ((i & h) == 0) {
        const float a = x[i], c = x[i + h];
        x[i] = a + c;
        x[i + h] = a - c;
      }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = lane & m;  // this lane holds the i + h half of each pair
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float o = __shfl_xor_sync(kFullMask, x[i], m);
      x[i] = upper ? o - x[i] : x[i] + o;
    }
  }
}


// ---- work schedule shared by the split and combine kernels
// Attended length of query row b of a decode call: the fused step attends
// pos[b] + 1 tokens, several queries per sequence read sequence q_to_seq[b]
// (outside [0, num_seqs): nothing), clamped to [0, min(max_seq_len, cap)].
__device__ __forceinline__ int decode_len(int b, const int32_t *seq_lens, const int32_t *pos,
                                          const int32_t *q_to_seq, int num_seqs, int max_seq_len,
                                          int cap) {
  const int bs = q_to_seq ? __ldg(q_to_seq + b) : b;
  const int raw =
      (bs < 0 || bs >= num_seqs) ? 0 : (pos ? __ldg(pos + b) + 1 : __ldg(seq_lens + b));
  return min(max(raw, 0), min(max_seq_len, cap));
}

// Balanced schedule over all (query row, head group) units of a call: unit
// u = b * n_hg + hg holds ceil(len_b / tile) tiles; the units' tiles are laid
// end to end and CTA c of G' = min(G, T) takes tiles [c T / G', (c + 1) T / G')
// (at least one each; CTAs c >= G' have none).  A CTA may cross unit
// boundaries; each (unit, CTA) overlap is one segment, whose partial records
// sit at slot u + c (u + c grows strictly along the tiles, so slots are unique
// and below n_units + G).
// tokens of work the fused append of the new token is counted as when the
// stream schedule shares a unit's tiles (it costs its CTA a few microseconds)
constexpr int kAppendTokens = 256;

struct StreamLoc {
  int total;   // T
  int unit;    // unit holding the probed tile (-1 if none)
  int start;   // first tile of that unit
  int want;    // first tile of the unit asked for (0 if none asked)
};
// the CTA of G' owning tile t
__device__ __forceinline__ int cta_of_tile(int t, int total, int ctas) {
  return (int)(((int64_t)(t + 1) * ctas - 1) / total);
}
// Block-wide (kThreads threads, all must call): T, the unit holding tile
// probe(T) (a functor of T, e.g. this CTA's first tile) and the first tile of
// unit want_unit.  sm: 2 * warps + 4 ints of shared memory.
template <int kThreads, class TilesFn, class ProbeFn>
__device__ StreamLoc stream_locate(int n_units, TilesFn tiles, ProbeFn probe, int want_unit,
                                   int *sm) {
  constexpr int kW = kThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n_units + kThreads - 1) / kThreads;
  const int u0 = min(n_units, tid * per), u1 = min(n_units, u0 + per);
  int local = 0;
  for (int u = u0; u < u1; u++) local += tiles(u);
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(kFullMask, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sm[warp] = incl;
  if (tid == 0) {
    sm[2 * kW] = -1;
    sm[2 * kW + 1] = 0;
    sm[2 * kW + 2] = 0;
  }
  __syncthreads();
  int base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kW; w++) {
    base += w < warp ? sm[w] : 0;
    total += sm[w];
  }
  const int p = probe(total);
  int S = base + incl - local;  // first tile of unit u0
  for (int u = u0; u < u1; u++) {
    const int n = tiles(u);
    if (n > 0 && S <= p && p < S + n) {
      sm[2 * kW] = u;
      sm[2 * kW + 1] = S;
    }
    if (u == want_unit) sm[2 * kW + 2] = S;
    S += n;
  }
  __syncthreads();
  StreamLoc r;
  r.total = total;
  r.unit = sm[2 * kW];
  r.start = sm[2 * kW + 1];
  r.want = sm[2 * kW + 2];
  __syncthreads();  // sm may be reused
  return r;
}

// ---- host: 2-D tensor maps over the cache planes (cached per plane)
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// rows x row_bytes uint8 plane, boxes of box_rows rows x box_cols bytes (the
// maps are cached per plane and box)
// planes > 1: the rows are cut into `planes` column planes of box_cols bytes
// (box_cols * planes == row_bytes), and one box brings box_rows rows of every
// plane, laid out plane after plane (a 3-D map whose outer dimension steps
// box_cols bytes along the row), the same shared-memory image as `planes`
// 2-D boxes at consecutive column offsets
inline bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t row_bytes,
                     uint32_t box_cols, uint32_t box_rows, bool swizzle, uint32_t planes = 1) {
  struct Entry {
    const void *base;
    uint64_t rows;
    uint32_t row_bytes, box_cols, box_rows, planes;
    CUtensorMap map;
  };
  static Entry cache[16];
  static int next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : cache)
    if (e.base == base && e.rows == rows && e.row_bytes == row_bytes && e.box_cols == box_cols &&
        e.box_rows == box_rows && e.planes == planes) {
      *m = e.map;
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  if (planes < 1 || (planes > 1 && box_cols * planes != row_bytes)) return false;
  const cuuint64_t dims[3] = {planes > 1 ? box_cols : row_bytes, rows, planes};
  const cuuint64_t strides[2] = {row_bytes, box_cols};
  const cuuint32_t box[3] = {box_cols, box_rows, planes};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, planes > 1 ? 3 : 2, const_cast<void *>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cache[next] = Entry{base, rows, row_bytes, box_cols, box_rows, planes, *m};
  next = (next + 1) % 16;
  return true;
}

}  // namespace dec
}  // namespace kvq
