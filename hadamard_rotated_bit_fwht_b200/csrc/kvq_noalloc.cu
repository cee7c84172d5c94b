// kvq_noalloc.cu -- kvq_decode_attn for callers that cannot provide device
// scratch memory.
//
// The split-K decode needs scratch for its per-split partial records.  Some
// callers have no way to obtain it: a plugin interface that hands the library
// only its input and output tensors, a C host program without a device
// allocator, or a latency-critical decode loop that must never call cudaMalloc
// (which is slow and can synchronize the device).  This entry point uses a
// fixed scratch array that lives in the library's own device memory instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Its
// device address is looked up once per device (cudaGetSymbolAddress) on the
// first call made with that device current; host code never passes the
// variable itself to a kernel, since in host code the name is only a host-side
// stand-in for the device symbol.  The cached address belongs to the device's
// primary context: after cudaDeviceReset the module is loaded again and the
// address may change, so this entry point must not be used on a device after
// that device has been reset in the same process.
#include <mutex>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = KVQ_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
float *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (nullptr on error).
float *scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = static_cast<float *>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

KVQ_API kvq_status kvq_decode_attn_noalloc(const kvq_cache *cache, const void *q,
                                           kvq_dtype dtype, int32_t batch,
                                           int32_t num_q_heads, const int32_t *d_seq_lens,
                                           int32_t max_seq_len, float scale, float *out,
                                           void *stream) {
  // The argument checks of kvq_decode_attn come first, so a bad argument gets
  // the status kvq_decode_attn would give it; only a valid shape whose
  // workspace exceeds the array gets KVQ_ERR_WORKSPACE.
  const kvq_status st = kvq::check_decode_args(cache, q, dtype, batch, num_q_heads, d_seq_lens,
                                               max_seq_len, scale, out);
  if (st != KVQ_OK || batch == 0) return st;
  const size_t need = kvq_decode_attn_workspace(cache, batch, num_q_heads, max_seq_len);
  if (need > kNoAllocScratchBytes) return KVQ_ERR_WORKSPACE;
  float *ws = scratch_for_current_device();
  if (ws == nullptr) return KVQ_ERR_CUDA;
  return kvq_decode_attn(cache, q, dtype, batch, num_q_heads, d_seq_lens, max_seq_len, scale,
                         out, ws, kNoAllocScratchBytes, stream);
}

}  // extern "C"
