// kvq_errors.cu -- the device error word: kernels record conditions they
// cannot return as a status (a bounded wait that gave up, a debug-build bounds
// check) with atomicOr into one 32-bit word per device, which
// kvq_device_errors reads and clears.  Also the poll limit of the decode
// kernels' bounded waits (kvq_set_wait_limit).
#include <atomic>
#include <mutex>

#include "kvq_internal.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDefaultPolls = 1 << 20;

static __device__ uint32_t g_device_errors;

std::mutex g_mu;
uint32_t *g_word[kMaxDevices] = {};
std::atomic<int> g_polls{kDefaultPolls};

}  // namespace

namespace kvq {

uint32_t *device_error_word() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_word[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_errors) != cudaSuccess) return nullptr;
    g_word[dev] = static_cast<uint32_t *>(p);
  }
  return g_word[dev];
}

int wait_poll_limit() { return g_polls.load(std::memory_order_relaxed); }

}  // namespace kvq

extern "C" {

KVQ_API kvq_status kvq_device_errors(uint32_t *flags) {
  if (flags == nullptr) return KVQ_ERR_INVALID_ARG;
  *flags = 0;
  uint32_t *word = kvq::device_error_word();
  if (word == nullptr) return KVQ_ERR_CUDA;
  // synchronous on purpose: the word is read after all work on the device
  uint32_t value = 0, zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaMemcpy(&value, word, sizeof(value), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return KVQ_ERR_CUDA;
  *flags = value;
  return KVQ_OK;
}

KVQ_API kvq_status kvq_set_wait_limit(int32_t polls) {
  if (polls < -1) return KVQ_ERR_INVALID_ARG;
  g_polls.store(polls == -1 ? kDefaultPolls : polls, std::memory_order_relaxed);
  return KVQ_OK;
}

}  // extern "C"
