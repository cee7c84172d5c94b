// octave_quant.cu -- dispatch of kvq_octave_quantize to the format instances
// (kernel and its description in octave_quant.cuh).
#include "octave_quant.cuh"

namespace kvq {

cudaError_t launch_octave_quantize(const OctaveParams &p, const void *key, const void *value,
                                   int bf16, int num_tokens, int n_kv_heads,
                                   const int64_t *slot_mapping, uint8_t *cache,
                                   int block_size, int64_t num_blocks, cudaStream_t s) {
  const int64_t items = (int64_t)num_tokens * n_kv_heads;
  if (items == 0) return cudaSuccess;
  if (p.head_size != 128 || p.rope_dim < 0 || p.rope_dim > 128 || p.rope_dim % 64)
    return cudaErrorInvalidValue;
  auto fn = bf16 ? (p.v_bits == 4 ? octave_quant_bf16_v4 : octave_quant_bf16_v3)
                 : (p.v_bits == 4 ? octave_quant_f32_v4 : octave_quant_f32_v3);
  return fn(p, key, value, items, n_kv_heads, slot_mapping, cache, block_size, num_blocks, s);
}

}  // namespace kvq
