// octave_quant_f32_v4.cu -- the Octave quantize instances for f32 inputs and
// 4-bit V codes (kernel in octave_quant.cuh).
#include "octave_quant.cuh"

namespace kvq {

KVQ_OCTQ_DECL(octave_quant_f32_v4) {
  using namespace octq;
  const int rb = p.rope_dim / 64;
#define KVQ_OCT_Q(C, R) \
  launch_one<false, C, 4, R>(p, key, value, items, n_kv_heads, slot_mapping, cache, block_size, \
                           num_blocks, s)
  if (p.compact) return KVQ_OCT_Q(true, 0);
  return rb == 0 ? KVQ_OCT_Q(false, 0) : rb == 1 ? KVQ_OCT_Q(false, 1) : KVQ_OCT_Q(false, 2);
#undef KVQ_OCT_Q
}

}  // namespace kvq
