// skip_rule.cuh -- the Skip-Softmax row test shared by the prefill and decode
// kernels.
//
// The TensorRT-LLM Skip-Softmax article ("Skip Softmax 的三步走算法" section)
// compares a block's local maximum logit with the running maximum and skips
// the block when the gap exceeds the threshold t = threshold_scale_factor / L
// ("实战演练" section).  In exp form a row passes when
// exp(m_local - m_run) < t.  The kernels keep logits pre-multiplied by log2(e),
// so the same test reads (m_local - m_run) < log2(t) in log2 units.
#pragma once

namespace sskip {

// m_local = -inf: the row sees no key in this tile; it passes iff t > 0.
// m_run = -inf with a finite m_local: nothing kept yet, so the row fails
// (the first visited tile of a row is never skipped).
__device__ __forceinline__ bool row_passes_log2(float m_local, float m_run, float log2_t,
                                                bool t_positive) {
  if (m_local == -INFINITY) return t_positive;
  if (m_run == -INFINITY) return false;
  return (m_local - m_run) < log2_t;
}

}  // namespace sskip
