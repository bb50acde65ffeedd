// merge_rule.cuh - the partial-output update rule in fp32, shared by the
// merge kernels and the attention epilogue.
//
// TokenRing review (pith.science, arXiv 2412.20501), "What carries the
// argument":
//     out <- out - sigma(block_lse - lse) * (out - block_out)
//     lse <- lse - ln sigma(lse - block_lse)
// Evaluated without overflow: with d = block_lse - lse and e = exp(-|d|),
//     sigma(d)            = 1 / (1 + e)  for d >= 0,   e / (1 + e)  for d < 0
//     -ln sigma(lse - bl) = max(d, 0) + log1p(e)
// lse = -inf marks an empty partial: merging an empty block changes nothing;
// merging into an empty state copies the block (where the literal formula
// would form -inf - (-inf)).
#pragma once

#include <math.h>

namespace ra {

struct MergeWeights {
  float w;     // weight of block_out
  float lse;   // merged lse
};

__device__ __forceinline__ MergeWeights merge_weights(float lse, float block_lse) {
  MergeWeights r;
  if (block_lse == -INFINITY) {  // empty block: keep the state
    r.w = 0.f;
    r.lse = lse;
  } else if (lse == -INFINITY) {  // empty state: take the block
    r.w = 1.f;
    r.lse = block_lse;
  } else {
    const float d = block_lse - lse;
    const float e = expf(-fabsf(d));
    const float inv = 1.f / (1.f + e);
    r.w = d >= 0.f ? inv : e * inv;
    r.lse = lse + fmaxf(d, 0.f) + log1pf(e);
  }
  return r;
}

__device__ __forceinline__ float merge_out(float out, float block_out, float w) {
  return out - w * (out - block_out);
}

}  // namespace ra
