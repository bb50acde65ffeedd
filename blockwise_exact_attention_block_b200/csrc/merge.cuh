// merge.cuh - HBM-bound kernels that apply the partial-output update rule
// (merge_rule.cuh) to whole tensors of rows.
//
// Layout: out / block_out [rows, D] fp32, lse / block_lse [rows] fp32.
// Each thread owns float4 column groups of rows; the D/4 threads of one row
// always sit in one warp (32 % (D/4) == 0 is required for the in-warp lse
// hand-off below, so D in {4, 8, 16, 32, 64, 128}), and the loop trip count is
// uniform across each warp so that __syncwarp() is legal.
#pragma once

#include "common.cuh"
#include "merge_rule.cuh"

namespace ra {

constexpr int kMergeThreads = 256;
constexpr int kMergeUnroll = 2;
constexpr int kMaxMergeInputs = 16;

// out, lse <- merge(out, lse; block_out, block_lse), in place.
__global__ void __launch_bounds__(kMergeThreads)
    merge_partial_kernel(float* __restrict__ out, float* __restrict__ lse,
                         const float* __restrict__ block_out, const float* __restrict__ block_lse,
                         long long rows, int vpr /* D / 4 */) {
  const long long nvec = rows * vpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * kMergeUnroll;
  const long long base0 = (static_cast<long long>(blockIdx.x) * blockDim.x * kMergeUnroll) + threadIdx.x;
  float4* o4 = reinterpret_cast<float4*>(out);
  const float4* b4 = reinterpret_cast<const float4*>(block_out);
  for (long long base = base0 - threadIdx.x % 32; base < nvec; base += stride) {
    // `base` is warp-uniform here: the warp's first vector of this sweep
    float4 ov[kMergeUnroll], bv[kMergeUnroll];
    float la[kMergeUnroll], lb[kMergeUnroll];
    long long iv[kMergeUnroll];
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      iv[u] = base + threadIdx.x % 32 + static_cast<long long>(u) * blockDim.x;
      if (iv[u] < nvec) {
        const long long row = iv[u] / vpr;
        ov[u] = o4[iv[u]];
        bv[u] = __ldcs(b4 + iv[u]);
        la[u] = lse[row];
        lb[u] = __ldcs(block_lse + row);
      }
    }
    __syncwarp();  // every lane has read lse[row] before any lane rewrites it
#pragma unroll
    for (int u = 0; u < kMergeUnroll; ++u) {
      if (iv[u] < nvec) {
        const MergeWeights mw = merge_weights(la[u], lb[u]);
        float4 r;
        r.x = merge_out(ov[u].x, bv[u].x, mw.w);
        r.y = merge_out(ov[u].y, bv[u].y, mw.w);
        r.z = merge_out(ov[u].z, bv[u].z, mw.w);
        r.w = merge_out(ov[u].w, bv[u].w, mw.w);
        o4[iv[u]] = r;
        if (iv[u] % vpr == 0) lse[iv[u] / vpr] = mw.lse;
      }
    }
  }
}

struct MergeList {
  const float* outs[kMaxMergeInputs];
  const float* lses[kMaxMergeInputs];
};

// k partials folded left to right on chip; one write of the result.
// out / lse may alias outs[0] / lses[0]: every lane reads its row's lse before
// the warp rewrites it (the lanes of a row share a warp; see the top note).
__global__ void __launch_bounds__(kMergeThreads)
    merge_partials_kernel(const __grid_constant__ MergeList in, int k, float* out, float* lse,
                          long long rows, int vpr) {
  const long long nvec = rows * vpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x % 32;
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x - lane; base < nvec;
       base += stride) {
    const long long i = base + lane;
    const bool act = i < nvec;
    const long long row = act ? i / vpr : 0;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = -INFINITY;
    if (act) {
      acc = reinterpret_cast<const float4*>(in.outs[0])[i];
      l = in.lses[0][row];
      for (int j = 1; j < k; ++j) {
        const float4 bo = __ldcs(reinterpret_cast<const float4*>(in.outs[j]) + i);
        const float bl = in.lses[j][row];
        const MergeWeights mw = merge_weights(l, bl);
        acc.x = merge_out(acc.x, bo.x, mw.w);
        acc.y = merge_out(acc.y, bo.y, mw.w);
        acc.z = merge_out(acc.z, bo.z, mw.w);
        acc.w = merge_out(acc.w, bo.w, mw.w);
        l = mw.lse;
      }
    }
    __syncwarp();
    if (act) {
      reinterpret_cast<float4*>(out)[i] = acc;
      if (i % vpr == 0) lse[row] = l;
    }
  }
}

}  // namespace ra
