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
constexpr int kMergeUnroll = 1;  // float4 vectors per lane and warp sweep (pairwise)
constexpr int kMaxMergeInputs = 16;

// Work split of the merge kernels: the vectors are cut into sweeps of one
// warp (32 * V vectors, whole rows since D / 4 divides 32), and the warps of
// the grid take the sweeps in turn (grid stride).  The grid holds many more
// blocks than are resident at once, so the block scheduler keeps every SM fed
// to the end even though SMs do not all stream at the same rate.  One vector
// per lane and sweep with a large grid (launch_merge in api.cu) measured best:
// many small independent warps keep more loads in flight early in a launch
// than a few warps that each hold two vectors.
// out, lse <- merge(out, lse; block_out, block_lse), in place.
__global__ void __launch_bounds__(kMergeThreads)
    merge_partial_kernel(float* __restrict__ out, float* __restrict__ lse,
                         const float* __restrict__ block_out, const float* __restrict__ block_lse,
                         long long rows, int vpr /* D / 4 */) {
  constexpr int V = kMergeUnroll;
  const long long nvec = rows * vpr;
  const long long sweeps = (nvec + 32 * V - 1) / (32 * V);
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  float4* o4 = reinterpret_cast<float4*>(out);
  const float4* b4 = reinterpret_cast<const float4*>(block_out);
  for (long long g = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < sweeps;
       g += nw) {
    const long long base = g * 32 * V;  // the warp's first vector of this sweep
    float4 ov[V], bv[V];
    float la[V], lb[V];
    long long iv[V];
    bool act[V];
#pragma unroll
    for (int u = 0; u < V; ++u) {
      iv[u] = base + 32 * u + lane;
      act[u] = iv[u] < nvec && RA_IN_BOUNDS(iv[u] / vpr, rows);
      if (act[u]) {
        const long long row = iv[u] / vpr;
        ov[u] = o4[iv[u]];
        bv[u] = __ldcs(b4 + iv[u]);
        la[u] = lse[row];
        lb[u] = __ldcs(block_lse + row);
      }
    }
    __syncwarp();  // every lane has read lse[row] before any lane rewrites it
#pragma unroll
    for (int u = 0; u < V; ++u) {
      if (act[u]) {
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

// k = K partials merged on chip; one write of the result.  Folding the
// update rule left to right k - 1 times gives, for every row,
//     lse = ln sum_j exp(lse_j),   out = sum_j exp(lse_j - lse) * out_j,
// the softmax merge of the k partials; this kernel evaluates that closed
// form (maximum, sum of exponentials, one logarithm, weighted sum), whose k
// exponentials are independent, instead of a chain of k - 1 dependent rule
// applications (the chain left the k = 16 kernel bound by instruction
// latency).  Partials with lse = -inf get weight 0; when every partial is
// empty the state stays partial 0, as the fold leaves it.
// K is a compile-time constant so that every partial's load is issued before
// any is used (K loads in flight per vector); one vector per lane and sweep.
// out / lse may alias outs[0] / lses[0]: every lane reads its row's lse before
// the warp rewrites it (the lanes of a row share a warp; see the top note).
template <int K>
__global__ void __launch_bounds__(kMergeThreads)
    merge_partials_kernel(const __grid_constant__ MergeList in, float* out, float* lse, long long rows, int vpr) {
  constexpr int V = 1;
  const long long nvec = rows * vpr;
  const long long sweeps = (nvec + 32 * V - 1) / (32 * V);
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (long long g = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < sweeps;
       g += nw) {
    const long long base = g * 32 * V;
    long long iv[V], row[V];
    bool act[V];
    float4 v[V][K];
    float l[V][K];
#pragma unroll
    for (int u = 0; u < V; ++u) {
      iv[u] = base + 32 * u + lane;
      act[u] = iv[u] < nvec && RA_IN_BOUNDS(iv[u] / vpr, rows);
      row[u] = act[u] ? iv[u] / vpr : 0;
      if (act[u]) {
#pragma unroll
        for (int j = 0; j < K; ++j) {
          v[u][j] = j == 0 ? reinterpret_cast<const float4*>(in.outs[0])[iv[u]]
                           : __ldcs(reinterpret_cast<const float4*>(in.outs[j]) + iv[u]);
          l[u][j] = in.lses[j][row[u]];
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < V; ++u) {
      if (!act[u]) continue;
      float m = l[u][0];
#pragma unroll
      for (int j = 1; j < K; ++j) m = fmaxf(m, l[u][j]);
      float4 acc = v[u][0];
      float la = -INFINITY;
      if (m != -INFINITY) {
        float e[K], ssum = 0.f;
#pragma unroll
        for (int j = 0; j < K; ++j) {
          e[j] = expf(l[u][j] - m);  // 0 for an empty partial
          ssum += e[j];
        }
        const float inv = 1.f / ssum;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < K; ++j) {
          const float w = e[j] * inv;
          if (w != 0.f) {
            acc.x = fmaf(w, v[u][j].x, acc.x);
            acc.y = fmaf(w, v[u][j].y, acc.y);
            acc.z = fmaf(w, v[u][j].z, acc.z);
            acc.w = fmaf(w, v[u][j].w, acc.w);
          }
        }
        la = m + logf(ssum);
      }
      reinterpret_cast<float4*>(out)[iv[u]] = acc;
      if (iv[u] % vpr == 0) lse[row[u]] = la;
    }
  }
}

}  // namespace ra
