// permute.cuh - token-row reordering between original order and block order
// (contiguous or zigzag partition), optionally fused with a dtype cast.
//
// TokenRing review (pith.science, arXiv 2412.20501), "If this is right": the
// zigzag causal partition.  The pages give no pseudo-code (same page, "minor
// comments, section 3.3.2"); the partition used here: chunk size
// c = S / (2n), block r holds chunk r followed by chunk 2n-1-r, so block-order
// row p = r*L + t holds original token
//     perm(p) = r*c + t              for t <  c
//               (2n-1-r)*c + (t - c) for t >= c.
// Rows are [H, D] elements, contiguous; every row moves as a whole.
#pragma once

#include "common.cuh"

namespace ra {

struct PermGeom {
  int S, L, c, n;
  int zigzag;
};

__device__ __forceinline__ int perm_of(const PermGeom& g, int p) {
  if (!g.zigzag) return p;
  const int r = p / g.L;
  const int t = p - r * g.L;
  return t < g.c ? r * g.c + t : (2 * g.n - 1 - r) * g.c + (t - g.c);
}

// Bit-exact row move with vector type V (row_vecs vectors of V per row).
//   inverse = 0: dst[b, p] = src[b, perm(p)];  inverse = 1: dst[b, perm(p)] = src[b, p]
template <typename V>
__global__ void __launch_bounds__(256)
    permute_rows_kernel(const V* __restrict__ src, V* __restrict__ dst, int B, PermGeom g,
                        long long row_vecs, int inverse) {
  const long long nvec = static_cast<long long>(B) * g.S * row_vecs;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    const long long row = i / row_vecs;
    const long long col = i - row * row_vecs;
    const int b = static_cast<int>(row / g.S);
    const int p = static_cast<int>(row - static_cast<long long>(b) * g.S);
    const long long other = (static_cast<long long>(b) * g.S + perm_of(g, p)) * row_vecs + col;
    if (inverse) dst[other] = __ldcs(src + i);
    else dst[i] = __ldcs(src + other);
  }
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Row move fused with a cast (fp32 -> bf16 round-to-nearest-even, or a plain
// copy when Tin == Tout).  8 elements per thread; row_elems % 8 == 0.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256)
    permute_cast_kernel(const Tin* __restrict__ src, Tout* __restrict__ dst, int B, PermGeom g,
                        long long row_elems, int inverse) {
  const long long row_oct = row_elems / 8;
  const long long noct = static_cast<long long>(B) * g.S * row_oct;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < noct; i += stride) {
    const long long row = i / row_oct;
    const long long col = i - row * row_oct;
    const int b = static_cast<int>(row / g.S);
    const int p = static_cast<int>(row - static_cast<long long>(b) * g.S);
    const long long orow = static_cast<long long>(b) * g.S + perm_of(g, p);
    const long long si = (inverse ? row : orow) * row_elems + col * 8;
    const long long di = (inverse ? orow : row) * row_elems + col * 8;
    Tout v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = from_f32<Tout>(to_f32<Tin>(src[si + e]));
    if constexpr (sizeof(Tout) == 2) {
      *reinterpret_cast<uint4*>(dst + di) = *reinterpret_cast<const uint4*>(v);
    } else {
      reinterpret_cast<uint4*>(dst + di)[0] = reinterpret_cast<const uint4*>(v)[0];
      reinterpret_cast<uint4*>(dst + di)[1] = reinterpret_cast<const uint4*>(v)[1];
    }
  }
}

}  // namespace ra
