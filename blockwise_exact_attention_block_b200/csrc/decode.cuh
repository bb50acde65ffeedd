// decode.cuh - decode-phase attention over a KV cache: a few query tokens
// against a long cache split into chunks, one partial (out, lse) per chunk,
// the partials stitched with the merge rule (merge_rule.cuh).
//
// TokenRing review (pith.science, arXiv 2412.20501), "Reading between the
// lines": the decode phase as KV-cache chunking, partial results merged by
// the same update rule as the prefill blocks.
//
// Queries are the last Tq tokens of the sequence: query token i has position
// Skv - Tq + i and, when causal, sees the cached keys j <= Skv - Tq + i.
//
// This path is bound by HBM: each cached K/V element is used by the
// gqa_groups * Tq (<= 64) query rows of its KV head only.  So the kernel
// streams the cache once, in 64-key tiles staged by TMA (128-byte swizzle)
// through an mbarrier ring, and computes the two small products with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) on fragments loaded by
// ldmatrix: with at most 64 rows the 128-row tcgen05 tiles would be mostly
// padding, and the instruction count, not the math, is what must stay small.
// Grid: (KV head, KV chunk, batch); the host sizes the chunks so the grid
// fills the GPU.  A second kernel folds each row's chunk partials with the
// merge rule.
#pragma once

#include "common.cuh"
#include "merge_rule.cuh"
#include "permute.cuh"

namespace ra {

constexpr int kDecThreads = 256;
constexpr int kDecKeys = 64;     // keys per KV tile
constexpr int kDecMaxRows = 64;  // query rows per KV head: gqa_groups * Tq
constexpr int kDecStages = 3;

struct DecodeArgs {
  int B, Tq, Skv, Hq, Hkv, groups, causal;
  int rows;     // gqa_groups * Tq: query rows of one KV head
  int chunk;    // keys per chunk, a multiple of kDecKeys
  float scale_log2;
  const __nv_bfloat16* q;  // [B, Tq, Hq, D]
  float* part_out;         // [n_splits][B * Tq * Hq][D]
  float* part_lse;         // [n_splits][B * Tq * Hq]
};

// Shared memory of the partial kernel with MT 16-row tiles of query rows.
template <int D, int MT>
struct DecSmem {
  static constexpr int kBox = kDecKeys * 128;    // 64 keys x 64 bf16: one TMA box, 8 KB
  static constexpr int kTile = kBox * (D / 64);  // one K or V tile
  static constexpr int kStage = 2 * kTile;       // K, then V
  static constexpr int kQStride = (D + 8) * 2;   // bytes per Q row (padded: conflict-free ldmatrix)
  static constexpr int kPStride = (kDecKeys + 8) * 2;
  static constexpr int kQ = kDecStages * kStage;               // bf16 [16 MT][D + 8]
  static constexpr int kP = kQ + 16 * MT * kQStride;           // bf16 [16 MT][64 + 8]
  static constexpr int kRedMax = kP + 16 * MT * kPStride;      // fp32 [8 warps][16 MT]
  static constexpr int kRedSum = kRedMax + 8 * 16 * MT * 4;    // fp32 [8 warps][16 MT]
  static constexpr int kBar = kRedSum + 8 * 16 * MT * 4;
  static constexpr int kAbort = kBar + kDecStages * 8;
  static constexpr int kBytes = kAbort + 16 + 1024;  // + slack to align the base to 1024
};

// Byte offset of (key j, column d), d a multiple of 8, in a K or V tile that
// TMA wrote with 128-byte swizzle: 16-byte chunk c of row j sits at chunk
// position c ^ (j % 8) of the row; columns 64.. are in the second box.
__device__ __forceinline__ uint32_t sw128_off(int j, int d) {
  return (d >> 6) * (kDecKeys * 128) + j * 128 + ((((d & 63) >> 3) ^ (j & 7)) << 4);
}

// Four 8x8 bf16 matrices from shared memory; lane l gives the address of row
// l % 8 of matrix l / 8 (plain or transposed distribution).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row-major) * B (16x8 bf16, column-major).
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One CTA: KV head g of batch b, keys [c * chunk, min((c + 1) * chunk, Skv)),
// against the rows = gqa_groups * Tq query rows of that head (row r = token
// r / groups, query head g * groups + r % groups), held as MT tiles of 16 rows
// (rows beyond `rows` are zero and never written).  Per 64-key tile:
//   S = Q K^T   warp w computes the 8 keys [8w, 8w + 8) for every row tile;
//   softmax     row maxima and sums combined across the 8 warps in shared
//               memory; P (bf16) to shared memory;
//   O += P V    warp w owns the D / 8 columns [w D/8, (w + 1) D/8).
// Tensor-core fragments follow mma.m16n8k16: lane l holds rows l / 4 and
// l / 4 + 8 of a tile and columns 2 (l % 4), 2 (l % 4) + 1 of an n8 block.
template <int D, int MT>
__global__ void __launch_bounds__(kDecThreads)
    decode_partial_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ DecodeArgs a) {
  using SL = DecSmem<D, MT>;
  constexpr int NT = D / 64;  // n8 column blocks per warp in the P V product
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* smem = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row / column-pair of this lane
  // heads fastest: the CTAs of one chunk run side by side and sweep the same
  // key rows (all KV heads of a key are adjacent in memory) together
  const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int rows = a.rows;
  const int k0 = split * a.chunk, k1 = min(k0 + a.chunk, a.Skv);
  const int ntiles = (k1 - k0 + kDecKeys - 1) / kDecKeys;
  float* red_max = reinterpret_cast<float*>(smem + SL::kRedMax);
  float* red_sum = reinterpret_cast<float*>(smem + SL::kRedSum);
  const uint32_t bar0 = sb + SL::kBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);

  int issued = 0;                // tiles whose copies thread 0 has issued
  auto load_tile = [&](int t) {  // K and V of tile t into stage t % kDecStages
    const int st = t % kDecStages;
    const uint32_t bar = bar0 + 8u * st;
    mbar_expect_tx(bar, SL::kStage);
    const int key = k0 + t * kDecKeys;
    for (int bx = 0; bx < D / 64; ++bx) {
      tma_load_4d(sb + st * SL::kStage + bx * SL::kBox, &tmK, bx * 64, g, key, b, bar);
      tma_load_4d(sb + st * SL::kStage + SL::kTile + bx * SL::kBox, &tmV, bx * 64, g, key, b, bar);
    }
    issued = t + 1;
  };
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(bar0 + 8u * s, 1);
    *abort_flag = grid_timed_out() ? 1 : 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // the query rows of this KV head (bf16), zero beyond `rows`
  for (int i = tid; i < 16 * MT * (D / 8); i += kDecThreads) {
    const int r = i / (D / 8), c8 = i % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows) {
      const int tok = r / a.groups, h = g * a.groups + r % a.groups;
      v = *reinterpret_cast<const uint4*>(a.q + ((static_cast<long long>(b) * a.Tq + tok) * a.Hq + h) * D + 8 * c8);
    }
    *reinterpret_cast<uint4*>(smem + SL::kQ + r * SL::kQStride + 16 * c8) = v;
  }
  __syncthreads();
  if (tid == 0 && !*abort_flag) {
    for (int t = 0; t < min(ntiles, kDecStages); ++t) load_tile(t);
  }

  // per lane: rows gq and gq + 8 of every row tile
  float m[MT][2], l[MT][2], o[MT][NT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    m[mt][0] = m[mt][1] = -INFINITY;
    l[mt][0] = l[mt][1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  }
  const int last_pos = a.Skv - a.Tq;  // position of query token 0
  // ldmatrix addresses: lane l reads row (l % 8) + 8 ((l / 8) % 2), column block l / 16
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lcol = 8 * (lane >> 4);
  int t = 0;
  for (; t < ntiles; ++t) {
    const int st = t % kDecStages;
    if (!*abort_flag && !mbar_wait(bar0 + 8u * st, (t / kDecStages) & 1, abort_flag)) *abort_flag = 1;
    const uint32_t kt = sb + st * SL::kStage;
    const uint32_t vt = kt + SL::kTile;
    // ---- S = Q K^T for the warp's 8 keys
    float sacc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) sacc[mt][0] = sacc[mt][1] = sacc[mt][2] = sacc[mt][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < D / 32; ++kp) {  // two k16 steps per ldmatrix.x4 of K
      uint32_t kb[4];  // keys 8w.. x columns 32kp + {0, 8, 16, 24}
      ldsm_x4(kt + sw128_off(8 * warp + (lane & 7), 32 * kp + 8 * (lane >> 3)), kb);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          uint32_t qa[4];
          ldsm_x4(sb + SL::kQ + (16 * mt + lrow) * SL::kQStride + 2 * (32 * kp + 16 * h + lcol), qa);
          mma_16816(sacc[mt], qa, kb[2 * h], kb[2 * h + 1]);
        }
      }
    }
    // ---- scale, mask, row maxima of the tile
    const int key0 = k0 + t * kDecKeys + 8 * warp + 2 * tq;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * mt + gq + 8 * hr;
        const int lim = a.causal ? min(k1, last_pos + r / a.groups + 1) : k1;  // keys < lim are visible
#pragma unroll
        for (int e = 0; e < 2; ++e)
          sacc[mt][2 * hr + e] = key0 + e < lim ? sacc[mt][2 * hr + e] * a.scale_log2 : -INFINITY;
        float mx = fmaxf(sacc[mt][2 * hr], sacc[mt][2 * hr + 1]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (tq == 0) red_max[warp * 16 * MT + r] = mx;
      }
    __syncthreads();
    // ---- exponentials against the raised maximum; P (bf16) and row sums
    float alpha[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * mt + gq + 8 * hr;
        float mt_ = red_max[r];
#pragma unroll
        for (int w = 1; w < 8; ++w) mt_ = fmaxf(mt_, red_max[w * 16 * MT + r]);
        const float mn = fmaxf(m[mt][hr], mt_);
        const float base = mn == -INFINITY ? 0.f : mn;
        alpha[mt][hr] = m[mt][hr] == -INFINITY ? 0.f : fast_exp2(m[mt][hr] - base);
        m[mt][hr] = mn;
        const float p0 = fast_exp2(sacc[mt][2 * hr] - base), p1 = fast_exp2(sacc[mt][2 * hr + 1] - base);
        *reinterpret_cast<uint32_t*>(smem + SL::kP + r * SL::kPStride + 2 * (8 * warp + 2 * tq)) =
            pack_bf16x2(p0, p1);
        float sm = p0 + p1;
        sm += __shfl_xor_sync(0xffffffffu, sm, 1);
        sm += __shfl_xor_sync(0xffffffffu, sm, 2);
        if (tq == 0) red_sum[warp * 16 * MT + r] = sm;
      }
    __syncthreads();
    // ---- O = alpha O + P V over the warp's columns
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * mt + gq + 8 * hr;
        float sm = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sm += red_sum[w * 16 * MT + r];
        l[mt][hr] = l[mt][hr] * alpha[mt][hr] + sm;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][2 * hr] *= alpha[mt][hr];
          o[mt][nt][2 * hr + 1] *= alpha[mt][hr];
        }
      }
    const int col0 = warp * (D / 8);
#pragma unroll
    for (int ks = 0; ks < kDecKeys / 16; ++ks) {
      // V^T fragments: keys 16ks.. (+8) x this warp's n8 blocks, transposed
      uint32_t vb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        uint32_t r4[4];
        const int nb = NT == 1 ? 0 : (lane >> 4);  // x4: two n8 blocks of 16 keys (D = 128)
        ldsm_x4_t(vt + sw128_off(16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1), col0 + 8 * (nt + nb)), r4);
        vb[nt][0] = r4[0];
        vb[nt][1] = r4[1];
        if (NT > 1) {
          vb[nt + 1][0] = r4[2];
          vb[nt + 1][1] = r4[3];
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t pa[4];
        ldsm_x4(sb + SL::kP + (16 * mt + lrow) * SL::kPStride + 2 * (16 * ks + lcol), pa);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(o[mt][nt], pa, vb[nt][0], vb[nt][1]);
      }
    }
    __syncthreads();  // the stage, P and the reductions are free
    if (*abort_flag) break;
    if (tid == 0 && t + kDecStages < ntiles) {
      fence_proxy_async_smem();  // this CTA's reads of the stage precede the copy into it
      load_tile(t + kDecStages);
    }
  }
  if (*abort_flag) {  // let every copy already issued land before shared memory is released
    if (tid == 0)
      for (int u = t; u < issued; ++u) mbar_drain(bar0 + 8u * (u % kDecStages), (u / kDecStages) & 1);
    return;
  }
  // ---- the chunk's partial: out = O / l, lse = ln 2 * (m + log2 l); -inf when empty
  const long long rows_all = static_cast<long long>(a.B) * a.Tq * a.Hq;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = 16 * mt + gq + 8 * hr;
      if (r >= rows) continue;
      const int tok = r / a.groups, h = g * a.groups + r % a.groups;
      const long long row = (static_cast<long long>(b) * a.Tq + tok) * a.Hq + h;
      const bool has = l[mt][hr] > 0.f;
      const float inv = has ? 1.f / l[mt][hr] : 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float2*>(a.part_out + (split * rows_all + row) * D + warp * (D / 8) + 8 * nt + 2 * tq) =
            make_float2(o[mt][nt][2 * hr] * inv, o[mt][nt][2 * hr + 1] * inv);
      if (warp == 0 && tq == 0)
        a.part_lse[split * rows_all + row] = has ? (m[mt][hr] + log2f(l[mt][hr])) * 0.6931471805599453f : -INFINITY;
    }
}

// Folds the n_splits partials of every row with the merge rule and writes
// out (fp32 or bf16, nearest even) and lse.  One CTA per row: warp w folds
// the chunks w, w + 8, w + 16, ... (lane i holds D / 32 columns, four chunks'
// loads in flight at a time), then warp 0 folds the eight warp results.  The
// rule is associative and commutative (each fold is a softmax-weighted mean
// over disjoint key sets), so the grouping only changes rounding.
template <int D, typename Tout>
__global__ void __launch_bounds__(256)
    decode_combine_kernel(const float* __restrict__ part_out, const float* __restrict__ part_lse, int n_splits,
                          long long rows, Tout* __restrict__ out, float* __restrict__ lse) {
  constexpr int kPer = D / 32;
  constexpr int kBatch = 4;
  __shared__ float s_out[8][D];
  __shared__ float s_lse[8];
  const long long row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[kPer], l = -INFINITY;
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  for (int s0 = warp; s0 < n_splits; s0 += 8 * kBatch) {
    float bl[kBatch], bo[kBatch][kPer];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int s = s0 + 8 * u;
      bl[u] = -INFINITY;
      if (s < n_splits) {
        bl[u] = part_lse[s * rows + row];
        const float* src = part_out + (s * rows + row) * D + kPer * lane;
#pragma unroll
        for (int e = 0; e < kPer; ++e) bo[u][e] = src[e];
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const MergeWeights mw = merge_weights(l, bl[u]);
      if (mw.w != 0.f)
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = merge_out(acc[e], bo[u][e], mw.w);
      l = mw.lse;
    }
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) s_out[warp][kPer * lane + e] = acc[e];
  if (lane == 0) s_lse[warp] = l;
  __syncthreads();
  if (warp != 0) return;
  l = s_lse[0];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = s_out[0][kPer * lane + e];
  for (int w = 1; w < 8; ++w) {
    const MergeWeights mw = merge_weights(l, s_lse[w]);
    if (mw.w != 0.f)
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = merge_out(acc[e], s_out[w][kPer * lane + e], mw.w);
    l = mw.lse;
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) out[row * D + kPer * lane + e] = from_f32<Tout>(acc[e]);
  if (lane == 0) lse[row] = l;
}

}  // namespace ra
