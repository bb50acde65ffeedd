// attn_bwd.cuh - gradients of exact blockwise attention on the 5th-generation
// tensor cores (sm_100a).
//
// Anthology of the SOTA, SOTA-181: ring attention trains models, so the
// blockwise computation has a backward pass; TokenRing review (pith.science,
// arXiv 2412.20501), "What carries the argument": the forward returns, per
// query row, the log-sum-exp of the whole row.  With that lse every
// (query block, KV block) pair's share of the gradient is independent of the
// other pairs, and the shares add up (s = 1 / sqrt(D)):
//     P  = exp(s Q K^T - lse)            (rebuilt, never stored)
//     dV += P^T dO                       dP = dO V^T
//     dS = P (dP - Delta)                Delta = rowsum(dO * O)
//     dQ += s dS K                       dK += s dS^T Q
// Two kernels, each owning the output rows it writes (no atomics):
//   bwd_dq_kernel:  one 128-row query tile of one head per CTA walks the KV
//                   tiles its rows see, KV blocks in the schedule's order
//                   (the query block stays, as in the ring);
//   bwd_dkv_kernel: one 128-key tile of one KV head per CTA walks the query
//                   tiles that see it, for every query head of its group
//                   (the KV block stays, as in TokenRing).
// bwd_prep_kernel first writes Delta and lse * log2(e) per (batch, head),
// contiguous over positions.
//
// Warp roles (320 threads):
//   warps 0-7  elementwise: thread (warp % 4) * 32 + lane owns TMEM lane /
//              tile row (warp % 4) * 32 + lane; warps 4w..4w+3 take columns
//              64h + 32w .. 64h + 32w + 31 of column half h = 0, 1 of the
//              128 x 128 score tile
//   warp 8     TMA producer
//   warp 9     TMEM allocator and MMA issuer (one thread)
// Each tile's elementwise pass first loads its scores into registers and
// signals "read"; the tensor core then starts the next tile's score-shaped
// products (both of them in the dQ kernel, dP^T in the dK/dV kernel) while
// the pass converts P and dS to bf16.  The pass converts column half 0 of the
// tile (all 8 warps, 32 columns each), signals it, then half 1, so the
// products that consume half 0 run while half 1 is converted.  All
// products are 128 wide: SS products of K-major SW128 tiles, and TS products
// with a bf16 A operand in tensor memory and an MN-major B tile, the operand
// forms of the forward kernel.
#pragma once

#include "attn_fwd.cuh"
#include "permute.cuh"

namespace ra {

constexpr int kBwdThreads = 320;
constexpr int kBwdElem = 256;  // elementwise threads (warps 0-7)
constexpr int kBwdProducer = 8;
constexpr int kBwdMma = 9;
// Tiles between drains of the tensor-core accumulators (see bwd_flush_row):
// bounds every accumulation to 256 x 8 products of 16.  A power of two.
constexpr int kFlushTiles = 256;

struct BwdArgs {
  int B, S, Hq, Hkv, groups, causal;
  int nblk;            // ring blocks
  int nseg;            // segments per block: 1 (contiguous) or 2 (zigzag)
  int seg_tiles;       // 128-row tiles per segment
  float scale;         // 1 / sqrt(D)
  float scale_log2;    // log2(e) / sqrt(D)
  const float* lse2;   // [B][Hq][S]: lse * log2(e)
  const float* delta;  // [B][Hq][S]
  float* dq;           // [B, S, Hq, D]
  float* dk;           // [B, S, Hkv, D]
  float* dv;           // [B, S, Hkv, D]
  Seg seg[kMaxBlocks][2];                     // segments of block r (queries and keys alike)
  signed char order[kMaxBlocks][kMaxBlocks];  // order[r][s]: s-th block that block r meets
  signed char seg_order[2 * kMaxBlocks];      // (r * nseg + e) of the CTA segments, heaviest first
  CtaTimeline timeline;  // per-CTA tracing (rec == nullptr: off); work units = tiles walked
};

// Shared memory of the dQ kernel: Q and dO stay; K and V stream through
// rings.  V(j) is free once dP(j) completes, K(j) only after dQ(j), so the K
// ring is deeper.
template <int D>
struct BwdQSmem {
  static constexpr int kBox = kBM * 128;  // 128 rows x 64 bf16: one TMA box, 16 KB
  static constexpr int kTile = kBox * (D / 64);
  static constexpr int kNK = D == 128 ? 3 : 6;
  static constexpr int kNV = D == 128 ? 2 : 4;
  static constexpr int kX = 0;  // Q, then dO
  static constexpr int kK = 2 * kTile;
  static constexpr int kV = kK + kNK * kTile;
  static constexpr int kBar = kV + kNV * kTile;
  // barriers: X, Kfull[NK], Kempty[NK], Vfull[NV], Vempty[NV], Sfull, Read, Done[2][2], Odone, End,
  // Flush full / empty, Sfull of half 1
  static constexpr int kNBar = 1 + 2 * kNK + 2 * kNV + 11;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;  // + slack to align the base to 1024
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(2 * kBM * (D / 2 + 4) * 4 <= kBar, "output staging fits in the tile buffers");
};

// Shared memory of the dK/dV kernel: K and V stay; Q and dO stream (dO(j+1)
// is needed first, as soon as tile j's scores are read, so its ring is the
// deeper one), plus the -lse2 / -Delta of the current query tile.
template <int D>
struct BwdKVSmem {
  static constexpr int kBox = kBM * 128;
  static constexpr int kTile = kBox * (D / 64);
  static constexpr int kNQ = D == 128 ? 2 : 4;
  static constexpr int kNO = D == 128 ? 3 : 4;
  static constexpr int kX = 0;  // K, then V
  static constexpr int kQ = 2 * kTile;
  static constexpr int kO = kQ + kNQ * kTile;
  static constexpr int kStat = kO + kNO * kTile;  // -lse2 x 128 | -delta x 128
  static constexpr int kBar = kStat + 2 * kBM * 4;
  // barriers: X, Qfull[NQ], Qempty[NQ], Ofull[NO], Oempty[NO], Sfull, Read, Done[2][2], Odone, End,
  // Flush full / empty, Sfull of half 1
  static constexpr int kNBar = 1 + 2 * kNQ + 2 * kNO + 11;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(2 * kBM * (D + 4) * 4 <= kStat, "output staging fits in the tile buffers");
};

// Tensor memory (512 columns).
//   dQ kernel:   S [0, 128), dP [128, 256), dQ [256, 256 + D),
//                bf16 dS of tile j at [384 + 64 (j & 1), + 64) (two buffers,
//                so tile j + 1's scores never wait for dQ(j) to read dS(j))
//   dK/dV kernel: S^T [0, 128), dP^T [128, 256), dV [256, 256 + D),
//                dK [384, 384 + D); the bf16 results of column half h go over
//                S^T once every warp has read it: P^T at [64h, 64h + 32),
//                dS^T at [64h + 32, 64h + 64)
constexpr int kTmS = 0, kTmP = 128, kTmAcc = 256, kTmDS = 384;

// Delta = rowsum(dO * O) and lse * log2(e), written as [B][Hq][S].  D / 4
// threads per row, 4 elements each.
template <typename TO>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const TO* __restrict__ out, const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                    int B, int S, int Hq, int D, float* __restrict__ delta, float* __restrict__ lse2) {
  const int tpr = D / 4;  // 16 or 32: a power of two dividing 32
  const long long rows = static_cast<long long>(B) * S * Hq;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  const int sub = threadIdx.x % tpr;
  // every lane of a warp runs the same number of iterations (the row range is
  // padded to whole warps), so the shuffles below see all 32 lanes
  const long long rows_pad = (rows * tpr + 31) / 32 * 32 / tpr;
  for (long long r = tid / tpr; r < rows_pad; r += nthreads / tpr) {
    float acc = 0.f;
    if (r < rows) {
      const long long e = r * D + 4 * sub;
      float o[4];
      if constexpr (sizeof(TO) == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(out + e));
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
      } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(out + e));
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&v);
        o[0] = __low2float(hv[0]), o[1] = __high2float(hv[0]), o[2] = __low2float(hv[1]), o[3] = __high2float(hv[1]);
      }
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(dout + e));
      const __nv_bfloat162* gv = reinterpret_cast<const __nv_bfloat162*>(&w);
      acc = o[0] * __low2float(gv[0]) + o[1] * __high2float(gv[0]) + o[2] * __low2float(gv[1]) +
            o[3] * __high2float(gv[1]);
    }
    for (int m = tpr / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (sub == 0 && r < rows) {
      const int h = static_cast<int>(r % Hq);
      const long long bs = r / Hq;
      const int s = static_cast<int>(bs % S), b = static_cast<int>(bs / S);
      const long long t = (static_cast<long long>(b) * Hq + h) * S + s;
      if (RA_IN_BOUNDS(t, rows)) {
        delta[t] = acc;
        lse2[t] = lse[r] * 1.4426950408889634f;
      }
    }
  }
}

// Keys of segment kv visible to a query at original position qpos (a prefix
// of the segment); qpos < 0 marks a padding row.
__device__ __forceinline__ int bwd_visible(const BwdArgs& a, const Seg& kv, int qpos) {
  if (qpos < 0) return 0;
  if (!a.causal) return kv.len;
  return min(max(qpos - kv.pos + 1, 0), kv.len);
}

// Two 32-column TMEM loads of this thread's lane, then one wait (warp-collective).
__device__ __forceinline__ void tmem_ld32x2_wait(uint32_t ta, uint32_t tb, uint32_t (&va)[32], uint32_t (&vb)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(va[0]), "=r"(va[1]), "=r"(va[2]), "=r"(va[3]), "=r"(va[4]), "=r"(va[5]), "=r"(va[6]), "=r"(va[7]),
        "=r"(va[8]), "=r"(va[9]), "=r"(va[10]), "=r"(va[11]), "=r"(va[12]), "=r"(va[13]), "=r"(va[14]),
        "=r"(va[15]), "=r"(va[16]), "=r"(va[17]), "=r"(va[18]), "=r"(va[19]), "=r"(va[20]), "=r"(va[21]),
        "=r"(va[22]), "=r"(va[23]), "=r"(va[24]), "=r"(va[25]), "=r"(va[26]), "=r"(va[27]), "=r"(va[28]),
        "=r"(va[29]), "=r"(va[30]), "=r"(va[31]), "=r"(vb[0]), "=r"(vb[1]), "=r"(vb[2]), "=r"(vb[3]), "=r"(vb[4]),
        "=r"(vb[5]), "=r"(vb[6]), "=r"(vb[7]), "=r"(vb[8]), "=r"(vb[9]), "=r"(vb[10]), "=r"(vb[11]), "=r"(vb[12]),
        "=r"(vb[13]), "=r"(vb[14]), "=r"(vb[15]), "=r"(vb[16]), "=r"(vb[17]), "=r"(vb[18]), "=r"(vb[19]),
        "=r"(vb[20]), "=r"(vb[21]), "=r"(vb[22]), "=r"(vb[23]), "=r"(vb[24]), "=r"(vb[25]), "=r"(vb[26]),
        "=r"(vb[27]), "=r"(vb[28]), "=r"(vb[29]), "=r"(vb[30]), "=r"(vb[31])
      : "r"(ta), "r"(tb)
      : "memory");
}

// AND of `pred` over the `count` threads that reach named barrier `id`.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// One warp's 32 rows of an fp32 128 x NC tile in TMEM (columns taddr ..
// taddr + NC), times `mul`, to global memory (added to what is there when
// `add`): through a padded staging buffer, then whole rows, 16 bytes per lane.  Row r of the tile goes to
// dst + (first_row + r * row_stride) * ld; rows r >= nrows are not written.
template <int NC>
__device__ __forceinline__ void bwd_store_rows(float* stage, uint32_t taddr, int quad, int lane, float* dst,
                                               long long first_row, long long row_stride, int ld, int nrows,
                                               float mul, bool add, long long dst_rows) {
  constexpr int kStride = NC + 4;
  const int row = quad * 32 + lane;
#pragma unroll
  for (int q = 0; q < NC / 32; ++q) {
    uint32_t v[32];
    tmem_ld32_wait(taddr + 32 * q, v);
#pragma unroll
    for (int i = 0; i < 32; i += 4)
      *reinterpret_cast<float4*>(stage + row * kStride + 32 * q + i) =
          make_float4(__uint_as_float(v[i]) * mul, __uint_as_float(v[i + 1]) * mul, __uint_as_float(v[i + 2]) * mul,
                      __uint_as_float(v[i + 3]) * mul);
  }
  __syncwarp();
  constexpr int lpr = NC / 4, rpi = 32 / lpr;  // lanes per row, rows per pass
  const int ci = lane % lpr, rl = lane / lpr;
#pragma unroll 4
  for (int r0 = 0; r0 < 32; r0 += rpi) {
    const int r = quad * 32 + r0 + rl;
    if (r < nrows && RA_IN_BOUNDS(first_row + r * row_stride, dst_rows)) {
      float4* p = reinterpret_cast<float4*>(dst + (first_row + r * row_stride) * ld + 4 * ci);
      float4 val = *reinterpret_cast<const float4*>(stage + r * kStride + 4 * ci);
      if (add) {
        const float4 old = *p;
        val.x += old.x, val.y += old.y, val.z += old.z, val.w += old.w;
      }
      *p = val;
    }
  }
  __syncwarp();
}

// The tensor core adds each product into its fp32 accumulator without
// rounding to nearest, so over very long sums (a key tile at the start of a
// 1M-token sequence meets ~8,000 query tiles per query head) the error
// drifts one way.  Every kFlushTiles tiles the accumulator is therefore
// drained into the fp32 output with ordinary (round-to-nearest) adds and the
// next product restarts it.  This thread's row, NC columns from taddr:
// dst[c] (+)= mul * acc[c].
template <int NC>
__device__ __forceinline__ void bwd_flush_row(uint32_t taddr, float* dst, bool valid, bool add, float mul) {
#pragma unroll
  for (int q = 0; q < NC / 32; ++q) {
    uint32_t v[32];
    tmem_ld32_wait(taddr + 32 * q, v);
    if (valid) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4* p = reinterpret_cast<float4*>(dst + 32 * q + i);
        float4 o = add ? *p : make_float4(0.f, 0.f, 0.f, 0.f);
        o.x += __uint_as_float(v[i]) * mul;
        o.y += __uint_as_float(v[i + 1]) * mul;
        o.z += __uint_as_float(v[i + 2]) * mul;
        o.w += __uint_as_float(v[i + 3]) * mul;
        *p = o;
      }
    }
  }
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// One 32-column chunk of a row: from fp32 scores s and dP (raw TMEM bits) to
// bf16 pairs of P = 2^(s * ss - lse2) and dS = P (dP - Delta), two columns per
// packed fp32x2 operation.  nl / nd: -lse2 and -Delta per column (COLS) or
// the row's own (nl[0], nd[0]).  MASK: columns c < lo or c >= hi get P = 0.
template <bool COLS, bool MASK, bool WANT_P>
__device__ __forceinline__ void bwd_convert(const uint32_t (&sv)[32], const uint32_t (&pv)[32], float ss,
                                            const float* nl, const float* nd, int lo, int hi, uint32_t (&pp)[16],
                                            uint32_t (&pd)[16]) {
  const uint64_t ss2 = f2_pack(ss, ss);
  const uint64_t nl_row = f2_pack(nl[0], nl[0]), nd_row = f2_pack(nd[0], nd[0]);
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    float4 l4, d4;
    if constexpr (COLS) {
      l4 = *reinterpret_cast<const float4*>(nl + i);
      d4 = *reinterpret_cast<const float4*>(nd + i);
    }
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const uint64_t nlv = COLS ? f2_pack(e ? l4.z : l4.x, e ? l4.w : l4.y) : nl_row;
      const uint64_t ndv = COLS ? f2_pack(e ? d4.z : d4.x, e ? d4.w : d4.y) : nd_row;
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[i + e]), __uint_as_float(sv[i + e + 1])), ss2, nlv), x0, x1);
      float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
      if constexpr (MASK) {
        const int c = i + e;
        p0 = c >= lo && c < hi ? p0 : 0.f;
        p1 = c + 1 >= lo && c + 1 < hi ? p1 : 0.f;
      }
      const uint64_t t = f2_add(f2_pack(__uint_as_float(pv[i + e]), __uint_as_float(pv[i + e + 1])), ndv);
      float d0, d1;
      f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
      if constexpr (WANT_P) pp[(i + e) / 2] = pack_bf16x2(p0, p1);
      pd[(i + e) / 2] = pack_bf16x2(d0, d1);
    }
  }
}

// Barrier indices of the ring pair (r0 ring of n0 stages, r1 ring of n1).
struct BwdBars {
  static constexpr int kX = 0;
  int n0, n1;
  __device__ int full0(int s) const { return 1 + s; }
  __device__ int empty0(int s) const { return 1 + n0 + s; }
  __device__ int full1(int s) const { return 1 + 2 * n0 + s; }
  __device__ int empty1(int s) const { return 1 + 2 * n0 + n1 + s; }
  __device__ int sfull() const { return 1 + 2 * n0 + 2 * n1; }
  __device__ int read() const { return 2 + 2 * n0 + 2 * n1; }
  // column half h of tile j converted (P / dS in bf16 written).  Tiles of
  // each parity have their own pair: in the dQ kernel the next tile's scores
  // are released before the MMA thread waits for this tile's halves, so one
  // barrier per half could complete twice before it is polled; a second
  // completion of done(h, j) needs tile j + 2's scores, which the MMA thread
  // only issues after it has consumed done(h, j).  Polled with parity
  // (j >> 1) & 1.
  __device__ int done(int h, int j) const { return 3 + 2 * n0 + 2 * n1 + 2 * (j & 1) + h; }
  __device__ int odone() const { return 7 + 2 * n0 + 2 * n1; }
  __device__ int end() const { return 8 + 2 * n0 + 2 * n1; }
  // accumulator drain (see bwd_flush_row): full = the products of the last
  // kFlushTiles tiles are complete; empty = the warps have read the accumulator
  __device__ int ffull() const { return 9 + 2 * n0 + 2 * n1; }
  __device__ int fempty() const { return 10 + 2 * n0 + 2 * n1; }
  // dK/dV kernel: the scores of query half h of the tile are ready (half 0
  // uses sfull())
  __device__ int sfull_h(int h) const { return h ? 11 + 2 * n0 + 2 * n1 : sfull(); }
};

// ------------------------------------------------------------------- dQ
// MMA issue order over the CTA's KV tiles j:
//   S(0) dP(0); then per j: [tile j read] S(j+1) dP(j+1), [dS(j) written] dQ += dS(j) K(j)
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ BwdArgs a) {
  using SL = BwdQSmem<D>;
  constexpr int NK = SL::kNK, NV = SL::kNV;
  extern __shared__ uint8_t bsm_raw[];
  uint8_t* smem = bsm_raw + ((1024u - (smem_u32(bsm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  timeline_begin(a.timeline);

  // tile: heads fastest, then batch, then query segments heaviest first,
  // then tiles of the segment, latest first
  int idx = blockIdx.x;
  const int h = idx % a.Hq;
  idx /= a.Hq;
  const int b = idx % a.B;
  idx /= a.B;
  const int so = a.seg_order[idx / a.seg_tiles];
  const int qt = a.seg_tiles - 1 - idx % a.seg_tiles;
  const int qi = so / a.nseg;
  const Seg qs = a.seg[qi][so % a.nseg];
  const int hk = h / a.groups;
  const int row0 = qt * kBM;
  const int rows = min(max(qs.len - row0, 0), kBM);
  const int last = rows > 0 ? qs.pos + row0 + rows - 1 : -1;
  // the walk: KV blocks in order, their segments, the tiles the last row sees
  auto nt_of = [&](int s_, int e_) { return (bwd_visible(a, a.seg[a.order[qi][s_]][e_], last) + kBN - 1) / kBN; };
  int total = 0;
  for (int s_ = 0; s_ < a.nblk; ++s_)
    for (int e_ = 0; e_ < a.nseg; ++e_) total += nt_of(s_, e_);

  const BwdBars ib{NK, NV};
  auto bar = [&](int i) -> uint32_t { return sb + SL::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);
  if (threadIdx.x == 0) {
    for (int i = 0; i < SL::kNBar; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(ib.read()), kBwdElem / 32);  // one arrival per elementwise warp
    for (int i = 0; i < 4; ++i) mbar_init(bar(ib.done(i & 1, i >> 1)), kBwdElem / 32);  // one arrival per warp
    mbar_init(bar(ib.fempty()), kBwdElem / 32);
    *abort_flag = grid_timed_out() ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kBwdMma) tmem_alloc(sb + SL::kTmemSlot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SL::kTmemSlot);
  const int work = *abort_flag || rows == 0 ? 0 : total;
  timeline_work(a.timeline, work);

  if (warp == kBwdProducer) {
    if (lane == 0 && work > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      // checked build: the CTA's rows and heads must lie inside the tensors
      const bool x_ok = RA_IN_BOUNDS(qs.mem + row0, a.S) && RA_IN_BOUNDS(h, a.Hq) && RA_IN_BOUNDS(hk, a.Hkv);
      if (!x_ok) *abort_flag = 1;
      if (x_ok) {
        mbar_expect_tx(bar(ib.kX), 2 * SL::kTile);
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_4d(sb + SL::kX + bx * SL::kBox, &tmQ, bx * 64, h, qs.mem + row0, b, bar(ib.kX));
          tma_load_4d(sb + SL::kX + SL::kTile + bx * SL::kBox, &tmdO, bx * 64, h, qs.mem + row0, b, bar(ib.kX));
        }
      }
      int j = 0, lastk[NK], lastv[NV];
      for (int s = 0; s < NK; ++s) lastk[s] = -1;
      for (int s = 0; s < NV; ++s) lastv[s] = -1;
      bool ok = true;
      for (int s_ = 0; s_ < a.nblk && ok; ++s_)
        for (int e_ = 0; e_ < a.nseg && ok; ++e_) {
          const Seg ks = a.seg[a.order[qi][s_]][e_];
          const int nt = nt_of(s_, e_);
          for (int t = 0; t < nt; ++t, ++j) {
            const int sk = j % NK, sv = j % NV, r = ks.mem + t * kBN;
            if (!mbar_wait(bar(ib.empty0(sk)), ((j / NK) & 1) ^ 1, abort_flag) || !RA_IN_BOUNDS(r, a.S)) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            mbar_expect_tx(bar(ib.full0(sk)), SL::kTile);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_4d(sb + SL::kK + sk * SL::kTile + bx * SL::kBox, &tmK, bx * 64, hk, r, b, bar(ib.full0(sk)));
            lastk[sk] = j;
            if (!mbar_wait(bar(ib.empty1(sv)), ((j / NV) & 1) ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar(ib.full1(sv)), SL::kTile);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_4d(sb + SL::kV + sv * SL::kTile + bx * SL::kBox, &tmV, bx * 64, hk, r, b, bar(ib.full1(sv)));
            lastv[sv] = j;
          }
        }
      // every copy issued lands before the CTA can release its shared memory
      if (x_ok) mbar_drain(bar(ib.kX), 0);
      for (int s = 0; s < NK; ++s)
        if (lastk[s] >= 0) mbar_drain(bar(ib.full0(s)), (lastk[s] / NK) & 1);
      for (int s = 0; s < NV; ++s)
        if (lastv[s] >= 0) mbar_drain(bar(ib.full1(s)), (lastv[s] / NV) & 1);
    }
  } else if (warp == kBwdMma) {
    if (lane == 0 && work > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t kIdescQ = idesc_bf16_f32(kBM, D, true);
      // Descriptors as bases plus compile-time offsets (one add per operand
      // and product: this one thread's work per product bounds how close the
      // products run to the tensor core's rate).
      const uint32_t dhi = desc_sw128_hi();
      const uint32_t lo_q = desc_sw128_lo(sb + SL::kX, 16), lo_do = desc_sw128_lo(sb + SL::kX + SL::kTile, 16);
      const uint32_t lo_k = desc_sw128_lo(sb + SL::kK, 16), lo_v = desc_sw128_lo(sb + SL::kV, 16);
      const uint32_t lo_kmn = desc_sw128_lo(sb + SL::kK, SL::kBox);
      // S = Q K(j)^T into [0, 128), dP = dO V(j)^T into [128, 256): K-major operands
      auto issue_sdp = [&](int j) -> bool {
        const int sk = j % NK, sv = j % NV;
        if (!mbar_wait(bar(ib.full0(sk)), (j / NK) & 1, abort_flag) ||
            !mbar_wait(bar(ib.full1(sv)), (j / NV) & 1, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t bk = lo_k + static_cast<uint32_t>(sk) * (SL::kTile >> 4);
        const uint32_t bv = lo_v + static_cast<uint32_t>(sv) * (SL::kTile >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * SL::kBox + (kk % 4) * 32) >> 4;
          mma_ss_lo(tmem + kTmS, lo_q + off, bk + off, dhi, kIdescS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * SL::kBox + (kk % 4) * 32) >> 4;
          mma_ss_lo(tmem + kTmP, lo_do + off, bv + off, dhi, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(ib.empty1(sv)));  // V(j) is read only by dP(j)
        tc_commit(bar(ib.sfull()));
        return true;
      };
      // dQ += dS_h(j) K_h(j) over keys 64h .. 64h + 63: A = bf16 dS in TMEM,
      // B = rows of K(j) read MN-major; after half 1, K(j) is free
      auto issue_dq = [&](int j, int hf) {
        const int sk = j % NK;
        const uint32_t bk = lo_kmn + static_cast<uint32_t>(sk) * (SL::kTile >> 4);
        const uint32_t ta = tmem + kTmDS + 64 * (j & 1) + 32 * hf;
        const bool acc = j % kFlushTiles > 0 || hf > 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_lo(tmem + kTmAcc, ta + kk * 8, bk + (((4 * hf + kk) * 2048) >> 4), dhi, kIdescQ,
                    (acc || kk > 0) ? 1u : 0u);
        if (hf == 1) tc_commit(bar(ib.empty0(sk)));
      };
      bool ok = mbar_wait(bar(ib.kX), 0, abort_flag) && issue_sdp(0);
      for (int j = 0; ok && j < work; ++j) {
        if (j + 1 < work) {
          ok = mbar_wait(bar(ib.read()), j & 1, abort_flag) && issue_sdp(j + 1);
          if (!ok) break;
        }
        constexpr int F = kFlushTiles;
        for (int hf = 0; hf < 2 && ok; ++hf) {
          ok = mbar_wait(bar(ib.done(hf, j)), (j >> 1) & 1, abort_flag);
          // the accumulator restarts at tile j: the previous sum has been drained
          if (ok && hf == 0 && j > 0 && j % F == 0) ok = mbar_wait(bar(ib.fempty()), (j / F - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_dq(j, hf);
        }
        if (ok && (j + 1) % F == 0 && j + 1 < work) tc_commit(bar(ib.ffull()));
      }
      tc_commit(bar(ib.odone()));
      tc_commit(bar(ib.end()));
      mbar_drain(bar(ib.end()), 0);
    }
  } else {
    // ---------------------------------------------------------- elementwise
    const int quad = warp & 3, half = warp >> 2;  // half: the 32-column slice of each column half
    const int row = quad * 32 + lane;
    const bool valid = row < rows;
    const int qpos = valid ? qs.pos + row0 + row : -1;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTmS + 32 * half, tP = tmem + lane_base + kTmP + 32 * half;
    const long long stat = (static_cast<long long>(b) * a.Hq + h) * a.S + max(qpos, 0);
    // padding rows: -lse2 = -inf, so every P is 0
    const float nl = valid ? -a.lse2[stat] : -INFINITY;
    const float nd = valid ? -a.delta[stat] : 0.f;
    const float ss = a.scale_log2;
    bool ok = work > 0;
    int j = 0;
    for (int s_ = 0; s_ < a.nblk && ok; ++s_)
      for (int e_ = 0; e_ < a.nseg && ok; ++e_) {
        const Seg ks = a.seg[a.order[qi][s_]][e_];
        const int nt = nt_of(s_, e_);
        const int lim = bwd_visible(a, ks, qpos);
        for (int t = 0; t < nt; ++t, ++j) {
          if (j > 0 && j % kFlushTiles == 0) {
            // drain the accumulator (tiles j - kFlushTiles .. j - 1) into dq
            ok = __all_sync(0xffffffffu, mbar_wait(bar(ib.ffull()), (j / kFlushTiles - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            constexpr int NC = D / 2;
            bwd_flush_row<NC>(tmem + lane_base + kTmAcc + half * NC,
                              a.dq + ((static_cast<long long>(b) * a.S + qs.pos + row0 + row) * a.Hq + h) * D +
                                  half * NC,
                              valid && RA_IN_BOUNDS((static_cast<long long>(b) * a.S + qs.pos + row0 + row) * a.Hq + h,
                                                    static_cast<long long>(a.B) * a.S * a.Hq),
                              j > kFlushTiles, a.scale);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(ib.fempty()));
          }
          ok = __all_sync(0xffffffffu, mbar_wait(bar(ib.sfull()), j & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
          uint32_t sv[2][32], pv[2][32];
          tmem_ld32x2_wait(tS, tS + 64, sv[0], sv[1]);
          tmem_ld32x2_wait(tP, tP + 64, pv[0], pv[1]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(ib.read()));  // S and dP may be overwritten now
          const uint32_t dst = tmem + lane_base + kTmDS + 64 * (j & 1) + 16 * half;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            // keys of this 32-column slice visible to the row: [0, cnt)
            const int cnt = lim - t * kBN - 64 * hf - 32 * half;
            uint32_t pk[16];
            if (__all_sync(0xffffffffu, !valid || cnt >= 32))
              bwd_convert<false, false, false>(sv[hf], pv[hf], ss, &nl, &nd, 0, 0, pk, pk);
            else
              bwd_convert<false, true, false>(sv[hf], pv[hf], ss, &nl, &nd, 0, cnt, pk, pk);
            tmem_st16(dst + 32 * hf, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(ib.done(hf, j)));
          }
        }
      }
    // ---- epilogue: this CTA's dQ rows; column half h of every row by warps 4h..4h+3
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(ib.odone()), 0, abort_flag));
    if (ok) {
      tc_fence_after();
      constexpr int NC = D / 2;
      // every product is complete (odone): the tile buffers are free; warps
      // 4w..4w+3 store column half w of the rows
      float* stage = reinterpret_cast<float*>(smem) + half * kBM * (NC + 4);
      bwd_store_rows<NC>(stage, tmem + lane_base + kTmAcc + half * NC, quad, lane, a.dq + half * NC,
                         (static_cast<long long>(b) * a.S + qs.pos + row0) * a.Hq + h, a.Hq, D, rows, a.scale,
                         work > kFlushTiles, static_cast<long long>(a.B) * a.S * a.Hq);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMma) tmem_dealloc(tmem, 512);
  timeline_end(a.timeline);
}

// ----------------------------------------------------------------- dK, dV
// MMA issue order over the CTA's query tiles j (half h = queries 64h .. 64h + 63):
//   dP^T(0), S^T_0(0), S^T_1(0); then per j:
//   [half 0 of tile j converted] dV, dK += half 0,
//   [tile j's scores read]       dP^T(j+1), S^T_0(j+1),
//   [half 1 converted]           dV, dK += half 1, S^T_1(j+1)
// S^T is issued in 64-query halves so that tile j+1's half-0 conversion runs
// while the tensor core finishes tile j's half 1.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                   const __grid_constant__ BwdArgs a) {
  using SL = BwdKVSmem<D>;
  constexpr int NQ = SL::kNQ, NO = SL::kNO;
  extern __shared__ uint8_t bsm_raw[];
  uint8_t* smem = bsm_raw + ((1024u - (smem_u32(bsm_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  timeline_begin(a.timeline);

  // tile: KV heads fastest, then batch, then key segments heaviest first,
  // then tiles of the segment, earliest first
  int idx = blockIdx.x;
  const int g = idx % a.Hkv;
  idx /= a.Hkv;
  const int b = idx % a.B;
  idx /= a.B;
  const int so = a.seg_order[idx / a.seg_tiles];
  const int kt = idx % a.seg_tiles;
  const int kj = so / a.nseg;
  const Seg ks = a.seg[kj][so % a.nseg];
  const int key0 = kt * kBN;
  const int krows = min(max(ks.len - key0, 0), kBN);
  const int first_k = ks.pos + key0;  // earliest key of the tile
  // query tile t of segment e_ of the s_-th query block this KV block meets:
  // its first position and rows; false when none of its rows sees this tile
  auto q_tile = [&](int s_, int e_, int t, int& q0, int& qrows) -> bool {
    const Seg qsg = a.seg[a.order[kj][s_]][e_];
    q0 = qsg.pos + t * kBM;
    qrows = min(qsg.len - t * kBM, kBM);
    if (qrows <= 0) return false;
    return !a.causal || q0 + qrows - 1 >= first_k;
  };
  auto q_mem = [&](int s_, int e_, int t) { return a.seg[a.order[kj][s_]][e_].mem + t * kBM; };
  int total = 0;
  for (int s_ = 0; s_ < a.nblk; ++s_)
    for (int e_ = 0; e_ < a.nseg; ++e_)
      for (int t = 0; t < a.seg_tiles; ++t) {
        int q0, qr;
        total += q_tile(s_, e_, t, q0, qr) ? 1 : 0;
      }
  total *= a.groups;

  const BwdBars ib{NQ, NO};
  auto bar = [&](int i) -> uint32_t { return sb + SL::kBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);
  if (threadIdx.x == 0) {
    for (int i = 0; i < SL::kNBar; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(ib.read()), kBwdElem / 32);
    for (int i = 0; i < 4; ++i) mbar_init(bar(ib.done(i & 1, i >> 1)), kBwdElem / 32);  // one arrival per warp
    mbar_init(bar(ib.fempty()), kBwdElem / 32);
    *abort_flag = grid_timed_out() ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kBwdMma) tmem_alloc(sb + SL::kTmemSlot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SL::kTmemSlot);
  const int work = *abort_flag || krows == 0 ? 0 : total;
  timeline_work(a.timeline, work);

  if (warp == kBwdProducer) {
    if (lane == 0 && work > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      // checked build: the CTA's keys and KV head must lie inside the tensors
      const bool x_ok = RA_IN_BOUNDS(ks.mem + key0, a.S) && RA_IN_BOUNDS(g, a.Hkv);
      if (!x_ok) *abort_flag = 1;
      if (x_ok) {
        mbar_expect_tx(bar(ib.kX), 2 * SL::kTile);
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_4d(sb + SL::kX + bx * SL::kBox, &tmK, bx * 64, g, ks.mem + key0, b, bar(ib.kX));
          tma_load_4d(sb + SL::kX + SL::kTile + bx * SL::kBox, &tmV, bx * 64, g, ks.mem + key0, b, bar(ib.kX));
        }
      }
      int j = 0, lastq[NQ], lasto[NO];
      for (int s = 0; s < NQ; ++s) lastq[s] = -1;
      for (int s = 0; s < NO; ++s) lasto[s] = -1;
      bool ok = true;
      for (int hh = 0; hh < a.groups && ok; ++hh)
        for (int s_ = 0; s_ < a.nblk && ok; ++s_)
          for (int e_ = 0; e_ < a.nseg && ok; ++e_)
            for (int t = 0; t < a.seg_tiles; ++t) {
              int q0, qr;
              if (!q_tile(s_, e_, t, q0, qr)) continue;
              const int hq = g * a.groups + hh, r = q_mem(s_, e_, t);
              const int sq = j % NQ, so_ = j % NO;
              // dO(j) first: dP^T(j) is issued before S^T(j)
              if (!mbar_wait(bar(ib.empty1(so_)), ((j / NO) & 1) ^ 1, abort_flag) || !RA_IN_BOUNDS(r, a.S) ||
                  !RA_IN_BOUNDS(hq, a.Hq)) {
                *abort_flag = 1;
                ok = false;
                break;
              }
              mbar_expect_tx(bar(ib.full1(so_)), SL::kTile);
              for (int bx = 0; bx < D / 64; ++bx)
                tma_load_4d(sb + SL::kO + so_ * SL::kTile + bx * SL::kBox, &tmdO, bx * 64, hq, r, b,
                            bar(ib.full1(so_)));
              lasto[so_] = j;
              if (!mbar_wait(bar(ib.empty0(sq)), ((j / NQ) & 1) ^ 1, abort_flag)) {
                ok = false;
                break;
              }
              mbar_expect_tx(bar(ib.full0(sq)), SL::kTile);
              for (int bx = 0; bx < D / 64; ++bx)
                tma_load_4d(sb + SL::kQ + sq * SL::kTile + bx * SL::kBox, &tmQ, bx * 64, hq, r, b, bar(ib.full0(sq)));
              lastq[sq] = j;
              ++j;
            }
      if (x_ok) mbar_drain(bar(ib.kX), 0);
      for (int s = 0; s < NQ; ++s)
        if (lastq[s] >= 0) mbar_drain(bar(ib.full0(s)), (lastq[s] / NQ) & 1);
      for (int s = 0; s < NO; ++s)
        if (lasto[s] >= 0) mbar_drain(bar(ib.full1(s)), (lasto[s] / NO) & 1);
    }
  } else if (warp == kBwdMma) {
    if (lane == 0 && work > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBN, kBM, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(kBN, D, true);
      // S^T_h = K Q_h(j)^T into [64h, 64h + 64): Q_h = rows 64h.. of the Q tile
      constexpr uint32_t kIdescS2 = idesc_bf16_f32(kBN, 64, false);
      // Descriptors as bases plus compile-time offsets (see the dQ kernel).
      const uint32_t dhi = desc_sw128_hi();
      const uint32_t lo_k = desc_sw128_lo(sb + SL::kX, 16), lo_v = desc_sw128_lo(sb + SL::kX + SL::kTile, 16);
      const uint32_t lo_q = desc_sw128_lo(sb + SL::kQ, 16), lo_o = desc_sw128_lo(sb + SL::kO, 16);
      const uint32_t lo_qmn = desc_sw128_lo(sb + SL::kQ, SL::kBox), lo_omn = desc_sw128_lo(sb + SL::kO, SL::kBox);
      auto issue_s = [&](int j, int hf) -> bool {
        const int sq = j % NQ;
        if (!mbar_wait(bar(ib.full0(sq)), (j / NQ) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t bq = lo_q + static_cast<uint32_t>(sq) * (SL::kTile >> 4) + ((hf * 64 * 128) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * SL::kBox + (kk % 4) * 32) >> 4;
          mma_ss_lo(tmem + kTmS + 64 * hf, lo_k + off, bq + off, dhi, kIdescS2, kk > 0 ? 1u : 0u);
        }
        return true;
      };
      // dP^T = V dO(j)^T into [128, 256)
      auto issue_dp = [&](int j) -> bool {
        const int so_ = j % NO;
        if (!mbar_wait(bar(ib.full1(so_)), (j / NO) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t bo = lo_o + static_cast<uint32_t>(so_) * (SL::kTile >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * SL::kBox + (kk % 4) * 32) >> 4;
          mma_ss_lo(tmem + kTmP, lo_v + off, bo + off, dhi, kIdescS, kk > 0 ? 1u : 0u);
        }
        return true;
      };
      // dV += P^T_h(j) dO_h(j), dK += dS^T_h(j) Q_h(j) over queries 64h .. 64h + 63:
      // A = bf16 in TMEM (P^T_h at [64h, 64h + 32), dS^T_h at [64h + 32, 64h + 64)),
      // B = rows of dO(j) / Q(j) read MN-major; after half 1 both tiles are free
      auto issue_dkv = [&](int j, int hf) {
        const uint32_t bq = lo_qmn + static_cast<uint32_t>(j % NQ) * (SL::kTile >> 4);
        const uint32_t bo = lo_omn + static_cast<uint32_t>(j % NO) * (SL::kTile >> 4);
        const bool acc = j % kFlushTiles > 0 || hf > 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_lo(tmem + kTmAcc, tmem + 64 * hf + 8 * kk, bo + (((4 * hf + kk) * 2048) >> 4), dhi, kIdescO,
                    (acc || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_lo(tmem + kTmAcc + 128, tmem + 64 * hf + 32 + 8 * kk, bq + (((4 * hf + kk) * 2048) >> 4), dhi,
                    kIdescO, (acc || kk > 0) ? 1u : 0u);
        if (hf == 1) {
          tc_commit(bar(ib.empty1(j % NO)));
          tc_commit(bar(ib.empty0(j % NQ)));
        }
      };
      bool ok = mbar_wait(bar(ib.kX), 0, abort_flag) && issue_dp(0) && issue_s(0, 0);
      if (ok) tc_commit(bar(ib.sfull_h(0)));
      ok = ok && issue_s(0, 1);
      if (ok) tc_commit(bar(ib.sfull_h(1)));
      constexpr int F = kFlushTiles;
      for (int j = 0; ok && j < work; ++j) {
        const bool more = j + 1 < work;
        // half 0 of tile j converted: its products (the accumulators restart
        // at a drain tile once the previous sums have been drained)
        ok = mbar_wait(bar(ib.done(0, j)), (j >> 1) & 1, abort_flag);
        if (ok && j > 0 && j % F == 0) ok = mbar_wait(bar(ib.fempty()), (j / F - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_dkv(j, 0);
        // tile j's scores are in registers: the next tile's dP^T and S^T half 0
        if (more) {
          ok = mbar_wait(bar(ib.read()), j & 1, abort_flag) && issue_dp(j + 1) && issue_s(j + 1, 0);
          if (!ok) break;
          tc_commit(bar(ib.sfull_h(0)));
        }
        ok = mbar_wait(bar(ib.done(1, j)), (j >> 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_dkv(j, 1);
        if ((j + 1) % F == 0 && more) tc_commit(bar(ib.ffull()));
        if (more) {
          ok = issue_s(j + 1, 1);
          if (!ok) break;
          tc_commit(bar(ib.sfull_h(1)));
        }
      }
      tc_commit(bar(ib.odone()));
      tc_commit(bar(ib.end()));
      mbar_drain(bar(ib.end()), 0);
    }
  } else {
    // ---------------------------------------------------------- elementwise
    // Thread (quad, lane) owns key row quad * 32 + lane; warps 4w..4w+3 own
    // query columns 64h + 32w .. 64h + 32w + 31 of column half h = 0, 1.
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int kpos = row < krows ? first_k + row : -1;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTmS, tP = tmem + lane_base + kTmP;
    float* set = reinterpret_cast<float*>(smem + SL::kStat);  // -lse2 x 128 | -delta x 128
    const float ss = a.scale_log2;
    bool ok = work > 0;
    int j = 0;
    for (int hh = 0; hh < a.groups && ok; ++hh)
      for (int s_ = 0; s_ < a.nblk && ok; ++s_)
        for (int e_ = 0; e_ < a.nseg && ok; ++e_)
          for (int t = 0; t < a.seg_tiles; ++t) {
            int q0, qrows;
            if (!q_tile(s_, e_, t, q0, qrows)) continue;
            if (j > 0 && j % kFlushTiles == 0) {
              // drain the accumulators (tiles j - kFlushTiles .. j - 1): dV by
              // warps 0-3, dK by warps 4-7
              // one decision for all 8 warps (they meet at named barriers below)
              ok = bar_and(1, kBwdElem, mbar_wait(bar(ib.ffull()), (j / kFlushTiles - 1) & 1, abort_flag));
              if (!ok) break;
              tc_fence_after();
              bwd_flush_row<D>(tmem + lane_base + kTmAcc + half * 128,
                               (half ? a.dk : a.dv) +
                                   ((static_cast<long long>(b) * a.S + ks.pos + key0 + row) * a.Hkv + g) * D,
                               row < krows && RA_IN_BOUNDS((static_cast<long long>(b) * a.S + ks.pos + key0 + row) * a.Hkv + g,
                                                           static_cast<long long>(a.B) * a.S * a.Hkv),
                               j > kFlushTiles, half ? a.scale : 1.f);
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(ib.fempty()));
            }
            // -lse2 (threads 0-127) and -delta (threads 128-255) of the tile's queries
            const int c = threadIdx.x & (kBM - 1);
            const long long at = (static_cast<long long>(b) * a.Hq + g * a.groups + hh) * a.S + q0 + c;
            const float v = threadIdx.x < kBM ? (c < qrows ? -a.lse2[at] : -INFINITY)
                                              : (c < qrows ? -a.delta[at] : 0.f);
            named_barrier_sync(1, kBwdElem);  // every warp is done with tile j - 1's values
            set[threadIdx.x] = v;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              // the scores of query half hf; the first decision also publishes `set`
              const bool w = mbar_wait(bar(ib.sfull_h(hf)), j & 1, abort_flag);
              ok = bar_and(1, kBwdElem, w);  // one decision for all 8 warps
              if (!ok) break;
              tc_fence_after();
              const int c0 = 64 * hf + 32 * half;
              uint32_t sv[32], pv[32];
              tmem_ld32x2_wait(tS + c0, tP + c0, sv, pv);
              tc_fence_before();
              __syncwarp();
              if (hf == 1 && lane == 0) mbar_arrive(bar(ib.read()));  // dP^T may be overwritten now
              named_barrier_sync(1, kBwdElem);  // every warp has read half hf of S^T: it may be overwritten
              tc_fence_after();
              // when causal, this key sees the slice's query columns [lo, 32)
              const int lo = a.causal && kpos >= 0 ? kpos - q0 - c0 : -32;
              uint32_t pp[16], pd[16];
              if (__all_sync(0xffffffffu, lo <= 0))
                bwd_convert<true, false, true>(sv, pv, ss, set + c0, set + kBM + c0, 0, 0, pp, pd);
              else
                bwd_convert<true, true, true>(sv, pv, ss, set + c0, set + kBM + c0, lo, 32, pp, pd);
              tmem_st16(tS + 64 * hf + 16 * half, pp);       // P^T_h
              tmem_st16(tS + 64 * hf + 32 + 16 * half, pd);  // dS^T_h
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(ib.done(hf, j)));
            }
            if (!ok) break;
            ++j;
          }
    // ---- epilogue: dV rows by warps 0-3, dK rows by warps 4-7
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(ib.odone()), 0, abort_flag));
    if (ok) {
      tc_fence_after();
      float* stage = reinterpret_cast<float*>(smem) + half * kBM * (D + 4);
      bwd_store_rows<D>(stage, tmem + lane_base + kTmAcc + half * 128, quad, lane, half ? a.dk : a.dv,
                        (static_cast<long long>(b) * a.S + ks.pos + key0) * a.Hkv + g, a.Hkv, D, krows,
                        half ? a.scale : 1.f, work > kFlushTiles, static_cast<long long>(a.B) * a.S * a.Hkv);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMma) tmem_dealloc(tmem, 512);
  timeline_end(a.timeline);
}

}  // namespace ra
