// attn_fwd.cuh - block attention on the 5th-generation tensor cores (sm_100a).
//
// One CTA runs two 128-row query tiles, A and B, of one (batch, query head)
// against a list of KV blocks (one block for ra_block_attn and the unfused
// schedule; every block, in schedule order, for the persistent schedule).
// Row-pair mode: A and B are 256 consecutive query rows and share every K/V
// tile load.  KV-split mode (grids too small to fill the GPU): A and B are
// the same 128 rows; A takes the first half of the KV tiles, B the second
// half, and the two partial results are stitched on chip with the merge rule
// (the rule the method uses between blocks, applied inside one block).
// Cluster mode (row pairs, still too few CTAs): two CTAs of a thread-block
// cluster run the same 256 rows over the two halves of the KV tiles; each
// stages its partial rows in shared memory, and CTA r finalises tile r by
// reading the peer's partial through distributed shared memory and merging.
//
// TokenRing review (pith.science, arXiv 2412.20501), "What carries the
// argument" / "Core claim": the flash-attention kernel that yields, for one
// query block and one key/value block, the softmax-normalised block_out and
// the per-row block_lse; "If this is right": grouped-query attention and the
// zigzag causal partition; Anthology of the SOTA, SOTA-181: exact attention.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile A: thread i owns row i of A (TMEM lane i)
//   warps 4-7  softmax of tile B (same lanes, its own TMEM columns)
//   warp 8     TMA producer: Q once, then K and V tiles into their rings
//   warp 9     TMEM allocator and MMA issuer (one thread):
//                S_X = Q_X K^T   (SS MMA, fp32 in TMEM)
//                O_X += P_X V    (TS MMA, P_X bf16 in TMEM over S_X)
//              issued in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so
//              the tensor core works on one tile while the other tile's
//              softmax runs.
//   warps 10-11 idle (they complete the third warpgroup).
// Registers: launched at 168 per thread (384 x 168 = 64512); the third
// warpgroup gives most of its share to the softmax warpgroups
// (2 x 128 x 216 + 128 x 72 = 64512), so the softmax keeps a whole score
// row and its exponentials in registers.
// Tensor memory (512 columns): S_A/P_A [0,128), S_B/P_B [128,256),
// O_A [256,256+D), O_B [384,384+D).
//
// Online softmax in fp32 with base-2 exponentials (scores pre-scaled by
// log2(e)/sqrt(D)).  The running maximum used for the exponentials is only
// raised when a tile's maximum exceeds it by more than 8 (a factor 256), so
// O is rescaled in TMEM rarely; the final out = O / l and
// lse = ln 2 * (m + log2 l) are exact for any such choice of m.
//
// The partition is an index map, not a data movement: every block is one
// (contiguous) or two (zigzag) segments of consecutive original positions,
// and tiles never straddle a segment, so each 128-row tile is one TMA box read
// straight from the caller's tensor.  Causal masking uses original positions;
// inside a segment the keys a query may see form a prefix, so the KV loop
// stops at the last tile the CTA's last row can see, tile A skips the KV tiles
// none of its rows can see, and only tiles cut by a row's prefix are masked
// element-wise.
#pragma once

#include "common.cuh"
#include "merge_rule.cuh"
#include "tmem_ld.cuh"

namespace ra {

constexpr int kBM = 128;        // query rows per tile = TMEM lanes
constexpr int kCtaRows = 256;   // two tiles per CTA
constexpr int kBN = 128;        // keys per KV tile
constexpr int kMaxBlocks = 16;  // ring size limit
constexpr int kAttnThreads = 384;
constexpr int kRegsLaunch = 168;  // per thread at launch (__launch_bounds__(384, 1))
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kAttnThreads * kRegsLaunch,
              "register reallocation must fit in the launch allocation");
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;

enum AttnMode : int {
  kModePartial = 0,  // write (block_out, block_lse) into acc rows
  kModeMerge = 1,    // merge (block_out, block_lse) into the acc rows in place
  kModeFinal = 2     // write (out, lse) at original token positions
};

// A run of consecutive original positions [pos, pos + len) stored at rows
// [mem, mem + len) of a tensor.
struct Seg {
  int mem, pos, len;
};

struct AttnArgs {
  int B, S;               // batch, full sequence length
  int Hq, Hkv, groups;    // query heads, KV heads, Hq / Hkv
  int causal;
  int nq;                 // query blocks covered by this launch
  int nkv;                // KV blocks each query block visits in this launch
  int nseg;               // segments per block: 1 (contiguous) or 2 (zigzag)
  int seg_tiles;          // CTAs per query segment: ceil(len / 256), or ceil(len / 128) in KV-split mode
  int kv_split;           // 1: KV-split mode (see the top of this file)
  int cluster;            // CTAs per cluster sharing one row pair (1 or 2; row pairs only;
                          // selects the kernel instantiation, see Tiling)
  float scale_log2;       // log2(e) / sqrt(D)
  int mode;               // AttnMode
  // kModePartial / kModeMerge: row = b * acc_brows + memory row of the query
  float* acc_out;
  float* acc_lse;
  long long acc_brows;
  // kModeFinal: row = b * S + original position of the query
  void* out;
  float* lse;
  int out_bf16;
  int fault_inject;       // 1: the producer withholds its second K tile (failure-path tests);
                          // 2 (checked build only): its second K tile's row is checked out of range
  int q_rows, kv_rows;    // rows per batch of the Q and K / V tensors the maps cover
  CtaTimeline timeline;   // per-CTA tracing (rec == nullptr: off); work units = KV tiles
  Seg qseg[kMaxBlocks][2];                      // segments of the i-th query block of the launch
  Seg kvseg[kMaxBlocks][2];                     // segments of KV block r
  signed char kv_list[kMaxBlocks][kMaxBlocks];  // kv_list[i][s]: s-th KV block met by query block i
  signed char seg_order[2 * kMaxBlocks];        // (i * nseg + e) of the query segments, heaviest first
};

// Shared memory: the Q tiles (two for row pairs, one for KV-split), then a
// ring of K tiles and a ring of V tiles sized to fill the 227 KB.  A stage of
// either ring is refilled once the products of its step have read it, and
// V(g) is needed at the start of step g while K(g + 1) is needed only after
// P_A V(g) has been issued, so V gets the deeper ring where they differ.
template <int D, bool SPLIT>
struct AttnSmem {
  static constexpr int kBox = kBM * 64 * 2;  // one TMA box: 128 rows x 64 bf16 (128 B) = 16 KB
  static constexpr int kNBox = D / 64;
  static constexpr int kTile = kBox * kNBox;
  static constexpr int kQTiles = SPLIT ? 1 : 2;
  static constexpr int kNSK = D == 128 ? (SPLIT ? 3 : 2) : (SPLIT ? 6 : 5);
  static constexpr int kNSV = D == 128 ? 3 : 6;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQTiles * kTile;
  static constexpr int kV = kK + kNSK * kTile;
  static constexpr int kBar = kV + kNSV * kTile;
  // barriers: Q, Kfull[NSK], Kempty[NSK], Vfull[NSV], Vempty[NSV], Sfull[2], Pfull[2] (first
  // half of P), Odone[2], End, Phalf[2] (second half of P)
  static constexpr int kNBar = 1 + 2 * kNSK + 2 * kNSV + 2 + 2 + 2 + 1 + 2;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kTotal = kAbort + 4;               // KV tiles of the CTA's sequence
  static constexpr int kSegTab = (kTotal + 4 + 15) & ~15;  // SegTile[2 * kMaxBlocks]
  static constexpr int kBytes = kSegTab + 2 * kMaxBlocks * 32 + 1024;  // + slack to align the base to 1024
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Keys of a KV segment visible to a query at original position qpos: a
// prefix of the segment.  qpos < 0 marks a padding row.
__device__ __forceinline__ int visible_count(const AttnArgs& a, const Seg& kv, int qpos) {
  if (qpos < 0) return 0;
  if (!a.causal) return kv.len;
  return min(max(qpos - kv.pos + 1, 0), kv.len);
}

__device__ __forceinline__ int tiles_for(const AttnArgs& a, const Seg& kv, int qpos) {
  return (visible_count(a, kv, qpos) + kBN - 1) / kBN;
}

// Bounded wait that ignores the abort flag, used only to drain work that is
// already in flight before the CTA frees its resources.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      set_status(RA_ERR_TIMEOUT);
      return;
    }
  }
}

// One KV segment of the CTA's sequence with its tile counts for the CTA's
// last row (nt) and the last rows of tiles A and B (na, nb); the kernel fills
// a table of these in shared memory once, one segment per lane.
struct SegTile {
  Seg seg;
  int nt, na, nb, pad[2];
};
static_assert(sizeof(SegTile) == 32, "segment table entry");

// A walk over the CTA's KV tiles in schedule order: segment sg (KV block
// s = sg / nseg of the CTA's list, segment e = sg % nseg) and tile t inside it,
// with the segment's tile counts for the CTA's last row (nt) and the last rows
// of tiles A and B (na, nb).  The segment table is only read when the walk
// enters a segment, so a step costs a few integer operations.
struct KvWalk {
  int sg, t;
  int nt, na, nb;
};

// Tiling modes (compile-time: each kernel instantiation carries only its own
// code).
enum Tiling : int { kTileRowPairs = 0, kTileKvSplit = 1, kTileCluster2 = 2 };

template <int D, int TILING>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  constexpr bool SPLIT = TILING == kTileKvSplit;
  constexpr int kCl = TILING == kTileCluster2 ? 2 : 1;  // CTAs per cluster
  using SL = AttnSmem<D, SPLIT>;
  constexpr int NSK = SL::kNSK;
  constexpr int NSV = SL::kNSV;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  timeline_begin(a.timeline);

  // ---- tile decode: heads fastest (heads of one KV group share K/V in L2),
  // then batch, then query tiles in decreasing position (heaviest first).
  int crank = 0;
  if constexpr (kCl > 1) crank = static_cast<int>(cluster_ctarank());
  int idx = blockIdx.x / kCl;
  const int h = idx % a.Hq;
  idx /= a.Hq;
  const int b = idx % a.B;
  idx /= a.B;
  const int so = a.seg_order[idx / a.seg_tiles];
  const int qt = a.seg_tiles - 1 - idx % a.seg_tiles;
  const int qi = so / a.nseg;
  const Seg qs = a.qseg[qi][so % a.nseg];
  const int hk = h / a.groups;
  constexpr bool split = SPLIT;
  const int t0 = qt * (split ? kBM : kCtaRows);  // CTA row offset inside the query segment
  // per tile X (A = 0, B = 1): first row in the segment, valid rows, last position
  const int row0_a = t0, row0_b = t0 + (split ? 0 : kBM);
  const int rows_a = min(max(qs.len - row0_a, 0), kBM), rows_b = min(max(qs.len - row0_b, 0), kBM);
  const int last_a = rows_a > 0 ? qs.pos + row0_a + rows_a - 1 : -1;
  const int last_b = rows_b > 0 ? qs.pos + row0_b + rows_b - 1 : -1;
  const int last_u = max(last_a, last_b);  // the CTA's last row: its KV range covers both tiles
  auto seg_of = [&](int s_, int e_) -> const Seg& { return a.kvseg[a.kv_list[qi][s_]][e_]; };

  // Walk helpers (see KvWalk): enter the segment sg (skipping segments the
  // CTA sees nothing of), start at the CTA's u-th tile, step to the next tile.
  const int nsg = a.nkv * a.nseg;
  const SegTile* seg_tab = reinterpret_cast<const SegTile*>(smem + SL::kSegTab);
  auto enter = [&](KvWalk& k) {
    for (; k.sg < nsg; ++k.sg) {
      const SegTile& e = seg_tab[k.sg];
      if (e.nt > 0) {
        k.nt = e.nt;
        k.na = e.na;
        k.nb = e.nb;
        return;
      }
    }
    k.nt = k.na = k.nb = 0;
  };
  auto walk_from = [&](int u) -> KvWalk {
    KvWalk k;
    k.sg = 0;
    enter(k);
    while (k.nt > 0 && u >= k.nt) {
      u -= k.nt;
      ++k.sg;
      enter(k);
    }
    k.t = u;
    return k;
  };
  auto walk_next = [&](KvWalk& k) {
    if (++k.t >= k.nt) {
      k.t = 0;
      ++k.sg;
      enter(k);
    }
  };

  auto bar = [&](int i) -> uint32_t { return sb + SL::kBar + 8u * i; };
  const int BQ = 0;
  auto BKF = [&](int s) { return 1 + s; };
  auto BKE = [&](int s) { return 1 + NSK + s; };
  auto BVF = [&](int s) { return 1 + 2 * NSK + s; };
  auto BVE = [&](int s) { return 1 + 2 * NSK + NSV + s; };
  auto BSF = [&](int x) { return 1 + 2 * NSK + 2 * NSV + x; };
  auto BPF = [&](int x) { return 3 + 2 * NSK + 2 * NSV + x; };
  auto BOD = [&](int x) { return 5 + 2 * NSK + 2 * NSV + x; };
  const int BEND = 7 + 2 * NSK + 2 * NSV;
  auto BPH = [&](int x) { return 8 + 2 * NSK + 2 * NSV + x; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SL::kNBar; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(BPF(0)), kBM / 32);  // one arrival per softmax warp
    mbar_init(bar(BPF(1)), kBM / 32);
    mbar_init(bar(BPH(0)), kBM / 32);
    mbar_init(bar(BPH(1)), kBM / 32);
    *abort_flag = grid_timed_out() ? 1 : 0;  // after a timeout elsewhere, do no work
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(sb + SL::kTmemSlot, 512);
  if (warp == kMmaWarp + 1) {
    // the segment table, one segment per lane, and the CTA's tile count
    int nt = 0;
    if (lane < nsg) {
      SegTile e;
      e.seg = seg_of(lane / a.nseg, lane % a.nseg);
      nt = e.nt = tiles_for(a, e.seg, last_u);
      e.na = tiles_for(a, e.seg, last_a);
      e.nb = tiles_for(a, e.seg, last_b);
      e.pad[0] = e.pad[1] = 0;
      reinterpret_cast<SegTile*>(smem + SL::kSegTab)[lane] = e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nt += __shfl_xor_sync(0xffffffffu, nt, o);
    if (lane == 0) *reinterpret_cast<int*>(smem + SL::kTotal) = nt;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SL::kTmemSlot);
  const int total = *reinterpret_cast<volatile int*>(smem + SL::kTotal);
  // this CTA's share [lo, hi) of the sequence (the cluster splits it in equal parts)
  const int lo = kCl > 1 ? crank * total / kCl : 0;
  const int hi = kCl > 1 ? (crank + 1) * total / kCl : total;
  int work = hi - lo;
  timeline_work(a.timeline, work);
  // Tile x's share of the CTA's KV tiles.  u = index in the CTA's sequence,
  // t = index inside the segment.  KV-split: A takes [0, half), B [half, total).
  const int half = (total + 1) / 2;
  if (*abort_flag) work = 0;

  // ---- staging buffers and the final row write (see the epilogue)
  constexpr int kStride = D + 4;                        // floats per staged row (bank-conflict-free)
  constexpr int kStageFloats = kBM * kStride + 2 * kBM; // rows, then per-row weight and lse
  static_assert(2 * kStageFloats * 4 <= SL::kBar - SL::kK, "staging buffers must fit in the K/V rings");
  auto stage_of = [&](int x) { return reinterpret_cast<float*>(smem + SL::kK) + x * kStageFloats; };
  // Final write of tile x's staged rows, in two parts.  commit_lse: each of
  // the tile's threads writes the lse of its own row (merged into the running
  // state in epilogue-fused mode, where it also records the row's weight).
  // store_rows: warp wi of nw warps writes rows [wi*128/nw, (wi+1)*128/nw)
  // as contiguous runs (16 bytes per lane).
  auto commit_lse = [&](int x) {
    float* stage = stage_of(x);
    float* stage_w = stage + kBM * kStride;
    const float* stage_l = stage_w + kBM;
    const int row = threadIdx.x & 127;
    const int my_row0 = x ? row0_b : row0_a;
    const int my_rows = x ? rows_b : rows_a;
    const long long row_base = a.mode == kModeFinal ? static_cast<long long>(b) * a.S + qs.pos + my_row0
                                                    : static_cast<long long>(b) * a.acc_brows + qs.mem + my_row0;
    const long long out_rows = a.mode == kModeFinal ? static_cast<long long>(a.B) * a.S
                                                    : static_cast<long long>(a.B) * a.acc_brows;
    (void)out_rows;  // read by the checks of the checked build only
    if (row < my_rows && RA_IN_BOUNDS(row_base + row, out_rows) && RA_IN_BOUNDS(h, a.Hq)) {
      float* lse_ptr = (a.mode == kModeFinal ? a.lse : a.acc_lse) + (row_base + row) * a.Hq + h;
      if (a.mode == kModeMerge) {
        const MergeWeights mw = merge_weights(*lse_ptr, stage_l[row]);
        *lse_ptr = mw.lse;
        stage_w[row] = mw.w;
      } else {
        *lse_ptr = stage_l[row];
      }
    }
  };
  auto store_rows = [&](int x, int wi, int nw) {
    const float* stage = stage_of(x);
    const float* stage_w = stage + kBM * kStride;
    const int my_row0 = x ? row0_b : row0_a;
    const int my_rows = x ? rows_b : rows_a;
    const long long row_base = a.mode == kModeFinal ? static_cast<long long>(b) * a.S + qs.pos + my_row0
                                                    : static_cast<long long>(b) * a.acc_brows + qs.mem + my_row0;
    const int per = kBM / nw;
    const int wr0 = wi * per;
    const long long first = (row_base + wr0) * a.Hq + h;  // output row index of row wr0
    if (kDebugBounds) {  // checked build: this warp's rows must lie inside the output
      const long long out_rows = a.mode == kModeFinal ? static_cast<long long>(a.B) * a.S
                                                      : static_cast<long long>(a.B) * a.acc_brows;
      const int last = min(per, my_rows - wr0) - 1;
      (void)out_rows;
      if (last >= 0 && !(RA_IN_BOUNDS(row_base + wr0, out_rows) && RA_IN_BOUNDS(row_base + wr0 + last, out_rows) &&
                         RA_IN_BOUNDS(h, a.Hq)))
        return;
    }
    const long long rstride = static_cast<long long>(a.Hq) * D;  // elements between consecutive rows
    if (a.mode == kModeFinal && a.out_bf16) {
      constexpr int lpr = D / 8, rpi = 32 / lpr;  // 16 B (8 bf16) per lane
      const int ci = lane % lpr, rl = lane / lpr;
      __nv_bfloat16* dst0 = static_cast<__nv_bfloat16*>(a.out) + first * D + 8 * ci;
#pragma unroll 4
      for (int r0 = 0; r0 < per; r0 += rpi) {
        const int r = r0 + rl;
        if (r < per && wr0 + r < my_rows) {
          const float* src = stage + (wr0 + r) * kStride + 8 * ci;
          const float4 lo4 = *reinterpret_cast<const float4*>(src);
          const float4 hi4 = *reinterpret_cast<const float4*>(src + 4);
          uint4 o;
          o.x = pack_bf16x2(lo4.x, lo4.y);
          o.y = pack_bf16x2(lo4.z, lo4.w);
          o.z = pack_bf16x2(hi4.x, hi4.y);
          o.w = pack_bf16x2(hi4.z, hi4.w);
          __stcs(reinterpret_cast<uint4*>(dst0 + r * rstride), o);
        }
      }
      return;
    }
    constexpr int lpr = D / 4, rpi = 32 / lpr;  // 16 B (4 floats) per lane
    const int ci = lane % lpr, rl = lane / lpr;
    float* dst0 = (a.mode == kModeFinal ? static_cast<float*>(a.out) : a.acc_out) + first * D + 4 * ci;
    if (a.mode != kModeMerge) {
#pragma unroll 4
      for (int r0 = 0; r0 < per; r0 += rpi) {
        const int r = r0 + rl;
        if (r < per && wr0 + r < my_rows)
          __stcs(reinterpret_cast<float4*>(dst0 + r * rstride),
                 *reinterpret_cast<const float4*>(stage + (wr0 + r) * kStride + 4 * ci));
      }
      return;
    }
    // epilogue-fused schedule: the staged block partial merged into the running rows
    for (int r0 = 0; r0 < per; r0 += rpi) {
      const int r = r0 + rl;
      if (r >= per || wr0 + r >= my_rows) continue;
      const float wr = stage_w[wr0 + r];
      if (wr == 0.f) continue;
      float4* dst = reinterpret_cast<float4*>(dst0 + r * rstride);
      float4 v = *reinterpret_cast<const float4*>(stage + (wr0 + r) * kStride + 4 * ci);
      const float4 old = *dst;
      v.x = merge_out(old.x, v.x, wr);
      v.y = merge_out(old.y, v.y, wr);
      v.z = merge_out(old.z, v.z, wr);
      v.w = merge_out(old.w, v.w, wr);
      *dst = v;
    }
  };

  if (warp >= 8) {
    // third warpgroup: TMA producer, MMA issuer, two idle warps
    regs_dec<kRegsOther>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && work > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int nqt = split ? 1 : 2;  // KV-split: both tiles read Q_A
      // checked build: the rows a tile uses must lie inside the Q tensor (a
      // tile with no rows, past a short segment's end, reads TMA's zero fill)
      bool q_ok = RA_IN_BOUNDS(h, a.Hq) && RA_IN_BOUNDS(b, a.B);
      for (int x = 0; x < nqt; ++x) {
        const int r0 = qs.mem + (x ? row0_b : row0_a), nr = x ? rows_b : rows_a;
        if (nr > 0) q_ok = q_ok && RA_IN_BOUNDS(r0, a.q_rows) && RA_IN_BOUNDS(r0 + nr - 1, a.q_rows);
        (void)r0;
      }
      if (!q_ok) *abort_flag = 1;  // checked build: the load is skipped and the CTA gives up
      if (q_ok) {
        mbar_expect_tx(bar(BQ), nqt * SL::kTile);
        for (int x = 0; x < nqt; ++x)
          for (int bx = 0; bx < SL::kNBox; ++bx)
            tma_load_4d(sb + SL::kQ + x * SL::kTile + bx * SL::kBox, &tmQ, bx * 64, h,
                        qs.mem + (x ? row0_b : row0_a), b, bar(BQ));
      }
      int g = 0;
      bool ok = true;
      // row pairs: one walk over [lo, hi); KV-split: A's tiles [0, half) and B's
      // [half, total), loaded alternately A0, B0, A1, B1, ...
      KvWalk wa = walk_from(split ? 0 : lo);
      KvWalk wb = walk_from(split ? half : total);
      int issued_k[NSK], issued_v[NSV];
      for (int s = 0; s < NSK; ++s) issued_k[s] = -1;
      for (int s = 0; s < NSV; ++s) issued_v[s] = -1;
      // L2 prefetch: when load g2 is issued into its ring stage, load
      // g2 + kL2Ahead is prefetched into L2, so that by the time its own stage
      // frees, its ring load reads L2 rather than HBM.  A second cursor walks
      // the load order kL2Ahead loads ahead of the ring loads.  One load
      // ahead: at 1,048,576 tokens (power-capped) two ahead ran the same
      // TFLOP/s per MHz but at a 52 MHz lower clock (1,120 against 1,145 -
      // 1,153 TFLOP/s); at 24,000 tokens the two are even.
      constexpr int kL2Ahead = 1;
      KvWalk pa = wa, pb = wb;
      int g_pf = 0;
      auto prefetch_next = [&]() {
        const bool pub = split && (g_pf & 1);
        KvWalk& pw = pub ? pb : pa;
        const int row = seg_tab[pw.sg].seg.mem + pw.t * kBN;
        for (int bx = 0; bx < SL::kNBox; ++bx) {
          tma_prefetch_l2_4d(&tmK, bx * 64, hk, row, b);
          tma_prefetch_l2_4d(&tmV, bx * 64, hk, row, b);
        }
        walk_next(pw);
        ++g_pf;
      };
      for (int i = 0; i < kL2Ahead && g_pf < work; ++i) walk_next(split && (g_pf & 1) ? pb : pa), ++g_pf;
      // load order: the CTA's sequence (row pairs), or A0, B0, A1, B1, ... (KV-split)
      for (int g2 = 0; g2 < work && ok; ++g2) {
        if (g_pf < work) prefetch_next();
        const bool use_b = split && (g2 & 1);
        const int t = use_b ? wb.t : wa.t;
        const Seg ks = seg_tab[use_b ? wb.sg : wa.sg].seg;
        const int sk = g % NSK, sv = g % NSV;
        if (!mbar_wait(bar(BKE(sk)), ((g / NSK) & 1) ^ 1, abort_flag)) { ok = false; break; }
        // checked build: the tile's row and heads must lie inside the K / V tensors
        const int row_chk = ks.mem + t * kBN + (kDebugBounds && a.fault_inject == 2 && g == 1 ? a.kv_rows : 0);
        (void)row_chk;
        if (!(RA_IN_BOUNDS(row_chk, a.kv_rows) && RA_IN_BOUNDS(hk, a.Hkv) && RA_IN_BOUNDS(use_b ? wb.sg : wa.sg, nsg))) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (!(a.fault_inject == 1 && g == 1)) {  // an injected fault: this K tile never arrives
          mbar_expect_tx(bar(BKF(sk)), SL::kTile);
          for (int bx = 0; bx < SL::kNBox; ++bx)
            tma_load_4d(sb + SL::kK + sk * SL::kTile + bx * SL::kBox, &tmK, bx * 64, hk, ks.mem + t * kBN, b,
                        bar(BKF(sk)));
          issued_k[sk] = g;
        }
        if (!mbar_wait(bar(BVE(sv)), ((g / NSV) & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(bar(BVF(sv)), SL::kTile);
        for (int bx = 0; bx < SL::kNBox; ++bx)
          tma_load_4d(sb + SL::kV + sv * SL::kTile + bx * SL::kBox, &tmV, bx * 64, hk, ks.mem + t * kBN, b,
                      bar(BVF(sv)));
        issued_v[sv] = g;
        ++g;
        if (use_b) walk_next(wb);
        else walk_next(wa);
      }
      if (!ok) {  // let every copy already issued land before shared memory is released
        if (q_ok) mbar_drain(bar(BQ), 0);
        for (int s = 0; s < NSK; ++s)
          if (issued_k[s] >= 0) mbar_drain(bar(BKF(s)), (issued_k[s] / NSK) & 1);
        for (int s = 0; s < NSV; ++s)
          if (issued_v[s] >= 0) mbar_drain(bar(BVF(s)), (issued_v[s] / NSV) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0 && work > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, true);
      const int qslot1 = split ? 0 : 1;  // Q tile of B
      // The tensor core takes 64 cycles for a 128 x 128 x 16 product and this
      // one thread shares its scheduler with two softmax warps, so its work per
      // product decides how close the products run to that rate.  Every
      // descriptor is therefore a base computed here plus a compile-time
      // offset added to its low half (see mma_ss_lo); the descriptors share
      // their high half (the 1024-byte atom stride and the swizzle mode).
      const uint64_t dq0 = smem_desc_sw128(sb + SL::kQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sb + SL::kK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sb + SL::kV, SL::kBox, 1024);
      const uint32_t hi_qk = static_cast<uint32_t>(dq0 >> 32), hi_v = static_cast<uint32_t>(dv0 >> 32);
      const uint32_t lo_q0 = static_cast<uint32_t>(dq0);
      const uint32_t lo_q1 = lo_q0 + static_cast<uint32_t>((qslot1 * SL::kTile) >> 4);
      const uint32_t lo_k = static_cast<uint32_t>(dk0), lo_v = static_cast<uint32_t>(dv0);
      auto issue_s = [&](int x, int st) {
        const uint32_t a = x ? lo_q1 : lo_q0;
        const uint32_t bk = lo_k + static_cast<uint32_t>(st) * (SL::kTile >> 4);
        const uint32_t td = tmem + x * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * SL::kBox + (kk % 4) * 32) >> 4;
          mma_ss_lo(td, a + off, bk + off, hi_qk, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(BSF(x)));
      };
      // O_X += P_X V in two halves of the keys: the first as soon as the
      // softmax has written P's first 64 columns (Pfull), the second once it
      // has written the rest (Phalf).  Returns false when a wait gave up.
      auto issue_pv = [&](int x, int st, bool acc, uint32_t parity) -> bool {
        const uint32_t bv = lo_v + static_cast<uint32_t>(st) * (SL::kTile >> 4);
        const uint32_t to = tmem + 256 + x * 128, tp = tmem + x * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait_spin(bar(h ? BPH(x) : BPF(x)), parity, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
            mma_ts_lo(to, tp + kk * 8, bv + ((kk * 2048) >> 4), hi_v, kIdescO, (acc || kk > 0) ? 1u : 0u);
        }
        return true;
      };

      if (split) {
        // KV-split: tile x's i-th KV tile is load 2i + x (A has half, B total - half tiles)
        const int n_of[2] = {half, total - half};
        bool okk = mbar_wait(bar(BQ), 0, abort_flag);
        for (int x = 0; x < 2 && okk; ++x) {
          if (n_of[x] == 0) continue;
          okk = mbar_wait(bar(BKF(x % NSK)), (x / NSK) & 1, abort_flag);
          if (!okk) break;
          tc_fence_after();
          issue_s(x, x % NSK);
          tc_commit(bar(BKE(x % NSK)));
        }
        for (int j = 0; j < half && okk; ++j) {
          for (int x = 0; x < 2; ++x) {
            if (j >= n_of[x]) continue;
            const int ld = 2 * j + x, st = ld % NSV;
            if (!mbar_wait(bar(BVF(st)), (ld / NSV) & 1, abort_flag)) { okk = false; break; }
            if (!issue_pv(x, st, j > 0, j & 1)) { okk = false; break; }
            tc_commit(bar(BVE(st)));
            if (j + 1 < n_of[x]) {
              const int ld1 = ld + 2, st1 = ld1 % NSK;
              if (!mbar_wait(bar(BKF(st1)), (ld1 / NSK) & 1, abort_flag)) { okk = false; break; }
              tc_fence_after();
              issue_s(x, st1);
              tc_commit(bar(BKE(st1)));
            }
          }
        }
        tc_commit(bar(BOD(0)));  // O_A and O_B are complete once every product is
        tc_commit(bar(BOD(1)));
        tc_commit(bar(BEND));
        mbar_drain(bar(BEND), 0);
      } else {
      KvWalk cur = walk_from(lo);  // this CTA's first tile (work > 0, so it exists)
      bool act[2] = {cur.t < cur.na, cur.t < cur.nb};
      int cnt[2] = {0, 0};  // P V products issued per tile
      bool ok = mbar_wait(bar(BQ), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(BKF(0)), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (act[x]) issue_s(x, 0);
        tc_commit(bar(BKE(0)));
      }
      for (int g = 0; ok && g < work; ++g) {
        const int st = g % NSV;                 // V stage of tile g
        const int sk1 = (g + 1) % NSK;          // K stage of tile g + 1
        const bool has_next = g + 1 < work;
        KvWalk nxt = cur;
        bool act1[2] = {false, false};
        if (has_next) {
          walk_next(nxt);
          act1[0] = nxt.t < nxt.na;
          act1[1] = nxt.t < nxt.nb;
        }
        if (!mbar_wait(bar(BVF(st)), (g / NSV) & 1, abort_flag)) break;
        bool k_ready = false;
        const int last_pv = act[1] ? 1 : 0;  // the step's last P V product reads V(g) last
        for (int x = 0; x < 2; ++x) {
          if (act[x]) {
            if (!issue_pv(x, st, cnt[x] > 0, cnt[x] & 1)) { ok = false; break; }
            ++cnt[x];
            if (x == last_pv) tc_commit(bar(BVE(st)));  // V(g) is free once that product is done
          }
          if (act1[x]) {
            if (!k_ready) {
              if (!mbar_wait(bar(BKF(sk1)), ((g + 1) / NSK) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              k_ready = true;
            }
            issue_s(x, sk1);
          }
        }
        if (!ok) break;
        if (has_next) tc_commit(bar(BKE(sk1)));
        cur = nxt;
        act[0] = act1[0];
        act[1] = act1[1];
      }
      tc_commit(bar(BOD(0)));  // O_A and O_B are complete once every product is
      tc_commit(bar(BOD(1)));
      // nothing may still write tensor memory when it is released
      tc_commit(bar(BEND));
      mbar_drain(bar(BEND), 0);
      }
    }
  }
  } else {
    // ------------------------------------------------------------- softmax
    regs_inc<kRegsSoftmax>();
    const int x = warp >> 2;            // tile A (0) or B (1)
    const int row = threadIdx.x & 127;  // row inside the tile = TMEM lane
    const int my_row0 = x ? row0_b : row0_a;
    const int my_rows = x ? rows_b : rows_a;
    const bool valid = row < my_rows;
    const int qpos = valid ? qs.pos + my_row0 + row : -1;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + x * 128;
    const uint32_t tO = tmem + lane_base + 256 + x * 128;
    const float sl2 = a.scale_log2;
    // Padding rows (beyond the segment) see no key: all their scores are
    // masked and, with a finite base, their exponentials are 0.
    float m_use = valid ? -INFINITY : 0.f;
    float l_sum = 0.f;
    bool ok = work > 0;
    int c = 0;  // tiles processed by this tile's softmax
    // This tile's KV tiles: row pairs, those of [lo, hi) its rows see;
    // KV-split, A's [0, half) or B's [half, total) of the CTA's sequence.
    KvWalk w = walk_from(split ? (x ? half : 0) : lo);
    const int n_walk = split ? (x ? total - half : half) : work;
    int lim_sg = -1, lim = 0;  // keys of the walk's segment this row sees
    for (int i = 0; i < n_walk && ok; ++i, walk_next(w)) {
      if (!split && w.t >= (x ? w.nb : w.na)) continue;
      if (w.sg != lim_sg) {
        lim_sg = w.sg;
        lim = visible_count(a, seg_tab[w.sg].seg, qpos);
      }
      const int t = w.t;
      ok = mbar_wait(bar(BSF(x)), c & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[kBN];
      const int cnt = lim - t * kBN;
      // S of this row from TMEM, with the keys it may not see set to -inf
      // (warp-uniform test: full tiles skip the masking code)
      tmem_ld128_wait(tS, sv);
      if (__any_sync(0xffffffffu, cnt < kBN)) {
#pragma unroll
        for (int j = 0; j < kBN; ++j) sv[j] = j < cnt ? sv[j] : __float_as_uint(-INFINITY);
      }
      // The row maximum first (3-input max, 8 independent chains of depth 8),
      // so that the base of the exponentials is settled before any of them is
      // taken: P can then go to the tensor core in two halves.  The base is
      // raised only when the tile maximum exceeds it by more than 8 (log2
      // units; every P value then stays <= 2^8), and O is rescaled in TMEM.
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = fmaxf(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1]));
#pragma unroll
      for (int j = 16; j < kBN; j += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          m8[q] = fmax3(m8[q], __uint_as_float(sv[j + 2 * q]), __uint_as_float(sv[j + 2 * q + 1]));
      const float mt =
          fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
      float alpha = 1.f;
      bool resc = false;
      if (mt > m_use + 8.f) {  // also a row's first visible keys (m_use = -inf)
        if (m_use != -INFINITY) {
          alpha = fast_exp2(m_use - mt);
          resc = true;
        }
        m_use = mt;
      }
      // O of this tile is stable here: S_X(c) was committed after the P V
      // product of tile c-1, so its completion implies that one's.
      if (c > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t ov[32];
          tmem_ld32_wait(tO + 32 * q, ov);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) ov[i2] = __float_as_uint(__uint_as_float(ov[i2]) * alpha);
          tmem_st32(tO + 32 * q, ov);
        }
      }
      // P = 2^(scale * S - base) as packed bf16 pairs, on the SFU (ex2.approx),
      // over the score columns [64h, 64h + 64), stored over S in this tile's
      // TMEM columns [32h, 32h + 32); returns the row sum of the fp32 values.
      // Each half is handed to the MMA thread as soon as it is in TMEM.
      const float base = m_use == -INFINITY ? 0.f : m_use;
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t nbase2 = f2_pack(-base, -base);
      float psum = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int ch = 2 * h; ch < 2 * h + 2; ++ch) {  // 32 scores -> 16 packed bf16 pairs per store
          uint32_t pk[16];
#pragma unroll
          for (int pp = 0; pp < 16; ++pp) {
            const int j = ch * 32 + 2 * pp;
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), sl2x2, nbase2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint64_t e2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
            acc[pp & 3] = f2_add(acc[pp & 3], e2);
            float p0, p1;
            f2_unpack(e2, p0, p1);
            pk[pp] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + ch * 16, pk);
        }
        const uint64_t acc2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float ps0, ps1;
        f2_unpack(acc2, ps0, ps1);
        psum += ps0 + ps1;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(h ? BPH(x) : BPF(x)));
      }
      l_sum = l_sum * alpha + psum;
      ++c;
    }

    // ------------------------------------------------------------ epilogue
    // Each tile's rows are normalised into a staging buffer in shared memory,
    // then every warp writes whole rows to HBM with coalesced stores.  The K/V
    // rings hold the staging buffers: they are idle once the last P V products
    // of both tiles have landed (barrier below).
    if (ok && c > 0) {
      ok = mbar_wait(bar(BOD(x)), 0, abort_flag);  // one commit, after the last product
      ok = __all_sync(0xffffffffu, ok);
    }
    const bool has = ok && l_sum > 0.f;
    const float inv = has ? 1.f / l_sum : 0.f;
    const float row_lse = has ? (m_use + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
    named_barrier_sync(1, 256);  // both tiles' MMAs are complete: the rings are free
    fence_proxy_async_smem();
    if (split) {
      // KV-split: both tiles hold a partial of the same 128 rows.  The two
      // warps of a row exchange (lse, 1/l) through shared memory, then each
      // stitches half of the columns with the merge rule, reading both
      // partials straight from tensor memory (same lanes).
      float* xch = stage_of(1);  // [tile][lse, 1/l][row]
      xch[x * 2 * kBM + row] = row_lse;
      xch[x * 2 * kBM + kBM + row] = inv;
      named_barrier_sync(1, 256);
      tc_fence_after();
      const float lse_a = xch[row], inv_a = xch[kBM + row];
      const float lse_b = xch[2 * kBM + row], inv_b = xch[3 * kBM + row];
      const bool has_a = lse_a != -INFINITY, has_b = lse_b != -INFINITY;
      // tensor-memory loads are warp-collective: guarded by warp-uniform tile counts
      const bool ld_a = ok && half > 0, ld_b = ok && total - half > 0;
      const MergeWeights mw = merge_weights(lse_a, lse_b);
      float* stage = stage_of(0);
      if (x == 0) stage[kBM * kStride + kBM + row] = mw.lse;
      const uint32_t tOa = tmem + lane_base + 256, tOb = tmem + lane_base + 384;
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        const int col = x * (D / 2) + 32 * q;  // this warpgroup's half of the columns
        uint32_t oa[32], ob[32];
        if (ld_a) tmem_ld32_wait(tOa + col, oa);
        if (ld_b) tmem_ld32_wait(tOb + col, ob);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float v[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float va = ld_a && has_a ? __uint_as_float(oa[i + k]) * inv_a : 0.f;
            const float vb = ld_b && has_b ? __uint_as_float(ob[i + k]) * inv_b : 0.f;
            v[k] = merge_out(va, vb, mw.w);
          }
          *reinterpret_cast<float4*>(stage + row * kStride + col + i) = make_float4(v[0], v[1], v[2], v[3]);
        }
      }
      if (x == 0 && (ok || work == 0)) commit_lse(0);
      named_barrier_sync(1, 256);  // every row is staged (and its merge weight recorded)
      if (ok || work == 0) store_rows(0, warp, 8);
    } else if (ok || work == 0) {
      // row pairs: each tile stages and writes its own rows
      float* stage = stage_of(x);
      stage[kBM * kStride + kBM + row] = row_lse;
      uint32_t ov[D];
      if (c > 0) {  // c is uniform across the warp
        tc_fence_after();
        if constexpr (D == 128) tmem_ld128_wait(tO, ov);
        else tmem_ld64_wait(tO, ov);
      }
#pragma unroll
      for (int i = 0; i < D; i += 4)
        *reinterpret_cast<float4*>(stage + row * kStride + i) =
            make_float4(has ? __uint_as_float(ov[i]) * inv : 0.f, has ? __uint_as_float(ov[i + 1]) * inv : 0.f,
                        has ? __uint_as_float(ov[i + 2]) * inv : 0.f, has ? __uint_as_float(ov[i + 3]) * inv : 0.f);
      if constexpr (kCl == 1) {
        commit_lse(x);
        __syncwarp();  // each warp stores the 32 rows it staged
        store_rows(x, warp & 3, 4);
      }
    }
  }

  if constexpr (kCl > 1) {
    // Cluster mode: CTA r finalises tile r.  Its row = own partial merged
    // with the peer CTA's partial of the same row (merge rule), read from the
    // peer's staging buffer through distributed shared memory.
    cluster_sync();  // both CTAs have staged both tiles
    if (warp < 8 && (warp >> 2) == crank) {
      const int x = crank;
      const int row = threadIdx.x & 127;
      float* stage = stage_of(x);
      float* stage_l = stage + kBM * kStride + kBM;
      const uint32_t peer = cluster_map(smem_u32(stage), static_cast<uint32_t>(crank ^ 1));
      const float peer_lse = ld_cluster_f32(peer + 4u * (kBM * kStride + kBM + row));
      const MergeWeights mw = merge_weights(stage_l[row], peer_lse);
      stage_l[row] = mw.lse;
      if (mw.w != 0.f) {
        float* own = stage + row * kStride;
#pragma unroll 8
        for (int i = 0; i < D; i += 4) {
          const float4 pv = ld_cluster_f4(peer + 4u * (row * kStride + i));
          float4 ov = *reinterpret_cast<float4*>(own + i);
          ov.x = merge_out(ov.x, pv.x, mw.w);
          ov.y = merge_out(ov.y, pv.y, mw.w);
          ov.z = merge_out(ov.z, pv.z, mw.w);
          ov.w = merge_out(ov.w, pv.w, mw.w);
          *reinterpret_cast<float4*>(own + i) = ov;
        }
      }
      commit_lse(x);
      __syncwarp();
      store_rows(x, warp & 3, 4);
    }
    cluster_sync();  // the peer has finished reading this CTA's staging buffers
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  timeline_end(a.timeline);
}

}  // namespace ra
