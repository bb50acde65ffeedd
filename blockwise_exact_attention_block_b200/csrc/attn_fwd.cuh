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
//
// TokenRing review (pith.science, arXiv 2412.20501), "What carries the
// argument" / "Core claim": the flash-attention kernel that yields, for one
// query block and one key/value block, the softmax-normalised block_out and
// the per-row block_lse; "If this is right": grouped-query attention and the
// zigzag causal partition; Anthology of the SOTA, SOTA-181: exact attention.
//
// Warp roles (320 threads):
//   warps 0-3  softmax of tile A: thread i owns row i of A (TMEM lane i)
//   warps 4-7  softmax of tile B (same lanes, its own TMEM columns)
//   warp 8     TMA producer: Q (A and B) once, then K and V into an NST ring
//   warp 9     TMEM allocator and MMA issuer (one thread):
//                S_X = Q_X K^T   (SS MMA, fp32 in TMEM)
//                O_X += P_X V    (TS MMA, P_X bf16 in TMEM over S_X)
//              issued in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so
//              the tensor core works on one tile while the other tile's
//              softmax runs.
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
constexpr int kAttnThreads = 320;
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
  Seg qseg[kMaxBlocks][2];                      // segments of the i-th query block of the launch
  Seg kvseg[kMaxBlocks][2];                     // segments of KV block r
  signed char kv_list[kMaxBlocks][kMaxBlocks];  // kv_list[i][s]: s-th KV block met by query block i
  signed char seg_order[2 * kMaxBlocks];        // (i * nseg + e) of the query segments, heaviest first
};

template <int D, int NST>
struct AttnSmem {
  static constexpr int kBox = kBM * 64 * 2;  // one TMA box: 128 rows x 64 bf16 (128 B) = 16 KB
  static constexpr int kNBox = D / 64;
  static constexpr int kTile = kBox * kNBox;
  static constexpr int kQ = 0;                // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kTile;
  static constexpr int kV = kK + NST * kTile;
  static constexpr int kBar = kV + NST * kTile;
  // barriers: Q, Kfull[NST], Vfull[NST], Kempty[NST], Vempty[NST], Sfull[2], Pfull[2], Odone[2], End
  static constexpr int kNBar = 1 + 4 * NST + 2 + 2 + 2 + 1;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;  // + slack to align the base to 1024
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

// Position of the CTA's g-th KV tile as (KV block index s, segment e, tile t).
struct KvCursor {
  int s, e, t, nt;
};

template <int D, int NST>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  using SL = AttnSmem<D, NST>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- tile decode: heads fastest (heads of one KV group share K/V in L2),
  // then batch, then query tiles in decreasing position (heaviest first).
  int idx = blockIdx.x;
  const int h = idx % a.Hq;
  idx /= a.Hq;
  const int b = idx % a.B;
  idx /= a.B;
  const int so = a.seg_order[idx / a.seg_tiles];
  const int qt = a.seg_tiles - 1 - idx % a.seg_tiles;
  const int qi = so / a.nseg;
  const Seg qs = a.qseg[qi][so % a.nseg];
  const int hk = h / a.groups;
  const bool split = a.kv_split != 0;
  const int t0 = qt * (split ? kBM : kCtaRows);  // CTA row offset inside the query segment
  int rows[2], last[2], row0[2];                 // per tile: valid rows, last position, first row
  for (int x = 0; x < 2; ++x) {
    row0[x] = t0 + (split ? 0 : x * kBM);
    rows[x] = min(max(qs.len - row0[x], 0), kBM);
    last[x] = rows[x] > 0 ? qs.pos + row0[x] + rows[x] - 1 : -1;
  }
  const int last_u = max(last[0], last[1]);  // the CTA's last row: its KV range covers both tiles
  auto seg_of = [&](int s_, int e_) -> const Seg& { return a.kvseg[a.kv_list[qi][s_]][e_]; };

  int total = 0;
  for (int s = 0; s < a.nkv; ++s)
    for (int e = 0; e < a.nseg; ++e) total += tiles_for(a, seg_of(s, e), last_u);
  // Tile x's share of the CTA's KV tiles.  u = index in the CTA's sequence,
  // t = index inside the segment.  KV-split: A takes [0, half), B [half, total).
  const int half = (total + 1) / 2;
  auto active = [&](int x, int u, int t, const Seg& ks) -> bool {
    if (split) return x == 0 ? u < half : u >= half;
    return t < tiles_for(a, ks, last[x]);
  };
  // The segment and in-segment tile of the CTA's u-th KV tile.
  auto locate = [&](int u, int& s_, int& e_, int& t_) {
    for (s_ = 0; s_ < a.nkv; ++s_)
      for (e_ = 0; e_ < a.nseg; ++e_) {
        const int nt = tiles_for(a, seg_of(s_, e_), last_u);
        if (u < nt) {
          t_ = u;
          return;
        }
        u -= nt;
      }
    t_ = 0;
  };

  auto bar = [&](int i) -> uint32_t { return sb + SL::kBar + 8u * i; };
  const int BQ = 0;
  auto BKF = [&](int s) { return 1 + s; };
  auto BVF = [&](int s) { return 1 + NST + s; };
  auto BKE = [&](int s) { return 1 + 2 * NST + s; };
  auto BVE = [&](int s) { return 1 + 3 * NST + s; };
  auto BSF = [&](int x) { return 1 + 4 * NST + x; };
  auto BPF = [&](int x) { return 3 + 4 * NST + x; };
  auto BOD = [&](int x) { return 5 + 4 * NST + x; };
  const int BEND = 7 + 4 * NST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SL::kNBar; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(BPF(0)), kBM);
    mbar_init(bar(BPF(1)), kBM);
    *abort_flag = grid_timed_out() ? 1 : 0;  // after a timeout elsewhere, do no work
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(sb + SL::kTmemSlot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SL::kTmemSlot);
  if (*abort_flag) total = 0;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int nqt = split ? 1 : 2;  // KV-split: both tiles read Q_A
      mbar_expect_tx(bar(BQ), nqt * SL::kTile);
      for (int x = 0; x < nqt; ++x)
        for (int bx = 0; bx < SL::kNBox; ++bx)
          tma_load_4d(sb + SL::kQ + x * SL::kTile + bx * SL::kBox, &tmQ, bx * 64, h, qs.mem + row0[x], b,
                      bar(BQ));
      int g = 0;
      bool ok = true;
      int issued_k[NST], issued_v[NST];
      for (int s = 0; s < NST; ++s) issued_k[s] = issued_v[s] = -1;
      // load order: the CTA's sequence (row pairs), or A0, B0, A1, B1, ... (KV-split)
      for (int g2 = 0; g2 < total && ok; ++g2) {
        int s, e, t;
        locate(split ? ((g2 & 1) ? half + (g2 >> 1) : (g2 >> 1)) : g2, s, e, t);
        const Seg ks = seg_of(s, e);
        const int st = g % NST;
        const uint32_t ph = (g / NST) & 1;
        if (!mbar_wait(bar(BKE(st)), ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(bar(BKF(st)), SL::kTile);
        for (int bx = 0; bx < SL::kNBox; ++bx)
          tma_load_4d(sb + SL::kK + st * SL::kTile + bx * SL::kBox, &tmK, bx * 64, hk, ks.mem + t * kBN, b,
                      bar(BKF(st)));
        issued_k[st] = g;
        if (!mbar_wait(bar(BVE(st)), ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(bar(BVF(st)), SL::kTile);
        for (int bx = 0; bx < SL::kNBox; ++bx)
          tma_load_4d(sb + SL::kV + st * SL::kTile + bx * SL::kBox, &tmV, bx * 64, hk, ks.mem + t * kBN, b,
                      bar(BVF(st)));
        issued_v[st] = g;
        ++g;
      }
      if (!ok) {  // let every copy already issued land before shared memory is released
        mbar_drain(bar(BQ), 0);
        for (int s = 0; s < NST; ++s) {
          if (issued_k[s] >= 0) mbar_drain(bar(BKF(s)), (issued_k[s] / NST) & 1);
          if (issued_v[s] >= 0) mbar_drain(bar(BVF(s)), (issued_v[s] / NST) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0 && total > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, true);
      const int qslot1 = split ? 0 : 1;  // Q tile of B
      auto issue_s = [&](int x, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * SL::kBox + (kk % 4) * 32;
          const uint64_t ad = smem_desc_sw128(sb + SL::kQ + (x ? qslot1 : 0) * SL::kTile + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sb + SL::kK + st * SL::kTile + off, 16, 1024);
          mma_ss(tmem + x * 128, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(BSF(x)));
      };
      auto issue_pv = [&](int x, int st, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(sb + SL::kV + st * SL::kTile + kk * 2048, SL::kBox, 1024);
          mma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, bd, kIdescO, (acc || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(BOD(x)));
      };
      // moves the cursor to the next KV tile that exists
      auto advance = [&](KvCursor& k) {
        ++k.t;
        while (k.t >= k.nt && k.s < a.nkv) {
          k.t = 0;
          if (++k.e == a.nseg) {
            k.e = 0;
            ++k.s;
          }
          k.nt = k.s < a.nkv ? tiles_for(a, seg_of(k.s, k.e), last_u) : 0;
        }
      };
      auto active_at = [&](const KvCursor& k, int x) { return k.t < tiles_for(a, seg_of(k.s, k.e), last[x]); };

      if (split) {
        // KV-split: tile x's i-th KV tile is load 2i + x (A has half, B total - half tiles)
        const int n_of[2] = {half, total - half};
        bool okk = mbar_wait(bar(BQ), 0, abort_flag);
        for (int x = 0; x < 2 && okk; ++x) {
          if (n_of[x] == 0) continue;
          okk = mbar_wait(bar(BKF(x % NST)), (x / NST) & 1, abort_flag);
          if (!okk) break;
          tc_fence_after();
          issue_s(x, x % NST);
          tc_commit(bar(BKE(x % NST)));
        }
        for (int j = 0; j < half && okk; ++j) {
          for (int x = 0; x < 2; ++x) {
            if (j >= n_of[x]) continue;
            const int ld = 2 * j + x, st = ld % NST;
            if (!mbar_wait(bar(BVF(st)), (ld / NST) & 1, abort_flag)) { okk = false; break; }
            if (!mbar_wait(bar(BPF(x)), j & 1, abort_flag)) { okk = false; break; }
            tc_fence_after();
            issue_pv(x, st, j > 0);
            tc_commit(bar(BVE(st)));
            if (j + 1 < n_of[x]) {
              const int ld1 = ld + 2, st1 = ld1 % NST;
              if (!mbar_wait(bar(BKF(st1)), (ld1 / NST) & 1, abort_flag)) { okk = false; break; }
              tc_fence_after();
              issue_s(x, st1);
              tc_commit(bar(BKE(st1)));
            }
          }
        }
        tc_commit(bar(BEND));
        mbar_drain(bar(BEND), 0);
      } else {
      KvCursor cur = {0, 0, -1, tiles_for(a, seg_of(0, 0), last_u)};
      advance(cur);  // first existing tile (total > 0, so there is one)
      bool act[2] = {active_at(cur, 0), active_at(cur, 1)};
      int cnt[2] = {0, 0};  // P V products issued per tile
      bool ok = mbar_wait(bar(BQ), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(BKF(0)), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (act[x]) issue_s(x, 0);
        tc_commit(bar(BKE(0)));
      }
      for (int g = 0; ok && g < total; ++g) {
        const int st = g % NST;
        const bool has_next = g + 1 < total;
        KvCursor nxt = cur;
        bool act1[2] = {false, false};
        if (has_next) {
          advance(nxt);
          act1[0] = active_at(nxt, 0);
          act1[1] = active_at(nxt, 1);
        }
        if (!mbar_wait(bar(BVF(st)), (g / NST) & 1, abort_flag)) break;
        bool k_ready = false;
        for (int x = 0; x < 2; ++x) {
          if (act[x]) {
            if (!mbar_wait(bar(BPF(x)), cnt[x] & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv(x, st, cnt[x] > 0);
            ++cnt[x];
          }
          if (act1[x]) {
            if (!k_ready) {
              if (!mbar_wait(bar(BKF((g + 1) % NST)), ((g + 1) / NST) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              k_ready = true;
            }
            issue_s(x, (g + 1) % NST);
          }
        }
        if (!ok) break;
        tc_commit(bar(BVE(st)));
        if (has_next) tc_commit(bar(BKE((g + 1) % NST)));
        cur = nxt;
        act[0] = act1[0];
        act[1] = act1[1];
      }
      // nothing may still write tensor memory when it is released
      tc_commit(bar(BEND));
      mbar_drain(bar(BEND), 0);
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2;            // tile A (0) or B (1)
    const int row = threadIdx.x & 127;  // row inside the tile = TMEM lane
    const bool valid = row < rows[x];
    const int qpos = valid ? qs.pos + row0[x] + row : -1;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + x * 128;
    const uint32_t tO = tmem + lane_base + 256 + x * 128;
    const float sl2 = a.scale_log2;
    float m_use = -INFINITY;
    float l_sum = 0.f;
    bool ok = total > 0;
    int c = 0;  // tiles processed by this tile's softmax
    int u = 0;  // position in the CTA's KV sequence
    for (int s = 0; s < a.nkv && ok; ++s)
      for (int e = 0; e < a.nseg && ok; ++e) {
        const Seg ks = seg_of(s, e);
        const int nt = tiles_for(a, ks, last_u);
        const int lim = visible_count(a, ks, qpos);
        for (int t = 0; t < nt; ++t, ++u) {
          if (!active(x, u, t, ks)) continue;
          ok = mbar_wait(bar(BSF(x)), c & 1, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          uint32_t sv[kBN];
          tmem_ld128_wait(tS, sv);
          const int cnt = lim - t * kBN;
          // row maximum with 8 independent chains (short dependency paths)
          float mx8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
          if (cnt < kBN) {
#pragma unroll
            for (int j = 0; j < kBN; ++j) {
              const float v = j < cnt ? __uint_as_float(sv[j]) : -INFINITY;
              sv[j] = __float_as_uint(v);
              mx8[j & 7] = fmaxf(mx8[j & 7], v);
            }
          } else {
#pragma unroll
            for (int j = 0; j < kBN; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(sv[j]));
          }
          const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          const float mt = mx * sl2;
          float alpha = 1.f;
          bool resc = false;
          if (mt > m_use + 8.f) {
            if (m_use != -INFINITY) {
              alpha = fast_exp2(m_use - mt);
              resc = true;
            }
            m_use = mt;
          }
          const float base = (m_use == -INFINITY) ? 0.f : m_use;
          float ps8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) ps8[i] = 0.f;
#pragma unroll
          for (int ch = 0; ch < kBN / 32; ++ch) {  // 32 scores -> 16 packed bf16 pairs per store
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch * 32 + j]), sl2, -base));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch * 32 + j + 1]), sl2, -base));
              ps8[(j >> 1) & 7] += p0 + p1;
              pk[j / 2] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + ch * 16, pk);
          }
          const float psum = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
          l_sum = l_sum * alpha + psum;
          tmem_wait_st();
          if (c > 0) {
            // O may only be touched once the previous P V product has landed.
            ok = mbar_wait(bar(BOD(x)), (c - 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (__any_sync(0xffffffffu, resc)) {
              tc_fence_after();
#pragma unroll
              for (int q = 0; q < D / 32; ++q) {
                uint32_t ov[32];
                tmem_ld32_wait(tO + 32 * q, ov);
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                tmem_st32(tO + 32 * q, ov);
              }
              tmem_wait_st();
            }
          }
          tc_fence_before();
          mbar_arrive(bar(BPF(x)));
          ++c;
        }
      }

    // ------------------------------------------------------------ epilogue
    if (ok && c > 0) {
      ok = mbar_wait(bar(BOD(x)), (c - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (split) {
      // Stitch B's partial into A's with the merge rule.  B writes its
      // normalised row and lse to shared memory (the K/V ring is idle once
      // both tiles' last P V product has landed), then A merges.
      float* xo = reinterpret_cast<float*>(smem + SL::kK);  // [128][D + 4]
      float* xl = xo + kBM * (D + 4);                        // [128]
      named_barrier_sync(1, 256);  // both tiles' MMAs are complete
      fence_proxy_async_smem();
      if (x == 1) {
        const bool has = ok && l_sum > 0.f;
        const float inv = has ? 1.f / l_sum : 0.f;
        xl[row] = has ? (m_use + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
        if (c > 0) tc_fence_after();
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t ov[32];
          if (ok && c > 0) tmem_ld32_wait(tO + 32 * q, ov);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(xo + row * (D + 4) + 32 * q + i) =
                make_float4(has ? __uint_as_float(ov[i]) * inv : 0.f, has ? __uint_as_float(ov[i + 1]) * inv : 0.f,
                            has ? __uint_as_float(ov[i + 2]) * inv : 0.f, has ? __uint_as_float(ov[i + 3]) * inv : 0.f);
        }
      }
      named_barrier_sync(1, 256);
    }
    // rows are written by every tile in row-pair mode, by A alone in KV-split mode
    if ((ok || total == 0) && !(split && x == 1)) {
      const bool has = l_sum > 0.f;
      const float inv = has ? 1.f / l_sum : 0.f;
      float row_lse = has ? (m_use + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
      MergeWeights mwb;  // KV-split: weight of B's partial in this row
      mwb.w = 0.f;
      if (split) {
        mwb = merge_weights(row_lse, reinterpret_cast<float*>(smem + SL::kK)[kBM * (D + 4) + row]);
        row_lse = mwb.lse;
      }
      if (c > 0) tc_fence_after();
      long long o_off = 0;
      float* lse_ptr = nullptr;
      if (a.mode == kModeFinal) {
        const long long orow = static_cast<long long>(b) * a.S + qpos;
        o_off = (orow * a.Hq + h) * D;
        lse_ptr = a.lse + orow * a.Hq + h;
      } else {
        const long long prow = static_cast<long long>(b) * a.acc_brows + qs.mem + row0[x] + row;
        o_off = (prow * a.Hq + h) * D;
        lse_ptr = a.acc_lse + prow * a.Hq + h;
      }
      MergeWeights mw;
      mw.w = 1.f;
      mw.lse = row_lse;
      if (valid && a.mode == kModeMerge) mw = merge_weights(*lse_ptr, row_lse);
      if (valid) *lse_ptr = mw.lse;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t ov[32];
        if (c > 0) tmem_ld32_wait(tO + 32 * q, ov);  // c is uniform across the warp
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(has ? __uint_as_float(ov[i]) * inv : 0.f);
        if (split && mwb.w != 0.f) {
          const float* xb = reinterpret_cast<const float*>(smem + SL::kK) + row * (D + 4) + 32 * q;
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(merge_out(__uint_as_float(ov[i]), xb[i], mwb.w));
        }
        if (!valid) continue;
        if (a.mode == kModeFinal && a.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + o_off + 32 * q);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]), __uint_as_float(ov[8 * i + 1]));
            w.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3]));
            w.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5]));
            w.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7]));
            dst[i] = w;
          }
        } else {
          float4* dst =
              reinterpret_cast<float4*>((a.mode == kModeFinal ? static_cast<float*>(a.out) : a.acc_out) + o_off + 32 * q);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 v = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                   __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
            if (a.mode == kModeMerge) {
              if (mw.w == 0.f) continue;
              const float4 old = dst[i];
              v.x = merge_out(old.x, v.x, mw.w);
              v.y = merge_out(old.y, v.y, mw.w);
              v.z = merge_out(old.z, v.z, mw.w);
              v.w = merge_out(old.w, v.w, mw.w);
            }
            dst[i] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace ra
