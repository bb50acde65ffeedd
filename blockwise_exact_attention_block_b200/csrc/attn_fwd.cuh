// attn_fwd.cuh - block attention on the 5th-generation tensor cores (sm_100a).
//
// One CTA computes one 128-row query tile of one (batch, query head) against
// a list of KV blocks (one block for ra_block_attn and the unfused schedule,
// every block in schedule order for the persistent schedule).
//
// TokenRing review (pith.science, arXiv 2412.20501), "What carries the
// argument" / "Core claim": the flash-attention kernel that yields, for one
// query block and one key/value block, the softmax-normalised block_out and
// the per-row block_lse; "If this is right": grouped-query attention and the
// zigzag causal partition; Anthology of the SOTA, SOTA-181: exact attention.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread i owns query row i of the tile (TMEM lane i).
//   warp 4     TMA producer: Q once, then K and V tiles into an NST-deep ring.
//   warp 5     TMEM allocator and MMA issuer (one thread):
//                S_j  = Q K_j^T       (SS MMA, fp32 into TMEM, two buffers)
//                O   += P_j V_j       (TS MMA, P_j bf16 in TMEM over S_j)
// Tensor memory (512 columns): S buffers at columns [0,128) and [128,256);
// P_j is written as packed bf16 into the first 64 columns of its S buffer;
// the O accumulator lives at columns [256, 256 + D).
//
// Online softmax in fp32 with base-2 exponentials (scores pre-scaled by
// log2(e)/sqrt(D)).  The running maximum used for the exponentials is only
// raised when a tile's maximum exceeds it by more than 8 (a factor 256), so
// O is rescaled in TMEM rarely; the final out = O / l and
// lse = ln 2 * (m + log2 l) are exact for any such choice of m.
//
// Causal masking uses original token positions.  Inside one block positions
// increase with the block-local row index (both partitions), so the keys a
// query may see form a prefix of each KV block: the tile loop stops at the
// last tile the tile's last row can see, and only tiles cut by a row's prefix
// are masked element-wise.
#pragma once

#include "common.cuh"
#include "merge_rule.cuh"
#include "tmem_ld.cuh"

namespace ra {

constexpr int kBM = 128;        // query rows per tile = TMEM lanes
constexpr int kBN = 128;        // keys per KV tile
constexpr int kMaxBlocks = 16;  // ring size limit
constexpr int kAttnThreads = 192;

enum AttnMode : int {
  kModePartial = 0,  // write (block_out, block_lse) into acc rows
  kModeMerge = 1,    // merge (block_out, block_lse) into the acc rows in place
  kModeFinal = 2     // write (out, lse) at original token positions
};

struct AttnArgs {
  int B, S, n, L, c;      // batch, sequence, ring size, block length, zigzag chunk
  int Hq, Hkv, groups;    // query heads, KV heads, Hq / Hkv
  int zigzag, causal;
  int nq;                 // query blocks covered by this launch
  int nkv;                // KV blocks each query block visits in this launch
  int tiles_per_block;    // ceil(L / 128)
  int q_bmul, q_rmul;     // TMA 4th coordinate of (batch b, block r) = b*bmul + r*rmul
  int kv_bmul, kv_rmul;
  float scale_log2;       // log2(e) / sqrt(D)
  int mode;               // AttnMode
  // kModePartial / kModeMerge: row = b * acc_brows + r * acc_rmul * L + t
  float* acc_out;
  float* acc_lse;
  long long acc_brows;
  int acc_rmul;
  // kModeFinal: row = b * S + pos (original order)
  void* out;
  float* lse;
  int out_bf16;
  signed char q_blocks[kMaxBlocks];
  signed char kv_list[kMaxBlocks][kMaxBlocks];  // kv_list[i][s]: s-th KV block of query block i
};

template <int D, int NST>
struct AttnSmem {
  static constexpr int kBox = kBM * 64 * 2;  // one TMA box: 128 rows x 64 bf16 (128 B) = 16 KB
  static constexpr int kNBox = D / 64;
  static constexpr int kTile = kBox * kNBox;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + NST * kTile;
  static constexpr int kBar = kV + NST * kTile;
  // barriers: Q, Kfull[NST], Vfull[NST], Kempty[NST], Vempty[NST], Sfull[2], Pfull[2], Odone, End
  static constexpr int kNBar = 1 + 4 * NST + 2 + 2 + 1 + 1;
  static constexpr int kTmemSlot = kBar + kNBar * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4 + 1024;  // + slack to align the base to 1024
  static_assert(kBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ int block_pos(const AttnArgs& a, int r, int t) {
  if (!a.zigzag) return r * a.L + t;
  return t < a.c ? r * a.c + t : (2 * a.n - 1 - r) * a.c + (t - a.c);
}

// Number of keys of KV block kvb visible to a query at original position qpos
// (they form a prefix of the block).  qpos < 0 marks a padding row.
__device__ __forceinline__ int visible_count(const AttnArgs& a, int kvb, int qpos) {
  if (qpos < 0) return 0;
  if (!a.causal) return a.L;
  if (!a.zigzag) return min(max(qpos - kvb * a.L + 1, 0), a.L);
  const int c1 = min(max(qpos - kvb * a.c + 1, 0), a.c);
  const int c2 = min(max(qpos - (2 * a.n - 1 - kvb) * a.c + 1, 0), a.c);
  return c1 + c2;
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
  // heaviest tiles first.
  int idx = blockIdx.x;
  const int h = idx % a.Hq;
  idx /= a.Hq;
  const int b = idx % a.B;
  idx /= a.B;
  int qi, qt;
  if (a.zigzag) {
    qt = a.tiles_per_block - 1 - idx / a.nq;
    qi = a.nq - 1 - idx % a.nq;
  } else {
    qi = a.nq - 1 - idx / a.tiles_per_block;
    qt = a.tiles_per_block - 1 - idx % a.tiles_per_block;
  }
  const int r = a.q_blocks[qi];
  const int hk = h / a.groups;
  const int t0 = qt * kBM;
  const int q_rows = min(kBM, a.L - t0);
  const int last_pos = block_pos(a, r, t0 + q_rows - 1);

  int total = 0;
  for (int s = 0; s < a.nkv; ++s)
    total += (visible_count(a, a.kv_list[qi][s], last_pos) + kBN - 1) / kBN;

  auto bar = [&](int i) -> uint32_t { return sb + SL::kBar + 8u * i; };
  const int BQ = 0;
  auto BKF = [&](int s) { return 1 + s; };
  auto BVF = [&](int s) { return 1 + NST + s; };
  auto BKE = [&](int s) { return 1 + 2 * NST + s; };
  auto BVE = [&](int s) { return 1 + 3 * NST + s; };
  auto BSF = [&](int i) { return 1 + 4 * NST + i; };
  auto BPF = [&](int i) { return 3 + 4 * NST + i; };
  const int BOD = 5 + 4 * NST;
  const int BEND = 6 + 4 * NST;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SL::kAbort);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SL::kNBar; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(BPF(0)), 128);
    mbar_init(bar(BPF(1)), 128);
    *abort_flag = grid_timed_out() ? 1 : 0;  // after a timeout elsewhere, do no work
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(sb + SL::kTmemSlot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SL::kTmemSlot);
  if (*abort_flag) total = 0;
  const uint32_t tO = tmem + 256;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar(BQ), SL::kTile);
      for (int x = 0; x < SL::kNBox; ++x)
        tma_load_4d(sb + SL::kQ + x * SL::kBox, &tmQ, x * 64, h, t0, b * a.q_bmul + r * a.q_rmul,
                    bar(BQ));
      int g = 0;
      bool ok = true;
      int issued_k[NST], issued_v[NST];
      for (int s = 0; s < NST; ++s) issued_k[s] = issued_v[s] = -1;
      for (int s = 0; s < a.nkv && ok; ++s) {
        const int kvb = a.kv_list[qi][s];
        const int nt = (visible_count(a, kvb, last_pos) + kBN - 1) / kBN;
        const int wc = b * a.kv_bmul + kvb * a.kv_rmul;
        for (int t = 0; t < nt; ++t, ++g) {
          const int st = g % NST;
          const uint32_t ph = (g / NST) & 1;
          if (!mbar_wait(bar(BKE(st)), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(bar(BKF(st)), SL::kTile);
          for (int x = 0; x < SL::kNBox; ++x)
            tma_load_4d(sb + SL::kK + st * SL::kTile + x * SL::kBox, &tmK, x * 64, hk, t * kBN, wc,
                        bar(BKF(st)));
          issued_k[st] = g;
          if (!mbar_wait(bar(BVE(st)), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(bar(BVF(st)), SL::kTile);
          for (int x = 0; x < SL::kNBox; ++x)
            tma_load_4d(sb + SL::kV + st * SL::kTile + x * SL::kBox, &tmV, x * 64, hk, t * kBN, wc,
                        bar(BVF(st)));
          issued_v[st] = g;
        }
      }
      if (!ok) {  // let every copy already issued land before shared memory is released
        mbar_drain(bar(BQ), 0);
        for (int s = 0; s < NST; ++s) {
          if (issued_k[s] >= 0) mbar_drain(bar(BKF(s)), (issued_k[s] / NST) & 1);
          if (issued_v[s] >= 0) mbar_drain(bar(BVF(s)), (issued_v[s] / NST) & 1);
        }
      }
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0 && total > 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, true);
      auto issue_s = [&](int g) {
        const int st = g % NST;
        const uint32_t dst = tmem + (g & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * SL::kBox + (kk % 4) * 32;
          const uint64_t ad = smem_desc_sw128(sb + SL::kQ + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sb + SL::kK + st * SL::kTile + off, 16, 1024);
          mma_ss(dst, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(BSF(g & 1)));
        tc_commit(bar(BKE(st)));
      };
      bool ok = mbar_wait(bar(BQ), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(BKF(0)), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int g = 0; ok && g < total; ++g) {
        if (g + 1 < total) {
          const int st1 = (g + 1) % NST;
          if (!mbar_wait(bar(BKF(st1)), ((g + 1) / NST) & 1, abort_flag)) break;
          tc_fence_after();
          issue_s(g + 1);
        }
        if (!mbar_wait(bar(BPF(g & 1)), (g >> 1) & 1, abort_flag)) break;
        const int st = g % NST;
        if (!mbar_wait(bar(BVF(st)), (g / NST) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t pcol = tmem + (g & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(sb + SL::kV + st * SL::kTile + kk * 2048, SL::kBox, 1024);
          mma_ts(tO, pcol + kk * 8, bd, kIdescO, (g > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(BOD));
        tc_commit(bar(BVE(st)));
      }
      // nothing may still write tensor memory when it is released
      tc_commit(bar(BEND));
      mbar_drain(bar(BEND), 0);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int row = threadIdx.x;  // 0..127
    const int tl = t0 + row;
    const bool valid = row < q_rows;
    const int qpos = valid ? block_pos(a, r, tl) : -1;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_use = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;
    int g = 0;
    for (int s = 0; s < a.nkv && ok; ++s) {
      const int kvb = a.kv_list[qi][s];
      const int nt = (visible_count(a, kvb, last_pos) + kBN - 1) / kBN;
      const int lim = visible_count(a, kvb, qpos);
      for (int t = 0; t < nt; ++t, ++g) {
        ok = mbar_wait(bar(BSF(g & 1)), (g >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[kBN];
        tmem_ld128_wait(tmem + lane_base + (g & 1) * 128, sv);
        const int cnt = lim - t * kBN;
        float mx = -INFINITY;
        if (cnt < kBN) {
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const float x = c < cnt ? __uint_as_float(sv[c]) : -INFINITY;
            sv[c] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBN; ++c) mx = fmaxf(mx, __uint_as_float(sv[c]));
        }
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
        float psum = 0.f;
        uint32_t pk[kBN / 2];
#pragma unroll
        for (int c = 0; c < kBN; c += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sv[c]), sl2, -base));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sv[c + 1]), sl2, -base));
          psum += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        l_sum = l_sum * alpha + psum;
        const uint32_t pdst = tmem + lane_base + (g & 1) * 128;
        tmem_st32(pdst, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        tmem_st32(pdst + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        tmem_wait_st();
        if (g > 0) {
          // O may only be touched once the previous P V product has landed.
          ok = mbar_wait(bar(BOD), (g - 1) & 1, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          if (__any_sync(0xffffffffu, resc)) {
            tc_fence_after();
            uint32_t ov[D];
            if constexpr (D == 128) tmem_ld128_wait(tO + lane_base, ov);
            else tmem_ld64_wait(tO + lane_base, ov);
#pragma unroll
            for (int i = 0; i < D; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
#pragma unroll
            for (int i = 0; i < D / 32; ++i)
              tmem_st32(tO + lane_base + 32 * i, *reinterpret_cast<const uint32_t(*)[32]>(&ov[32 * i]));
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(bar(BPF(g & 1)));
      }
    }

    // ------------------------------------------------------------ epilogue
    if (ok && total > 0) {
      ok = mbar_wait(bar(BOD), (total - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      uint32_t ov[D];
      if (total > 0) {
        tc_fence_after();
        if constexpr (D == 128) tmem_ld128_wait(tO + lane_base, ov);
        else tmem_ld64_wait(tO + lane_base, ov);
      }
      const bool has = l_sum > 0.f;
      const float inv = has ? 1.f / l_sum : 0.f;
      const float row_lse = has ? (m_use + log2f(l_sum)) * 0.6931471805599453f : -INFINITY;
#pragma unroll
      for (int i = 0; i < D; ++i) ov[i] = __float_as_uint(has ? __uint_as_float(ov[i]) * inv : 0.f);

      if (valid) {
        if (a.mode == kModeFinal) {
          const long long orow = static_cast<long long>(b) * a.S + qpos;
          const long long o = (orow * a.Hq + h) * D;
          a.lse[orow * a.Hq + h] = row_lse;
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + o);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]), __uint_as_float(ov[8 * i + 1]));
              w.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3]));
              w.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5]));
              w.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7]));
              dst[i] = w;
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.out) + o);
#pragma unroll
            for (int i = 0; i < D / 4; ++i)
              dst[i] = make_uint4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
          }
        } else {
          const long long prow =
              static_cast<long long>(b) * a.acc_brows + static_cast<long long>(r) * a.acc_rmul * a.L + tl;
          float* dst = a.acc_out + (prow * a.Hq + h) * D;
          float* dl = a.acc_lse + prow * a.Hq + h;
          if (a.mode == kModePartial) {
            *dl = row_lse;
#pragma unroll
            for (int i = 0; i < D / 4; ++i)
              reinterpret_cast<uint4*>(dst)[i] = make_uint4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
          } else {
            const MergeWeights mw = merge_weights(*dl, row_lse);
            *dl = mw.lse;
            if (mw.w != 0.f) {
#pragma unroll
              for (int i = 0; i < D / 4; ++i) {
                float4 cur = reinterpret_cast<float4*>(dst)[i];
                cur.x = merge_out(cur.x, __uint_as_float(ov[4 * i + 0]), mw.w);
                cur.y = merge_out(cur.y, __uint_as_float(ov[4 * i + 1]), mw.w);
                cur.z = merge_out(cur.z, __uint_as_float(ov[4 * i + 2]), mw.w);
                cur.w = merge_out(cur.w, __uint_as_float(ov[4 * i + 3]), mw.w);
                reinterpret_cast<float4*>(dst)[i] = cur;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, 512);
}

}  // namespace ra
