// api.cu - the C ABI of libra_b200.so (include/ra.h): argument validation,
// TMA tensor maps, and the block scheduler that replays the ring / TokenRing
// order on one GPU.  The whole library is this one translation unit, so the
// device status word in common.cuh has a single definition.
//
// Schedules (Anthology of the SOTA, SOTA-181: the query block stays, KV
// blocks pass around the ring; TokenRing review, "Core claim" and "major
// comments, Algorithm 1 (section 3.2)": the KV block stays, query blocks move
// forward and partial results move back):
//   ring:      query block r meets KV blocks r, r-1, r-2, ... (mod n)
//   TokenRing: query block r meets KV blocks r, r+1, r+2, ... (mod n)
// (TokenRing step s, 1-based, pairs KV block j with query block
// (j - s + 1) mod n, i.e. query block r with KV block (r + s - 1) mod n.)
#include <math.h>
#include <stdio.h>

#include <mutex>

#include "attn_fwd.cuh"
#include "attn_bwd.cuh"
#include "decode.cuh"
#include "merge.cuh"
#include "permute.cuh"

namespace {

using namespace ra;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor viewed as [NB][L][H][D] (innermost last), box = box_rows rows x
// 64 columns of one head, 128-byte swizzle.  Rows beyond L read as zero.  The
// 4th coordinate is the batch index.
bool make_map(CUtensorMap* m, const void* ptr, int D, int H, int L, int NB, int box_rows = kBM) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(NB)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2,
                                 static_cast<cuuint64_t>(L) * H * D * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline ra_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RA_OK : RA_ERR_CUDA; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

struct Geom {
  int B, S, n, L, c, Hq, Hkv, groups, D, zigzag, causal;
};

ra_status check_geom(int B, int S, int n, int Hq, int Hkv, int D, int partition, Geom* g) {
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || n < 1) return RA_ERR_INVALID_ARG;
  if (n > kMaxBlocks) return RA_ERR_UNSUPPORTED;
  if (partition != RA_PART_CONTIGUOUS && partition != RA_PART_ZIGZAG) return RA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return RA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if (S % n != 0) return RA_ERR_INVALID_ARG;
  if (partition == RA_PART_ZIGZAG && S % (2 * n) != 0) return RA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * n > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  g->B = B;
  g->S = S;
  g->n = n;
  g->L = S / n;
  g->c = S / (2 * n);
  g->Hq = Hq;
  g->Hkv = Hkv;
  g->groups = Hq / Hkv;
  g->D = D;
  g->zigzag = partition == RA_PART_ZIGZAG;
  g->causal = 0;
  return RA_OK;
}

inline int seg_len_of(const Geom& g) { return g.zigzag ? g.c : g.L; }

// Row pairs (256 query rows per CTA, shared K/V loads) unless that leaves
// fewer than two CTAs per SM; then KV-split (128 rows per CTA, the CTA's KV
// tiles halved between its two warpgroups and merged on chip), which doubles
// the CTA count and halves the longest CTA.  The two-CTA cluster split is
// available on request (measured slower for the small grids that need it).
void choose_tiling(const Geom& g, AttnArgs& a, ra_tiling tiling) {
  const int len = seg_len_of(g);
  const long long pairs = static_cast<long long>(a.Hq) * a.B * a.nq * a.nseg * ((len + kCtaRows - 1) / kCtaRows);
  if (tiling == RA_TILING_AUTO) tiling = pairs < 2LL * sm_count() ? RA_TILING_KV_SPLIT : RA_TILING_ROW_PAIRS;
  a.kv_split = tiling == RA_TILING_KV_SPLIT ? 1 : 0;
  a.cluster = tiling == RA_TILING_CLUSTER2 ? 2 : 1;
  a.seg_tiles = (len + (a.kv_split ? kBM : kCtaRows) - 1) / (a.kv_split ? kBM : kCtaRows);
}

// The per-CTA timeline set by ra_set_cta_timeline (process-wide; off while
// rec is null): the one kernel it is recorded for, its records and their count.
struct TimelineState {
  unsigned long long* rec;
  int max_ctas;
  int kernel;
};
TimelineState g_timeline = {nullptr, 0, 0};

CtaTimeline timeline_for(int kernel) {
  if (g_timeline.rec == nullptr || g_timeline.kernel != kernel) return CtaTimeline{nullptr, 0};
  return CtaTimeline{g_timeline.rec, g_timeline.max_ctas};
}

AttnArgs base_args(const Geom& g) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.timeline = timeline_for(RA_TIMELINE_ATTN_FWD);
  a.B = g.B;
  a.S = g.S;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.groups = g.groups;
  a.causal = g.causal;
  a.nseg = g.zigzag ? 2 : 1;
  a.seg_tiles = (seg_len_of(g) + kCtaRows - 1) / kCtaRows;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(g.D)));
  return a;
}

// Segments of block r: original positions, stored at the same rows (tensor
// in original order) or at block-local rows 0.. (tensor holding block r only).
void block_segments(const Geom& g, int r, bool block_local, Seg out[2]) {
  if (!g.zigzag) {
    out[0].pos = r * g.L;
    out[0].len = g.L;
    out[0].mem = block_local ? 0 : out[0].pos;
    return;
  }
  out[0].pos = r * g.c;
  out[1].pos = (2 * g.n - 1 - r) * g.c;
  out[0].len = out[1].len = g.c;
  out[0].mem = block_local ? 0 : out[0].pos;
  out[1].mem = block_local ? g.c : out[1].pos;
}

// Query segments of the launch, heaviest (latest positions) first when causal.
void order_segments(AttnArgs& a) {
  const int m = a.nq * a.nseg;
  for (int i = 0; i < m; ++i) a.seg_order[i] = static_cast<signed char>(i);
  if (!a.causal) return;
  for (int i = 1; i < m; ++i)
    for (int j = i; j > 0; --j) {
      const Seg& x = a.qseg[a.seg_order[j] / a.nseg][a.seg_order[j] % a.nseg];
      const Seg& y = a.qseg[a.seg_order[j - 1] / a.nseg][a.seg_order[j - 1] % a.nseg];
      if (x.pos > y.pos) {
        const signed char t = a.seg_order[j];
        a.seg_order[j] = a.seg_order[j - 1];
        a.seg_order[j - 1] = t;
      }
    }
}

template <int D, int TILING>
ra_status launch_attn_t(const AttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        cudaStream_t st) {
  using SL = AttnSmem<D, TILING == kTileKvSplit>;
  static int attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, TILING>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SL::kBytes);
    if (e != cudaSuccess) return RA_ERR_CUDA;
    attr_set[dev] = 1;
  }
  const long long grid = static_cast<long long>(a.Hq) * a.B * a.nq * a.nseg * a.seg_tiles * a.cluster;
  if (grid <= 0) return RA_OK;
  if (grid > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  if (TILING != kTileCluster2) {
    attn_fwd_kernel<D, TILING><<<static_cast<unsigned>(grid), kAttnThreads, SL::kBytes, st>>>(mq, mk, mv, a);
    return cuda_status(cudaGetLastError());
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = SL::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, attn_fwd_kernel<D, TILING>, mq, mk, mv, a));
}

template <int D>
ra_status launch_attn_d(const AttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        cudaStream_t st) {
  if (a.kv_split) return launch_attn_t<D, kTileKvSplit>(a, mq, mk, mv, st);
  if (a.cluster == 2) return launch_attn_t<D, kTileCluster2>(a, mq, mk, mv, st);
  return launch_attn_t<D, kTileRowPairs>(a, mq, mk, mv, st);
}

ra_status launch_attn(int D, const AttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mk,
                      const CUtensorMap& mv, cudaStream_t st) {
  return D == 128 ? launch_attn_d<128>(a, mq, mk, mv, st) : launch_attn_d<64>(a, mq, mk, mv, st);
}

int grid_for(long long work, int per_block) {
  const long long need = (work + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(sm_count()) * 16;
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

// Blocks per SM of a merge grid, as measured on the B200 over 4,096 ..
// 1,048,576 tokens x 32 heads x 128 (fp32): up to 4 partials, 32 per SM below
// 8M float4 vectors and 128 above (pairwise: 80 - 90 % of the copy bandwidth,
// where 16 per SM with two vectors per lane gave 71 - 86 %); more partials
// keep K loads in flight per lane and do best with 16.
int merge_cap(long long nvec, int k) {
  if (k > 4) return 16;
  return nvec <= (8ll << 20) ? 32 : 128;
}

// Grid of a merge kernel: one block per 8 warp sweeps, at most cap_per_sm
// blocks per SM (the kernels stride over the rest).
int merge_grid(long long sweeps, int cap_per_sm) {
  const long long need = (sweeps + (kMergeThreads / 32) - 1) / (kMergeThreads / 32);
  const long long cap = static_cast<long long>(sm_count()) * cap_per_sm;
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

ra_status launch_merge(float* out, float* lse, const float* bo, const float* bl, long long rows, int D,
                       cudaStream_t st) {
  const long long nvec = rows * (D / 4);
  merge_partial_kernel<<<merge_grid((nvec + 32 * kMergeUnroll - 1) / (32 * kMergeUnroll), merge_cap(nvec, 2)),
                         kMergeThreads, 0, st>>>(
      out, lse, bo, bl, rows, D / 4);
  return cuda_status(cudaGetLastError());
}

template <int K>
ra_status launch_merge_k(const MergeList& ml, float* out, float* lse, long long rows, int D, cudaStream_t st) {
  const long long nvec = rows * (D / 4);
  merge_partials_kernel<K><<<merge_grid((nvec + 31) / 32, merge_cap(nvec, K)), kMergeThreads, 0, st>>>(ml, out, lse, rows,
                                                                                               D / 4);
  return cuda_status(cudaGetLastError());
}

ra_status launch_merge_partials(const MergeList& ml, int k, float* out, float* lse, long long rows, int D,
                                cudaStream_t st) {
  switch (k) {
    case 1: return launch_merge_k<1>(ml, out, lse, rows, D, st);
    case 2: return launch_merge_k<2>(ml, out, lse, rows, D, st);
    case 3: return launch_merge_k<3>(ml, out, lse, rows, D, st);
    case 4: return launch_merge_k<4>(ml, out, lse, rows, D, st);
    case 5: return launch_merge_k<5>(ml, out, lse, rows, D, st);
    case 6: return launch_merge_k<6>(ml, out, lse, rows, D, st);
    case 7: return launch_merge_k<7>(ml, out, lse, rows, D, st);
    case 8: return launch_merge_k<8>(ml, out, lse, rows, D, st);
    case 9: return launch_merge_k<9>(ml, out, lse, rows, D, st);
    case 10: return launch_merge_k<10>(ml, out, lse, rows, D, st);
    case 11: return launch_merge_k<11>(ml, out, lse, rows, D, st);
    case 12: return launch_merge_k<12>(ml, out, lse, rows, D, st);
    case 13: return launch_merge_k<13>(ml, out, lse, rows, D, st);
    case 14: return launch_merge_k<14>(ml, out, lse, rows, D, st);
    case 15: return launch_merge_k<15>(ml, out, lse, rows, D, st);
    case 16: return launch_merge_k<16>(ml, out, lse, rows, D, st);
  }
  return RA_ERR_UNSUPPORTED;
}

// Row move between original and block order, bit-exact, for rows and base
// addresses that are multiples of 2 bytes.
ra_status launch_permute_bytes(const void* src, void* dst, int B, const PermGeom& pg, long long row_bytes,
                               int inverse, cudaStream_t st) {
  const long long rows = static_cast<long long>(B) * pg.S;
  // widest vector that divides the row size and both base addresses
  const unsigned long long mix = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                                 static_cast<unsigned long long>(row_bytes);
  const int width = (mix & 15) == 0 ? 16 : (mix & 7) == 0 ? 8 : (mix & 3) == 0 ? 4 : 2;
  if (width == 16) {
    const long long rv = row_bytes / 16;
    permute_rows_kernel<uint4><<<grid_for(rows * rv, 256), 256, 0, st>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), B, pg, rv, inverse);
  } else if (width == 8) {
    const long long rv = row_bytes / 8;
    permute_rows_kernel<uint2><<<grid_for(rows * rv, 256), 256, 0, st>>>(
        static_cast<const uint2*>(src), static_cast<uint2*>(dst), B, pg, rv, inverse);
  } else if (width == 4) {
    const long long rv = row_bytes / 4;
    permute_rows_kernel<uint32_t><<<grid_for(rows * rv, 256), 256, 0, st>>>(
        static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), B, pg, rv, inverse);
  } else {
    const long long rv = row_bytes / 2;
    permute_rows_kernel<uint16_t><<<grid_for(rows * rv, 256), 256, 0, st>>>(
        static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), B, pg, rv, inverse);
  }
  return cuda_status(cudaGetLastError());
}

// Workspace plan of ra_ring_attention; offsets in bytes.  The partition
// itself needs no copy (it is applied through the TMA coordinates); the
// workspace holds only the bf16 rounding of fp32 inputs, the fp32 running
// output when the output itself is bf16 (unfused / epilogue-fused), and the
// per-step partials of the unfused schedule.
struct Plan {
  ra_sched sched;
  bool cast_inputs;
  bool acc_in_ws;
  size_t q, k, v, acc_out, part_out, part_lse, total;
};

Plan make_plan(const Geom& g, ra_dtype in_dtype, ra_dtype out_dtype, const ra_options* opts) {
  Plan p;
  memset(&p, 0, sizeof(p));
  p.sched = opts ? opts->sched : RA_SCHED_AUTO;
  if (p.sched == RA_SCHED_AUTO) p.sched = RA_SCHED_PERSISTENT;
  p.cast_inputs = in_dtype == RA_F32;
  const size_t rows = static_cast<size_t>(g.B) * g.S;
  size_t off = 0;
  if (p.cast_inputs) {
    p.q = off;
    off = align256(off + rows * g.Hq * g.D * 2);
    p.k = off;
    off = align256(off + rows * g.Hkv * g.D * 2);
    p.v = off;
    off = align256(off + rows * g.Hkv * g.D * 2);
  }
  if (p.sched != RA_SCHED_PERSISTENT) {
    p.acc_in_ws = out_dtype != RA_F32;
    if (p.acc_in_ws) {
      p.acc_out = off;
      off = align256(off + rows * g.Hq * g.D * 4);
    }
    if (p.sched == RA_SCHED_UNFUSED) {
      p.part_out = off;
      off = align256(off + rows * g.Hq * g.D * 4);
      p.part_lse = off;
      off = align256(off + rows * g.Hq * 4);
    }
  }
  p.total = off;
  return p;
}

bool valid_opts(const ra_options* o) {
  if (!o) return true;
  if (o->order != RA_ORDER_RING && o->order != RA_ORDER_TOKENRING) return false;
  if (o->tiling < RA_TILING_AUTO || o->tiling > RA_TILING_CLUSTER2) return false;
  // 2: the checked build's injected out-of-range row (see AttnArgs)
  if (o->fault_inject != 0 && o->fault_inject != 1 && !(kDebugBounds && o->fault_inject == 2)) return false;
  return o->sched >= RA_SCHED_AUTO && o->sched <= RA_SCHED_PERSISTENT;
}

// Chunking of a decode call: chunk = keys per CTA (a multiple of the tile),
// n = chunks that cover the cache.  n_req = 0 picks the n that minimises
// waves x (tiles per chunk + 2), the time of a grid of n * B * Hkv CTAs when
// `per_sm` CTAs fit on each SM (from the kernel's shared memory) and each costs
// about two tiles beyond its own, over chunks of at least four tiles.
struct DecodePlan {
  int n, chunk;
  size_t part_out, part_lse, total;
};

int decode_smem_bytes(int D, int rows) {
  const int mt = (rows + 15) / 16 <= 1 ? 1 : ((rows + 15) / 16 <= 2 ? 2 : 4);
  if (D == 128) return mt == 1 ? DecSmem<128, 1>::kBytes : mt == 2 ? DecSmem<128, 2>::kBytes : DecSmem<128, 4>::kBytes;
  return mt == 1 ? DecSmem<64, 1>::kBytes : mt == 2 ? DecSmem<64, 2>::kBytes : DecSmem<64, 4>::kBytes;
}

DecodePlan decode_plan(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_req) {
  DecodePlan p;
  memset(&p, 0, sizeof(p));
  const long long tiles = (Skv + kDecKeys - 1) / kDecKeys;
  long long n = n_req;
  if (n <= 0) {
    const long long ctas = static_cast<long long>(B) * Hkv;
    const int smem = decode_smem_bytes(D, (Hq / Hkv) * Tq);
    int per_sm = 233472 / (smem + 1024);  // 228 KB of shared memory per SM, 1 KB reserved per CTA
    per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
    const long long slots = static_cast<long long>(sm_count()) * per_sm;
    const long long max_n = (tiles + 3) / 4 < 1 ? 1 : (tiles + 3) / 4;
    long long best = -1;
    for (long long c = 1; c <= max_n && c <= 65535; ++c) {
      const long long per = (tiles + c - 1) / c;                 // tiles per chunk
      if (c > 1 && (tiles + per - 1) / per != c) continue;       // the same chunking as a smaller count
      const long long waves = (c * ctas + slots - 1) / slots;
      const long long cost = waves * (per + 2);
      if (best < 0 || cost < best) {
        best = cost;
        n = c;
      }
    }
  }
  long long chunk = (Skv + n - 1) / n;
  chunk = (chunk + kDecKeys - 1) / kDecKeys * kDecKeys;
  p.n = static_cast<int>((Skv + chunk - 1) / chunk);
  if (p.n > 65535) {  // the chunk index is gridDim.y
    chunk = ((Skv + 65534) / 65535 + kDecKeys - 1) / kDecKeys * kDecKeys;
    p.n = static_cast<int>((Skv + chunk - 1) / chunk);
  }
  p.chunk = static_cast<int>(chunk);
  const size_t rows = static_cast<size_t>(B) * Tq * Hq;
  p.part_out = 0;
  p.part_lse = align256(static_cast<size_t>(p.n) * rows * D * 4);
  p.total = align256(p.part_lse + static_cast<size_t>(p.n) * rows * 4);
  return p;
}

ra_status check_decode(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_splits) {
  if (B < 1 || Tq < 1 || Skv < 1 || Hq < 1 || Hkv < 1 || n_splits < 0) return RA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || Tq > Skv) return RA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return RA_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * Tq > kDecMaxRows) return RA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

template <int D, int MT>
ra_status launch_decode_partial(const DecodeArgs& a, const DecodePlan& p, const CUtensorMap& mk,
                                const CUtensorMap& mv, cudaStream_t st) {
  using SL = DecSmem<D, MT>;
  static int attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(decode_partial_kernel<D, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SL::kBytes) != cudaSuccess)
      return RA_ERR_CUDA;
    attr_set[dev] = 1;
  }
  decode_partial_kernel<D, MT><<<dim3(a.Hkv, p.n, a.B), kDecThreads, SL::kBytes, st>>>(mk, mv, a);
  return cuda_status(cudaGetLastError());
}

template <int D>
ra_status launch_decode_d(const DecodeArgs& a, const DecodePlan& p, const CUtensorMap& mk, const CUtensorMap& mv,
                          void* out, ra_dtype out_dtype, float* lse, cudaStream_t st) {
  // 16-row tiles of query rows per KV head: 1, 2 or 4
  const int mt = (a.rows + 15) / 16;
  ra_status s = mt <= 1   ? launch_decode_partial<D, 1>(a, p, mk, mv, st)
                : mt <= 2 ? launch_decode_partial<D, 2>(a, p, mk, mv, st)
                          : launch_decode_partial<D, 4>(a, p, mk, mv, st);
  if (s != RA_OK) return s;
  const long long rows = static_cast<long long>(a.B) * a.Tq * a.Hq;
  const long long blocks = rows;  // one CTA per row
  if (blocks > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  if (out_dtype == RA_BF16)
    decode_combine_kernel<D, __nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        a.part_out, a.part_lse, p.n, rows, static_cast<__nv_bfloat16*>(out), lse);
  else
    decode_combine_kernel<D, float><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        a.part_out, a.part_lse, p.n, rows, static_cast<float*>(out), lse);
  return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------------ backward
// Workspace of ra_ring_attention_backward: Delta and lse * log2(e) as
// [B][Hq][S] fp32, then the bf16 rounding of q, k, v and dout when in_dtype
// is fp32.
struct BwdPlan {
  bool cast_inputs;
  size_t delta, lse2, q, k, v, dout, total;
};

BwdPlan bwd_plan(const Geom& g, ra_dtype in_dtype) {
  BwdPlan p;
  memset(&p, 0, sizeof(p));
  const size_t rows = static_cast<size_t>(g.B) * g.S;
  size_t off = 0;
  p.delta = off;
  off = align256(off + rows * g.Hq * 4);
  p.lse2 = off;
  off = align256(off + rows * g.Hq * 4);
  p.cast_inputs = in_dtype == RA_F32;
  if (p.cast_inputs) {
    p.q = off;
    off = align256(off + rows * g.Hq * g.D * 2);
    p.k = off;
    off = align256(off + rows * g.Hkv * g.D * 2);
    p.v = off;
    off = align256(off + rows * g.Hkv * g.D * 2);
    p.dout = off;
    off = align256(off + rows * g.Hq * g.D * 2);
  }
  p.total = off;
  return p;
}

// Segments of the backward launch in weight order: latest positions first
// (queries that see the most keys) or earliest first (keys seen by the most
// queries); every order is correct, this one shortens the tail of the grid.
void bwd_segment_order(BwdArgs& a, bool latest_first) {
  const int m = a.nblk * a.nseg;
  for (int i = 0; i < m; ++i) a.seg_order[i] = static_cast<signed char>(i);
  if (!a.causal) return;
  for (int i = 1; i < m; ++i)
    for (int j = i; j > 0; --j) {
      const Seg& x = a.seg[a.seg_order[j] / a.nseg][a.seg_order[j] % a.nseg];
      const Seg& y = a.seg[a.seg_order[j - 1] / a.nseg][a.seg_order[j - 1] % a.nseg];
      if (latest_first ? x.pos > y.pos : x.pos < y.pos) {
        const signed char t = a.seg_order[j];
        a.seg_order[j] = a.seg_order[j - 1];
        a.seg_order[j - 1] = t;
      }
    }
}

template <int D>
ra_status launch_bwd_d(const BwdArgs& adq, const BwdArgs& adkv, const CUtensorMap& mq, const CUtensorMap& mk,
                       const CUtensorMap& mv, const CUtensorMap& mdo, cudaStream_t st) {
  constexpr int kQBytes = BwdQSmem<D>::kBytes, kKVBytes = BwdKVSmem<D>::kBytes;
  static int attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kQBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kKVBytes) !=
            cudaSuccess)
      return RA_ERR_CUDA;
    attr_set[dev] = 1;
  }
  const long long tiles = static_cast<long long>(adq.B) * adq.nblk * adq.nseg * adq.seg_tiles;
  const long long gkv = tiles * adkv.Hkv, gq = tiles * adq.Hq;
  if (gq > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  bwd_dkv_kernel<D><<<static_cast<unsigned>(gkv), kBwdThreads, kKVBytes, st>>>(mq, mk, mv, mdo, adkv);
  ra_status s = cuda_status(cudaGetLastError());
  if (s != RA_OK) return s;
  bwd_dq_kernel<D><<<static_cast<unsigned>(gq), kBwdThreads, kQBytes, st>>>(mq, mk, mv, mdo, adq);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

const char* ra_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID_ARG: return "RA_ERR_INVALID_ARG";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED";
    case RA_ERR_WORKSPACE: return "RA_ERR_WORKSPACE";
    case RA_ERR_CUDA: return "RA_ERR_CUDA";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT";
    case RA_ERR_DEVICE_BOUNDS: return "RA_ERR_DEVICE_BOUNDS";
  }
  return "RA_ERR_UNKNOWN";
}

const char* ra_version(void) { return "ra_b200 0.1 (sm_100a)"; }

int ra_debug_build(void) { return kDebugBounds ? 1 : 0; }

ra_status ra_set_cta_timeline(uint64_t* records, int64_t max_ctas, ra_timeline_kernel kernel) {
  if (kernel != RA_TIMELINE_ATTN_FWD && kernel != RA_TIMELINE_BWD_DKV && kernel != RA_TIMELINE_BWD_DQ)
    return RA_ERR_INVALID_ARG;
  if (records == nullptr) {
    g_timeline = TimelineState{nullptr, 0, 0};
    return RA_OK;
  }
  if (max_ctas < 1 || max_ctas > (int64_t{1} << 24) || (reinterpret_cast<uintptr_t>(records) & 7u) != 0)
    return RA_ERR_INVALID_ARG;
  g_timeline = TimelineState{reinterpret_cast<unsigned long long*>(records), static_cast<int>(max_ctas),
                             static_cast<int>(kernel)};
  return RA_OK;
}

ra_status ra_get_bounds_record(int64_t record[3]) {
  if (!record) return RA_ERR_INVALID_ARG;
  record[0] = record[1] = record[2] = 0;
#ifdef RA_DEBUG_BOUNDS
  long long r[3];
  if (cudaMemcpyFromSymbol(r, g_bounds_record, sizeof(r)) != cudaSuccess) return RA_ERR_CUDA;
  const long long z[3] = {0, 0, 0};
  if (cudaMemcpyToSymbol(g_bounds_record, z, sizeof(z)) != cudaSuccess) return RA_ERR_CUDA;
  for (int i = 0; i < 3; ++i) record[i] = r[i];
#endif
  return RA_OK;
}

ra_status ra_get_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return RA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return RA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return RA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return RA_ERR_CUDA;
  }
  return static_cast<ra_status>(v);
}

ra_status ra_block_attn(const void* q, const void* k, const void* v, ra_dtype in_dtype, int B, int S,
                        int n_blocks, int q_block, int kv_block, int Hq, int Hkv, int D, int causal,
                        ra_partition partition, float* block_out, float* block_lse, void* stream) {
  Geom g;
  ra_status s = check_geom(B, S, n_blocks, Hq, Hkv, D, partition, &g);
  if (s != RA_OK) return s;
  if (in_dtype != RA_BF16) return in_dtype == RA_F32 ? RA_ERR_UNSUPPORTED : RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !block_out || !block_lse) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(block_out) || !aligned16(block_lse))
    return RA_ERR_INVALID_ARG;
  if (q_block < 0 || q_block >= n_blocks || kv_block < 0 || kv_block >= n_blocks) return RA_ERR_INVALID_ARG;
  g.causal = causal != 0;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, Hq, g.L, B) || !make_map(&mk, k, D, Hkv, g.L, B) || !make_map(&mv, v, D, Hkv, g.L, B))
    return RA_ERR_CUDA;
  AttnArgs a = base_args(g);
  a.nq = 1;
  a.nkv = 1;
  block_segments(g, q_block, true, a.qseg[0]);
  block_segments(g, kv_block, true, a.kvseg[kv_block]);
  a.kv_list[0][0] = static_cast<signed char>(kv_block);
  order_segments(a);
  choose_tiling(g, a, RA_TILING_AUTO);
  a.mode = kModePartial;
  a.acc_out = block_out;
  a.acc_lse = block_lse;
  a.acc_brows = g.L;
  a.q_rows = a.kv_rows = g.L;  // the maps cover block-local tensors
  return launch_attn(D, a, mq, mk, mv, static_cast<cudaStream_t>(stream));
}

ra_status ra_block_attn_merge(const void* q, const void* k, const void* v, ra_dtype in_dtype, int B, int S,
                              int n_blocks, int q_block, int kv_block, int Hq, int Hkv, int D, int causal,
                              ra_partition partition, float* out, float* lse, void* stream) {
  Geom g;
  ra_status s = check_geom(B, S, n_blocks, Hq, Hkv, D, partition, &g);
  if (s != RA_OK) return s;
  if (in_dtype != RA_BF16) return in_dtype == RA_F32 ? RA_ERR_UNSUPPORTED : RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID_ARG;
  if (q_block < 0 || q_block >= n_blocks || kv_block < 0 || kv_block >= n_blocks) return RA_ERR_INVALID_ARG;
  g.causal = causal != 0;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, Hq, g.L, B) || !make_map(&mk, k, D, Hkv, g.L, B) || !make_map(&mv, v, D, Hkv, g.L, B))
    return RA_ERR_CUDA;
  AttnArgs a = base_args(g);
  a.nq = 1;
  a.nkv = 1;
  block_segments(g, q_block, true, a.qseg[0]);
  block_segments(g, kv_block, true, a.kvseg[kv_block]);
  a.kv_list[0][0] = static_cast<signed char>(kv_block);
  order_segments(a);
  choose_tiling(g, a, RA_TILING_AUTO);
  // the epilogue folds this pair's partial into the running rows (merge rule)
  a.mode = kModeMerge;
  a.acc_out = out;
  a.acc_lse = lse;
  a.acc_brows = g.L;
  a.q_rows = a.kv_rows = g.L;  // the maps cover block-local tensors
  return launch_attn(D, a, mq, mk, mv, static_cast<cudaStream_t>(stream));
}

ra_status ra_merge_partial(float* out, float* lse, const float* block_out, const float* block_lse, int64_t rows,
                           int D, void* stream) {
  if (rows < 0 || D <= 0) return RA_ERR_INVALID_ARG;
  if (D % 4 != 0 || D > 128 || 32 % (D / 4) != 0) return RA_ERR_UNSUPPORTED;
  if (rows == 0) return RA_OK;
  if (!out || !lse || !block_out || !block_lse) return RA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(block_out) || (reinterpret_cast<uintptr_t>(lse) & 3) ||
      (reinterpret_cast<uintptr_t>(block_lse) & 3))
    return RA_ERR_INVALID_ARG;
  return launch_merge(out, lse, block_out, block_lse, rows, D, static_cast<cudaStream_t>(stream));
}

ra_status ra_merge_partials(const float* const* outs, const float* const* lses, int k, float* out, float* lse,
                            int64_t rows, int D, void* stream) {
  if (rows < 0 || D <= 0 || k < 1 || !outs || !lses) return RA_ERR_INVALID_ARG;
  if (k > kMaxMergeInputs) return RA_ERR_UNSUPPORTED;
  if (D % 4 != 0 || D > 128 || 32 % (D / 4) != 0) return RA_ERR_UNSUPPORTED;
  if (rows == 0) return RA_OK;
  if (!out || !lse || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3)) return RA_ERR_INVALID_ARG;
  MergeList ml;
  memset(&ml, 0, sizeof(ml));
  for (int j = 0; j < k; ++j) {
    if (!outs[j] || !lses[j] || !aligned16(outs[j]) || (reinterpret_cast<uintptr_t>(lses[j]) & 3))
      return RA_ERR_INVALID_ARG;
    ml.outs[j] = outs[j];
    ml.lses[j] = lses[j];
  }
  return launch_merge_partials(ml, k, out, lse, rows, D, static_cast<cudaStream_t>(stream));
}

ra_status ra_zigzag_permute(const void* src, void* dst, int B, int S, int H, int D, int elem_bytes, int n_blocks,
                            int inverse, void* stream) {
  if (!src || !dst || B < 1 || S < 1 || H < 1 || D < 1 || n_blocks < 1) return RA_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return RA_ERR_INVALID_ARG;
  if (S % (2 * n_blocks) != 0) return RA_ERR_INVALID_ARG;
  if (inverse != 0 && inverse != 1) return RA_ERR_INVALID_ARG;
  if (src == dst) return RA_ERR_INVALID_ARG;
  const long long row_bytes = static_cast<long long>(H) * D * elem_bytes;
  const char* s0 = static_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  const long long tot = static_cast<long long>(B) * S * row_bytes;
  if (s0 < d0 + tot && d0 < s0 + tot) return RA_ERR_INVALID_ARG;  // overlap
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & (elem_bytes - 1))
    return RA_ERR_INVALID_ARG;
  PermGeom pg;
  pg.S = S;
  pg.n = n_blocks;
  pg.L = S / n_blocks;
  pg.c = S / (2 * n_blocks);
  pg.zigzag = 1;
  return launch_permute_bytes(src, dst, B, pg, row_bytes, inverse, static_cast<cudaStream_t>(stream));
}

size_t ra_ring_attention_workspace(int B, int S, int Hq, int D, int n_blocks, int gqa_groups, ra_partition partition,
                                   ra_dtype in_dtype, ra_dtype out_dtype, const ra_options* opts) {
  if (gqa_groups < 1 || Hq % gqa_groups != 0) return static_cast<size_t>(-1);
  Geom g;
  if (check_geom(B, S, n_blocks, Hq, Hq / gqa_groups, D, partition, &g) != RA_OK) return static_cast<size_t>(-1);
  if (in_dtype != RA_F32 && in_dtype != RA_BF16) return static_cast<size_t>(-1);
  if (out_dtype != RA_F32 && out_dtype != RA_BF16) return static_cast<size_t>(-1);
  if (!valid_opts(opts)) return static_cast<size_t>(-1);
  return make_plan(g, in_dtype, out_dtype, opts).total;
}

ra_status ra_ring_attention(const void* q, const void* k, const void* v, ra_dtype in_dtype, int B, int S, int Hq,
                            int D, int n_blocks, int causal, ra_partition partition, int gqa_groups, void* out,
                            ra_dtype out_dtype, float* lse, void* workspace, size_t workspace_bytes,
                            const ra_options* opts, void* stream) {
  if (gqa_groups < 1 || Hq < 1 || Hq % gqa_groups != 0) return RA_ERR_INVALID_ARG;
  Geom g;
  ra_status s = check_geom(B, S, n_blocks, Hq, Hq / gqa_groups, D, partition, &g);
  if (s != RA_OK) return s;
  g.causal = causal != 0;
  if (in_dtype != RA_F32 && in_dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (out_dtype != RA_F32 && out_dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (!valid_opts(opts)) return RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RA_ERR_INVALID_ARG;
  const Plan p = make_plan(g, in_dtype, out_dtype, opts);
  if (p.total > 0) {
    if (!workspace || workspace_bytes < p.total) return RA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return RA_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const ra_order order = opts ? opts->order : RA_ORDER_RING;
  PermGeom ident;
  memset(&ident, 0, sizeof(ident));
  ident.S = S;
  ident.L = g.L;
  ident.n = g.n;

  // fp32 inputs are rounded to bf16 (nearest even) once, in original order
  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  if (p.cast_inputs) {
    struct { const void* src; size_t off; int H; } mv[3] = {{q, p.q, g.Hq}, {k, p.k, g.Hkv}, {v, p.v, g.Hkv}};
    for (auto& m : mv) {
      const long long row_elems = static_cast<long long>(m.H) * D;
      const long long rows = static_cast<long long>(B) * S;
      permute_cast_kernel<float, __nv_bfloat16><<<grid_for(rows * row_elems / 8, 256), 256, 0, st>>>(
          static_cast<const float*>(m.src), reinterpret_cast<__nv_bfloat16*>(ws + m.off), B, ident, row_elems, 0);
      s = cuda_status(cudaGetLastError());
      if (s != RA_OK) return s;
    }
    qb = ws + p.q;
    kb = ws + p.k;
    vb = ws + p.v;
  }

  // a2: the partition, as TMA coordinates into the tensors in original order
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qb, D, g.Hq, S, B) || !make_map(&mk, kb, D, g.Hkv, S, B) || !make_map(&mv, vb, D, g.Hkv, S, B))
    return RA_ERR_CUDA;

  // a7: the order in which each query block meets the KV blocks
  int kv_order[kMaxBlocks][kMaxBlocks];
  for (int r = 0; r < g.n; ++r)
    for (int t = 0; t < g.n; ++t)
      kv_order[r][t] = order == RA_ORDER_RING ? ((r - t) % g.n + g.n) % g.n : (r + t) % g.n;

  AttnArgs a = base_args(g);
  a.nq = g.n;
  for (int r = 0; r < g.n; ++r) {
    block_segments(g, r, false, a.qseg[r]);
    block_segments(g, r, false, a.kvseg[r]);
  }
  order_segments(a);
  choose_tiling(g, a, opts ? opts->tiling : RA_TILING_AUTO);
  a.fault_inject = opts ? opts->fault_inject : 0;
  a.q_rows = a.kv_rows = S;  // the maps cover the tensors in original order

  if (p.sched == RA_SCHED_PERSISTENT) {
    // a3-a6 in one launch: the running state is carried across block boundaries
    a.nkv = g.n;
    for (int r = 0; r < g.n; ++r)
      for (int t = 0; t < g.n; ++t) a.kv_list[r][t] = static_cast<signed char>(kv_order[r][t]);
    a.mode = kModeFinal;
    a.out = out;
    a.lse = lse;
    a.out_bf16 = out_dtype == RA_BF16;
    if (opts && opts->attn_event_begin) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_begin), st);
    s = launch_attn(D, a, mq, mk, mv, st);
    if (s == RA_OK && opts && opts->attn_event_end) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_end), st);
    return s;
  }

  // unfused / epilogue-fused: one launch per ring step over all n pairs of
  // the step; the running (out, lse) is kept in fp32, in original order
  float* acc_out = p.acc_in_ws ? reinterpret_cast<float*>(ws + p.acc_out) : static_cast<float*>(out);
  float* acc_lse = lse;
  const long long rows = static_cast<long long>(B) * S * g.Hq;
  a.nkv = 1;
  a.acc_brows = S;
  if (opts && opts->attn_event_begin) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_begin), st);
  for (int step = 0; step < g.n; ++step) {
    for (int r = 0; r < g.n; ++r) a.kv_list[r][0] = static_cast<signed char>(kv_order[r][step]);
    if (step == 0) {
      a.mode = kModePartial;
      a.acc_out = acc_out;
      a.acc_lse = acc_lse;
    } else if (p.sched == RA_SCHED_EPILOGUE_FUSED) {
      a.mode = kModeMerge;
      a.acc_out = acc_out;
      a.acc_lse = acc_lse;
    } else {
      a.mode = kModePartial;
      a.acc_out = reinterpret_cast<float*>(ws + p.part_out);
      a.acc_lse = reinterpret_cast<float*>(ws + p.part_lse);
    }
    s = launch_attn(D, a, mq, mk, mv, st);
    if (s != RA_OK) return s;
    if (step > 0 && p.sched == RA_SCHED_UNFUSED) {
      s = launch_merge(acc_out, acc_lse, a.acc_out, a.acc_lse, rows, D, st);
      if (s != RA_OK) return s;
    }
  }
  if (opts && opts->attn_event_end) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_end), st);
  // a8: the cast of out (fp32 -> bf16, nearest even); lse is already in place
  if (p.acc_in_ws) {
    const long long row_elems = static_cast<long long>(g.Hq) * D;
    permute_cast_kernel<float, __nv_bfloat16><<<grid_for(static_cast<long long>(B) * S * row_elems / 8, 256), 256, 0, st>>>(
        acc_out, static_cast<__nv_bfloat16*>(out), B, ident, row_elems, 0);
    s = cuda_status(cudaGetLastError());
  }
  return s;
}

size_t ra_decode_workspace(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_splits) {
  if (check_decode(B, Tq, Skv, Hq, Hkv, D, n_splits) != RA_OK) return static_cast<size_t>(-1);
  return decode_plan(B, Tq, Skv, Hq, Hkv, D, n_splits).total;
}

int ra_decode_splits(int B, int Tq, int Skv, int Hq, int Hkv, int D, int n_splits) {
  if (check_decode(B, Tq, Skv, Hq, Hkv, D, n_splits) != RA_OK) return -1;
  return decode_plan(B, Tq, Skv, Hq, Hkv, D, n_splits).n;
}

ra_status ra_decode_attention(const void* q, const void* k, const void* v, ra_dtype in_dtype, int B, int Tq, int Skv,
                              int Hq, int Hkv, int D, int causal, int n_splits, void* out, ra_dtype out_dtype,
                              float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  ra_status s = check_decode(B, Tq, Skv, Hq, Hkv, D, n_splits);
  if (s != RA_OK) return s;
  if (in_dtype != RA_BF16) return in_dtype == RA_F32 ? RA_ERR_UNSUPPORTED : RA_ERR_INVALID_ARG;
  if (out_dtype != RA_F32 && out_dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse) & 3))
    return RA_ERR_INVALID_ARG;
  const DecodePlan p = decode_plan(B, Tq, Skv, Hq, Hkv, D, n_splits);
  if (!workspace || workspace_bytes < p.total) return RA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return RA_ERR_INVALID_ARG;
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, D, Hkv, Skv, B, kDecKeys) || !make_map(&mv, v, D, Hkv, Skv, B, kDecKeys)) return RA_ERR_CUDA;
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B;
  a.Tq = Tq;
  a.Skv = Skv;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.groups = Hq / Hkv;
  a.causal = causal != 0;
  a.rows = a.groups * Tq;
  a.chunk = p.chunk;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.part_out = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.part_out);
  a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + p.part_lse);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch_decode_d<128>(a, p, mk, mv, out, out_dtype, lse, st)
                  : launch_decode_d<64>(a, p, mk, mv, out, out_dtype, lse, st);
}

size_t ra_ring_attention_backward_workspace(int B, int S, int Hq, int D, int n_blocks, int gqa_groups,
                                            ra_partition partition, ra_dtype in_dtype) {
  if (gqa_groups < 1 || Hq % gqa_groups != 0) return static_cast<size_t>(-1);
  Geom g;
  if (check_geom(B, S, n_blocks, Hq, Hq / gqa_groups, D, partition, &g) != RA_OK) return static_cast<size_t>(-1);
  if (in_dtype != RA_F32 && in_dtype != RA_BF16) return static_cast<size_t>(-1);
  return bwd_plan(g, in_dtype).total;
}

ra_status ra_ring_attention_backward(const void* q, const void* k, const void* v, ra_dtype in_dtype,
                                     const void* out, ra_dtype out_dtype, const float* lse, const void* dout,
                                     int B, int S, int Hq, int D, int n_blocks, int causal, ra_partition partition,
                                     int gqa_groups, float* dq, float* dk, float* dv, void* workspace,
                                     size_t workspace_bytes, const ra_options* opts, void* stream) {
  if (gqa_groups < 1 || Hq < 1 || Hq % gqa_groups != 0) return RA_ERR_INVALID_ARG;
  Geom g;
  ra_status s = check_geom(B, S, n_blocks, Hq, Hq / gqa_groups, D, partition, &g);
  if (s != RA_OK) return s;
  g.causal = causal != 0;
  if (in_dtype != RA_F32 && in_dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (out_dtype != RA_F32 && out_dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (!valid_opts(opts)) return RA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return RA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return RA_ERR_INVALID_ARG;
  const BwdPlan p = bwd_plan(g, in_dtype);
  if (!workspace || workspace_bytes < p.total) return RA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return RA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const long long rows = static_cast<long long>(B) * S;

  // fp32 inputs are rounded to bf16 (nearest even) once, as in the forward
  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  const void* dob = dout;
  if (p.cast_inputs) {
    PermGeom ident;
    memset(&ident, 0, sizeof(ident));
    ident.S = S;
    ident.L = g.L;
    ident.n = g.n;
    struct { const void* src; size_t off; int H; } mv[4] = {
        {q, p.q, g.Hq}, {k, p.k, g.Hkv}, {v, p.v, g.Hkv}, {dout, p.dout, g.Hq}};
    for (auto& m : mv) {
      const long long row_elems = static_cast<long long>(m.H) * D;
      permute_cast_kernel<float, __nv_bfloat16><<<grid_for(rows * row_elems / 8, 256), 256, 0, st>>>(
          static_cast<const float*>(m.src), reinterpret_cast<__nv_bfloat16*>(ws + m.off), B, ident, row_elems, 0);
      s = cuda_status(cudaGetLastError());
      if (s != RA_OK) return s;
    }
    qb = ws + p.q;
    kb = ws + p.k;
    vb = ws + p.v;
    dob = ws + p.dout;
  }

  // Delta = rowsum(dO * O) and lse * log2(e), per (batch, head) over positions
  float* delta = reinterpret_cast<float*>(ws + p.delta);
  float* lse2 = reinterpret_cast<float*>(ws + p.lse2);
  const long long prep_threads = rows * Hq * (D / 4);
  if (out_dtype == RA_F32)
    bwd_prep_kernel<float><<<grid_for(prep_threads, 256), 256, 0, st>>>(
        static_cast<const float*>(out), static_cast<const __nv_bfloat16*>(dob), lse, B, S, Hq, D, delta, lse2);
  else
    bwd_prep_kernel<__nv_bfloat16><<<grid_for(prep_threads, 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dob), lse, B, S, Hq, D, delta,
        lse2);
  s = cuda_status(cudaGetLastError());
  if (s != RA_OK) return s;

  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, qb, D, g.Hq, S, B) || !make_map(&mk, kb, D, g.Hkv, S, B) ||
      !make_map(&mv, vb, D, g.Hkv, S, B) || !make_map(&mdo, dob, D, g.Hq, S, B))
    return RA_ERR_CUDA;

  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B;
  a.S = S;
  a.Hq = Hq;
  a.Hkv = g.Hkv;
  a.groups = g.groups;
  a.causal = g.causal;
  a.nblk = g.n;
  a.nseg = g.zigzag ? 2 : 1;
  a.seg_tiles = (seg_len_of(g) + kBM - 1) / kBM;
  a.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(D)));
  a.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(D)));
  a.lse2 = lse2;
  a.delta = delta;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  for (int r = 0; r < g.n; ++r) block_segments(g, r, false, a.seg[r]);
  // dQ: query block r meets the KV blocks in the schedule's order (as in the
  // forward); dK/dV: KV block j meets the query blocks that meet it there
  const ra_order order = opts ? opts->order : RA_ORDER_RING;
  BwdArgs adq = a, adkv = a;
  adq.timeline = timeline_for(RA_TIMELINE_BWD_DQ);
  adkv.timeline = timeline_for(RA_TIMELINE_BWD_DKV);
  for (int r = 0; r < g.n; ++r)
    for (int t = 0; t < g.n; ++t) {
      const int fwd = order == RA_ORDER_RING ? r - t : r + t;
      const int bwd = order == RA_ORDER_RING ? r + t : r - t;
      adq.order[r][t] = static_cast<signed char>(((fwd % g.n) + g.n) % g.n);
      adkv.order[r][t] = static_cast<signed char>(((bwd % g.n) + g.n) % g.n);
    }
  bwd_segment_order(adq, true);
  bwd_segment_order(adkv, false);
  if (opts && opts->attn_event_begin) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_begin), st);
  s = D == 128 ? launch_bwd_d<128>(adq, adkv, mq, mk, mv, mdo, st) : launch_bwd_d<64>(adq, adkv, mq, mk, mv, mdo, st);
  if (s == RA_OK && opts && opts->attn_event_end) cudaEventRecord(static_cast<cudaEvent_t>(opts->attn_event_end), st);
  return s;
}

}  // extern "C"
