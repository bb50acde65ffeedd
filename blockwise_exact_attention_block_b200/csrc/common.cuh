// common.cuh - device helpers shared by the kernels of libra_b200.so:
// the device status word, bounded mbarrier waits, TMA tile loads and the
// tcgen05 (5th-generation tensor core / tensor memory) instructions, all as
// inline PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ra.h"

namespace ra {

// Device status word: 0 = fine; otherwise the first ra_status a kernel hit.
__device__ int g_status;

__device__ __forceinline__ void set_status(int s) { atomicCAS(&g_status, 0, s); }

// Index checks of the checked build (compiled with -DRA_DEBUG_BOUNDS): a
// failed check records RA_ERR_DEVICE_BOUNDS in the status word (the first
// error wins) with the source line, the index and its limit, and the caller
// skips the access.  The release build compiles every check to `true`.
#ifdef RA_DEBUG_BOUNDS
__device__ long long g_bounds_record[3];  // line, index, limit of the first failed check
__device__ __noinline__ bool bounds_failed(long long idx, long long limit, int line) {
  if (atomicCAS(&g_status, 0, RA_ERR_DEVICE_BOUNDS) == 0) {
    g_bounds_record[0] = line;
    g_bounds_record[1] = idx;
    g_bounds_record[2] = limit;
  }
  return false;
}
#define RA_IN_BOUNDS(idx, limit)                                                                          \
  ((static_cast<long long>(idx) >= 0 && static_cast<long long>(idx) < static_cast<long long>(limit)) \
       ? true                                                                                             \
       : ::ra::bounds_failed(static_cast<long long>(idx), static_cast<long long>(limit), __LINE__))
constexpr bool kDebugBounds = true;
#else
#define RA_IN_BOUNDS(idx, limit) true
constexpr bool kDebugBounds = false;
#endif

// Per-CTA timeline (tracing, off unless the host sets it for one kernel): the
// CTA's thread 0 writes four 64-bit words at rec[4 * blockIdx.x] for the CTAs
// below max_ctas: start and end in ns of the global timer, the SM id (low 32
// bits) with the CTA's work units (the tiles of its walk, high 32 bits), and
// the SM clock cycles from start to end (the fourth word holds the start
// cycle count until the end stamp replaces it by the difference).
struct CtaTimeline {
  unsigned long long* rec;
  int max_ctas;
};

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool timeline_on(const CtaTimeline& t) {
  return t.rec != nullptr && threadIdx.x == 0 && static_cast<int>(blockIdx.x) < t.max_ctas;
}

__device__ __forceinline__ void timeline_begin(const CtaTimeline& t) {
  if (timeline_on(t)) {
    t.rec[4ull * blockIdx.x] = global_ns();
    t.rec[4ull * blockIdx.x + 3] = static_cast<unsigned long long>(clock64());
  }
}

__device__ __forceinline__ void timeline_work(const CtaTimeline& t, int units) {
  if (timeline_on(t)) {
    unsigned int sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    t.rec[4ull * blockIdx.x + 2] = sm | (static_cast<unsigned long long>(static_cast<unsigned int>(units)) << 32);
  }
}

__device__ __forceinline__ void timeline_end(const CtaTimeline& t) {
  if (timeline_on(t)) {
    unsigned long long* r = t.rec + 4ull * blockIdx.x;
    r[3] = static_cast<unsigned long long>(clock64()) - r[3];
    r[1] = global_ns();
  }
}

// A bounded wait gives up after this many SM clock cycles (about one second
// at the B200's 1.9 GHz boost clock) and reports RA_ERR_TIMEOUT.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// True once any CTA has recorded a timeout: the rest of the grid then stops
// waiting at once instead of each CTA running out its own limit.
__device__ __forceinline__ bool grid_timed_out() {
  return *reinterpret_cast<volatile int*>(&g_status) == RA_ERR_TIMEOUT;
}

// Waits until the phase with the given parity has completed.  Returns false
// (and records RA_ERR_TIMEOUT, and raises *abort for the rest of the CTA) when
// the wait runs past kWaitLimitCycles, or another role of the CTA or another
// CTA has already given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort || grid_timed_out()) {
      *abort = 1;
      return false;
    }
    if (clock64() - t0 > kWaitLimitCycles) {
      set_status(RA_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Same contract as mbar_wait, but polls without letting the thread be
// suspended, for the single MMA-issuing thread whose reaction time is on the
// critical path.
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test_wait(bar, parity)) return true;
    if ((it & 255) == 0) {
      if (*abort || grid_timed_out()) {
        *abort = 1;
        return false;
      }
      if (clock64() - t0 > kWaitLimitCycles) {
        set_status(RA_ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 4-D tiled load of one box into shared memory; completion is signalled on
// `bar` as transaction bytes.  No multicast.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// L2 prefetch of one box of a 4-D tensor map: the box's lines are brought
// into L2 ahead of a later tiled load of the same box (no shared memory, no
// completion to wait for).  The same coordinate rules as a load; no multicast.
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* m, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Barrier over the first `count` threads' warps that execute it (id 1-15;
// id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Orders this thread's earlier async-proxy (TMA / tensor core) shared-memory
// accesses before its later generic ones.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------ thread-block clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Barrier over every thread of every CTA in the cluster (all threads call it).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address, in the cluster's shared window, of the same shared-memory offset
// in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Warpgroup-wide register reallocation (all 128 threads of the warpgroup).
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// --------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Whole-warp TMEM allocation; the base address is written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16; A is K-major in tensor memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same two products with each shared-memory descriptor passed as its
// 32-bit halves.  The low half holds the start address (addr >> 4) in its low
// 14 bits, and shared addresses stay below 2^18, so a caller can step a
// descriptor through a tile by adding (offset >> 4) to the low half alone:
// one integer add per operand and product.
__device__ __forceinline__ void mma_ss_lo(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t desc_hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(desc_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_lo(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

#define RA_S32(i) "r"(v[i])

// Stores 32 consecutive 32-bit TMEM columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      RA_S32(0), RA_S32(1), RA_S32(2), RA_S32(3), RA_S32(4), RA_S32(5), RA_S32(6), RA_S32(7),
      RA_S32(8), RA_S32(9), RA_S32(10), RA_S32(11), RA_S32(12), RA_S32(13), RA_S32(14),
      RA_S32(15), RA_S32(16), RA_S32(17), RA_S32(18), RA_S32(19), RA_S32(20), RA_S32(21),
      RA_S32(22), RA_S32(23), RA_S32(24), RA_S32(25), RA_S32(26), RA_S32(27), RA_S32(28),
      RA_S32(29), RA_S32(30), RA_S32(31)
      : "memory");
}

// Stores 16 consecutive 32-bit TMEM columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      RA_S32(0), RA_S32(1), RA_S32(2), RA_S32(3), RA_S32(4), RA_S32(5), RA_S32(6), RA_S32(7),
      RA_S32(8), RA_S32(9), RA_S32(10), RA_S32(11), RA_S32(12), RA_S32(13), RA_S32(14), RA_S32(15)
      : "memory");
}

#undef RA_S32

// Shared-memory matrix descriptor for a tile written by TMA with 128-byte
// swizzling (8 rows x 128 bytes per swizzle atom, atoms 1024 bytes apart).
//   lbo: byte distance between 64-element column groups (MN-major operands)
//   sbo: byte distance between consecutive 8-row groups
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Low half of smem_desc_sw128(saddr, lbo, 1024): the start address and the
// leading byte offset.  The high half is the same for every such descriptor
// (desc_sw128_hi): stepping a descriptor through a tile is one add of
// (offset >> 4) to its low half (see mma_ss_lo).
__device__ __forceinline__ uint32_t desc_sw128_lo(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint32_t>(smem_desc_sw128(saddr, lbo, 1024));
}
__device__ __forceinline__ uint32_t desc_sw128_hi() { return static_cast<uint32_t>(smem_desc_sw128(0, 16, 1024) >> 32); }

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
//   b_mn_major: B operand is MN-major (N contiguous) instead of K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)   // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------ packed fp32 pairs
// Blackwell executes these as one instruction on two fp32 lanes.

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace ra
