// noalloc.cu - ra_ring_attention_noalloc: the whole method with its scratch
// in a fixed device array that is part of this library, so the call needs no
// workspace from the caller and allocates nothing.
//
// Some callers cannot hand over a workspace or call cudaMalloc: code that runs
// after its host framework has reserved the device memory for its own pool
// (a fresh cudaMalloc there fails or fragments the pool), and latency-bound
// callers that cannot accept the implicit device synchronisation of
// cudaMalloc / cudaFree.  For them the scratch lives in g_noalloc_scratch
// below: every GPU that loads this library holds those bytes until the
// process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ra.h"

namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;  // 64 MiB

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct CtxFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();  // a missing entry point leaves no error behind
  });
  return f;
}

// Process-unique ID of the context current on this thread (0 if none is, or
// the driver cannot say).  A context that is destroyed and created again (after
// cudaDeviceReset, or when the primary context is released and retained
// anew) gets a new ID, even where its handle value repeats.
unsigned long long current_ctx_id() {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  void* addr;                 // device address of g_noalloc_scratch in that context
  unsigned long long ctx_id;  // the context it was looked up in
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in: a kernel given it would fault or
// read the wrong memory, so the address comes from cudaGetSymbolAddress with
// the device current.  The lookup runs once per device and context: when the
// context has changed since (a reset re-loads this library's module, possibly
// at another address), the address is looked up again.
ra_status scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return RA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = current_ctx_id();
  ScratchSlot& slot = g_scratch[dev];
  if (slot.addr == nullptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // leave no error for the next library call to mistake for its own
      slot.addr = nullptr;
      return RA_ERR_CUDA;
    }
    if (id == 0) id = current_ctx_id();  // the lookup made the device's context current
    slot.addr = p;
    slot.ctx_id = id;
    if (id == 0) {  // no context ID to key on: use the address for this call only
      slot.addr = nullptr;
      *addr = p;
      return RA_OK;
    }
  }
  *addr = slot.addr;
  return RA_OK;
}

}  // namespace

extern "C" {

size_t ra_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

ra_status ra_ring_attention_noalloc(const void* q, const void* k, const void* v, ra_dtype in_dtype, int B, int S,
                                    int Hq, int D, int n_blocks, int causal, ra_partition partition,
                                    int gqa_groups, void* out, ra_dtype out_dtype, float* lse,
                                    const ra_options* opts, void* stream) {
  const size_t need = ra_ring_attention_workspace(B, S, Hq, D, n_blocks, gqa_groups, partition, in_dtype,
                                                  out_dtype, opts);
  if (need == static_cast<size_t>(-1)) {
    // Invalid arguments: ra_ring_attention validates the same ones before it
    // touches the workspace or launches anything, so it returns the same
    // status code (RA_ERR_INVALID_ARG or RA_ERR_UNSUPPORTED) here.
    return ra_ring_attention(q, k, v, in_dtype, B, S, Hq, D, n_blocks, causal, partition, gqa_groups, out,
                             out_dtype, lse, nullptr, 0, opts, stream);
  }
  if (need > kNoAllocScratchBytes) return RA_ERR_WORKSPACE;  // does not fit in the fixed scratch
  void* ws = nullptr;
  if (need > 0) {
    const ra_status s = scratch_address(&ws);
    if (s != RA_OK) return s;
  }
  return ra_ring_attention(q, k, v, in_dtype, B, S, Hq, D, n_blocks, causal, partition, gqa_groups, out,
                           out_dtype, lse, ws, need, opts, stream);
}

}  // extern "C"
