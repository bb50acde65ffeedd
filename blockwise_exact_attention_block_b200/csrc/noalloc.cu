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
#include <cuda_runtime.h>

#include <mutex>

#include "ra.h"

namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;  // 64 MiB

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in: a kernel given it would fault or
// read the wrong memory, so the address comes from cudaGetSymbolAddress, once
// per device, with that device current.
ra_status scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return RA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
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
  if (need == static_cast<size_t>(-1)) return RA_ERR_INVALID_ARG;
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
