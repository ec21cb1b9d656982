// Ring attention forward for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc or to ask their framework
// for a workspace: a plugin running inside a host application that owns the
// whole device-memory budget and forbids allocation while it executes, or a
// latency-critical loop in which an allocation would stall the device.  For
// them this file adds cp_ring_attn_fwd_noalloc, which runs exactly the same
// kernels as cp_ring_attn_fwd but keeps the ring steps' partial results in a
// fixed scratch array compiled into the library instead of a caller
// workspace.  The caller still passes its inputs and outputs.
//
// The array is a file-scope __device__ object: every GPU on which the library
// is used holds its CP_NOALLOC_SCRATCH_BYTES bytes until the process exits.
// In host code `g_ring_scratch` only names the object; its device address is
// looked up with cudaGetSymbolAddress once per device (on the first call made
// with that device current) and that address is what the kernels receive.
// The cached address belongs to the device's primary context: after a
// cudaDeviceReset in the same process it would be stale, so the entry point
// is not meant to be used across a reset.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "cp_attn.h"

namespace cp {
void set_error_message(const char* msg);
}

namespace {

constexpr size_t kScratchBytes = CP_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_ring_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

cp_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cp::set_error_message("cp_ring_attn_fwd_noalloc: cudaGetDevice failed");
    return CP_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    cp::set_error_message("cp_ring_attn_fwd_noalloc: device index out of range");
    return CP_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ring_scratch);
    if (e != cudaSuccess || !p) {
      cp::set_error_message("cp_ring_attn_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed");
      return CP_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CP_OK;
}

}  // namespace

extern "C" cp_status cp_ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, cp_dtype dtype, int S,
                                              int hq, int hkv, int dh, int P, cp_layout layout, cp_mask mask,
                                              const int32_t* cu_seqlens_host, const int32_t* cu_seqlens_dev,
                                              int n_docs, float softmax_scale, float* o, float* lse,
                                              void* stream) {
  size_t need = 0;
  cp_status s = cp_ring_attn_workspace_size(S, hq, hkv, dh, P, layout, mask, dtype, cu_seqlens_host, n_docs, &need);
  if (s != CP_OK) return s;
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "cp_ring_attn_fwd_noalloc: this problem needs %zu bytes of scratch but the built-in scratch holds %zu; "
             "call cp_ring_attn_fwd with a workspace instead",
             need, kScratchBytes);
    cp::set_error_message(msg);
    return CP_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != CP_OK) return s;
  // Every partial row the merge reads is written by the attention launch of
  // the same call, so nothing in the scratch has to start at zero.
  return cp_ring_attn_fwd(q, k, v, dtype, S, hq, hkv, dh, P, layout, mask, cu_seqlens_host, cu_seqlens_dev, n_docs,
                          softmax_scale, o, lse, scratch, kScratchBytes, stream);
}
