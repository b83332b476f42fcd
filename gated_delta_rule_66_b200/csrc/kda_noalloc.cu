// kda_bwd_noalloc: the backward with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory at the time they run the
// backward: a plugin whose host framework owns every byte of device memory
// and hands it no workspace, or a serving/training loop that forbids
// allocator calls once it is running (cudaMalloc and cudaFree synchronise the
// device and can fail when another allocator has already reserved the
// memory).  For them this entry point takes its scratch (the chunk states,
// the chunk state-gradients and, with grouped heads, the fp32 dq/dk
// partials) from one statically sized __device__ array instead of a caller
// workspace.  It calls no allocating routine.
//
// The array is KDA_NOALLOC_SCRATCH_BYTES per GPU and stays resident on every
// GPU that loads the library until the process exits.  All calls share it:
// two calls whose kernels overlap on the GPU (different streams, or
// different host threads on one device) race on it and must be ordered by
// the caller.  Every byte a call reads from it is written earlier by the same
// call, so nothing needs clearing between calls.
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_kda_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_kda_scratch on the current device (looked up once per
// device; the host-side name g_kda_scratch is only a stand-in and must never
// be handed to a kernel).  The cached address belongs to the device's primary
// context: a cudaDeviceReset() destroys that context, and the address is not
// looked up again afterwards, so such a process must not call
// kda_bwd_noalloc again.
int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kda::set_cuda_error("kda_bwd_noalloc: cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices)
    return kda::set_error(KDA_ERR_ARG, "kda_bwd_noalloc: device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kda_scratch);
    if (e != cudaSuccess) return kda::set_cuda_error("kda_bwd_noalloc: cudaGetSymbolAddress", e);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" int kda_bwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* S0, const void* dO,
                               const float* dS_T, float scale, int B, int T, int H, int HV, int K,
                               int V, int dtype, void* dq, void* dk, void* dv, float* dg,
                               float* dbeta, float* dS0, void* stream) {
  const size_t need = kda_bwd_workspace_bytes(B, T, H, HV, K, V);
  if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "kda_bwd_noalloc: this problem needs %zu bytes of scratch, more than the fixed "
             "%zu-byte device array; use kda_bwd with a caller workspace",
             need, (size_t)KDA_NOALLOC_SCRATCH_BYTES);
    return kda::set_error(KDA_ERR_WORKSPACE, buf);
  }
  void* scratch = nullptr;
  if (need > 0) {
    int rc = scratch_for_current_device(&scratch);
    if (rc) return rc;
  }
  return kda_bwd(q, k, v, g, beta, S0, dO, dS_T, scale, B, T, H, HV, K, V, dtype, dq, dk, dv, dg,
                 dbeta, dS0, scratch, (size_t)KDA_NOALLOC_SCRATCH_BYTES, 0, stream);
}
