// sta_noalloc.cu -- sta_backward_noalloc: the backward pass with its scratch
// in a fixed, library-owned device array instead of a caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward pass: every byte of the device may already belong to another
// allocator (a framework's caching allocator that has reserved the pool), or
// the call sits on a path where an allocation is not allowed (latency-bound
// serving loops, code that must not change the memory footprint once it is
// set up).  Such a caller can still pass its inputs and outputs; the
// temporaries of the backward pass (the kernel status word, LSE * log2 e and
// D = rowsum(dO * O), plus tile-major copies of Q, K, V and dO when the tiles
// are not readable in place) then go to the array below.
//
// The array has a fixed size (kNoallocScratchBytes).  Every GPU that loads
// this library holds it in device memory until the process exits.  All calls
// share it and it keeps whatever the last call left there: everything a call
// reads from it is written earlier in the same call (the status word is
// cleared by STA_CALL_CHECK, the only reader of it).  Calls whose execution
// overlaps on the GPU (different streams, or different host threads on one
// device) race on the array and give wrong results; the caller must order
// them.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sta.h"
#include "sta_kernels.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

// File-scope device array.  In host code `g_noalloc_scratch` is only a host-side
// stand-in for the symbol, never a device address: the address kernels may use
// comes from cudaGetSymbolAddress, once per device, with that device current.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// The device address of the array on the current device (looked up once per
// device).  Called after the device check, so the current device is the
// plan's.
sta_status scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return STA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return STA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return STA_OK;
}

}  // namespace

extern "C" {

sta_status sta_backward_noalloc(sta_plan_t plan, const void *q, const void *k, const void *v, const void *o,
                                const float *lse, const void *dout, void *dq, void *dk, void *dv, void *stream,
                                uint32_t flags) {
  if (!plan) return STA_ERR_INVALID_ARG;
  size_t need = 0;
  sta_status st = sta_plan_workspace_size(plan, nullptr, &need);
  if (st != STA_OK) return st;
  if (need > kNoallocScratchBytes) return STA_ERR_WORKSPACE;
  // every other check of sta_backward, before the array is looked up
  const void *tensors[9] = {q, k, v, o, lse, dout, dq, dk, dv};
  st = sta::check_backward_call(plan, tensors, flags);
  if (st != STA_OK) return st;
  void *scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != STA_OK) return st;
  return sta_backward(plan, q, k, v, o, lse, dout, dq, dk, dv, scratch, kNoallocScratchBytes, stream, flags);
}

}  // extern "C"
