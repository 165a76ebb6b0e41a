// sparse_attn_build_mask_static: mask construction without any caller-side or
// library-side device allocation.
//
// Some callers cannot call cudaMalloc when they build a mask: code that runs
// inside another framework's execute/enqueue callback (inference-server
// plugins are handed a stream and must not allocate), code on a latency path
// where cudaMalloc/cudaFree may synchronize the device, and processes that
// reserve all their device memory once at start-up. For them this entry point
// takes its scratch from one file-scope __device__ array instead of the
// caller's scratch workspace. Everything else is the regular
// sparse_attn_build_mask: the same kernels, the same mask output.
//
// The array is SA_STATIC_SCRATCH_BYTES long; every GPU that loads this library
// holds it until the process exits. All calls share it, so two calls whose
// work overlaps on the GPU (different streams, no ordering) race on it; calls
// on one stream, or otherwise ordered, are safe. Each call clears the status
// word at the start of the array; every other byte a call reads it first
// writes itself.
#include <cuda_runtime.h>

#include "../../include/sparse_attn.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[SA_STATIC_SCRATCH_BYTES];

// Device address of the array in the current device's context. In host code
// the name g_static_scratch is only a host-side stand-in, never a device
// address, so the address is looked up with the device current. The lookup
// runs on every call: it allocates nothing, and a cached address would outlive
// a cudaDeviceReset or a switch to another context of the same device.
int static_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SA_ERR_CUDA;
  *out = p;
  return SA_OK;
}

}  // namespace

extern "C" int sparse_attn_build_mask_static(const sa_problem* problem, const sa_policy* policy,
                                             const void* q, const void* k, void* mask_ws,
                                             void* stream) {
  size_t mask_bytes = 0, scratch_bytes = 0;
  int e = sparse_attn_workspace_size(problem, policy, &mask_bytes, &scratch_bytes);
  if (e != SA_OK) return e;
  if (scratch_bytes > (size_t)SA_STATIC_SCRATCH_BYTES) return SA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  e = static_scratch(&scratch);
  if (e != SA_OK) return e;
  return sparse_attn_build_mask(problem, policy, q, k, mask_ws, scratch, stream);
}

extern "C" int sparse_attn_status_static(void* stream, int clear) {
  void* scratch = nullptr;
  const int e = static_scratch(&scratch);
  if (e != SA_OK) return e;
  return sparse_attn_status(scratch, stream, clear);
}
