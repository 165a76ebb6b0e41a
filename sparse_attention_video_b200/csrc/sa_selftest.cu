// Self-test of the device-side failure path shared by every kernel: a bounded
// mbarrier wait that nothing completes must give up, record a timeout in the
// status word and return, leaving the context usable.
#include <cuda_runtime.h>

#include "sa_ptx.cuh"

namespace {

__global__ void wait_nothing_kernel(uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    sa::mbar_init(&bar, 1);                 // one arrival expected, none will come
    abort = 0;
    sa::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = sa::mbar_wait(&bar, 0, &abort, status, 0x7E570000u | threadIdx.x);
  if (!ok && threadIdx.x == 0) status[2] = 1u;   // this kernel observed its own timeout
}

}  // namespace

extern "C" int sparse_attn_selftest_wait_timeout(void* scratch_ws, void* stream) {
  if (!scratch_ws || (reinterpret_cast<uintptr_t>(scratch_ws) % 256) != 0) return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  wait_nothing_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(scratch_ws));
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
