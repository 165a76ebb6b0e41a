// Launch interface of the E4M3 quantizer (library-internal).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

namespace sa {

struct QuantParams {
  const __nv_bfloat16* x;  // [n_tensors][n_elems]
  uint8_t* codes;          // [n_tensors][n_elems]
  float* inv;              // [n_tensors]; holds each tensor's amax bits until the last pass
  long long n_elems;       // a multiple of 8
  int n_tensors;
};

cudaError_t launch_quant_e4m3(const QuantParams& p, cudaStream_t st);

}  // namespace sa
