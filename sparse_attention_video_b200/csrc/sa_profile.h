// SVG online head profiler: attention of sampled query rows under the full,
// spatial and temporal patterns, and the per-head choice by output error.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

struct ProfileParams {
  const __nv_bfloat16* q;    // [BH][N][d]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int* rows;           // [BH][n_rows] sampled query tokens (original order)
  float* row_err;            // [BH][n_rows][2]: sum over d of (O_pattern - O_full)^2
  float* mse;                // [BH][2]: spatial, temporal (mean over rows and d)
  int8_t* is_temporal;       // [BH]
  uint32_t* status;          // device status word (bounds flag), may be null
  int BH, N, T, H, W, d, n_rows, block, sink_blocks, frame_radius;
  float scale_log2;          // log2(e) / sqrt(d)
};

cudaError_t launch_profile(const ProfileParams& p, cudaStream_t stream);

}  // namespace sa
