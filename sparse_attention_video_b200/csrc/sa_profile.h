// Sampled-row pattern evaluation: attention of sampled query rows over all
// keys and under several sparse patterns, and the per-head choice of the
// pattern with the lowest output error. Two uses: the SVG online head
// profiler (spatial vs temporal pattern) and the STA per-head window search
// (one pattern per candidate tile window).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

constexpr int kProfileMaxPatterns = 8;

struct ProfileParams {
  const __nv_bfloat16* q;    // [BH][N][d]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int* rows;           // [BH][n_rows] sampled query tokens (original order)
  float* row_err;            // [BH][n_rows][n_pat]: sum over d of (O_pattern - O_full)^2
  float* mse;                // [BH][n_pat]: mean over rows and d
  int8_t* choice;            // [BH]: pattern with the lowest error (ties: the first)
  uint32_t* status;          // device status word (bounds flag), may be null
  int BH, N, T, H, W, d, n_rows, block, sink_blocks, frame_radius;
  int mode;                  // 0: SVG spatial, temporal; 1: STA tile windows
  int n_pat;                 // 2, or the number of candidate windows
  int tile[3];               // STA: (bt, bh, bw), bt*bh*bw == block
  int win[kProfileMaxPatterns][3];   // STA: candidate windows (odd, in tiles)
  float scale_log2;          // log2(e) / sqrt(d)
  const float* o_full;       // [BH][n_rows][d] fp32: full attention of the sampled rows
};

cudaError_t launch_profile(const ProfileParams& p, cudaStream_t stream);

// dst[bh][r] = src[bh][rows[bh][r]] for r < n_rows, zero rows up to n_pad:
// the sampled query rows as a contiguous [BH][n_pad][d] bf16 tensor.
cudaError_t launch_gather_rows(const __nv_bfloat16* src, const int* rows, int BH, int N, int d,
                               int n_rows, int n_pad, __nv_bfloat16* dst, uint32_t* status,
                               cudaStream_t stream);

}  // namespace sa
