// Launch interface of the fine-grained M x 1 key-slice path (library-internal).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

struct FgBuildParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* qbar;             // [BH][G][d] group-mean queries
  uint32_t* hist;          // radix-select histograms
  uint32_t* sel;           // radix-select state per head
  uint32_t* bits;          // [BH][G][WN] kept slices
  float* tau;              // [BH] threshold
  uint32_t* status;
  int BH, N, d, group, G, WN;
  float keep_fraction;
};

struct FgAttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const uint32_t* bits;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* status;
  int BH, N, d, group, G, WN;
  float scale_log2;
};

size_t fg_qbar_bytes(int BH, int G, int d);
size_t fg_hist_bytes(int BH);
size_t fg_sel_bytes(int BH);
cudaError_t launch_fg_build(const FgBuildParams& p, cudaStream_t st);
cudaError_t launch_fg_attn(const FgAttnParams& p, cudaStream_t st);

}  // namespace sa
