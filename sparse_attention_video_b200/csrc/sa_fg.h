// Launch interface of the fine-grained M x 1 key-slice path (library-internal).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                             const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                             const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

enum { FG_MODE_HIST = 0, FG_MODE_BITS = 1 };

struct FgQbarParams {
  const __nv_bfloat16* q;
  __nv_bfloat16* qsplit;   // [3][BH][G_pad][d]: hi, mid, lo terms of q_avg
  int BH, N, d, group, G, G_pad;
};

struct FgScoreParams {
  uint32_t* bits;          // [BH][G][WN]
  uint32_t* hist;          // [BH][4096]
  const uint32_t* sel;     // [BH][4]: prefix key, rank left, R
  uint32_t* status;
  int mode;                // FG_MODE_*
  int bin_shift;           // HIST: bin = (key >> bin_shift) & bin_mask
  uint32_t bin_mask;
  uint32_t match_mask;     // HIST: count only keys with (key & match_mask) == prefix
  int BH, N, G, WN;
};

struct FgListParams {
  const uint32_t* bits;    // [BH][G][WN]
  uint32_t* counts;        // [BH][P]
  uint32_t* offsets;       // [BH][P + 1]
  uint32_t* list;          // [BH][cap]: key | in-first-group << 30 | in-second-group << 31
  uint32_t* status;
  long long cap_per_head;
  int BH, P, G, WN, groups_per_tile;
};

struct FgBuildParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __nv_bfloat16* qsplit;
  uint32_t* hist;
  uint32_t* sel;
  uint32_t* bits;
  float* tau;
  uint32_t* status;
  FgListParams lists;
  int BH, N, d, group, G, WN;
  float keep_fraction;
};

int fg_g_pad(int G);
size_t fg_qsplit_bytes(int BH, int G, int d);
size_t fg_hist_bytes(int BH);
size_t fg_sel_bytes(int BH);
long long fg_list_cap_per_head(int G, int N, float keep_fraction);
cudaError_t launch_fg_build(const FgBuildParams& p, EncodeFn enc, cudaStream_t st);
cudaError_t launch_fg_lists(const FgListParams& p, cudaStream_t st);

}  // namespace sa
