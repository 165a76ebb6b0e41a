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

// HIST: histogram level of the radix select. BITS: slice bitmask key >= tau.
// BITS_COLLECT: bitmask of the keys whose top 24 bits exceed the prefix the
// first two levels decided, plus a list of the keys that share it (the last
// 8 bits are then selected among those few by fg_fixup).
enum { FG_MODE_HIST = 0, FG_MODE_BITS = 1, FG_MODE_BITS_COLLECT = 2 };

// Candidate slots per head for the last select level; more than this (only
// with very many scores equal in their top 24 bits) falls back to the full
// third histogram pass.
constexpr uint32_t kFgCandCap = 65536;

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
  uint2* cand;             // BITS_COLLECT: [BH][kFgCandCap] (key index, group << 8 | low 8 bits)
  uint32_t* cand_count;    // [BH]
  const uint32_t* only_heads;  // if set: heads whose flag is 0 do nothing
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
  uint2* cand;             // [BH][kFgCandCap]
  uint32_t* cand_count;    // [BH]
  uint32_t* fallback;      // [BH]: 1 where the candidate list overflowed
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
size_t fg_cand_bytes(int BH);
long long fg_list_cap_per_head(int G, int N, float keep_fraction);
cudaError_t launch_fg_build(const FgBuildParams& p, EncodeFn enc, cudaStream_t st);
cudaError_t launch_fg_lists(const FgListParams& p, cudaStream_t st);

}  // namespace sa
