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
// CACHED: the B operand is 128 query rows instead of q_avg terms; a slice
// (group, key) is kept when one of the group's queries gives the key a
// full-attention probability above tau (FG-Attn review, the cached strategy).
// HIST_WIN: exact count of the keys above a per-head window (sel[0] its low
// end) and a 4,096-bin histogram of the keys inside it.
enum { FG_MODE_HIST = 0, FG_MODE_BITS = 1, FG_MODE_BITS_COLLECT = 2, FG_MODE_CACHED = 3,
       FG_MODE_HIST_WIN = 4 };

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
  uint2* cand;             // BITS_COLLECT: [BH][kFgCandCap] (key index, group << cs | low cs bits)
  uint32_t* cand_count;    // [BH]
  const uint32_t* only_heads;  // if set: heads whose flag is 0 do nothing
  const float* lse;        // CACHED: [BH][N] natural-log LSE of full attention
  float ln_tau;            // CACHED: ln(tau)
  float sqrt_d;            // CACHED: sqrt(d)
  int group;               // CACHED: queries per group (64 or 128)
  int row_tiles;           // 128-row tiles of the B operand (groups, or queries for CACHED)
  int BH, N, G, WN;
  int tile_stride;         // > 1: only every tile_stride-th key tile (a sample)
  int collect_shift;       // BITS_COLLECT: low key bits left to fg_fixup (0: 8)
  int win_shift;           // HIST_WIN: log2 of the keys per bin
  uint32_t* above;         // HIST_WIN: [BH] keys above the window
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
  uint32_t* win;           // [BH][4]: above-window count, window miss, window hit, overflow
  uint32_t* bits;
  float* tau;
  uint32_t* status;
  FgListParams lists;
  int BH, N, d, group, G, WN;
  float keep_fraction;
};

// The cached rule's bitmask and union lists from Q, K and the LSE of full
// attention: a slice is kept when max over its group's queries of
// exp(q.k / sqrt(d) - lse_q) > tau.
struct FgCachedParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const float* lse;        // [BH][N]
  uint32_t* bits;          // [BH][G][WN], cleared here first
  float* tau_out;          // [BH]: tau, for inspection
  uint32_t* status;
  FgListParams lists;
  int BH, N, d, group, G, WN;
  float tau;
};

int fg_g_pad(int G);
size_t fg_qsplit_bytes(int BH, int G, int d);
size_t fg_hist_bytes(int BH);
size_t fg_sel_bytes(int BH);
size_t fg_cand_bytes(int BH);
long long fg_list_cap_per_head(int G, int N, float keep_fraction);
cudaError_t launch_fg_build(const FgBuildParams& p, EncodeFn enc, cudaStream_t st);
cudaError_t launch_fg_lists(const FgListParams& p, cudaStream_t st);
cudaError_t launch_fg_cached(const FgCachedParams& p, EncodeFn enc, cudaStream_t st);

}  // namespace sa
