// Internal definitions shared by the library's host code and kernels:
// workspace layouts, per-launch parameter blocks and device status flags.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/sparse_attn.h"

#define SA_DEVFLAG_TIMEOUT 1u
#define SA_DEVFLAG_BOUNDS 2u

namespace sa {

constexpr int kMaxCand = 4;
constexpr int kMaxBlocks = 4096;  // blocks per head in one working layout
constexpr int kMaxHeads = 256;    // heads per problem with per-head policy data

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Where each part of the caller's mask workspace lives (byte offsets).
struct MaskLayout {
  int BH = 0;        // batch * heads
  int NB = 0;        // max blocks per head over the policy's layouts
  int W32 = 0;       // ceil(NB / 32)
  int G = 0;         // FG groups per head
  int WN = 0;        // FG: ceil(N / 32)
  size_t off_head = 0, off_counts = 0, off_cols = 0, off_bits = 0;
  int P = 0;         // FG: 128-query tiles per head
  long long cap = 0; // FG: union-list capacity per head
  size_t off_fg_bits = 0, off_fg_tau = 0;
  size_t off_fg_counts = 0, off_fg_offsets = 0, off_fg_list = 0;
  size_t total = 0;
};

// Where each part of the caller's scratch workspace lives (byte offsets).
struct ScratchLayout {
  size_t off_status = 0;           // uint32[64]: [0] flags, [1] first bad index
  size_t off_perm = 0;             // 3 x [BH][N_pad][d] bf16 (frame-major heads)
  size_t perm_stride = 0;          // bytes of one permuted tensor
  size_t off_qbar = 0, off_kbar = 0, off_sics = 0;  // [BH][C][NB][d] f32, [BH][C][NB] f32
  size_t off_scores = 0;           // [BH][NB][NB] f32
  size_t off_fg_qsplit = 0;        // [3][BH][G_pad][d] bf16 terms of q_avg
  size_t off_fg_hist = 0;          // [BH][4096] u32 radix histogram
  size_t off_fg_sel = 0;           // [BH][4] u32 radix-select state
  size_t off_fg_cand = 0;          // [BH][kFgCandCap] uint2 candidates, then [BH] count, [BH] fallback
  size_t total = 0;
};

// One block-sparse head's geometry (device view of sa_head_info).
struct HeadGeom {
  int layout, cand, bt, bh, bw, nt, nh, nw, nb, kept;
  float sics_total[4];
  int window;                       // STA: wt | wh << 8 | ww << 16 (0: the policy's window)
  int reserved;
};
static_assert(sizeof(HeadGeom) == sizeof(sa_head_info), "head info layout");

}  // namespace sa
