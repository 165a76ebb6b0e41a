// Launch interface of the mask-construction kernels (library-internal).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

struct HeadInitParams {
  HeadGeom* geo;                    // [BH]
  int BH, heads;
  int T, H, W, block;
  int layout;                       // SA_LAYOUT_* for every head unless temporal_bits
  int bt, bh, bw;                   // tile of SA_LAYOUT_TILE
  int has_temporal_bits;            // SPATIOTEMPORAL: layout per head from the bitset
  uint32_t temporal_bits[8];        // bit h set: head h is temporal (frame-major)
  int has_windows;                  // STA: a window per head
  int windows[kMaxHeads];           // wt | wh << 8 | ww << 16
};

struct PermuteParams {
  const HeadGeom* heads;
  const __nv_bfloat16* src[3];      // q, k, v [BH][N][d]
  __nv_bfloat16* dst[3];            // [BH][n_pad][d]
  int T, H, W, d, n_pad;
};

struct PoolParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  float* qbar;                      // [BH][C][NB][d]
  float* kbar;
  float* sics;                      // [BH][C][NB]
  int cand[kMaxCand][3];
  int C, NB, T, H, W, d;
  int Rt, Rh, Rw;                   // region: lcm of the candidates' tiles, <= 8 blocks each
  int nRt, nRh, nRw;                // regions covering every candidate's tile grid
  int At, Ah, Aw;                   // atom: gcd of the candidates' tiles (one block of each)
  int nA;                           // atoms per region; 0 = per-candidate kernel
  int summarizer;                   // SA_SUMMARIZER_*: per-channel mean, max or min
};

// Atoms per region the one-pass pooling kernel holds in shared memory.
constexpr int kMaxPoolAtoms = 128;

struct ChooseParams {
  const float* sics;
  HeadGeom* heads;
  int cand[kMaxCand][3];
  int C, NB, T, H, W;
};

struct ScoreParams {
  const HeadGeom* heads;
  const float* qbar;
  const float* kbar;
  float* scores;                    // [BH][NB][NB]
  int C, NB;
  float sqrt_d;
};

struct SelectParams {
  HeadGeom* heads;
  const float* scores;              // [BH][NB][NB] or null
  const uint32_t* explicit_bits;    // [BH][NB][W32] or null
  uint32_t* bits;                   // [BH][NB][W32]
  int* counts;                      // [BH][NB]
  int* cols;                        // [BH][NB][NB]
  int kind, NB, W32, T, H, W;
  int topk, keep_diagonal;
  int win[3];
  float top_p;
  int frame_radius, sink_blocks;
  uint32_t* status;                 // debug builds: index checks flag it
};

cudaError_t launch_head_init(const HeadInitParams& p, cudaStream_t st);
cudaError_t launch_permute_fm(const PermuteParams& p, int BH, cudaStream_t st);
cudaError_t launch_pool_sics(const PoolParams& p, int BH, int max_nb, cudaStream_t st);
cudaError_t launch_choose(const ChooseParams& p, int BH, cudaStream_t st);
cudaError_t launch_pooled_scores(const ScoreParams& p, int BH, int d, cudaStream_t st);
cudaError_t launch_select(const SelectParams& p, int BH, cudaStream_t st);
cudaError_t launch_zero_counts(int* counts, size_t n, cudaStream_t st);

}  // namespace sa
