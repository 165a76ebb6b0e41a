// Launch interface of the block-sparse attention kernel (library-internal).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_internal.h"

namespace sa {

// Tensor maps per source tensor. Index 0: the original [BH][N][d] tensor as a
// 3-D map (identity layout); 1: the frame-major permuted copy [BH][N_pad][d];
// 2 + c: the original tensor as a 5-D (d, W, H, T, BH) map whose box is the
// 3D tile of blocking candidate c. All use 128-byte boxes along d (64 bf16 or
// 128 E4M3 columns), 128-byte swizzle.
constexpr int kMapsPerTensor = 6;
struct AttnMaps {
  CUtensorMap q[kMapsPerTensor];
  CUtensorMap k[kMapsPerTensor];
  CUtensorMap v[kMapsPerTensor];
};

struct AttnParams {
  const HeadGeom* heads;   // [BH]
  const int* counts;       // [BH][NB] kept key blocks per query block
  const int* cols;         // [BH][NB][NB] kept key blocks, ascending
  __nv_bfloat16* o;        // [BH][N][d]
  float* lse;              // [BH][N]
  uint32_t* status;        // device status word
  int BH, NB, T, H, W, N;
  float scale_log2;        // log2(e) / sqrt(d)
  // gather mode (M x 1 key slices): maps.q[0] is the 3-D query map
  const __nv_bfloat16* k_rows; // gather mode: K and V [BH][N][d], rows copied by key index
  const __nv_bfloat16* v_rows;
  const uint32_t* fg_list;     // [BH][fg_cap]
  const uint32_t* fg_offsets;  // [BH][NB + 1]
  long long fg_cap;
  int fg_groups_per_tile;      // 2 for groups of 64, 1 for groups of 128
  // FP8 mode: per-(batch, head) inverse scales of the E4M3 codes (value = code / inv)
  const float* q_inv;
  const float* k_inv;
  const float* v_inv;
  // Sampled-row mode (the profilers' full pass): every head has geometry geo0
  // (heads is null), every query tile visits every key block of it in order
  // (dense), the query tiles are rows of the gathered tensor behind maps.q[0]
  // (q_tiles of them, q_rows valid per head), and O is written in fp32 to
  // o_f32 [BH][q_rows][d] (o and lse unused).
  HeadGeom geo0;
  int dense;
  int q_tiles;
  int q_rows;
  float* o_f32;
};

cudaError_t launch_attn_fwd(int head_dim, int block, const AttnMaps& maps, const AttnParams& p,
                            cudaStream_t stream);
// The one-warpgroup block kernel (two CTAs per SM), block mode only.
cudaError_t launch_attn_fwd_solo(int head_dim, int block, const AttnMaps& maps,
                                 const AttnParams& p, cudaStream_t stream);
// The one-warpgroup kernel on E4M3 codes (maps over uint8 tensors).
cudaError_t launch_attn_fwd_solo_fp8(int head_dim, int block, const AttnMaps& maps,
                                     const AttnParams& p, cudaStream_t stream);
// Q, K, V as E4M3 codes (maps over uint8 tensors, 128-column boxes).
cudaError_t launch_attn_fwd_fp8(int head_dim, int block, const AttnMaps& maps,
                               const AttnParams& p, cudaStream_t stream);
cudaError_t launch_attn_gather(int head_dim, const AttnMaps& maps, const AttnParams& p,
                               cudaStream_t stream);

}  // namespace sa
