// Host side of the C ABI declared in include/sparse_attn.h: argument checks,
// workspace layouts, TMA tensor maps and the launch sequence of each call.
// No device memory is allocated here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "sa_attn.h"
#include "sa_fg.h"
#include "sa_internal.h"
#include "sa_mask.h"
#include "sa_profile.h"
#include "sa_quant.h"

using namespace sa;

namespace {

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

bool is_tile_kind(int kind) { return kind == SA_MASK_TOPK || kind == SA_MASK_STA; }

// Blocks of a 3D tiling of the problem's grid.
int tile_blocks(const sa_problem& pr, const int* t) {
  return ceil_div(pr.T, t[0]) * ceil_div(pr.H, t[1]) * ceil_div(pr.W, t[2]);
}

long long n_tokens(const sa_problem& pr) { return (long long)pr.T * pr.H * pr.W; }

int check_problem(const sa_problem* pr) {
  if (!pr) return SA_ERR_INVALID_ARG;
  if (pr->batch < 1 || pr->heads < 1 || pr->T < 1 || pr->H < 1 || pr->W < 1)
    return SA_ERR_INVALID_ARG;
  if (pr->head_dim != 64 && pr->head_dim != 128) return SA_ERR_UNSUPPORTED;
  if (n_tokens(*pr) > (1ll << 30) / pr->head_dim) return SA_ERR_UNSUPPORTED;
  if ((long long)pr->batch * pr->heads > 65535) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

int check_tile(const sa_problem& pr, const int* t, int block) {
  if (t[0] < 1 || t[1] < 1 || t[2] < 1) return SA_ERR_INVALID_ARG;
  // product in 64 bits, stopped once it passes the block: no overflow for any int extents
  const long long t01 = (long long)t[0] * t[1];
  if (t01 > block || t01 * t[2] != block) return SA_ERR_INVALID_ARG;
  if (t[0] > 256 || t[1] > 256 || t[2] > 256) return SA_ERR_UNSUPPORTED;
  if (tile_blocks(pr, t) > kMaxBlocks) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

int check_policy(const sa_problem& pr, const sa_policy* po) {
  if (!po) return SA_ERR_INVALID_ARG;
  if (po->kind == SA_MASK_FG) {
    if (po->fg_group != 64 && po->fg_group != 128) return SA_ERR_UNSUPPORTED;
    if (!(po->fg_keep_fraction > 0.f && po->fg_keep_fraction <= 1.f)) return SA_ERR_INVALID_ARG;
    return SA_OK;
  }
  if (po->block != 128 && !(po->block == 64 && pr.head_dim == 64)) return SA_ERR_UNSUPPORTED;
  if ((po->kind == SA_MASK_TOPK || po->kind == SA_MASK_SPADE) &&
      (po->summarizer < SA_SUMMARIZER_MEAN || po->summarizer > SA_SUMMARIZER_MIN))
    return SA_ERR_INVALID_ARG;
  const long long N = n_tokens(pr);
  switch (po->kind) {
    case SA_MASK_TOPK:
      if (po->topk < 1) return SA_ERR_INVALID_ARG;
      return check_tile(pr, po->tile, po->block);
    case SA_MASK_STA:
      for (int i = 0; i < 3; ++i)
        if (po->window[i] < 1 || po->window[i] % 2 == 0) return SA_ERR_INVALID_ARG;
      if (po->head_windows) {
        if (pr.heads > kMaxHeads) return SA_ERR_UNSUPPORTED;
        for (int i = 0; i < 3 * pr.heads; ++i)
          if (po->head_windows[i] < 1 || po->head_windows[i] % 2 == 0 || po->head_windows[i] > 255)
            return SA_ERR_INVALID_ARG;
      }
      return check_tile(pr, po->tile, po->block);
    case SA_MASK_SPADE:
      if (po->n_candidates < 1 || po->n_candidates > kMaxCand) return SA_ERR_INVALID_ARG;
      if (!(po->top_p > 0.f && po->top_p <= 1.f)) return SA_ERR_INVALID_ARG;
      for (int i = 0; i < 3; ++i)
        if (po->window[i] < 1 || po->window[i] % 2 == 0) return SA_ERR_INVALID_ARG;
      for (int c = 0; c < po->n_candidates; ++c) {
        const int e = check_tile(pr, po->candidates[c], po->block);
        if (e) return e;
      }
      return SA_OK;
    case SA_MASK_SPATIOTEMPORAL:
      if (!po->head_is_temporal) return SA_ERR_INVALID_ARG;
      if (pr.heads > 256) return SA_ERR_UNSUPPORTED;
      if (po->sink_tokens < 0 || po->frame_radius < 0) return SA_ERR_INVALID_ARG;
      if (ceil_div(N, po->block) > kMaxBlocks) return SA_ERR_UNSUPPORTED;
      return SA_OK;
    case SA_MASK_EXPLICIT:
      if (!po->explicit_bits) return SA_ERR_INVALID_ARG;
      if (po->explicit_layout == SA_LAYOUT_TILE) return check_tile(pr, po->tile, po->block);
      if (po->explicit_layout != SA_LAYOUT_IDENTITY && po->explicit_layout != SA_LAYOUT_FRAME_MAJOR)
        return SA_ERR_INVALID_ARG;
      if (ceil_div(N, po->block) > kMaxBlocks) return SA_ERR_UNSUPPORTED;
      return SA_OK;
    default:
      return SA_ERR_INVALID_ARG;
  }
}

// Max blocks per head over every layout the policy can use.
int policy_nb(const sa_problem& pr, const sa_policy& po) {
  switch (po.kind) {
    case SA_MASK_TOPK:
    case SA_MASK_STA:
      return tile_blocks(pr, po.tile);
    case SA_MASK_SPADE: {
      int nb = 0;
      for (int c = 0; c < po.n_candidates; ++c) nb = std::max(nb, tile_blocks(pr, po.candidates[c]));
      return nb;
    }
    case SA_MASK_EXPLICIT:
      if (po.explicit_layout == SA_LAYOUT_TILE) return tile_blocks(pr, po.tile);
      return ceil_div(n_tokens(pr), po.block);
    case SA_MASK_SPATIOTEMPORAL:
      return ceil_div(n_tokens(pr), po.block);
    default:
      return 0;
  }
}

bool needs_frame_major(const sa_problem& pr, const sa_policy& po) {
  if (po.kind == SA_MASK_EXPLICIT) return po.explicit_layout == SA_LAYOUT_FRAME_MAJOR;
  if (po.kind != SA_MASK_SPATIOTEMPORAL) return false;
  for (int h = 0; h < pr.heads; ++h)
    if (po.head_is_temporal[h]) return true;
  return false;
}

int n_cand(const sa_policy& po) {
  if (po.kind == SA_MASK_SPADE) return po.n_candidates;
  if (po.kind == SA_MASK_TOPK) return 1;
  return 0;
}

MaskLayout mask_layout(const sa_problem& pr, const sa_policy& po) {
  MaskLayout L;
  L.BH = pr.batch * pr.heads;
  L.NB = policy_nb(pr, po);
  L.W32 = (L.NB + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  L.off_head = take(sizeof(HeadGeom) * L.BH);
  L.off_counts = take(sizeof(int) * (size_t)L.BH * L.NB);
  L.off_cols = take(sizeof(int) * (size_t)L.BH * L.NB * L.NB);
  L.off_bits = take(sizeof(uint32_t) * (size_t)L.BH * L.NB * L.W32);
  if (po.kind == SA_MASK_FG) {
    const long long N = n_tokens(pr);
    L.G = ceil_div(N, po.fg_group);
    L.WN = ceil_div(N, 32);
    L.P = ceil_div(N, 128);
    L.cap = fg_list_cap_per_head(L.G, (int)N, po.fg_keep_fraction);
    L.off_fg_bits = take(sizeof(uint32_t) * (size_t)L.BH * L.G * L.WN);
    L.off_fg_tau = take(sizeof(float) * (size_t)L.BH);
    L.off_fg_counts = take(sizeof(uint32_t) * (size_t)L.BH * L.P);
    L.off_fg_offsets = take(sizeof(uint32_t) * (size_t)L.BH * (L.P + 1));
    L.off_fg_list = take(sizeof(uint32_t) * (size_t)L.BH * L.cap);
  }
  L.total = std::max<size_t>(off, 256);
  return L;
}

ScratchLayout scratch_layout(const sa_problem& pr, const sa_policy& po, const MaskLayout& M) {
  ScratchLayout S;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  S.off_status = take(256);
  const int d = pr.head_dim;
  if (needs_frame_major(pr, po)) {
    const size_t n_pad = (size_t)ceil_div(n_tokens(pr), po.block) * po.block;
    S.perm_stride = align_up((size_t)M.BH * n_pad * d * 2, 256);
    S.off_perm = take(3 * S.perm_stride);
  }
  const int C = n_cand(po);
  if (C > 0) {
    S.off_qbar = take(sizeof(float) * (size_t)M.BH * C * M.NB * d);
    S.off_kbar = take(sizeof(float) * (size_t)M.BH * C * M.NB * d);
    S.off_sics = take(sizeof(float) * (size_t)M.BH * C * M.NB);
    S.off_scores = take(sizeof(float) * (size_t)M.BH * M.NB * M.NB);
  }
  if (po.kind == SA_MASK_FG) {
    S.off_fg_qsplit = take(fg_qsplit_bytes(M.BH, M.G, d));
    S.off_fg_hist = take(fg_hist_bytes(M.BH));
    S.off_fg_sel = take(fg_sel_bytes(M.BH));
    S.off_fg_cand = take(fg_cand_bytes(M.BH));
  }
  S.total = off;
  return S;
}

// ------------------------------------------------------------------ tensor maps
typedef EncodeFn EncodeTiledFn;

// Resolved once, on first use; a function-local static is initialised exactly
// once even when several host threads make their first call together.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return EncodeTiledFn(nullptr);
  }();
  return fn;
}

// 3-D map over [BH][rows][d] with a (128-byte, box_rows, 1) box: bf16 by
// default, E4M3 codes (one byte each) with ``bytes`` = 1.
bool map_3d(CUtensorMap* m, const void* base, int BH, long long rows, int d, int box_rows,
            int bytes = 2) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * bytes, (cuuint64_t)rows * d * bytes};
  cuuint32_t box[3] = {(cuuint32_t)(128 / bytes), (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapDataType dt = bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return encode_fn()(m, dt, 3, const_cast<void*>(base), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D map over [BH][T][H][W][d] whose box is one (bt, bh, bw) tile x 128 bytes
// of d (bf16, or E4M3 codes with ``bytes`` = 1).
bool map_5d(CUtensorMap* m, const void* base, const sa_problem& pr, const int* tile,
            int bytes = 2) {
  const int d = pr.head_dim;
  const cuuint64_t e = (cuuint64_t)bytes;
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)pr.W, (cuuint64_t)pr.H, (cuuint64_t)pr.T,
                        (cuuint64_t)pr.batch * pr.heads};
  cuuint64_t strides[4] = {d * e, (cuuint64_t)pr.W * d * e, (cuuint64_t)pr.H * pr.W * d * e,
                           (cuuint64_t)pr.T * pr.H * pr.W * d * e};
  cuuint32_t box[5] = {(cuuint32_t)(128 / bytes), (cuuint32_t)tile[2], (cuuint32_t)tile[1],
                       (cuuint32_t)tile[0], 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUtensorMapDataType dt = bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return encode_fn()(m, dt, 5, const_cast<void*>(base), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gcd_i(int a, int b) { return b ? gcd_i(b, a % b) : a; }
int lcm_i(int a, int b) { return a / gcd_i(a, b) * b; }

// Regions for the pooling kernel: the least common multiple of the candidate
// tiles along each axis, so every region holds whole blocks of every
// candidate; then grown along w, h, t (by doubling while it stays inside the
// grid) until the smallest candidate count per region reaches 8 blocks, one
// per warp of the CTA, without exceeding 8 for any candidate.
void pool_regions(PoolParams& pp) {
  int R[3] = {1, 1, 1};
  for (int c = 0; c < pp.C; ++c)
    for (int a = 0; a < 3; ++a) R[a] = lcm_i(R[a], pp.cand[c][a]);
  auto blocks = [&](int c) {
    return (R[0] / pp.cand[c][0]) * (R[1] / pp.cand[c][1]) * (R[2] / pp.cand[c][2]);
  };
  const int ext[3] = {pp.T, pp.H, pp.W};
  for (bool grew = true; grew;) {
    grew = false;
    int mx = 0, mn = 1 << 30;
    for (int c = 0; c < pp.C; ++c) { mx = std::max(mx, blocks(c)); mn = std::min(mn, blocks(c)); }
    if (mn >= 8 || 2 * mx > 8) break;
    for (int a = 2; a >= 0 && !grew; --a)
      if (2 * R[a] <= ext[a] + R[a] - 1) { R[a] *= 2; grew = true; }
  }
  pp.Rt = R[0]; pp.Rh = R[1]; pp.Rw = R[2];
  pp.nRt = ceil_div(pp.T, R[0]); pp.nRh = ceil_div(pp.H, R[1]); pp.nRw = ceil_div(pp.W, R[2]);
  // atoms: greatest common divisor of the tiles along each axis
  int A[3] = {pp.cand[0][0], pp.cand[0][1], pp.cand[0][2]};
  for (int c = 1; c < pp.C; ++c)
    for (int a = 0; a < 3; ++a) A[a] = gcd_i(A[a], pp.cand[c][a]);
  pp.At = A[0]; pp.Ah = A[1]; pp.Aw = A[2];
  const long long nA = (long long)(R[0] / A[0]) * (R[1] / A[1]) * (R[2] / A[2]);
  pp.nA = nA <= kMaxPoolAtoms ? (int)nA : 0;    // else the per-candidate kernel
}

// Top-K, tile windows and frame windows bound how many key blocks a row
// keeps, to a few dozen at the sizes these policies are used at. Their CTAs
// spend a large share of their time on setup, the Q load and the epilogue,
// which the one-warpgroup attention kernel hides by running two CTAs per SM.
// Top-P and caller-supplied masks can keep most of a row and run the
// two-warpgroup kernel, whose three K/V stages hide the loads of long rows.
bool bounded_rows(const sa_policy& po) {
  return po.kind == SA_MASK_TOPK || po.kind == SA_MASK_STA || po.kind == SA_MASK_SPATIOTEMPORAL;
}

int aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Union lists of the slice bitmask in the mask workspace (FG policies).
FgListParams fg_lists(const MaskLayout& M, const sa_policy& po, uint8_t* mw, uint32_t* status) {
  FgListParams lp{};
  lp.bits = reinterpret_cast<uint32_t*>(mw + M.off_fg_bits);
  lp.counts = reinterpret_cast<uint32_t*>(mw + M.off_fg_counts);
  lp.offsets = reinterpret_cast<uint32_t*>(mw + M.off_fg_offsets);
  lp.list = reinterpret_cast<uint32_t*>(mw + M.off_fg_list);
  lp.status = status;
  lp.cap_per_head = M.cap;
  lp.BH = M.BH; lp.P = M.P; lp.G = M.G; lp.WN = M.WN; lp.groups_per_tile = 128 / po.fg_group;
  return lp;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

}  // namespace

// ======================================================================== API
extern "C" int sparse_attn_workspace_size(const sa_problem* problem, const sa_policy* policy,
                                          size_t* mask_bytes, size_t* scratch_bytes) {
  int e = check_problem(problem);
  if (e) return e;
  e = check_policy(*problem, policy);
  if (e) return e;
  if (!mask_bytes || !scratch_bytes) return SA_ERR_INVALID_ARG;
  const MaskLayout M = mask_layout(*problem, *policy);
  const ScratchLayout S = scratch_layout(*problem, *policy, M);
  *mask_bytes = M.total;
  *scratch_bytes = S.total;
  return SA_OK;
}

extern "C" int sparse_attn_build_mask(const sa_problem* problem, const sa_policy* policy,
                                      const void* q, const void* k, void* mask_ws,
                                      void* scratch_ws, void* stream) {
  int e = check_problem(problem);
  if (e) return e;
  e = check_policy(*problem, policy);
  if (e) return e;
  const sa_problem& pr = *problem;
  const sa_policy& po = *policy;
  const bool needs_qk = po.kind == SA_MASK_TOPK || po.kind == SA_MASK_SPADE || po.kind == SA_MASK_FG;
  if (needs_qk && (!aligned(q, 16) || !aligned(k, 16))) return SA_ERR_INVALID_ARG;
  if (!aligned(mask_ws, 256) || !aligned(scratch_ws, 256)) return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const MaskLayout M = mask_layout(pr, po);
  const ScratchLayout S = scratch_layout(pr, po, M);
  uint8_t* mw = static_cast<uint8_t*>(mask_ws);
  uint8_t* sw = static_cast<uint8_t*>(scratch_ws);
  HeadGeom* heads = reinterpret_cast<HeadGeom*>(mw + M.off_head);
  const int N = (int)n_tokens(pr);
  const int d = pr.head_dim;
  const int BH = M.BH;

  if (cudaMemsetAsync(sw + S.off_status, 0, 256, st) != cudaSuccess) return SA_ERR_CUDA;

  if (po.kind == SA_MASK_FG) {
    if (!encode_fn()) return SA_ERR_CUDA;
    FgBuildParams fp{};
    fp.q = static_cast<const __nv_bfloat16*>(q);
    fp.k = static_cast<const __nv_bfloat16*>(k);
    fp.qsplit = reinterpret_cast<__nv_bfloat16*>(sw + S.off_fg_qsplit);
    fp.hist = reinterpret_cast<uint32_t*>(sw + S.off_fg_hist);
    fp.sel = reinterpret_cast<uint32_t*>(sw + S.off_fg_sel);
    fp.cand = reinterpret_cast<uint2*>(sw + S.off_fg_cand);
    fp.cand_count = reinterpret_cast<uint32_t*>(sw + S.off_fg_cand + sizeof(uint2) * (size_t)M.BH * kFgCandCap);
    fp.fallback = fp.cand_count + M.BH;
    fp.win = fp.fallback + M.BH;
    fp.bits = reinterpret_cast<uint32_t*>(mw + M.off_fg_bits);
    fp.tau = reinterpret_cast<float*>(mw + M.off_fg_tau);
    fp.status = reinterpret_cast<uint32_t*>(sw + S.off_status);
    fp.BH = BH; fp.N = N; fp.d = d; fp.group = po.fg_group; fp.G = M.G; fp.WN = M.WN;
    fp.keep_fraction = po.fg_keep_fraction;
    fp.lists = fg_lists(M, po, mw, fp.status);
    return cuda_status(launch_fg_build(fp, encode_fn(), st));
  }

  SelectParams sp{};
  sp.heads = heads;
  sp.bits = reinterpret_cast<uint32_t*>(mw + M.off_bits);
  sp.counts = reinterpret_cast<int*>(mw + M.off_counts);
  sp.cols = reinterpret_cast<int*>(mw + M.off_cols);
  sp.kind = po.kind; sp.NB = M.NB; sp.W32 = M.W32; sp.T = pr.T; sp.H = pr.H; sp.W = pr.W;
  sp.topk = po.topk; sp.keep_diagonal = po.keep_diagonal;
  for (int i = 0; i < 3; ++i) sp.win[i] = po.window[i];
  sp.top_p = po.top_p;
  sp.frame_radius = po.frame_radius;
  sp.sink_blocks = ceil_div(po.sink_tokens, po.block);
  sp.status = reinterpret_cast<uint32_t*>(sw + S.off_status);

  const int C = n_cand(po);
  if (C > 0) {
    PoolParams pp{};
    pp.q = static_cast<const __nv_bfloat16*>(q);
    pp.k = static_cast<const __nv_bfloat16*>(k);
    pp.qbar = reinterpret_cast<float*>(sw + S.off_qbar);
    pp.kbar = reinterpret_cast<float*>(sw + S.off_kbar);
    pp.sics = reinterpret_cast<float*>(sw + S.off_sics);
    for (int c = 0; c < C; ++c)
      for (int i = 0; i < 3; ++i) pp.cand[c][i] = po.kind == SA_MASK_SPADE ? po.candidates[c][i] : po.tile[i];
    pp.C = C; pp.NB = M.NB; pp.T = pr.T; pp.H = pr.H; pp.W = pr.W; pp.d = d;
    pp.summarizer = po.summarizer;
    pool_regions(pp);
    if ((e = cuda_status(launch_pool_sics(pp, BH, M.NB, st)))) return e;
    if (po.kind == SA_MASK_SPADE) {
      ChooseParams cp{};
      cp.sics = pp.sics; cp.heads = heads;
      std::memcpy(cp.cand, pp.cand, sizeof(cp.cand));
      cp.C = C; cp.NB = M.NB; cp.T = pr.T; cp.H = pr.H; cp.W = pr.W;
      if ((e = cuda_status(launch_choose(cp, BH, st)))) return e;
    }
  }
  if (po.kind != SA_MASK_SPADE) {
    HeadInitParams hp{};
    hp.geo = heads; hp.BH = BH; hp.heads = pr.heads;
    hp.T = pr.T; hp.H = pr.H; hp.W = pr.W; hp.block = po.block;
    hp.layout = po.kind == SA_MASK_EXPLICIT ? po.explicit_layout
              : (is_tile_kind(po.kind) ? SA_LAYOUT_TILE : SA_LAYOUT_IDENTITY);
    hp.bt = po.tile[0]; hp.bh = po.tile[1]; hp.bw = po.tile[2];
    if (po.kind == SA_MASK_SPATIOTEMPORAL) {
      hp.has_temporal_bits = 1;
      for (int h = 0; h < pr.heads; ++h)
        if (po.head_is_temporal[h]) hp.temporal_bits[h / 32] |= 1u << (h % 32);
    }
    if (po.kind == SA_MASK_STA && po.head_windows) {
      hp.has_windows = 1;
      for (int h = 0; h < pr.heads; ++h)
        hp.windows[h] = po.head_windows[3 * h] | (po.head_windows[3 * h + 1] << 8) |
                        (po.head_windows[3 * h + 2] << 16);
    }
    if ((e = cuda_status(launch_head_init(hp, st)))) return e;
  }
  if (C > 0) {
    ScoreParams sc{};
    sc.heads = heads;
    sc.qbar = reinterpret_cast<const float*>(sw + S.off_qbar);
    sc.kbar = reinterpret_cast<const float*>(sw + S.off_kbar);
    sc.scores = reinterpret_cast<float*>(sw + S.off_scores);
    sc.C = C; sc.NB = M.NB; sc.sqrt_d = sqrtf((float)d);
    if ((e = cuda_status(launch_pooled_scores(sc, BH, d, st)))) return e;
    sp.scores = sc.scores;
  }
  if (po.kind == SA_MASK_EXPLICIT) sp.explicit_bits = po.explicit_bits;
  return cuda_status(launch_select(sp, BH, st));
}

extern "C" int sparse_attn_build_mask_fg_cached(const sa_problem* problem,
                                                const sa_policy* policy, const void* q,
                                                const void* k, const float* lse, float tau,
                                                void* mask_ws, void* scratch_ws, void* stream) {
  int e = check_problem(problem);
  if (e) return e;
  e = check_policy(*problem, policy);
  if (e) return e;
  if (policy->kind != SA_MASK_FG) return SA_ERR_INVALID_ARG;
  if (!(tau >= 0.f && tau < 1.f)) return SA_ERR_INVALID_ARG;     // NaN fails too
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(lse, 4)) return SA_ERR_INVALID_ARG;
  if (!aligned(mask_ws, 256) || !aligned(scratch_ws, 256)) return SA_ERR_WORKSPACE;
  if (!encode_fn()) return SA_ERR_CUDA;
  const sa_problem& pr = *problem;
  const sa_policy& po = *policy;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const MaskLayout M = mask_layout(pr, po);
  const ScratchLayout S = scratch_layout(pr, po, M);
  uint8_t* mw = static_cast<uint8_t*>(mask_ws);
  uint8_t* sw = static_cast<uint8_t*>(scratch_ws);
  const long long N = n_tokens(pr);
  if (cudaMemsetAsync(sw + S.off_status, 0, 256, st) != cudaSuccess) return SA_ERR_CUDA;
  FgCachedParams cp{};
  cp.q = static_cast<const __nv_bfloat16*>(q);
  cp.k = static_cast<const __nv_bfloat16*>(k);
  cp.lse = lse;
  cp.bits = reinterpret_cast<uint32_t*>(mw + M.off_fg_bits);
  cp.tau_out = reinterpret_cast<float*>(mw + M.off_fg_tau);
  cp.status = reinterpret_cast<uint32_t*>(sw + S.off_status);
  cp.lists = fg_lists(M, po, mw, cp.status);
  cp.BH = M.BH; cp.N = (int)N; cp.d = pr.head_dim; cp.group = po.fg_group;
  cp.G = M.G; cp.WN = M.WN;
  // FG-Attn review, Sec. 5.1 as quoted by the referee: tau_cached = 0.5 / N
  cp.tau = tau > 0.f ? tau : (float)(0.5 / (double)N);
  return cuda_status(launch_fg_cached(cp, encode_fn(), st));
}

namespace {

struct CallCtx;
bool block_maps(const sa_problem& pr, const sa_policy& po, const CallCtx& c, const void* q,
                const void* k, const void* v, int bytes, AttnMaps* maps);

struct CallCtx {
  MaskLayout M;
  ScratchLayout S;
  const uint8_t* mw;
  uint8_t* sw;
  cudaStream_t st;
  int N, d, BH, n_pad;
};

int prepare_call(const sa_problem* problem, const sa_policy* policy, const void* q,
                 const void* k, const void* v, const void* mask_ws, void* scratch_ws,
                 void* stream, CallCtx* c) {
  int e = check_problem(problem);
  if (e) return e;
  e = check_policy(*problem, policy);
  if (e) return e;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return SA_ERR_INVALID_ARG;
  if (!aligned(mask_ws, 256) || !aligned(scratch_ws, 256)) return SA_ERR_WORKSPACE;
  c->M = mask_layout(*problem, *policy);
  c->S = scratch_layout(*problem, *policy, c->M);
  c->mw = static_cast<const uint8_t*>(mask_ws);
  c->sw = static_cast<uint8_t*>(scratch_ws);
  c->st = reinterpret_cast<cudaStream_t>(stream);
  c->N = (int)n_tokens(*problem);
  c->d = problem->head_dim;
  c->BH = c->M.BH;
  c->n_pad = policy->kind == SA_MASK_FG ? c->N : ceil_div(c->N, policy->block) * policy->block;
  return SA_OK;
}

// Tensor maps of the block kernel for Q, K, V (elements of ``bytes`` bytes):
// the original tensors (3-D), the frame-major copies in the scratch
// workspace, and one 5-D tile map per blocking candidate.
bool block_maps(const sa_problem& pr, const sa_policy& po, const CallCtx& c, const void* q,
                const void* k, const void* v, int bytes, AttnMaps* maps) {
  const void* src[3] = {q, k, v};
  const bool fm = needs_frame_major(pr, po);
  std::memset(maps, 0, sizeof(*maps));
  CUtensorMap* sets[3] = {maps->q, maps->k, maps->v};
  const bool tiled = po.kind == SA_MASK_SPADE || is_tile_kind(po.kind) ||
                     (po.kind == SA_MASK_EXPLICIT && po.explicit_layout == SA_LAYOUT_TILE);
  const int C = po.kind == SA_MASK_SPADE ? po.n_candidates : 1;
  for (int i = 0; i < 3; ++i) {
    if (!map_3d(&sets[i][0], src[i], c.BH, c.N, c.d, po.block, bytes)) return false;
    if (fm) {
      const void* perm = c.sw + c.S.off_perm + i * c.S.perm_stride;
      if (!map_3d(&sets[i][1], perm, c.BH, c.n_pad, c.d, po.block, bytes)) return false;
    } else {
      sets[i][1] = sets[i][0];
    }
    for (int cc = 0; cc < C; ++cc) {
      if (!tiled) { sets[i][2 + cc] = sets[i][0]; continue; }
      const int* tile = po.kind == SA_MASK_SPADE ? po.candidates[cc] : po.tile;
      if (!map_5d(&sets[i][2 + cc], src[i], pr, tile, bytes)) return false;
    }
  }
  return true;
}

}  // namespace

extern "C" int sparse_attn_permute(const sa_problem* problem, const sa_policy* policy,
                                   const void* q, const void* k, const void* v,
                                   const void* mask_ws, void* scratch_ws, void* stream) {
  CallCtx c;
  int e = prepare_call(problem, policy, q, k, v, mask_ws, scratch_ws, stream, &c);
  if (e) return e;
  if (!needs_frame_major(*problem, *policy)) return SA_OK;
  PermuteParams pp{};
  pp.heads = reinterpret_cast<const HeadGeom*>(c.mw + c.M.off_head);
  const void* src[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    pp.src[i] = static_cast<const __nv_bfloat16*>(src[i]);
    pp.dst[i] = reinterpret_cast<__nv_bfloat16*>(c.sw + c.S.off_perm + i * c.S.perm_stride);
  }
  pp.T = problem->T; pp.H = problem->H; pp.W = problem->W; pp.d = c.d; pp.n_pad = c.n_pad;
  return cuda_status(launch_permute_fm(pp, c.BH, c.st));
}

extern "C" int sparse_attn_attend(const sa_problem* problem, const sa_policy* policy,
                                  const void* q, const void* k, const void* v,
                                  const void* mask_ws, void* scratch_ws, void* o, float* lse,
                                  void* stream) {
  CallCtx c;
  int e = prepare_call(problem, policy, q, k, v, mask_ws, scratch_ws, stream, &c);
  if (e) return e;
  if (!aligned(o, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID_ARG;
  if (!encode_fn()) return SA_ERR_CUDA;
  const sa_problem& pr = *problem;
  const sa_policy& po = *policy;
  uint32_t* status = reinterpret_cast<uint32_t*>(c.sw + c.S.off_status);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)c.d);

  if (po.kind == SA_MASK_FG) {
    AttnMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!map_3d(&maps.q[0], q, c.BH, c.N, c.d, 128)) return SA_ERR_CUDA;
    AttnParams ap{};
    ap.o = static_cast<__nv_bfloat16*>(o);
    ap.lse = lse;
    ap.status = status;
    ap.BH = c.BH; ap.NB = c.M.P; ap.T = pr.T; ap.H = pr.H; ap.W = pr.W; ap.N = c.N;
    ap.scale_log2 = scale_log2;
    ap.k_rows = static_cast<const __nv_bfloat16*>(k);
    ap.v_rows = static_cast<const __nv_bfloat16*>(v);
    ap.fg_list = reinterpret_cast<const uint32_t*>(c.mw + c.M.off_fg_list);
    ap.fg_offsets = reinterpret_cast<const uint32_t*>(c.mw + c.M.off_fg_offsets);
    ap.fg_cap = c.M.cap;
    ap.fg_groups_per_tile = 128 / po.fg_group;
    return cuda_status(launch_attn_gather(c.d, maps, ap, c.st));
  }

  AttnMaps maps;
  if (!block_maps(pr, po, c, q, k, v, 2, &maps)) return SA_ERR_CUDA;
  AttnParams ap{};
  ap.heads = reinterpret_cast<const HeadGeom*>(c.mw + c.M.off_head);
  ap.counts = reinterpret_cast<const int*>(c.mw + c.M.off_counts);
  ap.cols = reinterpret_cast<const int*>(c.mw + c.M.off_cols);
  ap.o = static_cast<__nv_bfloat16*>(o);
  ap.lse = lse;
  ap.status = status;
  ap.BH = c.BH; ap.NB = c.M.NB; ap.T = pr.T; ap.H = pr.H; ap.W = pr.W; ap.N = c.N;
  ap.scale_log2 = scale_log2;
  return cuda_status(bounded_rows(po) ? launch_attn_fwd_solo(c.d, po.block, maps, ap, c.st)
                                      : launch_attn_fwd(c.d, po.block, maps, ap, c.st));
}

extern "C" int sparse_attn_forward(const sa_problem* problem, const sa_policy* policy,
                                   const void* q, const void* k, const void* v,
                                   const void* mask_ws, void* scratch_ws, void* o, float* lse,
                                   void* stream) {
  int e = sparse_attn_permute(problem, policy, q, k, v, mask_ws, scratch_ws, stream);
  if (e) return e;
  return sparse_attn_attend(problem, policy, q, k, v, mask_ws, scratch_ws, o, lse, stream);
}

extern "C" int sparse_attn_forward_host(const sa_problem* problem, const sa_policy* policy,
                                        const void* q_host, const void* k_host,
                                        const void* v_host, void* o_host, float* lse_host,
                                        void* qkv_dev, void* o_dev, float* lse_dev,
                                        void* mask_ws, void* scratch_ws, void* stream) {
  int e = check_problem(problem);
  if (e) return e;
  if (!policy) return SA_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !o_host || !qkv_dev || !o_dev) return SA_ERR_INVALID_ARG;
  if ((lse_host == nullptr) != (lse_dev == nullptr)) return SA_ERR_INVALID_ARG;
  if (!aligned(qkv_dev, 16) || !aligned(o_dev, 16) || (lse_dev && !aligned(lse_dev, 4)))
    return SA_ERR_INVALID_ARG;
  const size_t elems = (size_t)problem->batch * problem->heads * (size_t)n_tokens(*problem) *
                       problem->head_dim;
  const size_t bytes = elems * 2;                      // bf16
  uint8_t* qd = static_cast<uint8_t*>(qkv_dev);
  uint8_t* kd = qd + bytes;
  uint8_t* vd = kd + bytes;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // one copy per tensor, in and out, on the caller's stream
  const void* hin[3] = {q_host, k_host, v_host};
  uint8_t* din[3] = {qd, kd, vd};
  for (int i = 0; i < 3; ++i)
    if (cudaMemcpyAsync(din[i], hin[i], bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return SA_ERR_CUDA;
  e = sparse_attn_build_mask(problem, policy, qd, kd, mask_ws, scratch_ws, stream);
  if (e) return e;
  e = sparse_attn_forward(problem, policy, qd, kd, vd, mask_ws, scratch_ws, o_dev, lse_dev, stream);
  if (e) return e;
  if (cudaMemcpyAsync(o_host, o_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SA_ERR_CUDA;
  if (lse_host) {
    const size_t lbytes = sizeof(float) * (size_t)problem->batch * problem->heads *
                          (size_t)n_tokens(*problem);
    if (cudaMemcpyAsync(lse_host, lse_dev, lbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return SA_ERR_CUDA;
  }
  return SA_OK;
}

extern "C" int sparse_attn_permute_fp8(const sa_problem* problem, const sa_policy* policy,
                                       const void* q8, const void* k8, const void* v8,
                                       const void* mask_ws, void* scratch_ws, void* stream) {
  CallCtx c;
  int e = prepare_call(problem, policy, q8, k8, v8, mask_ws, scratch_ws, stream, &c);
  if (e) return e;
  if (c.d % 32 != 0) return SA_ERR_UNSUPPORTED;
  if (!needs_frame_major(*problem, *policy)) return SA_OK;
  // The permutation moves whole rows in 16-byte pieces: a row of d E4M3
  // codes is moved as a row of d / 2 bf16-sized elements.
  PermuteParams pp{};
  pp.heads = reinterpret_cast<const HeadGeom*>(c.mw + c.M.off_head);
  const void* src[3] = {q8, k8, v8};
  for (int i = 0; i < 3; ++i) {
    pp.src[i] = static_cast<const __nv_bfloat16*>(src[i]);
    pp.dst[i] = reinterpret_cast<__nv_bfloat16*>(c.sw + c.S.off_perm + i * c.S.perm_stride);
  }
  pp.T = problem->T; pp.H = problem->H; pp.W = problem->W; pp.d = c.d / 2; pp.n_pad = c.n_pad;
  return cuda_status(launch_permute_fm(pp, c.BH, c.st));
}

extern "C" int sparse_attn_attend_fp8(const sa_problem* problem, const sa_policy* policy,
                                      const void* q8, const void* k8, const void* v8,
                                      const float* q_inv, const float* k_inv, const float* v_inv,
                                      const void* mask_ws, void* scratch_ws, void* o, float* lse,
                                      void* stream) {
  CallCtx c;
  int e = prepare_call(problem, policy, q8, k8, v8, mask_ws, scratch_ws, stream, &c);
  if (e) return e;
  if (!aligned(o, 16) || (lse && !aligned(lse, 4))) return SA_ERR_INVALID_ARG;
  if (!q_inv || !k_inv || !v_inv || !aligned(q_inv, 4) || !aligned(k_inv, 4) ||
      !aligned(v_inv, 4))
    return SA_ERR_INVALID_ARG;
  const sa_policy& po = *policy;
  if (po.kind == SA_MASK_FG || c.d != 128 || po.block != 128) return SA_ERR_UNSUPPORTED;
  if (!encode_fn()) return SA_ERR_CUDA;
  AttnMaps maps;
  if (!block_maps(*problem, po, c, q8, k8, v8, 1, &maps)) return SA_ERR_CUDA;
  AttnParams ap{};
  ap.heads = reinterpret_cast<const HeadGeom*>(c.mw + c.M.off_head);
  ap.counts = reinterpret_cast<const int*>(c.mw + c.M.off_counts);
  ap.cols = reinterpret_cast<const int*>(c.mw + c.M.off_cols);
  ap.o = static_cast<__nv_bfloat16*>(o);
  ap.lse = lse;
  ap.status = reinterpret_cast<uint32_t*>(c.sw + c.S.off_status);
  ap.BH = c.BH; ap.NB = c.M.NB; ap.T = problem->T; ap.H = problem->H; ap.W = problem->W;
  ap.N = c.N;
  ap.scale_log2 = 1.4426950408889634f / sqrtf((float)c.d);
  ap.q_inv = q_inv; ap.k_inv = k_inv; ap.v_inv = v_inv;
  return cuda_status(bounded_rows(po) ? launch_attn_fwd_solo_fp8(c.d, po.block, maps, ap, c.st)
                                      : launch_attn_fwd_fp8(c.d, po.block, maps, ap, c.st));
}

extern "C" int sparse_attn_export_bytes(const sa_problem* problem, const sa_policy* policy,
                                        int what, size_t* bytes) {
  int e = check_problem(problem);
  if (e) return e;
  e = check_policy(*problem, policy);
  if (e) return e;
  if (!bytes) return SA_ERR_INVALID_ARG;
  const MaskLayout M = mask_layout(*problem, *policy);
  switch (what) {
    case SA_EXPORT_BLOCK_BITS: *bytes = sizeof(uint32_t) * (size_t)M.BH * M.NB * M.W32; break;
    case SA_EXPORT_HEAD_INFO: *bytes = sizeof(HeadGeom) * (size_t)M.BH; break;
    case SA_EXPORT_FG_BITS: *bytes = sizeof(uint32_t) * (size_t)M.BH * M.G * M.WN; break;
    case SA_EXPORT_FG_TAU: *bytes = policy->kind == SA_MASK_FG ? sizeof(float) * M.BH : 0; break;
    case SA_EXPORT_FG_TILE_KEYS: *bytes = sizeof(uint32_t) * (size_t)M.BH * M.P; break;
    default: return SA_ERR_INVALID_ARG;
  }
  return SA_OK;
}

extern "C" int sparse_attn_mask_export(const sa_problem* problem, const sa_policy* policy,
                                       const void* mask_ws, int what, void* host_dst,
                                       size_t bytes, void* stream) {
  size_t need = 0;
  int e = sparse_attn_export_bytes(problem, policy, what, &need);
  if (e) return e;
  if (!host_dst || bytes != need || !aligned(mask_ws, 256)) return SA_ERR_INVALID_ARG;
  const MaskLayout M = mask_layout(*problem, *policy);
  size_t off = 0;
  switch (what) {
    case SA_EXPORT_BLOCK_BITS: off = M.off_bits; break;
    case SA_EXPORT_HEAD_INFO: off = M.off_head; break;
    case SA_EXPORT_FG_BITS: off = M.off_fg_bits; break;
    case SA_EXPORT_FG_TAU: off = M.off_fg_tau; break;
    case SA_EXPORT_FG_TILE_KEYS: off = M.off_fg_counts; break;
  }
  if (need == 0) return SA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host_dst, static_cast<const uint8_t*>(mask_ws) + off, need,
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SA_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(st));
}

// ------------------------------------------------------------------ sampled rows
namespace {

// Scratch of the sampled-row calls: status words, the gathered query rows
// [BH][n_pad][d] bf16 (n_pad = n_rows rounded up to 128), and the full pass's
// fp32 O [BH][n_rows][d].
struct SampledLayout {
  size_t off_status = 0, off_qg = 0, off_ofull = 0, total = 0;
  int n_pad = 0;
};

SampledLayout sampled_layout(const sa_problem& pr, int n_rows) {
  SampledLayout L;
  const size_t BH = (size_t)pr.batch * pr.heads, d = (size_t)pr.head_dim;
  L.n_pad = ceil_div(n_rows, 128) * 128;
  L.off_status = 0;
  L.off_qg = 256;
  L.off_ofull = align_up(L.off_qg + BH * L.n_pad * d * 2, 256);
  L.total = align_up(L.off_ofull + BH * (size_t)n_rows * d * 4, 256);
  return L;
}

// The full pass of both sampled-row calls on the block-sparse attention
// kernel: gather the sampled rows into 128-row query tiles, then attend every
// tile to every key block of the identity layout, O in fp32.
int sampled_full_pass(const sa_problem& pr, const void* q, const void* k, const void* v,
                      const int32_t* rows, int n_rows, uint8_t* sw, cudaStream_t st,
                      const float** o_full) {
  if (!encode_fn()) return SA_ERR_CUDA;
  const SampledLayout L = sampled_layout(pr, n_rows);
  const int BH = pr.batch * pr.heads, d = pr.head_dim;
  const int N = (int)n_tokens(pr);
  uint32_t* status = reinterpret_cast<uint32_t*>(sw + L.off_status);
  __nv_bfloat16* qg = reinterpret_cast<__nv_bfloat16*>(sw + L.off_qg);
  float* of = reinterpret_cast<float*>(sw + L.off_ofull);
  if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return SA_ERR_CUDA;
  int e = cuda_status(launch_gather_rows(static_cast<const __nv_bfloat16*>(q), rows, BH, N, d,
                                         n_rows, L.n_pad, qg, status, st));
  if (e) return e;
  AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!map_3d(&maps.q[0], qg, BH, L.n_pad, d, 128) || !map_3d(&maps.k[0], k, BH, N, d, 128) ||
      !map_3d(&maps.v[0], v, BH, N, d, 128))
    return SA_ERR_CUDA;
  AttnParams ap{};
  ap.heads = nullptr;
  HeadGeom g{};
  g.layout = SA_LAYOUT_IDENTITY;
  g.bt = 1; g.bh = 1; g.bw = 128;
  g.nb = ceil_div(N, 128);
  g.nt = 1; g.nh = 1; g.nw = g.nb;
  ap.geo0 = g;
  ap.dense = 1;
  ap.q_tiles = L.n_pad / 128;
  ap.q_rows = n_rows;
  ap.o_f32 = of;
  ap.status = status;
  ap.BH = BH; ap.NB = ap.q_tiles; ap.T = pr.T; ap.H = pr.H; ap.W = pr.W; ap.N = N;
  ap.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  e = cuda_status(launch_attn_fwd(d, 128, maps, ap, st));
  if (e) return e;
  *o_full = of;
  return SA_OK;
}

}  // namespace

extern "C" int sparse_attn_profile_workspace_size(const sa_problem* problem, int n_rows,
                                                  size_t* bytes) {
  int e = check_problem(problem);
  if (e) return e;
  if (!bytes || n_rows < 1 || n_rows > n_tokens(*problem)) return SA_ERR_INVALID_ARG;
  *bytes = sampled_layout(*problem, n_rows).total;
  return SA_OK;
}

extern "C" int sparse_attn_profile_heads(const sa_problem* problem, const sa_policy* policy,
                                         const void* q, const void* k, const void* v,
                                         const int32_t* rows, int n_rows, float* row_err,
                                         float* mse, int8_t* is_temporal, void* scratch_ws,
                                         void* stream) {
  int e = check_problem(problem);
  if (e) return e;
  if (!policy || policy->kind != SA_MASK_SPATIOTEMPORAL) return SA_ERR_INVALID_ARG;
  const sa_problem& pr = *problem;
  const sa_policy& po = *policy;
  if (po.block != 128 && !(po.block == 64 && pr.head_dim == 64)) return SA_ERR_UNSUPPORTED;
  if (po.sink_tokens < 0 || po.frame_radius < 0) return SA_ERR_INVALID_ARG;
  const long long N = n_tokens(pr);
  if (n_rows < 1 || n_rows > N) return SA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return SA_ERR_INVALID_ARG;
  if (!aligned(rows, 4) || !aligned(row_err, 4) || !aligned(mse, 4) || !is_temporal)
    return SA_ERR_INVALID_ARG;
  if (!scratch_ws || !aligned(scratch_ws, 256)) return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float* o_full = nullptr;
  e = sampled_full_pass(pr, q, k, v, rows, n_rows, static_cast<uint8_t*>(scratch_ws), st, &o_full);
  if (e) return e;
  ProfileParams pp{};
  pp.o_full = o_full;
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.rows = rows;
  pp.row_err = row_err;
  pp.mse = mse;
  pp.choice = is_temporal;                    // pattern 1 (temporal) beats pattern 0
  pp.mode = 0;
  pp.n_pat = 2;
  pp.tile[0] = pp.tile[1] = 1;
  pp.tile[2] = po.block;
  pp.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(scratch_ws) +
                                         sampled_layout(pr, n_rows).off_status);
  pp.BH = pr.batch * pr.heads;
  pp.N = (int)N; pp.T = pr.T; pp.H = pr.H; pp.W = pr.W; pp.d = pr.head_dim;
  pp.n_rows = n_rows;
  pp.block = po.block;
  pp.sink_blocks = ceil_div(po.sink_tokens, po.block);
  pp.frame_radius = po.frame_radius;
  pp.scale_log2 = 1.4426950408889634f / sqrtf((float)pr.head_dim);
  return cuda_status(launch_profile(pp, st));
}

extern "C" int sparse_attn_sta_window_search(const sa_problem* problem, const sa_policy* policy,
                                             const void* q, const void* k, const void* v,
                                             const int32_t* rows, int n_rows,
                                             const int* candidates, int n_candidates,
                                             float* row_err, float* mse, int8_t* choice,
                                             void* scratch_ws, void* stream) {
  int e = check_problem(problem);
  if (e) return e;
  if (!policy || policy->kind != SA_MASK_STA) return SA_ERR_INVALID_ARG;
  const sa_problem& pr = *problem;
  const sa_policy& po = *policy;
  if (po.block != 128 && !(po.block == 64 && pr.head_dim == 64)) return SA_ERR_UNSUPPORTED;
  if ((e = check_tile(pr, po.tile, po.block))) return e;
  if (!candidates || n_candidates < 1 || n_candidates > kProfileMaxPatterns) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3 * n_candidates; ++i)
    if (candidates[i] < 1 || candidates[i] % 2 == 0 || candidates[i] > 255) return SA_ERR_INVALID_ARG;
  const long long N = n_tokens(pr);
  if (n_rows < 1 || n_rows > N) return SA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return SA_ERR_INVALID_ARG;
  if (!aligned(rows, 4) || !aligned(row_err, 4) || !aligned(mse, 4) || !choice)
    return SA_ERR_INVALID_ARG;
  if (!scratch_ws || !aligned(scratch_ws, 256)) return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float* o_full = nullptr;
  e = sampled_full_pass(pr, q, k, v, rows, n_rows, static_cast<uint8_t*>(scratch_ws), st, &o_full);
  if (e) return e;
  ProfileParams pp{};
  pp.o_full = o_full;
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.rows = rows;
  pp.row_err = row_err;
  pp.mse = mse;
  pp.choice = choice;
  pp.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(scratch_ws) +
                                         sampled_layout(pr, n_rows).off_status);
  pp.BH = pr.batch * pr.heads;
  pp.N = (int)N; pp.T = pr.T; pp.H = pr.H; pp.W = pr.W; pp.d = pr.head_dim;
  pp.n_rows = n_rows;
  pp.block = po.block;
  pp.mode = 1;
  pp.n_pat = n_candidates;
  for (int i = 0; i < 3; ++i) pp.tile[i] = po.tile[i];
  for (int c = 0; c < n_candidates; ++c)
    for (int i = 0; i < 3; ++i) pp.win[c][i] = candidates[3 * c + i];
  pp.scale_log2 = 1.4426950408889634f / sqrtf((float)pr.head_dim);
  return cuda_status(launch_profile(pp, st));
}

extern "C" int sparse_attn_quantize_e4m3(const void* x, long long n_elems, int n_tensors,
                                         uint8_t* codes, float* inv, void* stream) {
  if (n_elems < 8 || n_elems % 8 != 0 || n_tensors < 1 || n_tensors > 65535)
    return SA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(inv, 4)) return SA_ERR_INVALID_ARG;
  QuantParams qp{};
  qp.x = static_cast<const __nv_bfloat16*>(x);
  qp.codes = codes;
  qp.inv = inv;
  qp.n_elems = n_elems;
  qp.n_tensors = n_tensors;
  return cuda_status(launch_quant_e4m3(qp, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int sparse_attn_status(void* scratch_ws, void* stream, int clear) {
  if (!aligned(scratch_ws, 256)) return SA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, scratch_ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
  if (clear) {
    if (cudaMemsetAsync(scratch_ws, 0, 256, st) != cudaSuccess) return SA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
  }
  if (word & SA_DEVFLAG_TIMEOUT) return SA_ERR_DEVICE_TIMEOUT;
  if (word & SA_DEVFLAG_BOUNDS) return SA_ERR_DEVICE_BOUNDS;
  return SA_OK;
}

extern "C" const char* sparse_attn_strerror(int status) {
  switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported problem or policy";
    case SA_ERR_WORKSPACE: return "workspace pointer not 256-byte aligned";
    case SA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case SA_ERR_DEVICE_TIMEOUT: return "a device-side wait ran out (kernel gave up)";
    case SA_ERR_DEVICE_BOUNDS: return "a device-side index check failed";
    default: return "unknown status";
  }
}
