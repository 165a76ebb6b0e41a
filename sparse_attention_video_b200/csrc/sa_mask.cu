// Mask construction kernels for block-sparse policies (sm_100a, CUDA cores).
//
//   head_init      per-head working-layout geometry for static policies
//   permute_fm     token-major -> frame-major copy of Q, K, V for temporal heads
//   pool_sics      per block: mean of Q, mean of K, and SICS of K, for every
//                  blocking candidate (one pass over the block's tokens)
//   choose         per head: argmax over candidates of summed SICS
//   pooled_scores  per head: qbar_i . kbar_j / sqrt(d) over the chosen blocks
//   select         per query block: Top-K / Top-P + window / static rules,
//                  emitted as a bit row and an ascending list of key blocks
//
// All reductions run in a fixed order, so every result is deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sa_mask.h"
#include "sa_ptx.cuh"

namespace sa {

namespace {

__device__ __forceinline__ int tile_slot_token(int bt, int bh, int bw, int nh, int nw, int blk,
                                               int s, int T, int H, int W) {
  const int tw = blk % nw, th = (blk / nw) % nh, tt = blk / (nw * nh);
  const int lw = s % bw, lh = (s / bw) % bh, lt = s / (bw * bh);
  const int t = tt * bt + lt, h = th * bh + lh, w = tw * bw + lw;
  if (t >= T || h >= H || w >= W) return -1;
  return (t * H + h) * W + w;
}

// ------------------------------------------------------------------ head_init
__global__ void head_init_kernel(HeadInitParams p) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= p.BH) return;
  const int head = bh % p.heads;
  HeadGeom g{};
  const int N = p.T * p.H * p.W;
  int layout = p.layout;
  if (p.has_temporal_bits) {
    const bool temporal = (p.temporal_bits[head / 32] >> (head % 32)) & 1u;
    layout = temporal ? SA_LAYOUT_FRAME_MAJOR : SA_LAYOUT_IDENTITY;
  }
  g.layout = layout;
  g.cand = 0;
  if (layout == SA_LAYOUT_TILE) {
    g.bt = p.bt; g.bh = p.bh; g.bw = p.bw;
    g.nt = (p.T + p.bt - 1) / p.bt; g.nh = (p.H + p.bh - 1) / p.bh; g.nw = (p.W + p.bw - 1) / p.bw;
    g.nb = g.nt * g.nh * g.nw;
  } else {
    g.bt = 1; g.bh = 1; g.bw = p.block;
    g.nb = (N + p.block - 1) / p.block;
    g.nt = 1; g.nh = 1; g.nw = g.nb;
  }
  g.kept = 0;
  g.window = p.has_windows ? p.windows[head] : 0;
  p.geo[bh] = g;
}

// ------------------------------------------------------------------ permute_fm
// dst[bh][m] = src[bh][n(m)] for slot m of the frame-major order, zero rows for
// slots m >= N. One 16-byte vector per thread; rows are 2*d bytes.
__global__ void permute_fm_kernel(PermuteParams p) {
  const int bh = blockIdx.y;
  if (p.heads[bh].layout != SA_LAYOUT_FRAME_MAJOR) return;
  const int vec_per_row = p.d / 8;
  const int rows_per_cta = blockDim.x / vec_per_row;
  const int r = blockIdx.x * rows_per_cta + threadIdx.x / vec_per_row;
  const int c = threadIdx.x % vec_per_row;
  if (r >= p.n_pad) return;
  const int N = p.T * p.H * p.W;
  uint4 val[3] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  if (r < N) {
    const int pos = r / p.T, t = r - pos * p.T;
    const size_t src_row = (size_t)bh * N + (size_t)t * (p.H * p.W) + pos;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      val[i] = __ldg(reinterpret_cast<const uint4*>(p.src[i] + src_row * p.d) + c);
  }
  const size_t dst_row = (size_t)bh * p.n_pad + r;
#pragma unroll
  for (int i = 0; i < 3; ++i) reinterpret_cast<uint4*>(p.dst[i] + dst_row * p.d)[c] = val[i];
}

// ------------------------------------------------------------------ pool_sics
// One warp per (block, candidate, head), 8 warps per CTA. Half-warp h of the
// warp takes tokens h, h+2, h+4, ... of the block; lane i of a half-warp owns
// dimensions 8i..8i+7 (16-byte loads, one 256-byte row per half-warp), four
// token pairs in flight per step. Row norms come from shuffles inside the
// half-warp; the two halves are combined by one shuffle at the end. Every sum
// runs in a fixed order.
constexpr int kMaxPoolBlock = 128;   // tokens per block (64 or 128)

// Block summaries (SA_SUMMARIZER_*): the per-channel sum of the valid tokens
// (divided by their count at the end: the mean), or their maximum / minimum.
template <int kSum>
__device__ __forceinline__ float summ_init() {
  return kSum == SA_SUMMARIZER_MAX ? -INFINITY : (kSum == SA_SUMMARIZER_MIN ? INFINITY : 0.f);
}
template <int kSum>
__device__ __forceinline__ float summ_add(float a, float b) {
  return kSum == SA_SUMMARIZER_MAX ? fmaxf(a, b) : (kSum == SA_SUMMARIZER_MIN ? fminf(a, b) : a + b);
}
template <int kSum>
__device__ __forceinline__ float summ_final(float a, int n, float inv_n) {
  return n == 0 ? 0.f : (kSum == SA_SUMMARIZER_MEAN ? a * inv_n : a);
}

template <int D, int kSum>
__global__ void __launch_bounds__(256) pool_sics_kernel(PoolParams p) {
  static_assert(D == 128 || D == 64, "head_dim");
  constexpr int CH = D / 8;                 // lanes per token (16 or 8)
  constexpr int TPW = 32 / CH;              // tokens per warp step (2 or 4)
  constexpr int UNROLL = 4;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = blockIdx.x, region = blockIdx.y, bh = blockIdx.z;
  const int bt = p.cand[c][0], bhh = p.cand[c][1], bw = p.cand[c][2];
  const int nt = (p.T + bt - 1) / bt, nh = (p.H + bhh - 1) / bhh, nw = (p.W + bw - 1) / bw;
  // Local block ``warp`` of this candidate inside the region (regions are the
  // least common multiple of every candidate's tile, so each holds whole
  // blocks of every candidate; the candidates' CTAs of one region run next to
  // each other and read the same tokens while they are in L2).
  const int rw = region % p.nRw, rh = (region / p.nRw) % p.nRh, rt = region / (p.nRw * p.nRh);
  const int mt = p.Rt / bt, mh = p.Rh / bhh, mw = p.Rw / bw;
  __shared__ int slot_tok[8][kMaxPoolBlock];
  for (int lb = warp; lb < mt * mh * mw; lb += 8) {
  const int lw = lb % mw, lh = (lb / mw) % mh, lt = lb / (mw * mh);
  const int tt = rt * mt + lt, th = rh * mh + lh, tw = rw * mw + lw;
  if (tt >= nt || th >= nh || tw >= nw) continue;
  const int blk = (tt * nh + th) * nw + tw;
  const int BS = bt * bhh * bw;
  const int tl = lane / CH, dc = lane % CH;
  const int N = p.T * p.H * p.W;
  const __nv_bfloat16* q = p.q + (size_t)bh * N * D;
  const __nv_bfloat16* k = p.k + (size_t)bh * N * D;
  // token index of every slot of this warp's block, computed once (the
  // divisions by runtime tile sizes stay out of the streaming loop)
  int* st = slot_tok[warp];
  __syncwarp();
  for (int s = lane; s < BS; s += 32) st[s] = tile_slot_token(bt, bhh, bw, nh, nw, blk, s, p.T, p.H, p.W);
  __syncwarp();

  float qs[8], ks[8], us[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { qs[i] = summ_init<kSum>(); ks[i] = summ_init<kSum>(); us[i] = 0.f; }
  int n_valid = 0, n_unit = 0;
  for (int s0 = 0; s0 < BS; s0 += TPW * UNROLL) {
    uint4 qv[UNROLL], kv[UNROLL];
    int tok[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int s = s0 + u * TPW + tl;
      tok[u] = s < BS ? st[s] : -1;
      qv[u] = make_uint4(0, 0, 0, 0);
      kv[u] = make_uint4(0, 0, 0, 0);
      if (tok[u] >= 0) {
        qv[u] = __ldg(reinterpret_cast<const uint4*>(q + (size_t)tok[u] * D) + dc);
        kv[u] = __ldg(reinterpret_cast<const uint4*>(k + (size_t)tok[u] * D) + dc);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const __nv_bfloat16* qe = reinterpret_cast<const __nv_bfloat16*>(&qv[u]);
      const __nv_bfloat16* ke = reinterpret_cast<const __nv_bfloat16*>(&kv[u]);
      float kf[8], ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        kf[i] = __bfloat162float(ke[i]);
        ss = fmaf(kf[i], kf[i], ss);
      }
      // every lane joins; pad slots carry zeros
#pragma unroll
      for (int o = CH / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (tok[u] < 0) continue;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        qs[i] = summ_add<kSum>(qs[i], __bfloat162float(qe[i]));
        ks[i] = summ_add<kSum>(ks[i], kf[i]);
      }
      ++n_valid;
      if (ss > 0.f) {
        // one correctly rounded 1/||k|| per token, then products: within about
        // one ulp of k_i / ||k|| per component
        const float rn = 1.0f / sqrtf(ss);
#pragma unroll
        for (int i = 0; i < 8; ++i) us[i] = fmaf(kf[i], rn, us[i]);
        ++n_unit;
      }
    }
  }
  // combine the token lanes of the warp (same dimensions, lanes dc + CH*t)
#pragma unroll
  for (int o = CH; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qs[i] = summ_add<kSum>(qs[i], __shfl_xor_sync(0xffffffffu, qs[i], o));
      ks[i] = summ_add<kSum>(ks[i], __shfl_xor_sync(0xffffffffu, ks[i], o));
      us[i] += __shfl_xor_sync(0xffffffffu, us[i], o);
    }
    n_valid += __shfl_xor_sync(0xffffffffu, n_valid, o);
    n_unit += __shfl_xor_sync(0xffffffffu, n_unit, o);
  }
  // every lane of a token group counted that group's tokens, so summing over
  // the groups gives each lane the block's counts
  const size_t base = (((size_t)bh * p.C + c) * p.NB + blk);
  float usq = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) usq = fmaf(us[i], us[i], usq);
#pragma unroll
  for (int o = CH / 2; o >= 1; o >>= 1) usq += __shfl_xor_sync(0xffffffffu, usq, o);
  if (tl == 0) {
    const float nv = (float)n_valid;
    float* qo = p.qbar + base * D + dc * 8;
    float* ko = p.kbar + base * D + dc * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if constexpr (kSum == SA_SUMMARIZER_MEAN) {
        qo[i] = n_valid ? qs[i] / nv : 0.f;
        ko[i] = n_valid ? ks[i] / nv : 0.f;
      } else {
        qo[i] = n_valid ? qs[i] : 0.f;
        ko[i] = n_valid ? ks[i] : 0.f;
      }
    }
    if (dc == 0) p.sics[base] = usq - (float)n_unit;
  }
  }
}

// One pass over Q and K for every blocking candidate at once. A region (the
// least common multiple of the candidates' tiles) is cut into atoms, the
// greatest common divisor of the tiles along each axis: every atom lies in
// exactly one block of every candidate. Warps stream the atoms' tokens once
// (q, k, and the unit vector k / ||k|| with one approximate reciprocal
// square root per token), keep per-atom sums in shared memory, then every
// candidate block adds up its atoms: its mean q, mean k and
// SICS = ||sum of unit vectors||^2 - (number of nonzero keys).
constexpr int kPoolAtomThreads = 256;     // 8 warps; two CTAs per SM (shared memory)

// One token's 8 dimensions held by this lane (CH = D/8 lanes per token):
// the summaries of q and k, and the unit vector k / ||k|| for SICS. Every
// lane joins the ||k||^2 shuffles; lanes of a missing token (zeros) then add
// nothing.
template <int D, int kSum>
__device__ __forceinline__ void pool_token(const uint4& qv, const uint4& kv, bool valid,
                                           float (&qs)[8], float (&ks)[8], float (&us)[8],
                                           int& n_valid, int& n_unit) {
  constexpr int CH = D / 8;
  // bf16 -> fp32 is a shift: element 2e in the low half of word e
  const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
  const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
  float kf[8], qf[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    kf[2 * e] = __uint_as_float(kw[e] << 16);
    kf[2 * e + 1] = __uint_as_float(kw[e] & 0xFFFF0000u);
    qf[2 * e] = __uint_as_float(qw[e] << 16);
    qf[2 * e + 1] = __uint_as_float(qw[e] & 0xFFFF0000u);
  }
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    fma2(kf[2 * e], kf[2 * e + 1], kf[2 * e], kf[2 * e + 1], s0, s1, s0, s1);
  float ss = s0 + s1;
#pragma unroll
  for (int o = CH / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (!valid) return;
  if constexpr (kSum == SA_SUMMARIZER_MEAN) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      add2(qs[2 * e], qs[2 * e + 1], qf[2 * e], qf[2 * e + 1]);
      add2(ks[2 * e], ks[2 * e + 1], kf[2 * e], kf[2 * e + 1]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qs[i] = summ_add<kSum>(qs[i], qf[i]);
      ks[i] = summ_add<kSum>(ks[i], kf[i]);
    }
  }
  ++n_valid;
  if (ss > 0.f) {
    // approximate reciprocal square root (MUFU): the unit vectors differ
    // from k / sqrt(|k|^2) by a few ulp
    const float rn = rsqrtf(ss);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      fma2(kf[2 * e], kf[2 * e + 1], rn, rn, us[2 * e], us[2 * e + 1], us[2 * e], us[2 * e + 1]);
    ++n_unit;
  }
}

// The lanes of a warp's token groups combined (same dimensions, lanes
// dc + CH*t), then group 0 writes atom ``a``'s summaries.
template <int D, int kSum>
__device__ __forceinline__ void pool_store_atom(float* sums, int* cnt, int a, int lane,
                                                float (&qs)[8], float (&ks)[8], float (&us)[8],
                                                int n_valid, int n_unit) {
  constexpr int CH = D / 8;
  const int tl = lane / CH, dc = lane % CH;
#pragma unroll
  for (int o = CH; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qs[i] = summ_add<kSum>(qs[i], __shfl_xor_sync(0xffffffffu, qs[i], o));
      ks[i] = summ_add<kSum>(ks[i], __shfl_xor_sync(0xffffffffu, ks[i], o));
      us[i] += __shfl_xor_sync(0xffffffffu, us[i], o);
    }
    n_valid += __shfl_xor_sync(0xffffffffu, n_valid, o);
    n_unit += __shfl_xor_sync(0xffffffffu, n_unit, o);
  }
  if (tl == 0) {
    float* sa = sums + (size_t)a * 3 * D + dc * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) { sa[i] = qs[i]; sa[D + i] = ks[i]; sa[2 * D + i] = us[i]; }
    if (dc == 0) { cnt[2 * a] = n_valid; cnt[2 * a + 1] = n_unit; }
  }
}

// Every block of every candidate inside the region from the per-atom
// summaries: one warp per block, each lane D/32 dimensions.
template <int D, int kSum>
__device__ __forceinline__ void pool_combine(const PoolParams& p, const float* sums, const int* cnt,
                                             int warp, int lane, int rt, int rh, int rw, int bh,
                                             int mAh, int mAw) {
  constexpr int kWarps = kPoolAtomThreads / 32;
  constexpr int DL = D / 32;
  int first[kMaxCand + 1];
  first[0] = 0;
  for (int c = 0; c < p.C; ++c)
    first[c + 1] = first[c] + (p.Rt / p.cand[c][0]) * (p.Rh / p.cand[c][1]) * (p.Rw / p.cand[c][2]);
  for (int pi = warp; pi < first[p.C]; pi += kWarps) {
    int c = 0;
    while (pi >= first[c + 1]) ++c;
    const int bt = p.cand[c][0], bhh = p.cand[c][1], bw = p.cand[c][2];
    const int lb = pi - first[c];
    const int mw = p.Rw / bw, mh = p.Rh / bhh;
    const int lw = lb % mw, lh = (lb / mw) % mh, lt = lb / (mw * mh);
    const int nt = (p.T + bt - 1) / bt, nh = (p.H + bhh - 1) / bhh, nw = (p.W + bw - 1) / bw;
    const int tt = rt * (p.Rt / bt) + lt, th = rh * (p.Rh / bhh) + lh, tw = rw * (p.Rw / bw) + lw;
    if (tt >= nt || th >= nh || tw >= nw) continue;    // warp-uniform
    const int blk = (tt * nh + th) * nw + tw;
    float qv[DL], kv[DL], uv[DL];
#pragma unroll
    for (int i = 0; i < DL; ++i) { qv[i] = summ_init<kSum>(); kv[i] = summ_init<kSum>(); uv[i] = 0.f; }
    int nv = 0, nu = 0;
    const int ft = bt / p.At, fh = bhh / p.Ah, fw = bw / p.Aw;   // atoms per block along each axis
    for (int xt = 0; xt < ft; ++xt)
      for (int xh = 0; xh < fh; ++xh) {
        const int arow = ((lt * ft + xt) * mAh + (lh * fh + xh)) * mAw + lw * fw;
        for (int xw = 0; xw < fw; ++xw) {
          const int a = arow + xw;
          const float* sa = sums + (size_t)a * 3 * D + lane * DL;
#pragma unroll
          for (int i = 0; i < DL; ++i) {
            qv[i] = summ_add<kSum>(qv[i], sa[i]);
            kv[i] = summ_add<kSum>(kv[i], sa[D + i]);
            uv[i] += sa[2 * D + i];
          }
          nv += cnt[2 * a];
          nu += cnt[2 * a + 1];
        }
      }
    const size_t base = (((size_t)bh * p.C + c) * p.NB + blk);
    const float inv = nv ? 1.f / (float)nv : 0.f;
    float usq = 0.f;
#pragma unroll
    for (int i = 0; i < DL; ++i) {
      p.qbar[base * D + lane * DL + i] = summ_final<kSum>(qv[i], nv, inv);
      p.kbar[base * D + lane * DL + i] = summ_final<kSum>(kv[i], nv, inv);
      usq = fmaf(uv[i], uv[i], usq);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) usq += __shfl_xor_sync(0xffffffffu, usq, o);
    if (lane == 0) p.sics[base] = usq - (float)nu;
  }
}

template <int D, int kSum>
__global__ void __launch_bounds__(kPoolAtomThreads, 2) pool_atoms_kernel(PoolParams p) {
  constexpr int CH = D / 8;                 // lanes per token (16 or 8)
  constexpr int TPW = 32 / CH;              // tokens per warp step (2 or 4)
  constexpr int UNROLL = 8;                 // a 16-token atom's rows all in flight
  extern __shared__ float pool_sm[];        // [nA][3][D] sums, then [nA][2] counts
  float* sums = pool_sm;
  int* cnt = reinterpret_cast<int*>(pool_sm + (size_t)p.nA * 3 * D);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int region = blockIdx.x, bh = blockIdx.y;
  const int rw = region % p.nRw, rh = (region / p.nRw) % p.nRh, rt = region / (p.nRw * p.nRh);
  const int t0 = rt * p.Rt, h0 = rh * p.Rh, w0 = rw * p.Rw;
  const int mAh = p.Rh / p.Ah, mAw = p.Rw / p.Aw;
  const int tl = lane / CH, dc = lane % CH;
  const int N = p.T * p.H * p.W;
  const __nv_bfloat16* q = p.q + (size_t)bh * N * D;
  const __nv_bfloat16* k = p.k + (size_t)bh * N * D;
  // This lane's first token of an atom is token tl (atom order t, h, w); its
  // later ones follow TPW apart. The coordinates inside the atom are the same
  // for every atom, found once here and then advanced without division.
  const int iw0 = tl % p.Aw, ih0 = (tl / p.Aw) % p.Ah, it0 = tl / (p.Aw * p.Ah);

  constexpr int kWarps = kPoolAtomThreads / 32;
  // atom a = (at, ah, aw) of the region; this warp takes a = warp, warp + 8,
  // ... and advances the coordinates without division
  int aw = warp % mAw, ah = (warp / mAw) % mAh, at = warp / (mAw * mAh);
  for (int a = warp; a < p.nA; a += kWarps) {
    const int ta = t0 + at * p.At, ha = h0 + ah * p.Ah, wa = w0 + aw * p.Aw;
    aw += kWarps;
    while (aw >= mAw) {
      aw -= mAw;
      if (++ah == mAh) { ah = 0; ++at; }
    }
    if (ta >= p.T || ha >= p.H || wa >= p.W) {
      // an atom wholly in the padding: no token, so the identity summary
      if (tl == 0) {
        float* sa = sums + (size_t)a * 3 * D + dc * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) { sa[i] = summ_init<kSum>(); sa[D + i] = summ_init<kSum>(); sa[2 * D + i] = 0.f; }
        if (dc == 0) { cnt[2 * a] = 0; cnt[2 * a + 1] = 0; }
      }
      continue;
    }
    float qs[8], ks[8], us[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { qs[i] = summ_init<kSum>(); ks[i] = summ_init<kSum>(); us[i] = 0.f; }
    int n_valid = 0, n_unit = 0;
    int iw = iw0, ih = ih0, it = it0;
    // the warp's lanes stay in step: it < At for some lane until the last step
    while (__any_sync(0xffffffffu, it < p.At)) {
      uint4 qv[UNROLL], kv[UNROLL];
      int tok[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int t = ta + it, h = ha + ih, w = wa + iw;
        tok[u] = (it < p.At && t < p.T && h < p.H && w < p.W) ? (t * p.H + h) * p.W + w : -1;
        iw += TPW;
        while (iw >= p.Aw) {
          iw -= p.Aw;
          if (++ih == p.Ah) { ih = 0; ++it; }
        }
        qv[u] = make_uint4(0, 0, 0, 0);
        kv[u] = make_uint4(0, 0, 0, 0);
        if (tok[u] >= 0) {
          qv[u] = __ldg(reinterpret_cast<const uint4*>(q + (size_t)tok[u] * D) + dc);
          kv[u] = __ldg(reinterpret_cast<const uint4*>(k + (size_t)tok[u] * D) + dc);
        }
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u)
        pool_token<D, kSum>(qv[u], kv[u], tok[u] >= 0, qs, ks, us, n_valid, n_unit);
    }
    pool_store_atom<D, kSum>(sums, cnt, a, lane, qs, ks, us, n_valid, n_unit);
  }
  __syncthreads();

  pool_combine<D, kSum>(p, sums, cnt, warp, lane, rt, rh, rw, bh, mAh, mAw);
}

// ------------------------------------------------------------------ choose
__global__ void choose_kernel(ChooseParams p) {
  const int bh = blockIdx.x;
  __shared__ double part[256];
  __shared__ double totals[kMaxCand];
  for (int c = 0; c < p.C; ++c) {
    const int bt = p.cand[c][0], bhh = p.cand[c][1], bw = p.cand[c][2];
    const int nb = ((p.T + bt - 1) / bt) * ((p.H + bhh - 1) / bhh) * ((p.W + bw - 1) / bw);
    double s = 0.0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x)
      s += (double)p.sics[((size_t)bh * p.C + c) * p.NB + b];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w >= 1; w >>= 1) {
      if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) totals[c] = part[0];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int best = 0;
    for (int c = 1; c < p.C; ++c) {
      const double a = totals[best], b = totals[c];
      if (b > a + 1e-4 * fmax(fabs(a), fabs(b))) best = c;
    }
    HeadGeom g{};
    g.layout = SA_LAYOUT_TILE;
    g.cand = best;
    g.bt = p.cand[best][0]; g.bh = p.cand[best][1]; g.bw = p.cand[best][2];
    g.nt = (p.T + g.bt - 1) / g.bt; g.nh = (p.H + g.bh - 1) / g.bh; g.nw = (p.W + g.bw - 1) / g.bw;
    g.nb = g.nt * g.nh * g.nw;
    g.kept = 0;
    for (int c = 0; c < kMaxCand; ++c) g.sics_total[c] = c < p.C ? (float)totals[c] : 0.f;
    p.heads[bh] = g;
  }
}

// ------------------------------------------------------------------ pooled_scores
// 64 x 64 output tile per CTA, 256 threads, 4 x 4 outputs per thread. Each
// output is a sequential fp32 FMA chain over the d components.
template <int D>
__global__ void __launch_bounds__(256) pooled_scores_kernel(ScoreParams p) {
  const int bh = blockIdx.z;
  const HeadGeom g = p.heads[bh];
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  if (i0 >= g.nb || j0 >= g.nb) return;
  extern __shared__ float sm[];
  float* sq = sm;              // [64][D+1]
  float* sk = sm + 64 * (D + 1);
  const size_t cbase = ((size_t)bh * p.C + g.cand) * p.NB;
  for (int e = threadIdx.x; e < 64 * D; e += 256) {
    const int r = e / D, c = e % D;
    sq[r * (D + 1) + c] = (i0 + r < g.nb) ? p.qbar[(cbase + i0 + r) * D + c] : 0.f;
    sk[r * (D + 1) + c] = (j0 + r < g.nb) ? p.kbar[(cbase + j0 + r) * D + c] : 0.f;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int c = 0; c < D; ++c) {
    float qa[4], kb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) qa[a] = sq[(ty + 16 * a) * (D + 1) + c];
#pragma unroll
    for (int b = 0; b < 4; ++b) kb[b] = sk[(tx + 16 * b) * (D + 1) + c];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qa[a], kb[b], acc[a][b]);
  }
  const float rs = p.sqrt_d;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
      if (i < g.nb && j < g.nb) p.scores[((size_t)bh * p.NB + i) * p.NB + j] = acc[a][b] / rs;
    }
}

// ------------------------------------------------------------------ select
__device__ __forceinline__ bool block_valid(const HeadGeom& g, int blk, int T, int H, int W) {
  if (g.layout == SA_LAYOUT_TILE) {
    const int tw = blk % g.nw, th = (blk / g.nw) % g.nh, tt = blk / (g.nw * g.nh);
    return tt * g.bt < T && th * g.bh < H && tw * g.bw < W;
  }
  return blk * g.bw < T * H * W;
}

// Block-wide reductions over 256 threads (fixed tree).
__device__ __forceinline__ float block_max(float v, float* buf) {
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (threadIdx.x % 32 == 0) buf[threadIdx.x / 32] = v;
  __syncthreads();
  float r = buf[0];
  for (int i = 1; i < 8; ++i) r = fmaxf(r, buf[i]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_sum(float v, float* buf) {
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (threadIdx.x % 32 == 0) buf[threadIdx.x / 32] = v;
  __syncthreads();
  float r = buf[0];
  for (int i = 1; i < 8; ++i) r += buf[i];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256) select_kernel(SelectParams p) {
  const int i = blockIdx.x, bh = blockIdx.y;
  const HeadGeom g = p.heads[bh];
  if (i >= g.nb) return;
  __shared__ uint32_t bits[kMaxBlocks / 32];
  __shared__ uint32_t vbits[kMaxBlocks / 32];
  __shared__ float fbuf[8];
  const int nb = g.nb, W32 = (nb + 31) / 32;
  for (int w = threadIdx.x; w < W32; w += 256) { bits[w] = 0u; vbits[w] = 0u; }
  __syncthreads();
  // which key blocks hold at least one token, computed once per row
  for (int j = threadIdx.x; j < nb; j += 256)
    if (block_valid(g, j, p.T, p.H, p.W)) atomicOr(&vbits[j / 32], 1u << (j % 32));
  __syncthreads();
  auto kvalid = [&](int j) { return (vbits[j >> 5] >> (j & 31)) & 1u; };
  const bool qvalid = block_valid(g, i, p.T, p.H, p.W);
  const float* srow = p.scores ? p.scores + ((size_t)bh * p.NB + i) * p.NB : nullptr;

  if (qvalid) {
    if (p.kind == SA_MASK_TOPK) {
      // K rounds of block-wide argmax (score desc, index asc) over unchosen valid blocks.
      for (int r = 0; r < p.topk; ++r) {
        unsigned long long best = 0ull;
        for (int j = threadIdx.x; j < nb; j += 256) {
          if (!kvalid(j) || ((bits[j / 32] >> (j % 32)) & 1u)) continue;
          uint32_t f = __float_as_uint(srow[j]);
          f = (f & 0x80000000u) ? ~f : (f | 0x80000000u);         // order-preserving
          // nonzero for every non-NaN score, so 0 can stand for "none"
          const unsigned long long key = ((unsigned long long)f << 32) | (0xFFFFFFFFu - (uint32_t)j);
          if (key > best) best = key;
        }
        for (int o = 16; o >= 1; o >>= 1) {
          const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
          best = other > best ? other : best;
        }
        __shared__ unsigned long long wbest[8];
        if (threadIdx.x % 32 == 0) wbest[threadIdx.x / 32] = best;
        __syncthreads();
        if (threadIdx.x == 0) {
          unsigned long long b = 0ull;
          for (int w = 0; w < 8; ++w) b = wbest[w] > b ? wbest[w] : b;
          if (b) {
            const int j = (int)(0xFFFFFFFFu - (uint32_t)(b & 0xFFFFFFFFull));
            bits[j / 32] |= 1u << (j % 32);
          }
        }
        __syncthreads();
      }
      if (threadIdx.x == 0 && p.keep_diagonal && i < nb && block_valid(g, i, p.T, p.H, p.W))
        bits[i / 32] |= 1u << (i % 32);
    } else if (p.kind == SA_MASK_STA || p.kind == SA_MASK_SPADE) {
      // clipped tile window around query tile i (the head's own window if it has one)
      const int wwin = g.window;
      const int rt = (wwin ? (wwin & 0xFF) : p.win[0]) / 2;
      const int rh = (wwin ? ((wwin >> 8) & 0xFF) : p.win[1]) / 2;
      const int rw = (wwin ? ((wwin >> 16) & 0xFF) : p.win[2]) / 2;
      const int iw = i % g.nw, ih = (i / g.nw) % g.nh, it = i / (g.nw * g.nh);
      const int wt = 2 * rt + 1, wh = 2 * rh + 1, ww = 2 * rw + 1;
      for (int e = threadIdx.x; e < wt * wh * ww; e += 256) {
        const int jt = it - rt + e / (wh * ww), jh = ih - rh + (e / ww) % wh, jw = iw - rw + e % ww;
        if (jt < 0 || jh < 0 || jw < 0 || jt >= g.nt || jh >= g.nh || jw >= g.nw) continue;
        const int j = (jt * g.nh + jh) * g.nw + jw;
        if (kvalid(j)) atomicOr(&bits[j / 32], 1u << (j % 32));
      }
      __syncthreads();
      if (p.kind == SA_MASK_SPADE) {
        // Softmax over the valid key blocks, then the shortest prefix by
        // descending probability (ties to the lower index) whose mass reaches
        // top_p. The prefix is found by a radix select over the order key
        // (probability bits above the complemented block index), 8 bits per
        // level from the top: each level histograms the count and the mass of
        // the keys that share the prefix fixed so far, and the bin where the
        // mass (from the highest bin down) reaches what is still needed
        // becomes the new prefix. Masses are summed in 2^-31 fixed point
        // (every probability rounded to a multiple of 2^-31, at most 4,096 of
        // them: the total stays below 2^32), so the sums, and the cut, do not
        // depend on the order of the atomics; they differ from a float32
        // running sum by far less than that sum's own rounding.
        float mx = -INFINITY;
        for (int j = threadIdx.x; j < nb; j += 256)
          if (kvalid(j)) mx = fmaxf(mx, srow[j]);
        mx = block_max(mx, fbuf);
        // probabilities, once: exp(s - max) first, normalised below
        __shared__ float prob[kMaxBlocks];
        float se = 0.f;
        for (int j = threadIdx.x; j < nb; j += 256) {
          const float e = kvalid(j) ? expf(srow[j] - mx) : 0.f;
          prob[j] = e;
          se += e;
        }
        se = block_sum(se, fbuf);                       // ends with a barrier
        for (int j = threadIdx.x; j < nb; j += 256) prob[j] = prob[j] / se;
        __syncthreads();
        constexpr float kFix = 2147483648.f;            // 2^31
        // order key of valid block j: probability bits above ~j
        auto order_key = [&](int j) {
          return ((unsigned long long)__float_as_uint(prob[j]) << 32) | (0xFFFFFFFFu - (uint32_t)j);
        };
        auto mass = [&](int j) { return __float2uint_rn(prob[j] * kFix); };
        const uint32_t target = __float2uint_ru(p.top_p * kFix);
        __shared__ uint32_t h_mass[256], w_mass[8], s_above;
        __shared__ uint32_t h_cnt[256], s_cnt;
        __shared__ int s_bin, s_all;
        if (threadIdx.x == 0) s_all = 0;
        unsigned long long prefix = 0ull;                // fixed key bits
        uint32_t above = 0u;                             // mass of the keys above them
        int shift = 56;
        bool all = false;
        for (;; shift -= 8) {
          h_mass[threadIdx.x] = 0u;
          h_cnt[threadIdx.x] = 0u;
          __syncthreads();
          const unsigned long long hi = shift == 56 ? 0ull : (~0ull << (shift + 8));
          for (int j = threadIdx.x; j < nb; j += 256) {
            if (!kvalid(j)) continue;
            const unsigned long long k = order_key(j);
            if ((k & hi) == prefix) {
              const int bin = (int)((k >> shift) & 255u);
              atomicAdd(&h_mass[bin], mass(j));
              atomicAdd(&h_cnt[bin], 1u);
            }
          }
          __syncthreads();
          // thread t takes bin 255 - t: inclusive scan of the mass from the top bin
          const int bin = 255 - (int)threadIdx.x;
          const uint32_t m = h_mass[bin];
          uint32_t incl = m;
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if ((threadIdx.x & 31) >= (unsigned)o) incl += t;
          }
          if ((threadIdx.x & 31) == 31) w_mass[threadIdx.x >> 5] = incl;
          __syncthreads();
          for (int w = 0; w < (int)(threadIdx.x >> 5); ++w) incl += w_mass[w];
          const uint32_t need = target - above;            // > 0: above < target
          if (incl >= need && incl - m < need) {
            s_bin = bin;
            s_above = above + (incl - m);
            s_cnt = h_cnt[bin];
          }
          // the whole valid mass falls short of top_p (rounding): keep every valid block
          if (threadIdx.x == 255 && incl < need) s_all = 1;
          __syncthreads();
          if (s_all) { all = true; break; }
          prefix |= (unsigned long long)s_bin << shift;
          above = s_above;
          if (s_cnt == 1u || shift == 0) break;
        }
        // kept: every key at or above the cut's prefix
        for (int j = threadIdx.x; j < nb; j += 256)
          if (kvalid(j) && (all || (order_key(j) >> shift) >= (prefix >> shift)))
            atomicOr(&bits[j / 32], 1u << (j % 32));
      }
    } else if (p.kind == SA_MASK_SPATIOTEMPORAL) {
      const int N = p.T * p.H * p.W, BS = g.bw, HW = p.H * p.W;
      const int lo_i = i * BS, hi_i = min(N, lo_i + BS) - 1;
      for (int j = threadIdx.x; j < nb; j += 256) {
        const int lo_j = j * BS, hi_j = min(N, lo_j + BS) - 1;
        bool keep;
        if (g.layout == SA_LAYOUT_FRAME_MAJOR) {
          // shared spatial position: slot m holds position m / T
          keep = !(hi_j / p.T < lo_i / p.T || hi_i / p.T < lo_j / p.T);
        } else {
          // frame ranges within frame_radius
          const int fi0 = lo_i / HW, fi1 = hi_i / HW, fj0 = lo_j / HW, fj1 = hi_j / HW;
          const int gap = max(0, max(fj0 - fi1, fi0 - fj1));
          keep = gap <= p.frame_radius;
        }
        if (j < p.sink_blocks) keep = true;
        if (keep) atomicOr(&bits[j / 32], 1u << (j % 32));
      }
    } else if (p.kind == SA_MASK_EXPLICIT) {
      const uint32_t* src = p.explicit_bits + ((size_t)bh * p.NB + i) * p.W32;
      for (int w = threadIdx.x; w < W32; w += 256) {
        uint32_t word = src[w];
        if (32 * w + 32 > nb) word &= (nb - 32 * w) >= 32 ? 0xffffffffu : ((1u << (nb - 32 * w)) - 1u);
        for (int b = 0; b < 32; ++b)
          if (((word >> b) & 1u) && !kvalid(32 * w + b)) word &= ~(1u << b);
        bits[w] = word;
      }
    }
  }
  __syncthreads();
  // emit: bit row, ascending list, count
  uint32_t* brow = p.bits + ((size_t)bh * p.NB + i) * p.W32;
  for (int w = threadIdx.x; w < p.W32; w += 256) brow[w] = w < W32 ? bits[w] : 0u;
  __shared__ int wcount[kMaxBlocks / 32 + 1];
  for (int w = threadIdx.x; w < W32; w += 256) wcount[w] = __popc(bits[w]);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int w = 0; w < W32; ++w) { const int c = wcount[w]; wcount[w] = run; run += c; }
    wcount[W32] = run;
    p.counts[(size_t)bh * p.NB + i] = run;
    atomicAdd(&p.heads[bh].kept, run);
  }
  __syncthreads();
  int* crow = p.cols + ((size_t)bh * p.NB + i) * p.NB;
  for (int w = threadIdx.x; w < W32; w += 256) {
    uint32_t word = bits[w];
    int pos = wcount[w];
    while (word) {
      const int b = __ffs(word) - 1;
      if (dbg_in_range(pos, p.NB, p.status)) crow[pos] = 32 * w + b;
      ++pos;
      word &= word - 1;
    }
  }
}

__global__ void zero_counts_kernel(int* counts, size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x)
    counts[e] = 0;
}

}  // namespace

cudaError_t launch_head_init(const HeadInitParams& p, cudaStream_t st) {
  head_init_kernel<<<(p.BH + 127) / 128, 128, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_permute_fm(const PermuteParams& p, int BH, cudaStream_t st) {
  const int vec_per_row = p.d / 8;
  const int rows_per_cta = 256 / vec_per_row;
  dim3 grid((p.n_pad + rows_per_cta - 1) / rows_per_cta, BH);
  permute_fm_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <int D, int kSum>
static cudaError_t launch_pool(const PoolParams& p, int BH, cudaStream_t st) {
  if (p.nA > 0 && p.nA <= kMaxPoolAtoms) {
    const size_t smem = (size_t)p.nA * (3 * p.d + 2) * sizeof(float);
    dim3 grid(p.nRt * p.nRh * p.nRw, BH);
    cudaError_t e = cudaFuncSetAttribute(pool_atoms_kernel<D, kSum>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    pool_atoms_kernel<D, kSum><<<grid, kPoolAtomThreads, smem, st>>>(p);
    return cudaGetLastError();
  }
  dim3 grid(p.C, p.nRt * p.nRh * p.nRw, BH);
  pool_sics_kernel<D, kSum><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_pool_d(const PoolParams& p, int BH, cudaStream_t st) {
  switch (p.summarizer) {
    case SA_SUMMARIZER_MEAN: return launch_pool<D, SA_SUMMARIZER_MEAN>(p, BH, st);
    case SA_SUMMARIZER_MAX: return launch_pool<D, SA_SUMMARIZER_MAX>(p, BH, st);
    case SA_SUMMARIZER_MIN: return launch_pool<D, SA_SUMMARIZER_MIN>(p, BH, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_pool_sics(const PoolParams& p, int BH, int max_nb, cudaStream_t st) {
  (void)max_nb;
  if (p.d == 128) return launch_pool_d<128>(p, BH, st);
  if (p.d == 64) return launch_pool_d<64>(p, BH, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_choose(const ChooseParams& p, int BH, cudaStream_t st) {
  choose_kernel<<<BH, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_pooled_scores(const ScoreParams& p, int BH, int d, cudaStream_t st) {
  dim3 grid((p.NB + 63) / 64, (p.NB + 63) / 64, BH);
  const size_t sm = 2 * 64 * (d + 1) * sizeof(float);
  if (d == 128) {
    const cudaError_t e = cudaFuncSetAttribute(pooled_scores_kernel<128>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    pooled_scores_kernel<128><<<grid, 256, sm, st>>>(p);
  } else if (d == 64) {
    pooled_scores_kernel<64><<<grid, 256, sm, st>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectParams& p, int BH, cudaStream_t st) {
  dim3 grid(p.NB, BH);
  select_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_zero_counts(int* counts, size_t n, cudaStream_t st) {
  zero_counts_kernel<<<256, 256, 0, st>>>(counts, n);
  return cudaGetLastError();
}

}  // namespace sa
