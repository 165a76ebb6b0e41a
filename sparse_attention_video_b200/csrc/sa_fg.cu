// Fine-grained M x 1 key slices (FG-Attn review: key machinery, and skeptic
// critique / referee major comment 2 on Sec. 4.4).
//
// Mask (sparse_attn_build_mask):
//   fg_qbar      q_avg of every group of M contiguous queries (fp32), written
//                as three bf16 terms hi + mid + lo whose sum is q_avg to about
//                2^-24 relative; each bf16 x bf16 product is exact in fp32.
//   fg_score     tcgen05 GEMM: D[key][group] = sum_terms k . term, the slice
//                score times sqrt(d), in tensor memory. One kernel, two uses:
//                  HIST  histogram of 12 (or 8) bits of the order-preserving
//                        key of D among the scores that match the prefix
//                        decided so far (an exact radix select of the R-th
//                        largest score, R = ceil(f * G * N));
//                  BITS  slice bitmask D >= tau (ties at tau are kept).
//                Every pass recomputes the same D values (same operands, same
//                MMA order), so the passes agree bit for bit.
//   fg_select    one CTA per head: turns a histogram into the next bits of the
//                threshold key and the rank left inside the chosen bin.
// Attention (sparse_attn_attend):
//   fg_pair_count / fg_offsets / fg_compact  the union of the kept keys of the
//                groups that share a 128-query tile, ascending, with one
//                membership bit per group, packed per head.
//   the gather variant of attn_fwd_kernel (sa_attn.cu) consumes that list.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "sa_fg.h"
#include "sa_ptx.cuh"

namespace sa {

namespace {

constexpr int kScoreThreads = 640;   // warps 4-19: epilogue, four per key lane quarter
constexpr int kEpiParts = 4;         // group columns split into 128 / kEpiParts per warp
constexpr int kKeyTilesPerCta = 64;      // 8192 keys per CTA
constexpr int kBins = 4096;
constexpr int kAcc = 4;              // score tiles in tensor memory (128 columns each)
constexpr int kKStages = 3;          // key tiles in flight
constexpr int kHists = 2;            // shared-memory histogram copies (two lane quarters each)

// Unsigned key with the order of the floats: negative values have every bit
// flipped, non-negative ones only the sign bit (two instructions).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// The warp's 32 words as a 32 x 32 bit matrix (row = lane), transposed by
// five block swaps: on return bit l of lane e's word is bit e of lane l's.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
  const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int j = 16 >> i;
    const uint32_t m = masks[i];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
    x = (lane & j) ? ((x & ~m) | ((y & ~m) >> j)) : ((x & m) | ((y & m) << j));
  }
  return x;
}

// ------------------------------------------------------------------ q_avg
// One CTA of 128 threads per (group, head). d/8 lanes cover one query row
// with 16-byte loads (8 dimensions each), so 1,024 / d rows are read per
// step, all of a group's rows in flight at once; the per-lane partial sums
// are then added in a fixed order through shared memory.
constexpr int kQbarThreads = 128;

__global__ void __launch_bounds__(kQbarThreads) fg_qbar_kernel(FgQbarParams p) {
  __shared__ float part[kQbarThreads * 8];          // [row slot][d]
  const int g = blockIdx.x, bh = blockIdx.y;
  const int lanes = p.d / 8, rows = kQbarThreads / lanes;
  const int piece = threadIdx.x % lanes, slot = threadIdx.x / lanes;
  const int t0 = g * p.group, t1 = min(t0 + p.group, p.N);
  const __nv_bfloat16* q = p.q + (size_t)bh * p.N * p.d + piece * 8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 8
  for (int t = t0 + slot; t < t1; t += rows) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q + (size_t)t * p.d));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[slot * p.d + piece * 8 + i] = acc[i];
  __syncthreads();
  const int c = threadIdx.x;
  if (c >= p.d) return;
  float s = 0.f;
  for (int r = 0; r < rows; ++r) s += part[r * p.d + c];
  const int n = t1 > t0 ? t1 - t0 : 0;
  const float mean = n ? s / (float)n : 0.f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
  const float r1 = mean - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
  const size_t row = ((size_t)bh * p.G_pad + g) * p.d + c;
  const size_t term = (size_t)p.BH * p.G_pad * p.d;
  p.qsplit[row] = hi;
  p.qsplit[term + row] = mid;
  p.qsplit[2 * term + row] = lo;
}

// ------------------------------------------------------------------ scoring GEMM
template <int D>
struct ScoreSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kTerm = kHalves * 128 * 128;          // one q_avg term tile, 128 groups
  static constexpr int kKTile = kHalves * 128 * 128;          // 128 keys
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 3 * kTerm;
  static constexpr int kOffHist = kOffK + kKStages * kKTile;
  static constexpr int kOffBar = kOffHist + kHists * kBins * 4;
  static constexpr int kAlloc = kOffBar + 256 + 1024;
};

struct ScoreBars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t acc_full[kAcc], acc_free[kAcc];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1)
fg_score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                const FgScoreParams p) {
  using L = ScoreSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kOffQ;
  uint8_t* sK = smem + L::kOffK;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L::kOffHist);
  ScoreBars* bars = reinterpret_cast<ScoreBars*>(smem + L::kOffBar);

  const int chunk = blockIdx.x, gt = blockIdx.y, bh = blockIdx.z;
  const int n_tiles_total = (p.N + 127) / 128;
  // key tiles tile0, tile0 + stride, ... (stride > 1: a sample of the keys)
  const int stride = p.tile_stride > 1 ? p.tile_stride : 1;
  const int tile0 = chunk * kKeyTilesPerCta * stride;
  const int n_tiles = min(kKeyTilesPerCta, (n_tiles_total - tile0 + stride - 1) / stride);
  if (n_tiles <= 0 || grid_aborted(p.status)) return;
  if (p.only_heads && p.only_heads[bh] == 0u) return;     // uniform across the CTA
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Selection state of this head (HIST level > 0 and BITS read the prefix).
  const uint32_t prefix = p.mode == FG_MODE_HIST ? p.sel[bh * 4 + 0] : 0u;
  // (CACHED has no selection state: sel is null there)
  const uint32_t tau_key = p.mode == FG_MODE_CACHED ? 0u : p.sel[bh * 4 + 0];
  // Bitmask thresholds as floats: the order key is monotonic in the float
  // value, so key >= t  <=>  value >= key_to_float(t) (zeros aside: -0 and
  // +0 compare equal as floats, which only matters when the threshold is a
  // zero, a tie either way).
  // BITS: keep >= tau. BITS_COLLECT: keep >= the first key above the 24-bit
  // prefix bin, list the scores inside the bin.
  const float f_tau = key_to_float(tau_key);
  const int cs = p.collect_shift > 0 ? p.collect_shift : 8;      // low bits left to fg_fixup
  const uint32_t hib = tau_key >> cs;
  const float f_bin_lo = key_to_float(hib << cs);
  const float f_bin_hi = hib >= (0xFFFFFFFFu >> cs) ? INFINITY : key_to_float((hib + 1u) << cs);
  // HIST_WIN: the window [win_lo, win_lo + 2^(12 + win_shift)) is histogrammed
  // in 4,096 bins of 2^win_shift keys; keys above it are counted in registers
  const uint32_t win_lo = p.mode == FG_MODE_HIST_WIN ? p.sel[bh * 4 + 0] : 0u;
  const uint32_t win_span = 1u << (12 + p.win_shift);
  const uint32_t win_hi = win_lo <= 0xFFFFFFFFu - win_span ? win_lo + win_span : 0xFFFFFFFFu;
  uint32_t n_above = 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 1); }
    for (int i = 0; i < kAcc; ++i) {
      mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_free[i], 4 * kEpiParts);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (p.mode == FG_MODE_HIST || p.mode == FG_MODE_HIST_WIN)
    for (int i = threadIdx.x; i < kHists * kBins; i += kScoreThreads) hist[i] = 0u;
  // CACHED: exp(s/sqrt(d) - lse) > tau  <=>  s > sqrt(d) * (lse + ln tau), one
  // threshold per query column, staged where the histogram would be. A query
  // past the end (a zero row of the TMA fill) never keeps a slice.
  const int n_terms = p.mode == FG_MODE_CACHED ? 1 : 3;
  if (p.mode == FG_MODE_CACHED) {
    float* thr = reinterpret_cast<float*>(hist);
    for (int i = threadIdx.x; i < 128; i += kScoreThreads) {
      const int qi = gt * 128 + i;
      thr[i] = qi < p.N ? p.sqrt_d * (p.lse[(size_t)bh * p.N + qi] + p.ln_tau) : INFINITY;
    }
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 128 * kAcc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;
  uint32_t* status = p.status;

  if (warp == 0) {
    if (lane == 0) {
      // q_avg terms for this group tile: 3 terms x D/64 boxes of (64 x 128
      // groups); CACHED: one term, the 128 query rows of this tile
      mbar_arrive_expect_tx(&bars->q_full, n_terms * L::kTerm);
      for (int t = 0; t < n_terms; ++t)
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(sQ + t * L::kTerm + h * 16384, &qmap, &bars->q_full, h * 64, gt * 128,
                      t * p.BH + bh);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kKStages;
        if (!mbar_wait(&bars->k_empty[st], ((j / kKStages) & 1) ^ 1, abort, status, 0x04010000u | j))
          break;
        mbar_arrive_expect_tx(&bars->k_full[st], L::kKTile);
        for (int h = 0; h < L::kHalves; ++h)
          tma_load_3d(sK + st * L::kKTile + h * 16384, &kmap, &bars->k_full[st], h * 64,
                      (tile0 + j * stride) * 128, bh);
        issued = j + 1;
      }
      if (*abort)
        for (int j = max(0, issued - kKStages); j < issued; ++j)
          mbar_drain(&bars->k_full[j % kKStages], (j / kKStages) & 1);
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop (waits and branches warp-uniform);
    // one elected lane issues each MMA and commit, so the descriptors stay
    // warp-uniform values and the issue keeps ahead of the tensor pipe.
    {
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128, false, false);
      // Descriptors formed once: the q_avg terms' are fixed, a K stage's
      // differ from stage 0's by a constant; each MMA adds a compile-time
      // offset, so the issuing thread spends its time issuing.
      const uint64_t dK0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      uint64_t dq[3][D / 16];
#pragma unroll
      for (int t = 0; t < 3; ++t)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          dq[t][kk] = umma_desc_sw128(smem_u32(sQ) + t * L::kTerm + (kk / 4) * 16384 + (kk % 4) * 32,
                                      16, 1024);
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait<false>(&bars->q_full, 0, abort, status, 0x05050000u));
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kKStages, ab = j % kAcc;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->k_full[st], (j / kKStages) & 1, abort,
                                                      status, 0x05060000u | j)))
          break;
        if (j >= kAcc &&
            !__all_sync(0xffffffffu, mbar_wait<false>(&bars->acc_free[ab], ((j / kAcc) - 1) & 1,
                                                      abort, status, 0x05070000u | j)))
          break;
        const uint64_t dk = umma_desc_advance(dK0, st * L::kKTile);
        uint64_t da[D / 16];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) da[kk] = umma_desc_advance(dk, (kk / 4) * 16384 + (kk % 4) * 32);
        tc_fence_after();
        const uint32_t d_tmem = tmem + ab * 128;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          if (t >= n_terms) break;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_bf16_ss_elect(d_tmem, da[kk], dq[t][kk], idesc, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_elect(&bars->acc_full[ab]);
        umma_commit_elect(&bars->k_empty[st]);
      }
      umma_commit_elect(&bars->drain);
      mbar_drain(&bars->drain, 0);
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- epilogue
    // Warp w reads tensor-memory lanes 32*(w%4).. (its keys) and part
    // (w-4)/4 of the 128 group columns; the warps of lane quarters q and
    // q + 2 share one histogram.
    constexpr int kCols = 128 / kEpiParts;
    const int quarter = warp & 3, half = (warp - 4) >> 2;
    const int r = 32 * quarter + lane;                 // key lane within the tile
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    uint32_t* whist = hist + (quarter % kHists) * kBins;
    const int g_base = gt * 128;
    const int g_lim = min(128, p.G - g_base);
    for (int j = 0; j < n_tiles; ++j) {
      const int ab = j % kAcc;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_full[ab], (j / kAcc) & 1, abort, status,
                                             0x06080000u | j)))
        break;
      tc_fence_after();
      const int key = (tile0 + j * stride) * 128 + r;
      const bool kvalid = key < p.N;
      uint32_t words[kCols / 32];
#pragma unroll
      for (int i = 0; i < kCols / 32; ++i) words[i] = 0u;
#pragma unroll
      for (int cc = 0; cc < kCols; cc += 32) {
        const int c0 = half * kCols + cc;
        float v[32];
        tmem_ld32(tmem + ab * 128 + lane_off + c0, v);
        tmem_wait_ld();
        // all 32 columns real (the usual case): no per-score bounds tests
        const int n_ok = kvalid ? min(32, g_lim - c0) : 0;
        if (p.mode == FG_MODE_HIST) {
          if (n_ok == 32) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t kk = order_key(v[e]);
              if ((kk & p.match_mask) == prefix) atomicAdd(&whist[(kk >> p.bin_shift) & p.bin_mask], 1u);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t kk = order_key(v[e]);
              if (e < n_ok && (kk & p.match_mask) == prefix)
                atomicAdd(&whist[(kk >> p.bin_shift) & p.bin_mask], 1u);
            }
          }
        } else if (p.mode == FG_MODE_HIST_WIN) {
          // fine bins: neighbouring keys' scores rarely share one. The
          // window test is one unsigned compare of the offset (a key below
          // the window wraps to a large offset) and the count is branch-free:
          // nested branches here ran the pass 1.5x slower, and so did float
          // compares against the window's bounds that left the key to the
          // scores inside it.
          const uint32_t wsize = 1u << (12 + p.win_shift);
          if (n_ok == 32) {
            // keys at or above win_hi lie above the window (win_hi is the
            // all-ones key, which no finite score has, when the window
            // reaches the top)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t kk = order_key(v[e]);
              n_above += kk >= win_hi ? 1u : 0u;
              const uint32_t off = kk - win_lo;
              if (off < wsize) atomicAdd(&whist[off >> p.win_shift], 1u);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t kk = order_key(v[e]);
              const uint32_t off = kk - win_lo;
              const bool ok_e = e < n_ok;
              n_above += (ok_e && off >= wsize && kk >= win_lo) ? 1u : 0u;
              if (ok_e && off < wsize) atomicAdd(&whist[off >> p.win_shift], 1u);
            }
          }
        } else if (p.mode == FG_MODE_CACHED) {
          // this lane's key against the warp's 32 query columns, which all
          // belong to one group (32 divides the group size): kept when one
          // of them passes its threshold; lane e of the ballot is key e of
          // this lane quarter, so the ballot is the bitmask word itself
          const float* thr = reinterpret_cast<const float*>(hist) + c0;
          bool any = false;
#pragma unroll
          for (int e = 0; e < 32; ++e) any |= v[e] > thr[e];
          const uint32_t word = __ballot_sync(0xffffffffu, kvalid && any);
          const int g = (gt * 128 + c0) / p.group;
          const int kw = ((tile0 + j * stride) * 128 + 32 * quarter) / 32;
          if (lane == 0 && word != 0u && g < p.G && kw < p.WN)
            atomicOr(p.bits + ((size_t)bh * p.G + g) * p.WN + kw, word);
        } else {
          const float f_keep = p.mode == FG_MODE_BITS ? f_tau : f_bin_hi;
          // bit e of kb: this lane's key is kept for column c0 + e; of lb:
          // its score is at least the collected bin's lower edge
          uint32_t kb = 0u, lb = 0u;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (v[e] >= f_keep) kb |= 1u << e;
            if (p.mode == FG_MODE_BITS_COLLECT && v[e] >= f_bin_lo) lb |= 1u << e;
          }
          const uint32_t okm = n_ok >= 32 ? 0xFFFFFFFFu : (n_ok > 0 ? (1u << n_ok) - 1u : 0u);
          kb &= okm;
          const uint32_t cand = lb & ~kb & okm;
          // lane e: the warp's 32 keys for column c0 + e, the bitmask word
          words[cc / 32] = warp_transpose32(kb, lane);
          if (p.mode == FG_MODE_BITS_COLLECT && __any_sync(0xffffffffu, cand != 0u)) {
            // rare: scores that share their top 24 bits with the threshold
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if ((cand >> e) & 1u) {
                const uint32_t pos = atomicAdd(p.cand_count + bh, 1u);
                if (pos < kFgCandCap)
                  p.cand[(size_t)bh * kFgCandCap + pos] = make_uint2(
                      (uint32_t)key, ((uint32_t)(g_base + c0 + e) << cs) |
                                         (order_key(v[e]) & ((1u << cs) - 1u)));
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_free[ab]);
      if (p.mode == FG_MODE_BITS || p.mode == FG_MODE_BITS_COLLECT) {
        // lane e holds this warp's 32 keys for groups half*kCols + 32*i + e
        const int kw = ((tile0 + j * stride) * 128 + 32 * quarter) / 32;
#pragma unroll
        for (int i = 0; i < kCols / 32; ++i) {
          const int gl = half * kCols + lane + 32 * i;
          if (gl < g_lim && kw < p.WN)
            p.bits[((size_t)bh * p.G + g_base + gl) * p.WN + kw] = words[i];
        }
      }
    }
  }
  if (p.mode == FG_MODE_HIST_WIN) {
    // this CTA's count of keys above the window, one global add per warp
    for (int o = 16; o >= 1; o >>= 1) n_above += __shfl_xor_sync(0xffffffffu, n_above, o);
    if (warp >= 4 && lane == 0 && n_above) atomicAdd(p.above + bh, n_above);
  }
  tc_fence_before();
  __syncthreads();
  if (p.mode == FG_MODE_HIST || p.mode == FG_MODE_HIST_WIN) {
    uint32_t* gh = p.hist + (size_t)bh * kBins;
    for (int b = threadIdx.x; b <= (int)p.bin_mask; b += kScoreThreads) {
      uint32_t c = 0;
#pragma unroll
      for (int h = 0; h < kHists; ++h) c += hist[h * kBins + b];
      if (c) atomicAdd(&gh[b], c);
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128 * kAcc);
  }
}

// ------------------------------------------------------------------ select
// sel[bh*4 + 0] prefix key so far, [1] rank left (1-based, counted from the
// largest), [2] number of slices kept (after the final level: R plus ties is
// only known after BITS; [2] holds R).
__global__ void fg_select_init_kernel(uint32_t* sel, uint32_t* hist, uint32_t* cand_count,
                                      int BH, uint32_t rank, const uint32_t* only_heads) {
  const int bh = blockIdx.x;
  if (only_heads && only_heads[bh] == 0u) return;
  if (threadIdx.x == 0) {
    sel[bh * 4 + 0] = 0u; sel[bh * 4 + 1] = rank; sel[bh * 4 + 2] = rank;
    cand_count[bh] = 0u;
  }
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) hist[(size_t)bh * kBins + b] = 0u;
}

__global__ void fg_select_kernel(uint32_t* sel, uint32_t* hist, int nbins, int shift,
                                 float* tau, float inv_sqrt_d, int final_level,
                                 const uint32_t* only_heads) {
  const int bh = blockIdx.x;
  if (only_heads && only_heads[bh] == 0u) return;
  __shared__ uint32_t counts[kBins];
  uint32_t* h = hist + (size_t)bh * kBins;
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) { counts[b] = h[b]; h[b] = 0u; }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t rank = sel[bh * 4 + 1];
    uint32_t acc = 0;
    int b = nbins - 1;
    for (; b > 0; --b) {                     // from the largest keys down
      if (acc + counts[b] >= rank) break;
      acc += counts[b];
    }
    sel[bh * 4 + 0] |= (uint32_t)b << shift;
    sel[bh * 4 + 1] = rank - acc;
    if (final_level) tau[bh] = key_to_float(sel[bh * 4 + 0]) * inv_sqrt_d;
  }
}

// ------------------------------------------------------------------ window
// Level 0 is first taken on a sample of the key tiles (every 16th), which
// only places tau roughly. The exact pass then counts the keys above a window
// of two level-0 bins around that place in registers and histograms the
// keys inside it in 4,096 fine bins; fine bins seldom collide in the
// shared-memory atomics that bind the full level-0 histogram, and a narrow
// window keeps most scores out of them. A head whose tau lies outside the
// window takes the three-level path instead.
// win arrays: above[BH], miss[BH], hit[BH], ovf[BH] (and fallback[BH]).
constexpr int kWinBins0 = 2;         // level-0 bins in the window
constexpr int kWinShift = 9;         // 2^(12 + 9) = 2 level-0 bins of 2^20 keys

__global__ void fg_win_init_kernel(uint32_t* sel, uint32_t* hist, uint32_t* cand_count,
                                   uint32_t* win, uint32_t* fallback, int BH, uint32_t rank) {
  const int bh = blockIdx.x;
  if (threadIdx.x == 0) {
    sel[bh * 4 + 0] = 0u; sel[bh * 4 + 1] = rank; sel[bh * 4 + 2] = rank;
    cand_count[bh] = 0u;
    fallback[bh] = 0u;
    for (int a = 0; a < 4; ++a) win[a * BH + bh] = 0u;
  }
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) hist[(size_t)bh * kBins + b] = 0u;
}

// From the sampled level-0 histogram: the bin b holding the sampled rank, and
// the window of two bins around it: b .. b + 1 when the sampled rank falls
// in the upper half of b's sampled count, else b - 1 .. b (clamped), so that
// tau keeps at least half a bin of margin on either side (about 1 % of the
// scores near a 15 % cut, against a sampling error in the rank of about
// 10^-4 of them).
__global__ void fg_window_kernel(uint32_t* sel, uint32_t* hist, uint32_t rank_sampled) {
  const int bh = blockIdx.x;
  __shared__ uint32_t counts[kBins];
  uint32_t* h = hist + (size_t)bh * kBins;
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) { counts[b] = h[b]; h[b] = 0u; }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t acc = 0;
    int b = kBins - 1;
    for (; b > 0; --b) {
      if (acc + counts[b] >= rank_sampled) break;
      acc += counts[b];
    }
    const bool upper = rank_sampled - acc <= (counts[b] + 1u) / 2u;   // near b's top
    const int lo = min(max(upper ? b : b - 1, 0), kBins - kWinBins0);
    sel[bh * 4 + 0] = (uint32_t)lo << 20;
  }
}

// After the exact windowed pass: tau's fine bin (a 23-bit prefix) and the
// rank left inside it, or a miss when tau lies above or below the window.
__global__ void fg_select_win_kernel(uint32_t* sel, uint32_t* hist, uint32_t* win, int BH) {
  const int bh = blockIdx.x;
  __shared__ uint32_t counts[kBins];
  uint32_t* h = hist + (size_t)bh * kBins;
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) { counts[b] = h[b]; h[b] = 0u; }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t rank = sel[bh * 4 + 1];
    uint32_t acc = win[0 * BH + bh];                    // keys above the window
    int found = -1;
    if (acc < rank) {
      for (int b = kBins - 1; b >= 0; --b) {
        if (acc + counts[b] >= rank) { found = b; break; }
        acc += counts[b];
      }
    }
    if (found >= 0) {
      sel[bh * 4 + 0] += (uint32_t)found << kWinShift;
      sel[bh * 4 + 1] = rank - acc;
      win[1 * BH + bh] = 0u;
      win[2 * BH + bh] = 1u;
    } else {
      win[1 * BH + bh] = 1u;
      win[2 * BH + bh] = 0u;
    }
  }
}

// Last select level over the collected candidates (keys sharing the top 24
// bits decided so far): histogram of their low 8 bits, the bin holding the
// rank left is tau's low byte; candidates at or above it get their bit. A
// head whose list overflowed is flagged for the full third level instead.
// ``cs`` low key bits are left (8 after the two 12-bit levels, kWinShift after
// the window); heads whose only_heads flag is 0 are not touched.
__global__ void fg_fixup_kernel(uint32_t* sel, const uint2* cand, const uint32_t* cand_count,
                                uint32_t* fallback, uint32_t* bits, float* tau, float inv_sqrt_d,
                                int G, int WN, int cs, const uint32_t* only_heads) {
  const int bh = blockIdx.x;
  if (only_heads && only_heads[bh] == 0u) return;
  __shared__ uint32_t counts[1 << kWinShift];
  __shared__ uint32_t low;
  const uint32_t nb = 1u << cs, lmask = nb - 1u;
  const uint32_t n = cand_count[bh];
  if (n > kFgCandCap) {
    if (threadIdx.x == 0) fallback[bh] = 1u;
    return;
  }
  for (uint32_t b = threadIdx.x; b < nb; b += blockDim.x) counts[b] = 0u;
  __syncthreads();
  const uint2* c = cand + (size_t)bh * kFgCandCap;
  for (uint32_t i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&counts[c[i].y & lmask], 1u);
  __syncthreads();
  if (threadIdx.x == 0) {
    fallback[bh] = 0u;
    const uint32_t rank = sel[bh * 4 + 1];
    uint32_t acc = 0;
    int b = (int)nb - 1;
    for (; b > 0; --b) {                     // from the largest keys down
      if (acc + counts[b] >= rank) break;
      acc += counts[b];
    }
    low = (uint32_t)b;
    sel[bh * 4 + 0] |= (uint32_t)b;
    sel[bh * 4 + 1] = rank - acc;
    tau[bh] = key_to_float(sel[bh * 4 + 0]) * inv_sqrt_d;
  }
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n; i += blockDim.x) {
    const uint2 e = c[i];
    if ((e.y & lmask) < low) continue;
    const uint32_t g = e.y >> cs, key = e.x;
    if ((int)g < G && (int)(key >> 5) < WN)
      atomicOr(bits + ((size_t)bh * G + g) * WN + (key >> 5), 1u << (key & 31u));
  }
}

// ------------------------------------------------------------------ compaction
// Union of the kept keys of the groups in one 128-query tile, per (tile, head).
__global__ void fg_pair_count_kernel(FgListParams p) {
  const int tile = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int bh = blockIdx.y, lane = threadIdx.x % 32;
  if (tile >= p.P) return;
  const int g0 = tile * p.groups_per_tile;
  const uint32_t* r0 = p.bits + ((size_t)bh * p.G + g0) * p.WN;
  const uint32_t* r1 = (p.groups_per_tile == 2 && g0 + 1 < p.G) ? r0 + p.WN : nullptr;
  int c = 0;
  for (int w = lane; w < p.WN; w += 32) c += __popc(r0[w] | (r1 ? r1[w] : 0u));
  for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) p.counts[(size_t)bh * p.P + tile] = c;
}

// Per head: exclusive scan of the tiles' union sizes, 1,024 tiles per pass
// (warp shuffles, then the warp totals). Offsets are clamped to the list
// capacity, so a head whose union lists would overflow it (only possible with
// very many ties at tau) writes no entry out of bounds; that case is flagged
// in the status word.
__global__ void __launch_bounds__(1024) fg_offsets_kernel(FgListParams p) {
  __shared__ unsigned long long wsum[32];
  const int bh = blockIdx.x, lane = threadIdx.x % 32, wi = threadIdx.x / 32;
  const uint32_t* cnt = p.counts + (size_t)bh * p.P;
  uint32_t* off = p.offsets + (size_t)bh * (p.P + 1);
  const unsigned long long cap = (unsigned long long)p.cap_per_head;
  unsigned long long carry = 0;
  for (int t0 = 0; t0 < p.P; t0 += 1024) {
    const int t = t0 + (int)threadIdx.x;
    const unsigned long long c = t < p.P ? cnt[t] : 0ull;
    unsigned long long incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[wi] = incl;
    __syncthreads();
    unsigned long long before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      const unsigned long long v = wsum[w];
      if (w < wi) before += v;
      total += v;
    }
    const unsigned long long run = carry + before + incl - c;
    if (t < p.P) off[t] = (uint32_t)(run < cap ? run : cap);
    carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    off[p.P] = (uint32_t)(carry < cap ? carry : cap);
    if (carry > cap) atomicOr(p.status, (uint32_t)SA_DEVFLAG_BOUNDS);
  }
}

// One warp per (tile, head) lists the tile's union in ascending key order,
// 1,024 keys (32 bitmask words) at a time: lane l expands the set bits of
// word l into a per-warp staging buffer in shared memory at its prefix
// position, then the warp copies the chunk's entries out with consecutive
// lanes on consecutive list slots (coalesced stores).
constexpr int kListWarps = 8;

__global__ void __launch_bounds__(32 * kListWarps) fg_compact_kernel(FgListParams p) {
  __shared__ uint32_t stage[kListWarps][1024];
  const int wi = threadIdx.x / 32;
  const int tile = blockIdx.x * kListWarps + wi;
  const int bh = blockIdx.y, lane = threadIdx.x % 32;
  if (tile >= p.P) return;
  const int g0 = tile * p.groups_per_tile;
  const uint32_t* r0 = p.bits + ((size_t)bh * p.G + g0) * p.WN;
  const uint32_t* r1 = (p.groups_per_tile == 2 && g0 + 1 < p.G) ? r0 + p.WN : nullptr;
  uint32_t* out = p.list + (size_t)bh * p.cap_per_head;
  uint32_t* sb = stage[wi];
  uint32_t pos = p.offsets[(size_t)bh * (p.P + 1) + tile];
  const uint32_t end = p.offsets[(size_t)bh * (p.P + 1) + tile + 1];
  for (int w0 = 0; w0 < p.WN; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t a = w < p.WN ? r0[w] : 0u;
    const uint32_t b = (w < p.WN && r1) ? r1[w] : 0u;
    uint32_t u = a | b;
    const uint32_t c = __popc(u);
    uint32_t incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    uint32_t* dst = sb + (incl - c);
    const uint32_t kbase = 32u * (uint32_t)w;
    while (u) {
      const uint32_t low = u & (0u - u);               // lowest set bit
      u ^= low;
      *dst++ = (kbase + (uint32_t)__popc(low - 1u)) | ((a & low) ? (1u << 30) : 0u) |
               ((b & low) ? (1u << 31) : 0u);
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
    for (uint32_t i = lane; i < total; i += 32)
      if (pos + i < end) out[pos + i] = sb[i];
    __syncwarp();
    pos += total;
  }
}

bool encode_3d(CUtensorMap* m, const void* base, long long d0, long long d1, long long d2,
               int box1, CUresult (*enc)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                         const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                         const cuuint32_t*, CUtensorMapInterleave,
                                         CUtensorMapSwizzle, CUtensorMapL2promotion,
                                         CUtensorMapFloatOOBfill)) {
  cuuint64_t dims[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t strides[2] = {(cuuint64_t)d0 * 2, (cuuint64_t)d0 * d1 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_score(const CUtensorMap& km, const CUtensorMap& qm, const FgScoreParams& p,
                         cudaStream_t st) {
  using L = ScoreSmem<D>;
  cudaError_t e = cudaFuncSetAttribute(fg_score_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const int n_tiles = (p.N + 127) / 128;
  const int per_cta = kKeyTilesPerCta * (p.tile_stride > 1 ? p.tile_stride : 1);
  dim3 grid((n_tiles + per_cta - 1) / per_cta, p.row_tiles, p.BH);
  fg_score_kernel<D><<<grid, kScoreThreads, L::kAlloc, st>>>(km, qm, p);
  return cudaGetLastError();
}

}  // namespace

int fg_g_pad(int G) { return (G + 127) / 128 * 128; }
size_t fg_qsplit_bytes(int BH, int G, int d) { return 3ull * BH * fg_g_pad(G) * d * 2; }
size_t fg_hist_bytes(int BH) { return sizeof(uint32_t) * (size_t)BH * kBins; }
size_t fg_sel_bytes(int BH) { return sizeof(uint32_t) * (size_t)BH * 4; }
// candidates, then cand_count [BH], fallback [BH] and the window state
// (above, miss, hit, ovf: 4 x [BH])
size_t fg_cand_bytes(int BH) {
  return sizeof(uint2) * (size_t)BH * kFgCandCap + 6 * sizeof(uint32_t) * (size_t)BH;
}
long long fg_list_cap_per_head(int G, int N, float f) {
  return (long long)ceil((double)f * (double)G * (double)N) + N + 32;
}

cudaError_t launch_fg_build(const FgBuildParams& b, EncodeFn enc, cudaStream_t st) {
  const int G_pad = fg_g_pad(b.G);
  cudaError_t e;
  // q_avg terms (pad groups stay zero: clear the whole buffer first)
  if ((e = cudaMemsetAsync(b.qsplit, 0, fg_qsplit_bytes(b.BH, b.G, b.d), st)) != cudaSuccess) return e;
  FgQbarParams qp{b.q, b.qsplit, b.BH, b.N, b.d, b.group, b.G, G_pad};
  fg_qbar_kernel<<<dim3(b.G, b.BH), kQbarThreads, 0, st>>>(qp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  CUtensorMap km, qm;
  if (!encode_3d(&km, b.k, b.d, b.N, b.BH, 128, enc)) return cudaErrorInvalidValue;
  if (!encode_3d(&qm, b.qsplit, b.d, G_pad, 3LL * b.BH, 128, enc)) return cudaErrorInvalidValue;

  const double total = (double)b.G * (double)b.N;
  const uint32_t rank = (uint32_t)ceil((double)b.keep_fraction * total);
  uint32_t* above = b.win;
  uint32_t* miss = b.win + b.BH;
  uint32_t* hit = b.win + 2 * b.BH;
  uint32_t* ovf = b.win + 3 * b.BH;
  fg_win_init_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, b.cand_count, b.win, b.fallback, b.BH,
                                           rank);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  FgScoreParams sp{};
  sp.bits = b.bits; sp.hist = b.hist; sp.sel = b.sel; sp.status = b.status;
  sp.cand = b.cand; sp.cand_count = b.cand_count;
  sp.BH = b.BH; sp.N = b.N; sp.G = b.G; sp.WN = b.WN;
  sp.row_tiles = G_pad / 128;
  sp.above = above;
  const float inv_sqrt_d = 1.0f / sqrtf((float)b.d);
  auto score = [&]() {
    return b.d == 128 ? launch_score<128>(km, qm, sp, st) : launch_score<64>(km, qm, sp, st);
  };
  // Radix select of the rank-th largest key: bits 31..20, 19..8, then 7..0.
  const int shifts[3] = {20, 8, 0};
  const int widths[3] = {12, 12, 8};
  auto hist_level = [&](int lv, const uint32_t* only) -> cudaError_t {
    sp.mode = FG_MODE_HIST;
    sp.tile_stride = 1;
    sp.bin_shift = shifts[lv];
    sp.bin_mask = (1u << widths[lv]) - 1u;
    sp.match_mask = lv == 0 ? 0u : (0xFFFFFFFFu << shifts[lv - 1]);
    sp.only_heads = only;
    cudaError_t err = score();
    if (err != cudaSuccess) return err;
    fg_select_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, 1 << widths[lv], shifts[lv], b.tau,
                                           inv_sqrt_d, lv == 2, only);
    return cudaGetLastError();
  };

  // 1. Level 0 on every kSampleStride-th key tile: where tau roughly lies.
  constexpr int kSampleStride = 16;
  const int n_tiles = (b.N + 127) / 128;
  long long n_sampled = 0;
  for (int t = 0; t < n_tiles; t += kSampleStride) n_sampled += std::min(128, b.N - 128 * t);
  const uint32_t rank_s = (uint32_t)std::max<double>(
      1.0, ceil((double)rank * (double)n_sampled / (double)b.N));
  sp.mode = FG_MODE_HIST;
  sp.tile_stride = kSampleStride;
  sp.bin_shift = 20;
  sp.bin_mask = 0xFFFu;
  sp.match_mask = 0u;
  sp.only_heads = nullptr;
  if ((e = score()) != cudaSuccess) return e;
  fg_window_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, rank_s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 2. Every key: the exact count above the window and its fine histogram.
  sp.mode = FG_MODE_HIST_WIN;
  sp.tile_stride = 1;
  sp.win_shift = kWinShift;
  if ((e = score()) != cudaSuccess) return e;
  fg_select_win_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, b.win, b.BH);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 3. The bitmask pass settles every score outside tau's fine bin and lists
  // the scores inside it; fg_fixup selects the last kWinShift bits among them.
  sp.mode = FG_MODE_BITS_COLLECT;
  sp.collect_shift = kWinShift;
  sp.only_heads = hit;
  if ((e = score()) != cudaSuccess) return e;
  fg_fixup_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.cand, b.cand_count, ovf, b.bits, b.tau,
                                        inv_sqrt_d, b.G, b.WN, kWinShift, hit);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Window heads whose candidate list overflowed: a histogram of the last
  // kWinShift bits over every key, then the plain bitmask pass.
  sp.mode = FG_MODE_HIST;
  sp.bin_shift = 0;
  sp.bin_mask = (1u << kWinShift) - 1u;
  sp.match_mask = 0xFFFFFFFFu << kWinShift;
  sp.only_heads = ovf;
  if ((e = score()) != cudaSuccess) return e;
  fg_select_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, 1 << kWinShift, 0, b.tau, inv_sqrt_d, 1,
                                         ovf);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sp.mode = FG_MODE_BITS;
  if ((e = score()) != cudaSuccess) return e;

  // Heads whose tau fell outside the window: the three-level path.
  fg_select_init_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.hist, b.cand_count, b.BH, rank, miss);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int lv = 0; lv < 2; ++lv)
    if ((e = hist_level(lv, miss)) != cudaSuccess) return e;
  // The bitmask pass settles every score outside the 24-bit prefix bin and
  // lists the few inside it; fg_fixup selects the last 8 bits among them.
  sp.mode = FG_MODE_BITS_COLLECT;
  sp.collect_shift = 8;
  sp.only_heads = miss;
  if ((e = score()) != cudaSuccess) return e;
  fg_fixup_kernel<<<b.BH, 256, 0, st>>>(b.sel, b.cand, b.cand_count, b.fallback, b.bits, b.tau,
                                        inv_sqrt_d, b.G, b.WN, 8, miss);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Heads whose candidate list overflowed: the full third level and the plain
  // bitmask pass (every other head's CTAs return at once).
  if ((e = hist_level(2, b.fallback)) != cudaSuccess) return e;
  sp.mode = FG_MODE_BITS;
  sp.only_heads = b.fallback;
  if ((e = score()) != cudaSuccess) return e;
  return launch_fg_lists(b.lists, st);
}

namespace {
__global__ void fill_f32_kernel(float* dst, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = v;
}
}  // namespace

cudaError_t launch_fg_cached(const FgCachedParams& b, EncodeFn enc, cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(b.bits, 0, sizeof(uint32_t) * (size_t)b.BH * b.G * b.WN, st)) != cudaSuccess)
    return e;
  fill_f32_kernel<<<(b.BH + 255) / 256, 256, 0, st>>>(b.tau_out, b.BH, b.tau);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap km, qm;
  if (!encode_3d(&km, b.k, b.d, b.N, b.BH, 128, enc)) return cudaErrorInvalidValue;
  if (!encode_3d(&qm, b.q, b.d, b.N, b.BH, 128, enc)) return cudaErrorInvalidValue;
  FgScoreParams sp{};
  sp.mode = FG_MODE_CACHED;
  sp.bits = b.bits; sp.status = b.status;
  sp.lse = b.lse;
  sp.ln_tau = logf(b.tau);
  sp.sqrt_d = sqrtf((float)b.d);
  sp.group = b.group;
  sp.row_tiles = (b.N + 127) / 128;
  sp.BH = b.BH; sp.N = b.N; sp.G = b.G; sp.WN = b.WN;
  e = b.d == 128 ? launch_score<128>(km, qm, sp, st) : launch_score<64>(km, qm, sp, st);
  if (e != cudaSuccess) return e;
  return launch_fg_lists(b.lists, st);
}

cudaError_t launch_fg_lists(const FgListParams& p, cudaStream_t st) {
  const int warps = kListWarps;
  dim3 grid((p.P + warps - 1) / warps, p.BH);
  fg_pair_count_kernel<<<grid, 32 * warps, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fg_offsets_kernel<<<p.BH, 1024, 0, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  fg_compact_kernel<<<grid, 32 * warps, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
