// Block-sparse flash attention on tcgen05 tensor cores (sm_100a).
//
// For one head and one query block of a working layout, the kernel visits the
// kept key blocks in ascending order and computes
//   S = Q K^T (tcgen05.mma, bf16 in, fp32 accumulate in tensor memory),
//   P = exp(S / sqrt(d) - m) with a running row maximum m (online softmax),
//   O += P V (tcgen05.mma, P written back over S in tensor memory as bf16),
// then writes O / l and LSE = ln(l) + m to the query tokens' original rows.
// This is the flash block-sparse kernel with online softmax of the SPADE
// review ("What carries the argument") and the dense-tile-only executor of the
// Sliding Tile Attention review (key machinery: every computed block is dense,
// the mask logic lives in the loader); online softmax is exact (SPADE review,
// axiom ledger), so the result equals masked softmax attention.
//
// Roles (320 threads):
//   warps 0-7   softmax, two groups of four warps. Group g takes the key
//               blocks j with j % 2 == g, one thread per row (warp w reads
//               tensor-memory lanes 32*(w%4)..): its own running maximum and
//               sum, and its own O accumulator that the PV MMAs of its blocks
//               fill. While one group waits for its next S, the other is in
//               its exponentials. The running maximum only moves when it
//               grows by more than 2^8, so O is rescaled rarely; P and l use
//               the same reference, which keeps the result exact. The
//               1/sqrt(d) scale is folded into one FFMA before exp2.
//               Epilogue: the groups trade (m, l) through shared memory, and
//               each thread writes half of its row's columns of
//               (a0 O_0 + a1 O_1) / (a0 l0 + a1 l1) in bf16 at the query's
//               original token row (the inverse permutation is fused here).
//   warp 8      TMA producer: Q once, then K and V of each kept key block into
//               a 3-stage ring. 3D tile layouts are gathered by one 5-D box per
//               64 columns (no separate permutation pass); identity and
//               frame-major layouts by a 3-D box.
//   warp 9      allocates tensor memory and issues all MMAs, the whole warp
//               converged and one elected lane per instruction: QK_0, QK_1,
//               then PV_j, QK_{j+2} for every j. S_j goes to buffer j % 2,
//               O_j % 2 accumulates P_j V_j.
//   warps 10-11 (M x 1 slices only) copy the kept keys' K and V rows with
//               cp.async; warp 8 then only builds the per-group masks.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "sa_attn.h"
#include "sa_ptx.cuh"

namespace sa {

namespace {

constexpr int kThreads = 320;
// M x 1 slice mode runs 384 threads (two more copy warps) with a register
// split (setmaxnreg): the softmax warpgroups take 208, warpgroup 2
// (producer, MMA issuer, copy warps) 88. The shares add up to the launch's
// 168 per thread.
constexpr uint32_t kRegsLaunch = 168, kRegsSoftmax = 208, kRegsOther = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == (kThreads + 64) * kRegsLaunch,
              "register split must equal the launch total");
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kCopyWarp0 = 10;             // gather mode: warps 10-11 copy K/V rows
constexpr int kStages = 3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows > 2^8
// Every exp2 runs on MUFU. Moving a quarter to three eighths of them to an
// FMA-pipe polynomial (Cody-Waite split plus a cubic) was measured slower on
// every workload, with the single-lane and the warp-uniform MMA issuer alike.

// FP8 operands (E4M3): every product runs as tcgen05.mma kind::f8f6f4 on
// the same tiles at one byte per element; P is E4M3 of 2^4 P (the reference
// moves when a row's maximum passes it by more than 2^4, so 2^4 P <= 2^8 stays
// below 448 and probabilities down to 2^-13 keep a normal code).
constexpr float kRescaleThresholdFp8 = 4.0f;
constexpr float kPOffsetFp8 = 4.0f;

// ES: bytes per element (2 bf16, 1 E4M3). A 128-byte swizzle row holds
// 128 / ES columns of d.
template <int D, int BN, int ES = 2>
struct Smem {
  static constexpr int kHalvesD = D * ES / 128;           // 128-byte column groups of d
  static constexpr int kQBytes = kHalvesD * 128 * 128;    // 128 rows, M of the MMA
  static constexpr int kKVHalf = BN * 128;                // one 64-column half of a K/V tile
  static constexpr int kKVBytes = kHalvesD * kKVHalf;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  static constexpr int kBytes = kOffBar + 512;
  static constexpr int kAlloc = kBytes + 1024;            // slack for 1024-byte alignment
  // S (one buffer per softmax group) and one O accumulator per group
  static constexpr uint32_t kTmemCols = (2 * BN + 2 * D) <= 256 ? 256 : 512;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages], v_full[kStages];
  uint64_t kv_empty[kStages];       // stage free: PV of its block (hence its QK) completed
  uint64_t s_full[2];
  uint64_t p_full[2];               // P_j written into S buffer j & 1 (by group j & 1)
  uint64_t drain;
  uint64_t m_full[2], m_empty[2];   // gather mode: per-chunk group-membership masks
  uint32_t masks[2][8];             // [chunk & 1][first group words 0-3, second group 4-7]
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(Bars) <= 512, "barrier block must fit its shared-memory slot");

// Which tensor map and which coordinates fetch block ``blk`` of head ``bh``.
__device__ __forceinline__ void block_source(const HeadGeom& g, int blk, int BN, int& map,
                                             int& c1, int& c2, int& c3) {
  if (g.layout == SA_LAYOUT_TILE) {
    map = 2 + g.cand;
    const int tw = blk % g.nw, th = (blk / g.nw) % g.nh, tt = blk / (g.nw * g.nh);
    c1 = tw * g.bw; c2 = th * g.bh; c3 = tt * g.bt;
  } else {
    map = g.layout;  // 0 identity (original tensor), 1 frame-major (permuted copy)
    c1 = blk * BN; c2 = 0; c3 = 0;
  }
}

template <int D, int BN, int ES = 2>
__device__ __forceinline__ void load_block(const CUtensorMap* maps, const HeadGeom& g, int bh,
                                           int blk, uint8_t* dst, uint64_t* bar) {
  constexpr int kBoxCols = 128 / ES;           // one 128-byte swizzle row per box row
  int map, c1, c2, c3;
  block_source(g, blk, BN, map, c1, c2, c3);
  const CUtensorMap* m = maps + map;
#pragma unroll
  for (int h = 0; h < D / kBoxCols; ++h) {
    uint8_t* d = dst + h * (BN * 128);
    if (map >= 2) tma_load_5d(d, m, bar, h * kBoxCols, c1, c2, c3, bh);
    else tma_load_3d(d, m, bar, h * kBoxCols, c1, bh);
  }
}

// Slot ``s`` of block ``blk`` -> original token index, or -1 for padding.
__device__ __forceinline__ int slot_to_token(const HeadGeom& g, int blk, int s, int BN, int T,
                                             int H, int W) {
  const int N = T * H * W;
  if (g.layout == SA_LAYOUT_TILE) {
    const int tw = blk % g.nw, th = (blk / g.nw) % g.nh, tt = blk / (g.nw * g.nh);
    const int lw = s % g.bw, lh = (s / g.bw) % g.bh, lt = s / (g.bw * g.bh);
    const int t = tt * g.bt + lt, h = th * g.bh + lh, w = tw * g.bw + lw;
    if (t >= T || h >= H || w >= W) return -1;
    return (t * H + h) * W + w;
  }
  const int m = blk * BN + s;
  if (m >= N) return -1;
  if (g.layout == SA_LAYOUT_FRAME_MAJOR) {
    const int pos = m / T, t = m - pos * T;
    return t * (H * W) + pos;
  }
  return m;
}

// Validity of the BN slots of block ``blk`` as a bit mask (bit c = slot c holds
// a token). Computed arithmetically from the block's position, so every
// softmax thread can form it alone. Returns false when the block has no pad.
template <int BN>
__device__ __forceinline__ bool block_pad_mask(const HeadGeom& g, int blk, int T, int H, int W,
                                               uint32_t (&bits)[BN / 32]) {
#pragma unroll
  for (int i = 0; i < BN / 32; ++i) bits[i] = 0u;
  if (g.layout == SA_LAYOUT_TILE) {
    const int tw = blk % g.nw, th = (blk / g.nw) % g.nh, tt = blk / (g.nw * g.nh);
    const int lt_n = min(g.bt, T - tt * g.bt), lh_n = min(g.bh, H - th * g.bh);
    const int lw_n = min(g.bw, W - tw * g.bw);
    if (lt_n == g.bt && lh_n == g.bh && lw_n == g.bw) return false;
    for (int lt = 0; lt < lt_n; ++lt)
      for (int lh = 0; lh < lh_n; ++lh) {
        const int a = (lt * g.bh + lh) * g.bw, b = a + lw_n;   // slots [a, b) are tokens
#pragma unroll
        for (int i = 0; i < BN / 32; ++i) {
          const int lo = max(a, 32 * i), hi = min(b, 32 * i + 32);
          if (hi > lo) {
            const uint32_t width = (uint32_t)(hi - lo);
            const uint32_t ones = width >= 32 ? 0xffffffffu : ((1u << width) - 1u);
            bits[i] |= ones << (lo - 32 * i);
          }
        }
      }
    return true;
  }
  const int lim = T * H * W - blk * BN;                // slots [0, lim) are tokens
  if (lim >= BN) return false;
#pragma unroll
  for (int i = 0; i < BN / 32; ++i) {
    const int width = min(max(lim - 32 * i, 0), 32);
    bits[i] = width >= 32 ? 0xffffffffu : ((1u << width) - 1u);
  }
  return true;
}

// Timeout site code recorded in status word 1: role (1 producer, 2 MMA,
// 3 softmax), barrier id, key-block iteration.
__device__ __forceinline__ uint32_t site(uint32_t role, uint32_t bar, int j) {
  return (role << 24) | (bar << 16) | ((uint32_t)j & 0xFFFFu);
}

// kGather = false: blocks of a working layout, kept key blocks from the mask's
// ascending lists. kGather = true (M x 1 key slices): the query tile is 128
// contiguous queries (one or two groups); its keys are the union list of those
// groups, copied 128 rows at a time by the copy warps (cp.async), and each
// row masks keys outside its own group.
// kFp8 (block mode, D = BN = 128): Q, K, V are E4M3 codes, one scale per
// (batch, head) tensor; both products run on kind::f8f6f4.
template <int D, int BN, bool kGather, bool kFp8 = false>
__global__ void __launch_bounds__(kGather || kFp8 ? kThreads + 64 : kThreads, 1)
attn_fwd_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  static_assert(!kFp8 || (!kGather && D == 128 && BN == 128), "FP8: block mode, d = 128");
  constexpr int ES = kFp8 ? 1 : 2;
  constexpr bool kSplitRegs = kGather || kFp8;
  using L = Smem<D, BN, ES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kOffQ;
  uint8_t* sK = smem + L::kOffK;
  uint8_t* sV = smem + L::kOffV;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kOffBar);

  const int qb = blockIdx.x;
  const int bh = blockIdx.y;
  HeadGeom g{};
  int n_keys = 0;
  const int* cols = nullptr;
  uint32_t list_count = 0;
  const uint32_t* list = nullptr;
  if constexpr (kGather) {
    g.layout = SA_LAYOUT_IDENTITY;
    g.bt = 1; g.bh = 1; g.bw = BN; g.nt = 1; g.nh = 1; g.nw = p.NB; g.nb = p.NB;
    if (qb >= p.NB || grid_aborted(p.status)) return;
    const uint32_t* off = p.fg_offsets + (size_t)bh * (p.NB + 1);
    const uint32_t begin = off[qb];
    list_count = off[qb + 1] - begin;
    list = p.fg_list + (size_t)bh * p.fg_cap + begin;
    n_keys = (int)((list_count + BN - 1) / BN);
  } else {
    g = p.heads ? p.heads[bh] : p.geo0;
    // uniform across the CTA, before any allocation
    const int n_q = p.q_tiles > 0 ? p.q_tiles : g.nb;
    if (qb >= n_q || grid_aborted(p.status)) return;
    if (p.dense) {
      n_keys = g.nb;
    } else {
      const size_t row_base = ((size_t)bh * p.NB + qb);
      n_keys = p.counts[row_base];
      cols = p.cols + row_base * p.NB;
    }
  }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    // gather mode: K/V stages are filled by the two copy warps, not by TMA
    const uint32_t fill_arrivals = kGather ? 2u : 1u;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], fill_arrivals); mbar_init(&bars->v_full[s], fill_arrivals);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&bars->s_full[b], 1);
    for (int b = 0; b < 2; ++b) mbar_init(&bars->p_full[b], kSoftmaxWarps / 2);
    mbar_init(&bars->drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->m_full[b], 1);
      mbar_init(&bars->m_empty[b], kSoftmaxWarps / 2);
    }
    bars->abort = 0;
    fence_barrier_init();
  }
  if constexpr (BN < 128) {
    // Rows BN..127 of the 128-row MMA operand carry no query; keep them finite.
    constexpr int kVecPerHalf = (128 - BN) * 8;
    for (int i = threadIdx.x; i < kVecPerHalf * L::kHalvesD; i += blockDim.x) {
      const int h = i / kVecPerHalf, rem = i % kVecPerHalf;
      reinterpret_cast<uint4*>(sQ + h * 16384 + BN * 128)[rem] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tS[2] = {tmem, tmem + BN};
  const uint32_t tO = tmem + 2 * BN;              // O_0 at tO, O_1 at tO + D
  volatile int* abort = &bars->abort;
  uint32_t* status = p.status;

  if (warp >= 8) {
  // Slice mode: warpgroup 2 gives registers back at one point that dominates
  // all of its role code; the softmax warpgroups take them in the other branch.
  if constexpr (kSplitRegs) regs_dec<kRegsOther>();
  if (warp == kProducerWarp && kGather) {
    // ------------------------------------------------------------ producer (gather)
    if (n_keys > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->q_full, L::kHalvesD * BN * 128);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(sQ + h * (BN * 128), &maps.q[0], &bars->q_full, h * 64, qb * BN, bh);
      }
      // list entries j*128 + lane + 32*s; key index in the low 30 bits, one
      // membership bit per group of the tile in bits 30 and 31. The next
      // chunk's entries are loaded while this chunk waits on its barriers.
      uint32_t en[4];
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {
        const uint32_t idx = (uint32_t)lane + 32 * s4;
        en[s4] = idx < list_count ? __ldg(list + idx) : 0u;
      }
      for (int j = 0; j < n_keys; ++j) {
        const int mb = j & 1;
        uint32_t e[4];
        bool val[4];
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const uint32_t idx = (uint32_t)j * BN + lane + 32 * s4;
          val[s4] = idx < list_count;
          e[s4] = en[s4];
          const uint32_t nidx = idx + BN;
          en[s4] = nidx < list_count ? __ldg(list + nidx) : 0u;
        }
        uint32_t m0[4], m1[4];
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          m0[s4] = __ballot_sync(0xffffffffu, val[s4] && ((e[s4] >> 30) & 1u));
          m1[s4] = p.fg_groups_per_tile == 2
                       ? __ballot_sync(0xffffffffu, val[s4] && ((e[s4] >> 31) & 1u)) : m0[s4];
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->m_empty[mb], ((j >> 1) & 1) ^ 1, abort,
                                               status, site(1, 3, j))))
          break;
        if (lane == 0) {
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) { bars->masks[mb][s4] = m0[s4]; bars->masks[mb][4 + s4] = m1[s4]; }
          mbar_arrive(&bars->m_full[mb]);
        }
      }
    }
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_keys > 0) {
      const CUtensorMap* qmaps = maps.q;
      const CUtensorMap* kmaps = maps.k;
      const CUtensorMap* vmaps = maps.v;
      mbar_arrive_expect_tx(&bars->q_full, L::kHalvesD * BN * 128);
      // gathered query rows (sampled-row mode) are a plain row tensor
      HeadGeom gq = g;
      if (p.q_tiles > 0) gq.layout = SA_LAYOUT_IDENTITY;
      load_block<D, BN, ES>(qmaps, gq, bh, qb, sQ, &bars->q_full);
      int issued = 0;
      for (int j = 0; j < n_keys; ++j) {
        const int st = j % kStages, rnd = j / kStages;
        const int kb = p.dense ? j : cols[j];
        if (kb < 0 || kb >= g.nb) { atomicOr(status, SA_DEVFLAG_BOUNDS); *abort = 1; break; }
        if (!mbar_wait(&bars->kv_empty[st], (rnd & 1) ^ 1, abort, status, site(1, 1, j))) break;
        mbar_arrive_expect_tx(&bars->k_full[st], L::kKVBytes);
        load_block<D, BN, ES>(kmaps, g, bh, kb, sK + st * L::kKVBytes, &bars->k_full[st]);
        mbar_arrive_expect_tx(&bars->v_full[st], L::kKVBytes);
        load_block<D, BN, ES>(vmaps, g, bh, kb, sV + st * L::kKVBytes, &bars->v_full[st]);
        issued = j * 2 + 2;
      }
      if (*abort) {
        // Let copies already in flight land before the CTA's memory is released.
        for (int j = (issued / 2 > kStages ? issued / 2 - kStages : 0); j < (issued + 1) / 2; ++j) {
          const int st = j % kStages, par = (j / kStages) & 1;
          mbar_drain(&bars->k_full[st], par);
          if (2 * j + 1 < issued) mbar_drain(&bars->v_full[st], par);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (every wait and branch warp-uniform);
    // one elected lane issues each MMA and commit.
    if (n_keys > 0) {
      constexpr uint32_t idesc_qk = kFp8 ? umma_idesc_e4m3(128, BN, false, false)
                                         : umma_idesc_bf16(128, BN, false, false);
      constexpr uint32_t idesc_pv = kFp8 ? umma_idesc_e4m3(128, D, false, true)
                                         : umma_idesc_bf16(128, D, false, true);
      // Every MMA takes 32 bytes of its K dimension: 16 bf16 or 32 E4M3.
      constexpr int kKQ = D * ES / 32;             // QK MMAs along d
      constexpr int kKeysPerMma = 32 / ES;         // PV: keys per MMA
      constexpr int kKP = BN / kKeysPerMma;        // PV MMAs per block
      constexpr int kMmaPerChunk = 64 / kKeysPerMma;
      auto mma_ss = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (kFp8) umma_e4m3_ss_elect(d, a, b, id, acc);
        else umma_bf16_ss_elect(d, a, b, id, acc);
      };
      auto mma_ts = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (kFp8) umma_e4m3_ts_elect(d, a, b, id, acc);
        else umma_bf16_ts_elect(d, a, b, id, acc);
      };
      // Descriptors are formed once; each MMA only advances a base by a
      // compile-time offset, so the issuing thread spends its time issuing.
      const uint64_t dQ = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = umma_desc_sw128(smem_u32(sV), L::kKVHalf, 1024);
      uint64_t da[kKQ];
#pragma unroll
      for (int kk = 0; kk < kKQ; ++kk)           // 32 bytes of K inside a 128-byte row
        da[kk] = umma_desc_advance(dQ, (kk / 4) * 16384 + (kk % 4) * 32);
      // QK_j into S buffer j & 1 (softmax group j & 1 reads it).
      auto issue_qk = [&](int j) -> bool {
        const int st = j % kStages;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->k_full[st], (j / kStages) & 1, abort,
                                                      status, site(2, 6, j))))
          return false;
        const uint64_t dk = umma_desc_advance(dK0, st * L::kKVBytes);
        uint64_t db[kKQ];
#pragma unroll
        for (int kk = 0; kk < kKQ; ++kk)
          db[kk] = umma_desc_advance(dk, (kk / 4) * L::kKVHalf + (kk % 4) * 32);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKQ; ++kk)
          mma_ss(tS[j & 1], da[kk], db[kk], idesc_qk, kk > 0 ? 1u : 0u);
        umma_commit_elect(&bars->s_full[j & 1]);
        return true;
      };
      // PV_j: O_{j&1} += P_j V_j, P_j read from S buffer j & 1.
      auto issue_pv = [&](int i) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->p_full[i & 1], (i >> 1) & 1, abort,
                                                      status, site(2, 3, i))))
          return false;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->v_full[i % kStages], (i / kStages) & 1,
                                                      abort, status, site(2, 4, i))))
          return false;
        const uint64_t dv = umma_desc_advance(dV0, (i % kStages) * L::kKVBytes);
        uint64_t db[kKP];
#pragma unroll
        for (int kk = 0; kk < kKP; ++kk) db[kk] = umma_desc_advance(dv, kk * kKeysPerMma * 128);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKP; ++kk) {
          // A = P in tensor memory: 8 packed columns per step (16 bf16 keys,
          // two per column, or 32 E4M3 keys, four per column). The P of keys
          // 64c..64c+63 sits at the start of their own S columns 64c.. (where
          // their scores were). B = V (MN-major: d contiguous). O_{i&1} is
          // first written by block i & 1.
          mma_ts(tO + (i & 1) * D,
                 tS[i & 1] + (kk / kMmaPerChunk) * 64 + (kk % kMmaPerChunk) * 8, db[kk],
                 idesc_pv, (i > 1 || kk > 0) ? 1u : 0u);
        }
        umma_commit_elect(&bars->kv_empty[i % kStages]);
        return true;
      };
      // Order: QK_0, QK_1, then PV_j, QK_{j+2} for every j. S buffer j & 1
      // is rewritten by QK_{j+2} only after PV_j (issued first) read P_j, and
      // the commit of S_{j+2} also covers PV_j: once a softmax group sees
      // S_{j+2}, its O accumulator holds every block before j + 2.
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait<false>(&bars->q_full, 0, abort, status, site(2, 5, 0)));
      for (int j = 0; ok && j < 2 && j < n_keys; ++j) ok = issue_qk(j);
      for (int j = 0; ok && j < n_keys; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < n_keys) ok = issue_qk(j + 2);
      }
      // Every MMA issued above must finish before tensor memory is freed.
      umma_commit_elect(&bars->drain);
      mbar_drain(&bars->drain, 0);
      __syncwarp();
    }
  } else if (kGather && warp >= kCopyWarp0) {
    // ------------------------------------------------------------ K/V row copies (gather)
    // Copy warp cw fills rows 64cw..64cw+63 of every chunk with 16-byte
    // cp.async pieces straight into the 128-byte-swizzled tiles the MMA
    // reads. D/8 consecutive lanes copy one whole row (coalesced: a warp
    // instruction moves 32/(D/8) full rows), the key index of each row comes
    // by shuffle from the lane that loaded it. Before each announcement the
    // warp waits for its own copies and makes the generic-proxy writes
    // visible to the tensor core's async proxy.
    constexpr int kPieces = D / 8;                  // 16-byte pieces per row
    constexpr int kRowsPerStep = 32 / kPieces;      // rows per warp instruction
    const int cw = warp - kCopyWarp0;
    const int piece = lane % kPieces, sub = lane / kPieces;
    const __nv_bfloat16* kbase = p.k_rows + (size_t)bh * p.N * D + piece * 8;
    const __nv_bfloat16* vbase = p.v_rows + (size_t)bh * p.N * D + piece * 8;
    for (int j = 0; j < n_keys; ++j) {
      const int st = j % kStages, rnd = j / kStages;
      // lane l holds the keys of rows 64cw + l and 64cw + 32 + l
      int kl[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t idx = (uint32_t)j * BN + 64 * cw + 32 * i + lane;
        kl[i] = idx < list_count ? (int)(__ldg(list + idx) & 0x3FFFFFFFu) : 0;
        if (!dbg_in_range(kl[i], p.N, status)) kl[i] = 0;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->kv_empty[st], (rnd & 1) ^ 1, abort, status,
                                             site(4, 1, j)))) {
        break;
      }
      uint8_t* dk = sK + st * L::kKVBytes + (piece / 8) * (BN * 128);
      uint8_t* dv = sV + st * L::kKVBytes + (piece / 8) * (BN * 128);
      // K first, then V, as two cp.async groups: QK_j needs only K_j, so K is
      // announced as soon as it has landed; V follows.
      int keys[64 / kRowsPerStep];
#pragma unroll
      for (int i = 0; i < 64 / kRowsPerStep; ++i) {
        const int rl = i * kRowsPerStep + sub;       // row within this warp's 64
        keys[i] = __shfl_sync(0xffffffffu, kl[(i * kRowsPerStep) / 32], rl % 32);
        const int r = 64 * cw + rl;
        cp_async16(dk + r * 128 + (((piece % 8) ^ (r & 7)) << 4), kbase + (size_t)keys[i] * D);
      }
      cp_async_commit();
#pragma unroll
      for (int i = 0; i < 64 / kRowsPerStep; ++i) {
        const int r = 64 * cw + i * kRowsPerStep + sub;
        cp_async16(dv + r * 128 + (((piece % 8) ^ (r & 7)) << 4), vbase + (size_t)keys[i] * D);
      }
      cp_async_commit();
      cp_async_wait<1>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->k_full[st]);
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->v_full[st]);
    }
    // own copies land before anything else (also on the abort path)
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
  }
  } else {
    if constexpr (kSplitRegs) regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax + epilogue
    // Group grp = warp / 4 takes the key blocks j with j % 2 == grp; thread r
    // of a group owns row r of those blocks: its own running maximum m, sum
    // l and accumulator O_grp. The two groups work on different blocks at the
    // same time, so one group's loads, reductions and barrier waits overlap
    // the other's exponentials. The epilogue merges the two partial softmaxes:
    //   O = (a0 O_0 + a1 O_1) / (a0 l0 + a1 l1),  a_g = 2^(m_g - max(m0, m1)).
    constexpr int kChunks = BN / 64;
    const int grp = warp >> 2;
    const int r = (warp & 3) * 32 + lane;             // row == tensor-memory lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tSg = tS[grp] + lane_off;
    const uint32_t tOg = tO + grp * D + lane_off;
    // FP8: scores of the codes times the two tensors' scales
    const float scale = kFp8 ? p.scale_log2 / (p.q_inv[bh] * p.k_inv[bh]) : p.scale_log2;
    float m = -INFINITY;                              // reference maximum, log2 units
    float l = 0.f;                                    // sum of P over this group's blocks
    float s[64];
    bool ok = true;
    // key block of this group's next block, loaded one block ahead
    int kb_next = (!kGather && grp < n_keys) ? (p.dense ? grp : cols[grp]) : 0;
    for (int j = grp; j < n_keys; j += 2) {
      const uint32_t par = (uint32_t)(j >> 1) & 1u;
      uint32_t pw[BN / 32];
      bool pad = true;
      if constexpr (kGather) {
        // this row's group-membership bits for the chunk's keys
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->m_full[grp], par, abort, status,
                                               site(3, 11, j)))) {
          ok = false;
          break;
        }
        // the words stay in shared memory until this block is done (they are
        // read chunk by chunk below; m_empty is signalled after the block)
      } else {
        const int kb = kb_next;
        if (j + 2 < n_keys) kb_next = p.dense ? j + 2 : cols[j + 2];
        pad = block_pad_mask<BN>(g, kb, p.T, p.H, p.W, pw);
      }
      // a warp either waits out a barrier together or gives up together
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[grp], par, abort, status,
                                             site(3, 8, j)))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // One pass over the row, 64 columns at a time: load, chunk maximum,
      // exp2 against the running reference m, P back into tensor memory. The
      // reference moves only when a chunk's maximum passes it by more than
      // 2^8; then everything already summed against the old reference (l,
      // this block's partial sum, this block's stored P chunks and O) is
      // scaled by 2^(m_old - m_new). O holds blocks up to j - 2, all
      // complete (S_j was committed after PV_{j-2}), and PV_j waits for this
      // group's arrival below, so touching O needs no wait.
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (kFp8) {
        // FP8: the whole row in registers, one maximum and one rescale
        // decision per block, so no stored E4M3 P is ever rescaled. O is
        // rescaled before any of P_j is stored (PV_j waits for the arrival
        // below; O holds this group's blocks up to j - 2, all complete).
        float sr[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32) tmem_ld32(tSg + c, sr + c);
        tmem_wait_ld();
        if (pad) {
#pragma unroll
          for (int c = 0; c < BN; ++c) sr[c] = ((pw[c / 32] >> (c % 32)) & 1u) ? sr[c] : -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(sr[2 * e], sr[2 * e + 1]);
#pragma unroll
        for (int c = 16; c < BN; c += 16) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], sr[c + 2 * e], sr[c + 2 * e + 1]);
        }
        const float cm = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7])) * scale;
        const bool move = cm > m + kRescaleThresholdFp8;
        const bool had = move && m != -INFINITY;
        const float alpha = had ? ex2_approx(m - cm) : 1.f;
        if (move) { l *= alpha; m = cm; }
        if (__any_sync(0xffffffffu, had)) {
          float o[16];
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            tmem_ld16(tOg + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= alpha;
            tmem_st16(tOg + c, o);
          }
        }
        // 2^4 P, so that E4M3 keeps probabilities down to 2^-13 in its
        // normal range; l sums the same values and the epilogue removes 2^4
        const float neg = (m == -INFINITY ? 0.f : -m) + kPOffsetFp8;
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          float* sc = sr + ch * 64;
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float x0, x1;
            fma2(sc[c], sc[c + 1], scale, scale, neg, neg, x0, x1);
            sc[c] = ex2_approx(x0);
            sc[c + 1] = ex2_approx(x1);
          }
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            add2(rs4[0], rs4[1], sc[c], sc[c + 1]);
            add2(rs4[2], rs4[3], sc[c + 2], sc[c + 3]);
          }
          // four E4M3 codes per column, key 4i + b in byte b of column i
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(sc[4 * i], sc[4 * i + 1]),
                                                         __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(sc[4 * i + 2], sc[4 * i + 3]),
                                                         __NV_SATFINITE, __NV_E4M3);
            pk[i] = lo | (hi << 16);
          }
          tmem_st16(tSg + ch * 64, reinterpret_cast<const float*>(pk));
        }
      } else {
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
        tmem_ld32(tSg + ch * 64, s);
        tmem_ld32(tSg + ch * 64 + 32, s + 32);
        tmem_wait_ld();
        if (pad) {
          uint32_t w2[2];
#pragma unroll
          for (int w = 0; w < 2; ++w)
            w2[w] = kGather ? bars->masks[grp][(r < 64 ? 0 : 4) + ch * 2 + w] : pw[ch * 2 + w];
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = ((w2[c / 32] >> (c % 32)) & 1u) ? s[c] : -INFINITY;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          mx4[0] = fmax3(mx4[0], s[c], s[c + 1]);
          mx4[1] = fmax3(mx4[1], s[c + 2], s[c + 3]);
          mx4[2] = fmax3(mx4[2], s[c + 4], s[c + 5]);
          mx4[3] = fmax3(mx4[3], s[c + 6], s[c + 7]);
        }
        const float cm = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * scale;
        // m = -inf and cm finite counts as moving (the first key of the row)
        const bool move = cm > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, move)) {
          // warp-collective tensor-memory traffic: lanes that keep their
          // reference scale by 1
          const bool had = move && m != -INFINITY;
          const float alpha = had ? ex2_approx(m - cm) : 1.f;
          l *= alpha;
#pragma unroll
          for (int e = 0; e < 4; ++e) rs4[e] *= alpha;
          if (__any_sync(0xffffffffu, had)) {
            float o[32];
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              tmem_ld32(tOg + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= alpha;
              tmem_st32(tOg + c, o);
            }
#pragma unroll
            for (int pc = 0; pc < ch; ++pc) {
              // this block's P chunks stored so far: packed bf16 pairs
              tmem_ld32(tSg + pc * 64, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const uint32_t b = __float_as_uint(o[e]);
                o[e] = __uint_as_float(pack_bf16x2(__uint_as_float(b << 16) * alpha,
                                                   __uint_as_float(b & 0xFFFF0000u) * alpha));
              }
              tmem_st32(tSg + pc * 64, o);
            }
          }
          if (move) m = cm;
        }
        // masked keys are -inf and give exactly +0 on MUFU; a row whose
        // reference is still -inf has only masked keys so far. Scale and
        // shift, and the partial sums, run two columns per instruction.
        const float neg = m == -INFINITY ? 0.f : -m;
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1;
          fma2(s[c], s[c + 1], scale, scale, neg, neg, x0, x1);
          s[c] = ex2_approx(x0);
          s[c + 1] = ex2_approx(x1);
        }
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          add2(rs4[0], rs4[1], s[c], s[c + 1]);
          add2(rs4[2], rs4[3], s[c + 2], s[c + 3]);
        }
        // P as packed bf16 pairs over the first 32 of the chunk's own 64 S
        // columns (the A operand of the PV MMA is read from tensor memory);
        // packed in place: entry c only reads entries 2c and 2c+1
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(pack_bf16x2(s[2 * c], s[2 * c + 1]));
        tmem_st32(tSg + ch * 64, s);
      }
      }
      l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      if constexpr (kGather) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->m_empty[grp]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[grp]);
    }
    // ------------------------------------------------------------ epilogue
    // Once ``drain`` completes every MMA of the CTA has completed, so the Q
    // tile is free: the two groups trade (m, l) of each row through it.
    if (ok && n_keys > 0) {
      // the MMA warp commits ``drain`` after its last PV
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->drain, 0, abort, status, site(3, 10, n_keys)));
      tc_fence_after();
    }
    float* xch = reinterpret_cast<float*>(sQ);        // [group][m, l][128 rows]
    xch[(grp * 2 + 0) * 128 + r] = m;
    xch[(grp * 2 + 1) * 128 + r] = l;
    named_barrier_sync(1, kSoftmaxWarps * 32);
    const float m_o = xch[((grp ^ 1) * 2 + 0) * 128 + r];
    const float l_o = xch[((grp ^ 1) * 2 + 1) * 128 + r];
    // sampled-row mode: row qb*BN + r of the gathered rows, O in fp32
    const bool rows_f32 = p.o_f32 != nullptr;
    int tok = rows_f32 ? ((r < BN && qb * BN + r < p.q_rows) ? qb * BN + r : -1)
                             : ((r < BN) ? slot_to_token(g, qb, r, BN, p.T, p.H, p.W) : -1);
    if (tok >= 0 && !dbg_in_range(tok, rows_f32 ? p.q_rows : p.N, status)) tok = -1;
    if (ok) {
      const float m0 = grp == 0 ? m : m_o, l0 = grp == 0 ? l : l_o;
      const float m1 = grp == 0 ? m_o : m, l1 = grp == 0 ? l_o : l;
      const float mm = fmaxf(m0, m1);
      // a group with no block (or only masked keys) has m = -inf and an O
      // that was never written: weight 0, and its O is not read
      const float a0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - mm);
      const float a1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - mm);
      const float l_tot = a0 * l0 + a1 * l1;
      const float inv_l = (n_keys > 0 && l_tot > 0.f) ? 1.f / l_tot : 0.f;
      // FP8: the V codes' scale folds into the output weights
      const float osc = kFp8 ? 1.f / p.v_inv[bh] : 1.f;
      const float w0 = a0 * inv_l * osc, w1 = a1 * inv_l * osc;
      const bool use0 = n_keys > 0 && w0 != 0.f, use1 = n_keys > 1 && w1 != 0.f;
      // this thread writes output columns [grp*D/2, grp*D/2 + D/2)
      constexpr int HD = D / 2;
      __nv_bfloat16* orow = rows_f32 ? nullptr
                                     : p.o + ((size_t)bh * p.N + (tok < 0 ? 0 : tok)) * D + grp * HD;
      float* frow = rows_f32 ? p.o_f32 + ((size_t)bh * p.q_rows + (tok < 0 ? 0 : tok)) * D + grp * HD
                             : nullptr;
#pragma unroll
      for (int c = 0; c < HD; c += 16) {
        float o0[16], o1[16];
        // tcgen05.ld is warp-collective: load whenever any lane needs it
        if (__any_sync(0xffffffffu, use0)) tmem_ld16(tO + lane_off + grp * HD + c, o0);
        if (__any_sync(0xffffffffu, use1)) tmem_ld16(tO + D + lane_off + grp * HD + c, o1);
        tmem_wait_ld();
        if (tok >= 0 && rows_f32) {
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            float4 v;
            v.x = (use0 ? o0[e] * w0 : 0.f) + (use1 ? o1[e] * w1 : 0.f);
            v.y = (use0 ? o0[e + 1] * w0 : 0.f) + (use1 ? o1[e + 1] * w1 : 0.f);
            v.z = (use0 ? o0[e + 2] * w0 : 0.f) + (use1 ? o1[e + 2] * w1 : 0.f);
            v.w = (use0 ? o0[e + 3] * w0 : 0.f) + (use1 ? o1[e + 3] * w1 : 0.f);
            *reinterpret_cast<float4*>(frow + c + e) = v;
          }
        } else if (tok >= 0) {
#pragma unroll
          for (int e = 0; e < 16; e += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              v[u] = (use0 ? o0[e + u] * w0 : 0.f) + (use1 ? o1[e + u] * w1 : 0.f);
            uint4 w;
            w.x = pack_bf16x2(v[0], v[1]);
            w.y = pack_bf16x2(v[2], v[3]);
            w.z = pack_bf16x2(v[4], v[5]);
            w.w = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4*>(orow + c + e) = w;
          }
        }
      }
      if (tok >= 0 && grp == 0 && p.lse && !rows_f32)
        p.lse[(size_t)bh * p.N + tok] =
            (n_keys > 0 && l_tot > 0.f)
                ? (mm + __log2f(l_tot) - (kFp8 ? kPOffsetFp8 : 0.f)) * 0.69314718055994530942f
                : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}


// ------------------------------------------------------------------ solo CTAs
// A lighter block kernel for rows with few kept blocks: one softmax
// warpgroup, one K and one V stage (freed separately: K after its QK, V after
// its PV), 256 tensor-memory columns (S and O) and 192 threads, so that two
// CTAs fit on an SM and one CTA's setup, first loads and epilogue run under
// the other's blocks. Same arithmetic as attn_fwd_kernel's block mode: S, the
// lazily rescaled online softmax per 64-column chunk, P over S in tensor
// memory, O += P V.
//   warps 0-3  softmax and epilogue (thread r owns row r)
//   warp 4     TMA producer
//   warp 5     tensor memory and the MMAs (converged, elect.sync)
constexpr int kSoloThreads = 192;
constexpr int kSoloProducer = 4;
constexpr int kSoloMma = 5;

// ES: bytes per element (2 bf16, 1 E4M3 codes).
template <int D, int BN, int ES = 2>
struct SoloSmem {
  static constexpr int kHalvesD = D * ES / 128;           // 128-byte column groups of d
  static constexpr int kQBytes = kHalvesD * 128 * 128;
  static constexpr int kKVHalf = BN * 128;
  static constexpr int kKVBytes = kHalvesD * kKVHalf;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffBar = kOffV + kKVBytes;
  static constexpr int kBytes = kOffBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 256;              // S at 0, O at 128
};

struct SoloBars {
  uint64_t q_full, k_full, v_full, k_empty, v_empty, s_full, p_full, drain;
  uint32_t tmem_base;
  int abort;
};

// kFp8 (D = BN = 128): Q, K, V are E4M3 codes with one scale per (batch,
// head) tensor and both products run on kind::f8f6f4. The softmax takes the
// block's row maximum first (a pass over S without exponentials), so the
// reference moves before any P is stored and no stored E4M3 P is rescaled.
template <int D, int BN, bool kFp8 = false>
__global__ void __launch_bounds__(kSoloThreads, 2)
attn_solo_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
  static_assert(!kFp8 || (D == 128 && BN == 128), "FP8: d = 128, 128-token blocks");
  constexpr int ES = kFp8 ? 1 : 2;
  using L = SoloSmem<D, BN, ES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kOffQ;
  uint8_t* sK = smem + L::kOffK;
  uint8_t* sV = smem + L::kOffV;
  SoloBars* bars = reinterpret_cast<SoloBars*>(smem + L::kOffBar);
  const int qb = blockIdx.x, bh = blockIdx.y;
  const HeadGeom g = p.heads[bh];
  if (qb >= g.nb || grid_aborted(p.status)) return;
  const size_t row_base = (size_t)bh * p.NB + qb;
  const int n_keys = p.counts[row_base];
  const int* cols = p.cols + row_base * p.NB;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->k_full, 1); mbar_init(&bars->v_full, 1);
    mbar_init(&bars->k_empty, 1); mbar_init(&bars->v_empty, 1);
    mbar_init(&bars->s_full, 1); mbar_init(&bars->p_full, 4);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if constexpr (BN < 128) {
    constexpr int kVecPerHalf = (128 - BN) * 8;
    for (int i = threadIdx.x; i < kVecPerHalf * L::kHalvesD; i += blockDim.x) {
      const int h = i / kVecPerHalf, rem = i % kVecPerHalf;
      reinterpret_cast<uint4*>(sQ + h * 16384 + BN * 128)[rem] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == kSoloMma) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;
  volatile int* abort = &bars->abort;
  uint32_t* status = p.status;

  if (warp == kSoloProducer) {
    if (lane == 0 && n_keys > 0) {
      mbar_arrive_expect_tx(&bars->q_full, L::kHalvesD * BN * 128);
      load_block<D, BN, ES>(maps.q, g, bh, qb, sQ, &bars->q_full);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_keys; ++j) {
        const int kb = cols[j];
        if (kb < 0 || kb >= g.nb) { atomicOr(status, SA_DEVFLAG_BOUNDS); *abort = 1; break; }
        // K_j once QK_{j-1} has read the stage, V_j once PV_{j-1} has
        if (!mbar_wait(&bars->k_empty, (j & 1) ^ 1, abort, status, site(1, 1, j))) break;
        mbar_arrive_expect_tx(&bars->k_full, L::kKVBytes);
        load_block<D, BN, ES>(maps.k, g, bh, kb, sK, &bars->k_full);
        k_issued = j + 1;
        if (!mbar_wait(&bars->v_empty, (j & 1) ^ 1, abort, status, site(1, 2, j))) break;
        mbar_arrive_expect_tx(&bars->v_full, L::kKVBytes);
        load_block<D, BN, ES>(maps.v, g, bh, kb, sV, &bars->v_full);
        v_issued = j + 1;
      }
      if (*abort) {
        if (k_issued > 0) mbar_drain(&bars->k_full, (k_issued - 1) & 1);
        if (v_issued > 0) mbar_drain(&bars->v_full, (v_issued - 1) & 1);
      }
    }
  } else if (warp == kSoloMma) {
    if (n_keys > 0) {
      constexpr uint32_t idesc_qk = kFp8 ? umma_idesc_e4m3(128, BN, false, false)
                                         : umma_idesc_bf16(128, BN, false, false);
      constexpr uint32_t idesc_pv = kFp8 ? umma_idesc_e4m3(128, D, false, true)
                                         : umma_idesc_bf16(128, D, false, true);
      // every MMA takes 32 bytes of its K dimension: 16 bf16 or 32 E4M3
      constexpr int kKeysPerMma = 32 / ES;
      constexpr int kMmaPerChunk = 64 / kKeysPerMma;
      const uint64_t dQ = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = umma_desc_sw128(smem_u32(sV), L::kKVHalf, 1024);
      auto qk = [&](int j) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->k_full, j & 1, abort, status,
                                                      site(2, 6, j))))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D * ES / 32; ++kk) {
          const uint64_t da = umma_desc_advance(dQ, (kk / 4) * 16384 + (kk % 4) * 32);
          const uint64_t db = umma_desc_advance(dK, (kk / 4) * L::kKVHalf + (kk % 4) * 32);
          if constexpr (kFp8) umma_e4m3_ss_elect(tS, da, db, idesc_qk, kk > 0 ? 1u : 0u);
          else umma_bf16_ss_elect(tS, da, db, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(&bars->s_full);
        umma_commit_elect(&bars->k_empty);
        return true;
      };
      auto pv = [&](int j) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->p_full, j & 1, abort, status,
                                                      site(2, 3, j))))
          return false;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bars->v_full, j & 1, abort, status,
                                                      site(2, 4, j))))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / kKeysPerMma; ++kk) {
          // A = P in tensor memory, 8 packed columns per MMA, at the start of
          // the 64 S columns of its chunk; B = V, MN-major
          const uint32_t ta = tS + (kk / kMmaPerChunk) * 64 + (kk % kMmaPerChunk) * 8;
          const uint64_t db = umma_desc_advance(dV, kk * kKeysPerMma * 128);
          if constexpr (kFp8) umma_e4m3_ts_elect(tO, ta, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          else umma_bf16_ts_elect(tO, ta, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_elect(&bars->v_empty);
        return true;
      };
      // QK_0, then PV_j, QK_{j+1}: S is rewritten only after PV_j read P_j,
      // and S_{j+1}'s commit covers PV_j, so O holds every earlier block
      // when the softmax sees S_{j+1}.
      bool ok = __all_sync(0xffffffffu,
                           mbar_wait<false>(&bars->q_full, 0, abort, status, site(2, 5, 0)));
      if (ok) ok = qk(0);
      for (int j = 0; ok && j < n_keys; ++j) {
        ok = pv(j);
        if (ok && j + 1 < n_keys) ok = qk(j + 1);
      }
      umma_commit_elect(&bars->drain);
      mbar_drain(&bars->drain, 0);
      __syncwarp();
    }
  } else if (warp < 4) {
    constexpr int kChunks = BN / 64;
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tSg = tS + lane_off, tOg = tO + lane_off;
    // FP8: scores of the codes times the two tensors' scales
    const float scale = kFp8 ? p.scale_log2 / (p.q_inv[bh] * p.k_inv[bh]) : p.scale_log2;
    float m = -INFINITY, l = 0.f;
    float s[64];
    bool ok = true;
    int kb_next = n_keys > 0 ? cols[0] : 0;
    for (int j = 0; j < n_keys; ++j) {
      uint32_t pw[BN / 32];
      const int kb = kb_next;
      if (j + 1 < n_keys) kb_next = cols[j + 1];
      const bool pad = block_pad_mask<BN>(g, kb, p.T, p.H, p.W, pw);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort, status, site(3, 8, j)))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (kFp8) {
        // the block's row maximum (chunk kChunks - 1 stays in registers)
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          tmem_ld32(tSg + ch * 64, s);
          tmem_ld32(tSg + ch * 64 + 32, s + 32);
          tmem_wait_ld();
          if (pad) {
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = ((pw[ch * 2 + c / 32] >> (c % 32)) & 1u) ? s[c] : -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            mx4[0] = fmax3(mx4[0], s[c], s[c + 1]);
            mx4[1] = fmax3(mx4[1], s[c + 2], s[c + 3]);
            mx4[2] = fmax3(mx4[2], s[c + 4], s[c + 5]);
            mx4[3] = fmax3(mx4[3], s[c + 6], s[c + 7]);
          }
        }
        const float cm = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * scale;
        const bool move = cm > m + kRescaleThresholdFp8;
        const bool had = move && m != -INFINITY;
        const float alpha = had ? ex2_approx(m - cm) : 1.f;
        if (move) { l *= alpha; m = cm; }
        if (__any_sync(0xffffffffu, had)) {
          // O holds the complete earlier blocks (S_j's commit covers PV_{j-1})
          float o[32];
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            tmem_ld32(tOg + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tOg + c, o);
          }
        }
        // 2^4 P, so that E4M3 keeps probabilities down to 2^-13 in its
        // normal range; l sums the same values and the epilogue removes 2^4
        const float neg = (m == -INFINITY ? 0.f : -m) + kPOffsetFp8;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          const int ch = kChunks - 1 - i;
          if (i > 0) {
            tmem_ld32(tSg + ch * 64, s);
            tmem_ld32(tSg + ch * 64 + 32, s + 32);
            tmem_wait_ld();
            if (pad) {
#pragma unroll
              for (int c = 0; c < 64; ++c) s[c] = ((pw[ch * 2 + c / 32] >> (c % 32)) & 1u) ? s[c] : -INFINITY;
            }
          }
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float x0, x1;
            fma2(s[c], s[c + 1], scale, scale, neg, neg, x0, x1);
            s[c] = ex2_approx(x0);
            s[c + 1] = ex2_approx(x1);
          }
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            add2(rs4[0], rs4[1], s[c], s[c + 1]);
            add2(rs4[2], rs4[3], s[c + 2], s[c + 3]);
          }
          // four E4M3 codes per column, key 4i + b in byte b of column i;
          // chunk ch's 16 columns start at its own S column 64 ch (the S of
          // the chunk still to be reloaded is in columns it does not touch)
          uint32_t pk[16];
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(s[4 * q4], s[4 * q4 + 1]),
                                                         __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(s[4 * q4 + 2], s[4 * q4 + 3]),
                                                         __NV_SATFINITE, __NV_E4M3);
            pk[q4] = lo | (hi << 16);
          }
          tmem_st16(tSg + ch * 64, reinterpret_cast<const float*>(pk));
        }
      } else {
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
        tmem_ld32(tSg + ch * 64, s);
        tmem_ld32(tSg + ch * 64 + 32, s + 32);
        tmem_wait_ld();
        if (pad) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = ((pw[ch * 2 + c / 32] >> (c % 32)) & 1u) ? s[c] : -INFINITY;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          mx4[0] = fmax3(mx4[0], s[c], s[c + 1]);
          mx4[1] = fmax3(mx4[1], s[c + 2], s[c + 3]);
          mx4[2] = fmax3(mx4[2], s[c + 4], s[c + 5]);
          mx4[3] = fmax3(mx4[3], s[c + 6], s[c + 7]);
        }
        const float cm = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * scale;
        const bool move = cm > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, move)) {
          const bool had = move && m != -INFINITY;
          const float alpha = had ? ex2_approx(m - cm) : 1.f;
          l *= alpha;
#pragma unroll
          for (int e = 0; e < 4; ++e) rs4[e] *= alpha;
          if (__any_sync(0xffffffffu, had)) {
            float o[32];
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              tmem_ld32(tOg + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= alpha;
              tmem_st32(tOg + c, o);
            }
#pragma unroll
            for (int pc = 0; pc < ch; ++pc) {
              tmem_ld32(tSg + pc * 64, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const uint32_t b = __float_as_uint(o[e]);
                o[e] = __uint_as_float(pack_bf16x2(__uint_as_float(b << 16) * alpha,
                                                   __uint_as_float(b & 0xFFFF0000u) * alpha));
              }
              tmem_st32(tSg + pc * 64, o);
            }
          }
          if (move) m = cm;
        }
        const float neg = m == -INFINITY ? 0.f : -m;
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1;
          fma2(s[c], s[c + 1], scale, scale, neg, neg, x0, x1);
          s[c] = ex2_approx(x0);
          s[c + 1] = ex2_approx(x1);
        }
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          add2(rs4[0], rs4[1], s[c], s[c + 1]);
          add2(rs4[2], rs4[3], s[c + 2], s[c + 3]);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(pack_bf16x2(s[2 * c], s[2 * c + 1]));
        tmem_st32(tSg + ch * 64, s);
      }
      }
      l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok && n_keys > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->drain, 0, abort, status, site(3, 10, n_keys)));
      tc_fence_after();
    }
    int tok = r < BN ? slot_to_token(g, qb, r, BN, p.T, p.H, p.W) : -1;
    if (tok >= 0 && !dbg_in_range(tok, p.N, status)) tok = -1;
    if (ok) {
      // FP8: the V codes' scale folds into the output weight
      const float inv_l = (n_keys > 0 && l > 0.f) ? (kFp8 ? 1.f / (l * p.v_inv[bh]) : 1.f / l) : 0.f;
      const bool use = n_keys > 0;
      __nv_bfloat16* orow = p.o + ((size_t)bh * p.N + (tok < 0 ? 0 : tok)) * D;
#pragma unroll
      for (int c = 0; c < D; c += 16) {
        float o0[16];
        if (use) tmem_ld16(tOg + c, o0);             // warp-uniform (n_keys is per CTA)
        tmem_wait_ld();
        if (tok >= 0) {
#pragma unroll
          for (int e = 0; e < 16; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(use ? o0[e] * inv_l : 0.f, use ? o0[e + 1] * inv_l : 0.f);
            w.y = pack_bf16x2(use ? o0[e + 2] * inv_l : 0.f, use ? o0[e + 3] * inv_l : 0.f);
            w.z = pack_bf16x2(use ? o0[e + 4] * inv_l : 0.f, use ? o0[e + 5] * inv_l : 0.f);
            w.w = pack_bf16x2(use ? o0[e + 6] * inv_l : 0.f, use ? o0[e + 7] * inv_l : 0.f);
            *reinterpret_cast<uint4*>(orow + c + e) = w;
          }
        }
      }
      if (tok >= 0 && p.lse)
        p.lse[(size_t)bh * p.N + tok] =
            (n_keys > 0 && l > 0.f)
                ? (m + __log2f(l) - (kFp8 ? kPOffsetFp8 : 0.f)) * 0.69314718055994530942f
                : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kSoloMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace

template <int D, int BN, bool kGather, bool kFp8 = false>
static cudaError_t launch_one(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  using L = Smem<D, BN, kFp8 ? 1 : 2>;
  auto kern = attn_fwd_kernel<D, BN, kGather, kFp8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid(p.NB, p.BH);
  kern<<<grid, kGather || kFp8 ? kThreads + 64 : kThreads, L::kAlloc, stream>>>(maps, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(int head_dim, int block, const AttnMaps& maps, const AttnParams& p,
                            cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_one<128, 128, false>(maps, p, stream);
  if (head_dim == 64 && block == 128) return launch_one<64, 128, false>(maps, p, stream);
  if (head_dim == 64 && block == 64) return launch_one<64, 64, false>(maps, p, stream);
  return cudaErrorInvalidValue;
}

template <int D, int BN, bool kFp8 = false>
static cudaError_t launch_solo(const AttnMaps& maps, const AttnParams& p, cudaStream_t stream) {
  using L = SoloSmem<D, BN, kFp8 ? 1 : 2>;
  auto kern = attn_solo_kernel<D, BN, kFp8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  kern<<<dim3(p.NB, p.BH), kSoloThreads, L::kAlloc, stream>>>(maps, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_solo(int head_dim, int block, const AttnMaps& maps,
                                 const AttnParams& p, cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_solo<128, 128>(maps, p, stream);
  if (head_dim == 64 && block == 128) return launch_solo<64, 128>(maps, p, stream);
  if (head_dim == 64 && block == 64) return launch_solo<64, 64>(maps, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_fwd_solo_fp8(int head_dim, int block, const AttnMaps& maps,
                                     const AttnParams& p, cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_solo<128, 128, true>(maps, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_fwd_fp8(int head_dim, int block, const AttnMaps& maps,
                               const AttnParams& p, cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_one<128, 128, false, true>(maps, p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_gather(int head_dim, const AttnMaps& maps, const AttnParams& p,
                               cudaStream_t stream) {
  if (head_dim == 128) return launch_one<128, 128, true>(maps, p, stream);
  if (head_dim == 64) return launch_one<64, 128, true>(maps, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sa
