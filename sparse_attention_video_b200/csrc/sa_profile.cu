// Sampled-row pattern evaluation. For every head, on a sample of its query
// rows, attention is evaluated over all keys and under each of several
// sparse patterns; the head takes the pattern whose output has the lowest
// mean squared error against the full output (ties: the earlier pattern).
//   mode 0, SVG online head profiler (Sparse VideoGen review, key machinery;
//     Algorithm 1): the block masks of the spatial / temporal heads
//     (identity layout, frames within +-frame_radius; frame-major layout, a
//     shared spatial position), both with the sink blocks.
//   mode 1, STA per-head window search (Sliding Tile Attention review, key
//     machinery; Algorithm 1): one sliding tile window per candidate, on the
//     3D tile layout.
//
// The full pass (every sampled row against every key, the bulk of the work)
// runs on the tcgen05 block-sparse attention kernel: the sampled rows are
// gathered into 128-row query tiles, every tile visits every key block, and
// the kernel writes O in fp32. The masked passes then run here: one warp owns
// 16 sampled rows; keys pass through XOR-swizzled shared-memory tiles filled
// by cp.async (double-buffered); ldmatrix forms the fragments and mma.sync
// m16n8k16 (bf16 in, fp32 accumulate) computes S = Q K^T and O += P V with an
// online softmax in registers. The spatial pass walks key blocks in original
// order and the temporal pass in frame-major order (K/V rows gathered by
// token), per warp, each visiting only the blocks that some row of the warp
// keeps.
#include "sa_profile.h"
#include "sa_ptx.cuh"

namespace sa {

namespace {

constexpr int kProfWarps = 4;
constexpr int kRowsPerWarp = 16;
constexpr int kStepKeys = 16;

// Shared memory of a CTA: one K/V region cut into one double-buffered 16-key
// K/V pair per warp, then per warp its Q tile and the fp32 O of the full pass.
template <int D>
struct ProfSmem {
  static constexpr int kRow = D * 2;                       // one bf16 row
  static constexpr int kTile16 = kStepKeys * kRow;         // 16 rows (one step)
  static constexpr int kKV = kProfWarps * 4 * kTile16;     // K, V x 2 buffers per warp
  static constexpr int kOffWarp = kKV;
  static constexpr int kQ = kTile16;
  static constexpr int kPerWarp = kQ + kRowsPerWarp * D * 4;
  static constexpr int kBytes = kKV + kProfWarps * kPerWarp;
};

// Byte offset of 16-byte chunk c of row r in a tile of D bf16 per row: chunks
// XOR-swizzled by r % 8 so that the eight row addresses of an ldmatrix land
// in different banks.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(p)));
}

// D (16x8, fp32) += A (16x16, bf16, row) * B (16x8, bf16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct PatternGeo {
  int N, T, HW, BS, sink_blocks, radius;
};

// Spatial pattern, identity layout: query token's block and key block b keep
// each other when their frame ranges are at most ``radius`` apart.
__device__ __forceinline__ bool spatial_keep(const PatternGeo& g, int qtok, int b) {
  if (b < g.sink_blocks) return true;
  const int qb = qtok / g.BS;
  const int f_lo = (qb * g.BS) / g.HW, f_hi = (min(g.N, qb * g.BS + g.BS) - 1) / g.HW;
  const int k_lo = (b * g.BS) / g.HW, k_hi = (min(g.N, b * g.BS + g.BS) - 1) / g.HW;
  return max(0, max(k_lo - f_hi, f_lo - k_hi)) <= g.radius;
}

// Temporal pattern, frame-major layout (slot = (h*W + w)*T + t): the query
// token's block and key block b keep each other when they share a position.
__device__ __forceinline__ bool temporal_keep(const PatternGeo& g, int qtok, int b) {
  if (b < g.sink_blocks) return true;
  const int qb = ((qtok % g.HW) * g.T + qtok / g.HW) / g.BS;
  const int p_lo = (qb * g.BS) / g.T, p_hi = (min(g.N, qb * g.BS + g.BS) - 1) / g.T;
  const int k_lo = (b * g.BS) / g.T, k_hi = (min(g.N, b * g.BS + g.BS) - 1) / g.T;
  return !(k_hi < p_lo || p_hi < k_lo);
}

// STA window: key tile b (raster, tw fastest) against the query's tile.
__device__ __forceinline__ bool window_keep(int b, int nh, int nw, int qt, int qh, int qw,
                                            const int (&win)[3]) {
  const int kt = b / (nh * nw), kh = (b / nw) % nh, kw = b % nw;
  return abs(kt - qt) <= win[0] / 2 && abs(kh - qh) <= win[1] / 2 && abs(kw - qw) <= win[2] / 2;
}

template <int D>
__global__ void __launch_bounds__(32 * kProfWarps) profile_kernel(ProfileParams p) {
  using L = ProfSmem<D>;
  constexpr int kChunks = D / 8;                           // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t prof_smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y;
  const int row0 = (blockIdx.x * kProfWarps + warp) * kRowsPerWarp;
  const bool has_rows = row0 < p.n_rows;                   // warp-uniform
  uint8_t* kv = prof_smem;
  uint8_t* sQ = prof_smem + L::kOffWarp + warp * L::kPerWarp;
  float* sO = reinterpret_cast<float*>(sQ + L::kQ);
  const size_t head = (size_t)bh * p.N * D;
  const __nv_bfloat16* q = p.q + head;
  const __nv_bfloat16* k = p.k + head;
  const __nv_bfloat16* v = p.v + head;
  const PatternGeo geo{p.N, p.T, p.H * p.W, p.block, p.sink_blocks, p.frame_radius};
  const int nb = (p.N + p.block - 1) / p.block;
  const int subs = p.block / kStepKeys;

  // lane r < 16 holds the token of the warp's row r (-1: no row)
  int my_tok = -1;
  if (has_rows && lane < kRowsPerWarp && row0 + lane < p.n_rows) {
    my_tok = p.rows[(size_t)bh * p.n_rows + row0 + lane];
    if (my_tok < 0 || my_tok >= p.N) {
      if (p.status) atomicOr(p.status, SA_DEVFLAG_BOUNDS);
      my_tok = -1;
    }
  }
  // Q tile, then its A fragments for every 16-wide k step
  for (int e = lane; e < kRowsPerWarp * kChunks; e += 32) {
    const int r = e / kChunks, c = e % kChunks;
    const int t = __shfl_sync(0xffffffffu, my_tok, r);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t >= 0) val = __ldg(reinterpret_cast<const uint4*>(q + (size_t)t * D) + c);
    *reinterpret_cast<uint4*>(sQ + tile_off<D>(r, c)) = val;
  }
  __syncwarp();
  uint32_t qa[D / 16][4];
  {
    const int m = lane / 8, i = lane % 8;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
      ldsm_x4(sQ + tile_off<D>((m & 1) * 8 + i, 2 * ks + (m >> 1)), qa[ks][0], qa[ks][1],
              qa[ks][2], qa[ks][3]);
  }
  const int g = lane / 4, cq = 2 * (lane % 4);             // fragment row and column pair

  float acc[D / 8][4];
  float m0, m1, l0, l1;                                    // rows g and g + 8
  auto reset = [&]() {
#pragma unroll
    for (int j = 0; j < D / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  };
  // One step of 16 keys from 16-row tiles tK, tV; rows outside ``rmask`` and
  // keys outside ``kvm`` are masked.
  // kvm: bit i set when key i of the step exists (not padding)
  auto step16 = [&](const uint8_t* tK, const uint8_t* tV, uint32_t kvm, uint32_t rmask) {
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int m = lane / 8, i = lane % 8;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t b00, b01, b10, b11;
        ldsm_x4(tK + tile_off<D>((m >> 1) * 8 + i, 2 * ks + (m & 1)), b00, b01, b10, b11);
        mma16816(s0, qa[ks], b00, b01);
        mma16816(s1, qa[ks], b10, b11);
      }
    }
    const bool keep0 = (rmask >> g) & 1u, keep1 = (rmask >> (g + 8)) & 1u;
    const bool v00 = (kvm >> cq) & 1u, v01 = (kvm >> (cq + 1)) & 1u;
    const bool v10 = (kvm >> (8 + cq)) & 1u, v11 = (kvm >> (9 + cq)) & 1u;
    float x[8];
    x[0] = keep0 && v00 ? s0[0] * p.scale_log2 : -INFINITY;   // row g,     key cq
    x[1] = keep0 && v01 ? s0[1] * p.scale_log2 : -INFINITY;   // row g,     key cq + 1
    x[2] = keep1 && v00 ? s0[2] * p.scale_log2 : -INFINITY;   // row g + 8, key cq
    x[3] = keep1 && v01 ? s0[3] * p.scale_log2 : -INFINITY;
    x[4] = keep0 && v10 ? s1[0] * p.scale_log2 : -INFINITY;   // row g,     key 8 + cq
    x[5] = keep0 && v11 ? s1[1] * p.scale_log2 : -INFINITY;
    x[6] = keep1 && v10 ? s1[2] * p.scale_log2 : -INFINITY;   // row g + 8, key 8 + cq
    x[7] = keep1 && v11 ? s1[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[4], x[5]));
    float mx1 = fmaxf(fmaxf(x[2], x[3]), fmaxf(x[6], x[7]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
    const float a0 = ex2_approx(m0 - u0), a1 = ex2_approx(m1 - u1);   // 0 while m = -inf
    m0 = n0;
    m1 = n1;
    float pr[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) pr[e] = ex2_approx(x[e] - ((e & 2) ? u1 : u0));
    l0 = l0 * a0 + (pr[0] + pr[1]) + (pr[4] + pr[5]);
    l1 = l1 * a1 + (pr[2] + pr[3]) + (pr[6] + pr[7]);
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      acc[j][0] *= a0; acc[j][1] *= a0;
      acc[j][2] *= a1; acc[j][3] *= a1;
    }
    // P as the A fragment of the 16-key step (the accumulator layout of the
    // two n-tiles is the A layout of one k16 step)
    const uint32_t pa[4] = {pack_bf16x2(pr[0], pr[1]), pack_bf16x2(pr[2], pr[3]),
                            pack_bf16x2(pr[4], pr[5]), pack_bf16x2(pr[6], pr[7])};
    const int m = lane / 8, i = lane % 8;
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(tV + tile_off<D>((m & 1) * 8 + i, 2 * np + (m >> 1)), v0, v1, v2, v3);
      mma16816(acc[2 * np], pa, v0, v1);
      mma16816(acc[2 * np + 1], pa, v2, v3);
    }
  };
  // rows' sums over the four lanes that share them, O = acc / l; a masked
  // pass writes each row's squared error against the full pass's O
  auto finish = [&](int pass) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    float e0 = 0.f, e1 = 0.f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const int col = 8 * j + cq;
      // rounded products (no contraction into the subtraction below)
      const float o00 = __fmul_rn(acc[j][0], i0), o01 = __fmul_rn(acc[j][1], i0);
      const float o10 = __fmul_rn(acc[j][2], i1), o11 = __fmul_rn(acc[j][3], i1);
      const float* f0 = sO + g * D + col;
      const float* f1 = sO + (g + 8) * D + col;
      const float d00 = o00 - f0[0], d01 = o01 - f0[1], d10 = o10 - f1[0], d11 = o11 - f1[1];
      e0 += d00 * d00 + d01 * d01;
      e1 += d10 * d10 + d11 * d11;
    }
    e0 += __shfl_xor_sync(0xffffffffu, e0, 1);
    e0 += __shfl_xor_sync(0xffffffffu, e0, 2);
    e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
    e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
    if ((lane & 3) == 0) {
      float* re = p.row_err + ((size_t)bh * p.n_rows + row0) * p.n_pat + (pass - 1);
      if (row0 + g < p.n_rows) re[(size_t)g * p.n_pat] = e0;
      if (row0 + g + 8 < p.n_rows) re[(size_t)(g + 8) * p.n_pat] = e1;
    }
  };

  // ---- full pass: every key of every sampled row was attended by the
  // block-sparse attention kernel (tcgen05, a dense key list over gathered
  // query rows) before this kernel; its fp32 O of this warp's rows is the
  // reference the masked passes are measured against.
  if (has_rows) {
    for (int e = lane; e < kRowsPerWarp * D; e += 32) {
      const int r = e / D, c = e % D;
      sO[r * D + c] = row0 + r < p.n_rows ? p.o_full[((size_t)bh * p.n_rows + row0 + r) * D + c]
                                          : 0.f;
    }
    __syncwarp();
  }
  __syncthreads();
  if (!has_rows) return;
  uint8_t* sK = kv + warp * 4 * L::kTile16;                // 2 K buffers, then 2 V buffers
  uint8_t* sV = sK + 2 * L::kTile16;

  // ---- masked passes, per warp. Mode 0: spatial (original order) and
  // temporal (frame-major order); mode 1: one tile window per candidate (3D
  // tile order, padding slots inside tiles masked)
  const int bt = p.tile[0], bhh = p.tile[1], bw = p.tile[2];
  const int tnh = (p.H + bhh - 1) / bhh, tnw = (p.W + bw - 1) / bw;
  const int tnb = ((p.T + bt - 1) / bt) * tnh * tnw;
  int qt = 0, qh = 0, qw = 0;                              // the row's tile (mode 1)
  if (p.mode == 1 && my_tok >= 0) {
    qt = my_tok / geo.HW / bt;
    qh = (my_tok / p.W) % p.H / bhh;
    qw = my_tok % p.W / bw;
  }
  // slot s of the pass's order -> token, or -1 for a padding slot
  auto slot_token = [&](int pass, int slot) -> int {
    if (p.mode == 0) {
      if (slot >= p.N) return -1;
      return pass == 2 ? (slot % p.T) * geo.HW + slot / p.T : slot;
    }
    const int b = slot / p.block, s = slot % p.block;
    const int t = b / (tnh * tnw) * bt + s / (bhh * bw);
    const int h = (b / tnw) % tnh * bhh + (s / bw) % bhh;
    const int w = b % tnw * bw + s % bw;
    return (t < p.T && h < p.H && w < p.W) ? (t * p.H + h) * p.W + w : -1;
  };
  const int nb_pass = p.mode == 0 ? nb : tnb;
  // one pattern per CTA along grid z (the full pass's O is in global memory,
  // so the patterns are independent)
  for (int pass = 1 + (int)blockIdx.z; pass <= p.n_pat; pass += (int)gridDim.z) {
    int win[3] = {1, 1, 1};
    if (p.mode == 1) { win[0] = p.win[pass - 1][0]; win[1] = p.win[pass - 1][1]; win[2] = p.win[pass - 1][2]; }
    // rows (bits 0..15) that keep key block b under this pass's pattern
    auto keeps = [&](int b) -> uint32_t {
      bool kp = false;
      if (my_tok >= 0) {
        if (p.mode == 1) kp = window_keep(b, tnh, tnw, qt, qh, qw, win);
        else kp = pass == 1 ? spatial_keep(geo, my_tok, b) : temporal_keep(geo, my_tok, b);
      }
      return __ballot_sync(0xffffffffu, kp) & 0xFFFFu;
    };
    auto next_block = [&](int from, uint32_t& rmask) -> int {
      for (int x = from; x < nb_pass; ++x) {
        const uint32_t mk = keeps(x);
        if (mk) { rmask = mk; return x; }
      }
      return nb_pass;
    };
    // keys of step (b, sub) that exist
    auto step_keys = [&](int b, int sub) -> uint32_t {
      const bool ok = lane < kStepKeys && slot_token(pass, b * p.block + sub * kStepKeys + lane) >= 0;
      return __ballot_sync(0xffffffffu, ok) & 0xFFFFu;
    };
    // 16 key rows of step (b, sub) into buffer ``buf``; padding slots are zero
    auto load_step = [&](int buf, int b, int sub) {
      for (int e = lane; e < kStepKeys * kChunks; e += 32) {
        const int r = e / kChunks, c = e % kChunks;
        const int tok = slot_token(pass, b * p.block + sub * kStepKeys + r);
        uint8_t* dk = sK + buf * L::kTile16 + tile_off<D>(r, c);
        uint8_t* dv = sV + buf * L::kTile16 + tile_off<D>(r, c);
        if (tok >= 0) {
          cp_async16(dk, k + (size_t)tok * D + c * 8);
          cp_async16(dv, v + (size_t)tok * D + c * 8);
        } else {
          *reinterpret_cast<uint4*>(dk) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(dv) = make_uint4(0, 0, 0, 0);
        }
      }
      cp_async_commit();
    };
    reset();
    uint32_t rmask = 0;
    int b = next_block(0, rmask), sub = 0, buf = 0;
    if (b < nb_pass) load_step(0, b, 0);
    while (b < nb_pass) {
      int b2 = b, s2 = sub + 1;
      uint32_t rm2 = rmask;
      if (s2 == subs) { s2 = 0; b2 = next_block(b + 1, rm2); }
      if (b2 < nb_pass) {
        load_step(buf ^ 1, b2, s2);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      step16(sK + buf * L::kTile16, sV + buf * L::kTile16, step_keys(b, sub), rmask);
      __syncwarp();                                       // tile free for the load two steps on
      buf ^= 1;
      b = b2;
      sub = s2;
      rmask = rm2;
    }
    finish(pass);
  }
}

// Per head and pattern, the rows' errors summed in a fixed order
// (lane-strided partial sums, then a fixed shuffle tree), and the pattern
// with the lowest mean error (ties: the earlier one).
__global__ void profile_reduce_kernel(ProfileParams p) {
  const int bh = blockIdx.x, lane = threadIdx.x;
  const float* re = p.row_err + (size_t)bh * p.n_rows * p.n_pat;
  const float n = (float)p.n_rows * (float)p.d;
  int best = 0;
  float best_v = 0.f;
  for (int c = 0; c < p.n_pat; ++c) {
    float s = 0.f;
    for (int r = lane; r < p.n_rows; r += 32) s += re[(size_t)r * p.n_pat + c];
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float m = s / n;
    if (lane == 0) p.mse[bh * p.n_pat + c] = m;
    if (c == 0 || m < best_v) { best = c; best_v = m; }
  }
  if (lane == 0) p.choice[bh] = (int8_t)best;
}

}  // namespace

template <int D>
static cudaError_t launch_profile_d(const ProfileParams& p, cudaStream_t st) {
  using L = ProfSmem<D>;
  cudaError_t e = cudaFuncSetAttribute(profile_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::kBytes);
  if (e != cudaSuccess) return e;
  const int rows_per_cta = kProfWarps * kRowsPerWarp;
  dim3 grid((p.n_rows + rows_per_cta - 1) / rows_per_cta, p.BH, p.n_pat);
  profile_kernel<D><<<grid, 32 * kProfWarps, L::kBytes, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  profile_reduce_kernel<<<p.BH, 32, 0, st>>>(p);
  return cudaGetLastError();
}

namespace {

// One 16-byte piece per thread: piece c of row r of head bh.
__global__ void gather_rows_kernel(const __nv_bfloat16* src, const int* rows, int N, int d,
                                   int n_rows, int n_pad, __nv_bfloat16* dst, uint32_t* status) {
  const int bh = blockIdx.y;
  const int pieces = d / 8;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int r = (int)(i / pieces), c = (int)(i % pieces);
  if (r >= n_pad) return;
  uint4 val = make_uint4(0, 0, 0, 0);
  if (r < n_rows) {
    const int t = rows[(size_t)bh * n_rows + r];
    if (t >= 0 && t < N) {
      val = __ldg(reinterpret_cast<const uint4*>(src + ((size_t)bh * N + t) * d) + c);
    } else if (status) {
      atomicOr(status, SA_DEVFLAG_BOUNDS);
    }
  }
  reinterpret_cast<uint4*>(dst + ((size_t)bh * n_pad + r) * d)[c] = val;
}

}  // namespace

cudaError_t launch_gather_rows(const __nv_bfloat16* src, const int* rows, int BH, int N, int d,
                               int n_rows, int n_pad, __nv_bfloat16* dst, uint32_t* status,
                               cudaStream_t stream) {
  const long long pieces = (long long)n_pad * (d / 8);
  dim3 grid((unsigned)((pieces + 255) / 256), BH);
  gather_rows_kernel<<<grid, 256, 0, stream>>>(src, rows, N, d, n_rows, n_pad, dst, status);
  return cudaGetLastError();
}

cudaError_t launch_profile(const ProfileParams& p, cudaStream_t stream) {
  if (p.d == 128) return launch_profile_d<128>(p, stream);
  if (p.d == 64) return launch_profile_d<64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sa
