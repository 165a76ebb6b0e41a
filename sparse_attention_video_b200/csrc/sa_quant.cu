// FP8 (E4M3) operands with one scale per tensor (Sparse VideoGen review: the
// optional FP8 quantization of attention). E4M3 as in "FP8 Formats for Deep
// Learning" (Micikevicius et al.): bias 7, 3 mantissa bits, largest finite
// value 448, no infinity.
//
// Three stream-ordered passes over n_tensors contiguous bf16 tensors:
//   amax      max |x| per tensor; the float bits of a non-negative float
//             order like unsigned integers, so CTAs combine with atomicMax
//             on the (zeroed) inv buffer;
//   encode    inv = 448 / amax and y = x * inv, each one correctly rounded
//             float32 operation, then y to E4M3 (round to nearest even,
//             saturating at 448): eight codes per 16-byte load;
//   finalize  the inv buffer's amax bits become inv (1 for an all-zero tensor).
// HBM-bound: 2 bytes read (twice) and 1 byte written per element.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "sa_quant.h"

namespace sa {

namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float inv_scale(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
}

__global__ void __launch_bounds__(kQuantThreads) amax_kernel(const __nv_bfloat16* x,
                                                             long long n, uint32_t* amax_bits) {
  const int t = blockIdx.y;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * n);
  const long long nv = n / 8;
  uint32_t m = 0u;                       // |x| bits: the sign bit cleared
  for (long long i = blockIdx.x * (long long)kQuantThreads + threadIdx.x; i < nv;
       i += (long long)gridDim.x * kQuantThreads) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m = max(m, (w[e] << 16) & 0x7FFFFFFFu);
      m = max(m, w[e] & 0x7FFF0000u);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t wm[kQuantThreads / 32];
  if (threadIdx.x % 32 == 0) wm[threadIdx.x / 32] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0u;
#pragma unroll
    for (int i = 0; i < kQuantThreads / 32; ++i) r = max(r, wm[i]);
    atomicMax(amax_bits + t, r);
  }
}

__global__ void __launch_bounds__(kQuantThreads) encode_kernel(const __nv_bfloat16* x, long long n,
                                                               const uint32_t* amax_bits,
                                                               uint8_t* codes) {
  const int t = blockIdx.y;
  const float inv = inv_scale(amax_bits[t]);
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * n);
  uint2* dst = reinterpret_cast<uint2*>(codes + (size_t)t * n);
  const long long nv = n / 8;
  for (long long i = blockIdx.x * (long long)kQuantThreads + threadIdx.x; i < nv;
       i += (long long)gridDim.x * kQuantThreads) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t half[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // element 2e is the low half of word e; the pair's first code is the
      // low byte of the conversion
      const float lo = __fmul_rn(__uint_as_float(w[e] << 16), inv);
      const float hi = __fmul_rn(__uint_as_float(w[e] & 0xFFFF0000u), inv);
      half[e] = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    }
    dst[i] = make_uint2(half[0] | (half[1] << 16), half[2] | (half[3] << 16));
  }
}

__global__ void finalize_kernel(uint32_t* amax_bits, int n_tensors) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n_tensors) {
    const float inv = inv_scale(amax_bits[t]);
    reinterpret_cast<float*>(amax_bits)[t] = inv;
  }
}

}  // namespace

cudaError_t launch_quant_e4m3(const QuantParams& p, cudaStream_t st) {
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(p.inv);
  cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t) * (size_t)p.n_tensors, st);
  if (e != cudaSuccess) return e;
  // about four CTAs of 256 threads per SM over all tensors, at least one per
  // tensor, none without a full vector of work
  const long long nv = p.n_elems / 8;
  long long per = (4LL * 148 + p.n_tensors - 1) / p.n_tensors;
  per = std::min<long long>(per, (nv + kQuantThreads - 1) / kQuantThreads);
  per = std::max<long long>(per, 1);
  const dim3 grid((unsigned)per, (unsigned)p.n_tensors);
  amax_kernel<<<grid, kQuantThreads, 0, st>>>(p.x, p.n_elems, amax_bits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  encode_kernel<<<grid, kQuantThreads, 0, st>>>(p.x, p.n_elems, amax_bits, p.codes);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  finalize_kernel<<<(p.n_tensors + 255) / 256, 256, 0, st>>>(amax_bits, p.n_tensors);
  return cudaGetLastError();
}

}  // namespace sa
