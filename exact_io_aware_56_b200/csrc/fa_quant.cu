// e4m3 block quantization for the FP8 forward (FlashAttention: IO-aware
// exact attention, "The generations": FP8 support with block scaling).
//
// A block is 128 consecutive rows of one (batch, head) of a [BH][N][d] bf16
// tensor (Q and K), or the whole head (V). Its scale is s = amax / 448 (448
// = the largest finite e4m3), and its codes are e4m3(x * (448 / amax)),
// rounded to nearest even and saturated; the reciprocal and the product are
// each one correctly rounded fp32 operation. An all-zero block gets s = 1
// and zero codes. Three launches, all HBM-bound:
//   1. block (or head) amax, written over the scale array (a head's amax
//      through an atomic max on the bit pattern: non-negative floats order
//      like their bits, and the array starts at zero);
//   2. the codes, one CTA per block;
//   3. amax -> scale in place.

#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kQuantRows = 128;
constexpr int kQuantThreads = 256;

// Elements of block `blk` of head `bh`: rows [blk * 128, min(N, blk * 128 + 128))
// of that head, d contiguous elements each, contiguous in memory.
__device__ __forceinline__ void block_range(int bh, int blk, int N, int d, long long* start, int* count) {
  const int r0 = blk * kQuantRows;
  const int rows = min(kQuantRows, N - r0);
  *start = (static_cast<long long>(bh) * N + r0) * d;
  *count = rows * d;
}

__global__ void __launch_bounds__(kQuantThreads) quant_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   float* __restrict__ amax, int N, int d,
                                                                   int nb, int per_head) {
  const int bh = static_cast<int>(blockIdx.x / nb), blk = static_cast<int>(blockIdx.x % nb);
  long long start;
  int count;
  block_range(bh, blk, N, d, &start, &count);
  const uint4* src = reinterpret_cast<const uint4*>(x + start);  // 8 bf16 per vector; d is 64 or 128
  float m = 0.f;
  for (int i = threadIdx.x; i < count / 8; i += kQuantThreads) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
      m = fmaxf(m, fmaxf(fabsf(__low2float(h)), fabsf(__high2float(h))));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float part[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, part[i]);
    if (per_head)
      atomicMax(reinterpret_cast<unsigned int*>(amax) + bh, __float_as_uint(m));
    else
      amax[static_cast<long long>(bh) * nb + blk] = m;
  }
}

__global__ void __launch_bounds__(kQuantThreads) quant_codes_kernel(const __nv_bfloat16* __restrict__ x,
                                                                    uint8_t* __restrict__ codes,
                                                                    const float* __restrict__ amax, int N, int d,
                                                                    int nb, int per_head) {
  const int bh = static_cast<int>(blockIdx.x / nb), blk = static_cast<int>(blockIdx.x % nb);
  long long start;
  int count;
  block_range(bh, blk, N, d, &start, &count);
  const float am = per_head ? amax[bh] : amax[static_cast<long long>(bh) * nb + blk];
  uint2* dst = reinterpret_cast<uint2*>(codes + start);
  if (!(am > 0.f)) {  // all-zero block: zero codes (also for -0.0 inputs)
    for (int i = threadIdx.x; i < count / 8; i += kQuantThreads) dst[i] = make_uint2(0u, 0u);
    return;
  }
  const float inv = __fdiv_rn(448.f, am);
  const uint4* src = reinterpret_cast<const uint4*>(x + start);
  for (int i = threadIdx.x; i < count / 8; i += kQuantThreads) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float y[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
      y[2 * k] = __fmul_rn(__low2float(h), inv);
      y[2 * k + 1] = __fmul_rn(__high2float(h), inv);
    }
    dst[i] = make_uint2(pack_e4m3x4(y[0], y[1], y[2], y[3]), pack_e4m3x4(y[4], y[5], y[6], y[7]));
  }
}

__global__ void quant_scales_kernel(float* __restrict__ s, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s[i] = s[i] > 0.f ? __fdiv_rn(s[i], 448.f) : 1.f;
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* x, void* codes, float* scales, int BH, int N, int d, int per_head,
                                cudaStream_t stream) {
  const int nb = (N + kQuantRows - 1) / kQuantRows;
  const int n_scales = per_head ? BH : BH * nb;
  cudaError_t e;
  if (per_head && (e = cudaMemsetAsync(scales, 0, sizeof(float) * n_scales, stream)) != cudaSuccess) return e;
  const long long blocks = static_cast<long long>(nb) * BH;  // one CTA per (head, block), head-major
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const unsigned grid = static_cast<unsigned>(blocks);
  quant_amax_kernel<<<grid, kQuantThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), scales, N, d, nb,
                                                        per_head);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  quant_codes_kernel<<<grid, kQuantThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                         static_cast<uint8_t*>(codes), scales, N, d, nb, per_head);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  quant_scales_kernel<<<(n_scales + 255) / 256, 256, 0, stream>>>(scales, n_scales);
  return cudaGetLastError();
}

}  // namespace fa
