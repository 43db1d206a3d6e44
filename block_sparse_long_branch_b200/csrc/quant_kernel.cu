// quant_kernel.cu -- e4m3 index tensors for the quantised Index Branch.
//
// The pages report the sparse attention's indexer and main branch moving
// from Q8KV8 to Q8KV4 in a later model (dot-ai "MiniMax M3.1 Flashとは？428Bの
// MoEモデルがウェイト公開", the passage on the ModelScope model card's
// quantisation); the number format is not given.  The reading used here quantises the Index Branch's
// inputs to e4m3 with one fp32 scale per index-query row and one per 128-key
// block of index keys:
//   s = max|x| / 448 (fp32, round to nearest; 1 if max|x| = 0)
//   x8 = e4m3(x / s)  (fp32 division, round to nearest even, saturating)
// The selection ranks blocks by s_j * <q8, k8>: a query row's own scale is a
// positive constant of the row and cannot change its ranking, so only the key
// scales are kept.
#include <cuda_fp8.h>

#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ uint8_t to_e4m3(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float scale_of(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
}

// one warp per row of DI values (DI / 32 per lane); the row's scale is written
// to `scale` when it is given
template <int DI>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                         int64_t rows, uint8_t* __restrict__ x8,
                                                         float* __restrict__ scale) {
  constexpr int PER = DI / 32;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* src = x + r * DI + lane * PER;
  float v[PER];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = __bfloat162float(src[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = scale_of(amax);
  if (scale && lane == 0) scale[r] = s;
#pragma unroll
  for (int i = 0; i < PER; ++i) x8[r * DI + lane * PER + i] = to_e4m3(__fdiv_rn(v[i], s));
}

// one CTA per 128-key block of the index keys
template <int DI>
__global__ void __launch_bounds__(256) quant_blocks_kernel(const __nv_bfloat16* __restrict__ k,
                                                           int64_t N, uint8_t* __restrict__ k8,
                                                           float* __restrict__ kscale) {
  __shared__ float red[8];
  const int64_t j = blockIdx.x;
  const int64_t r0 = j * 128;
  const int nrows = (int)min64(128, N - r0);
  const int n = nrows * DI;
  const __nv_bfloat16* src = k + r0 * DI;
  float amax = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) amax = fmaxf(amax, fabsf(__bfloat162float(src[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = scale_of(amax);
  if (threadIdx.x == 0) kscale[j] = s;
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    k8[r0 * DI + i] = to_e4m3(__fdiv_rn(__bfloat162float(src[i]), s));
}

}  // namespace

cudaError_t launch_quantize_index(const QuantLaunch& p, cudaStream_t s) {
  const int64_t rows = p.N * p.G;
  const int64_t nb = (p.N + 127) / 128;
  if (p.d_idx != 128) return cudaErrorInvalidValue;
  const auto* q = static_cast<const __nv_bfloat16*>(p.q_idx);
  const auto* k = static_cast<const __nv_bfloat16*>(p.k_idx);
  quant_rows_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      q, rows, static_cast<uint8_t*>(p.q_idx8), nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  quant_blocks_kernel<128><<<(unsigned)nb, 256, 0, s>>>(k, p.N, static_cast<uint8_t*>(p.k_idx8),
                                                        p.kscale);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const void* x, int64_t rows, void* x8, float* scale,
                                 cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  quant_rows_kernel<128><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), rows, static_cast<uint8_t*>(x8), scale);
  return cudaGetLastError();
}

}  // namespace msa
