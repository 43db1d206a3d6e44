// mx_kernel.cu -- MX block formats for the quantised Main Branch ("Q8KV4").
//
// The pages report the sparse attention moving from Q8KV8 to Q8KV4 in a later
// model (dot-ai "MiniMax M3.1 Flashとは？428BのMoEモデルがウェイト公開", the
// passage on the ModelScope model card's quantisation) and name no number
// format.  The reading used: the OCP Microscaling (MX) formats, version 1.0.
// Every 32 consecutive values along d share one power-of-two scale 2^X, kept
// as an E8M0 byte (X + 127):
//   X = floor(log2(max|x|)) - emax_elem   (emax_elem 8 for e4m3, 2 for e2m1;
//                                          -127 for an all-zero block;
//                                          clamped to [-127, 127])
//   element = nearest value of the element format to x / 2^X (ties to even),
//             saturating at its largest magnitude (448 for e4m3, 6 for e2m1).
// Q is MXFP8 (e4m3 elements, one byte each); K and V are MXFP4 (e2m1
// elements, two per byte, element 2i in the low nibble).
//
// The prefill dequantises them exactly to bf16 in its workspace (an e4m3 or
// e2m1 value times a power of two has at most 4 significant bits, and the
// exponents stay within bf16's range for scales the quantiser writes) and
// runs the unchanged Main Branch on the result.
#include <cuda_fp8.h>

#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kMxBlock = 32;
constexpr int kPer = 8;  // elements per thread: 4 threads per block of 32

// floor(log2(a)) of a finite a > 0, from its fp32 bit pattern (exact, also
// for subnormal a)
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int e = (int)(b >> 23);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(b & 0x7FFFFF))) - 149;
}

// nearest e2m1 code of y (ties to the even code, saturating at 6); the sign
// bit is y's own
__device__ __forceinline__ uint32_t to_e2m1(float y) {
  const float a = fabsf(y);
  uint32_t c;
  if (a <= 0.25f) c = 0;        // tie at 0.25 -> 0 (code 0)
  else if (a < 0.75f) c = 1;    // 0.5
  else if (a <= 1.25f) c = 2;   // 1.0 (ties at 0.75 and 1.25 -> code 2)
  else if (a < 1.75f) c = 3;    // 1.5
  else if (a <= 2.5f) c = 4;    // 2.0 (ties at 1.75 and 2.5 -> code 4)
  else if (a < 3.5f) c = 5;     // 3.0
  else if (a <= 5.0f) c = 6;    // 4.0 (ties at 3.5 and 5 -> code 6)
  else c = 7;                   // 6.0
  return c | ((__float_as_uint(y) >> 31) << 3);
}

__device__ __forceinline__ float from_e2m1(uint32_t c) {
  const uint32_t m = c & 7;
  const float mag = m < 4 ? 0.5f * (float)m : (float)(1u << ((m >> 1) - 1)) * (1.f + 0.5f * (float)(m & 1));
  return (c & 8) ? -mag : mag;
}

__device__ __forceinline__ float from_e4m3(uint32_t c) {
  const __nv_fp8_e4m3 v = *reinterpret_cast<const __nv_fp8_e4m3*>(&c);
  return (float)v;
}

// x [n_blocks * 32] bf16 -> codes and scales.  Thread t handles elements
// 8t .. 8t+7; the 4 threads of a block share its maximum by shuffles.
template <int FMT>
__global__ void __launch_bounds__(256) mx_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                       int64_t n_blocks, uint8_t* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  constexpr int kEmax = FMT == kMxE4m3 ? 8 : 2;
  const int64_t n_threads = n_blocks * (kMxBlock / kPer);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // every warp covers whole blocks (32 threads = 8 blocks), so the shuffles
  // below run with the full warp active
  for (int64_t t0 = (int64_t)blockIdx.x * blockDim.x; t0 < n_threads; t0 += stride) {
    const int64_t t = t0 + threadIdx.x;
    const bool on = t < n_threads;
    float v[kPer];
    float amax = 0.f;
    if (on) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x) + t);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        v[i] = __bfloat162float(h[i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (!on) continue;
    int X = amax > 0.f ? floor_log2(amax) - kEmax : -127;
    X = X < -127 ? -127 : (X > 127 ? 127 : X);
    // 2^-X is a normal fp32 power of two here: X >= -127, and X <= 119 (e4m3)
    // or 125 (e2m1) because a finite amax is below 2^128
    const float inv = __uint_as_float((uint32_t)(127 - X) << 23);
    if ((threadIdx.x & 3) == 0) scales[t >> 2] = (uint8_t)(X + 127);
    if (FMT == kMxE4m3) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lo |= (uint32_t)__nv_cvt_float_to_fp8(v[i] * inv, __NV_SATFINITE, __NV_E4M3) << (8 * i);
        hi |= (uint32_t)__nv_cvt_float_to_fp8(v[4 + i] * inv, __NV_SATFINITE, __NV_E4M3) << (8 * i);
      }
      reinterpret_cast<uint2*>(codes)[t] = make_uint2(lo, hi);
    } else {
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < kPer; ++i) w |= to_e2m1(v[i] * inv) << (4 * i);
      reinterpret_cast<uint32_t*>(codes)[t] = w;
    }
  }
}

// codes and scales -> bf16, exactly (see the file header).  Thread t handles
// chunk t: elements 8t .. 8t+7 of block t/4, that is 8 (e4m3) or 4 (e2m1)
// bytes of codes in and 16 bytes of bf16 out, so a warp's loads and stores
// each cover one contiguous run.  A thread issues the loads of kDqDepth chunks
// (one grid stride apart) before it converts any of them.  The grid is one
// resident wave (kDqCtasPerSm CTAs per SM), so no CTA waits for a second wave.
constexpr int kDqDepth = 8;
constexpr int kDqCtasPerSm = 6;

template <int FMT>
__global__ void __launch_bounds__(256, kDqCtasPerSm)
    mx_dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                      int64_t n_blocks, __nv_bfloat16* __restrict__ out) {
  const int64_t n_chunks = n_blocks * (kMxBlock / kPer);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c0 < n_chunks;
       c0 += kDqDepth * stride) {
    uint2 w[kDqDepth];  // e4m3: 8 codes in x and y; e2m1: 8 nibbles in x
    uint32_t sx[kDqDepth / 4] = {};  // the chunks' scale bytes, four to a word
#pragma unroll
    for (int u = 0; u < kDqDepth; ++u) {
      const int64_t c = c0 + u * stride;
      w[u] = make_uint2(0, 0);
      if (c < n_chunks) {
        if (FMT == kMxE4m3)
          w[u] = __ldg(reinterpret_cast<const uint2*>(codes) + c);
        else
          w[u].x = __ldg(reinterpret_cast<const uint32_t*>(codes) + c);
        sx[u / 4] |= (uint32_t)__ldg(scales + (c >> 2)) << (8 * (u % 4));
      }
    }
#pragma unroll
    for (int u = 0; u < kDqDepth; ++u) {
      const int64_t c = c0 + u * stride;
      if (c >= n_chunks) break;
      const int X = (int)((sx[u / 4] >> (8 * (u % 4))) & 0xFF) - 127;
      // v * 2^X by one multiply, exact while 2^X and the product stay normal
      // (elements are at least 2^-9 in magnitude, or zero); ldexpf otherwise
      const bool mul = X >= -110 && X <= 120;
      const float p2 = __uint_as_float((uint32_t)(mul ? X + 127 : 127) << 23);
      float v[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (FMT == kMxE4m3)
          v[i] = from_e4m3(((i < 4 ? w[u].x : w[u].y) >> (8 * (i % 4))) & 0xFF);
        else
          v[i] = from_e2m1((w[u].x >> (4 * i)) & 0xF);
        v[i] = mul ? v[i] * p2 : ldexpf(v[i], X);
      }
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        ow[i] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      reinterpret_cast<uint4*>(out)[c] = o;
    }
  }
}

unsigned grid_for(int64_t n_threads, int sms, int ctas_per_sm = 16) {
  const int64_t want = (n_threads + 255) / 256;
  const int64_t cap = (int64_t)sms * ctas_per_sm;
  return (unsigned)(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

cudaError_t launch_mx_quantize(const void* x, int64_t n_blocks, int fmt, void* codes,
                               uint8_t* scales, int sms, cudaStream_t s) {
  if (n_blocks <= 0) return cudaSuccess;
  const unsigned g = grid_for(n_blocks * 4, sms);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* c = static_cast<uint8_t*>(codes);
  if (fmt == kMxE4m3)
    mx_quant_kernel<kMxE4m3><<<g, 256, 0, s>>>(xb, n_blocks, c, scales);
  else
    mx_quant_kernel<kMxE2m1><<<g, 256, 0, s>>>(xb, n_blocks, c, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_dequantize(const void* codes, const uint8_t* scales, int64_t n_blocks,
                                 int fmt, void* out, int sms, cudaStream_t s) {
  if (n_blocks <= 0) return cudaSuccess;
  const unsigned g = grid_for((n_blocks * 4 + kDqDepth - 1) / kDqDepth, sms, kDqCtasPerSm);
  const auto* c = static_cast<const uint8_t*>(codes);
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (fmt == kMxE4m3)
    mx_dequant_kernel<kMxE4m3><<<g, 256, 0, s>>>(c, scales, n_blocks, o);
  else
    mx_dequant_kernel<kMxE2m1><<<g, 256, 0, s>>>(c, scales, n_blocks, o);
  return cudaGetLastError();
}

}  // namespace msa
