// merge_kernel.cu -- combines the per-block partial softmaxes of each query.
//
// The Main Branch is one exact softmax over all selected keys (ai-tool-zukan
// "MiniMax MSA guide", section "Index BranchとMain Branchの役割分担").  The
// key-block-outer kernel produces it in pieces, one per selected block r:
// o_r (normalised over block r) and lse_r = log sum_{s in r} exp(logit_s).
// The exact result is  out = sum_r exp(lse_r - L) o_r  with  L = log sum_r
// exp(lse_r),  i.e. the standard log-sum-exp split of a softmax.
//
// One warp per (query t, group g).  The group's H/G heads x d values of one
// slot are contiguous (2 KiB for 8 heads of 128): lane l owns CPL consecutive
// 16-byte chunks, all inside one head, so it needs one set of weights and
// issues the loads of every slot before it uses them.  HBM-bound.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;

template <int CPL, int KMAX>
__global__ void __launch_bounds__(kWarps * 32)
    merge_kernel(const __half* __restrict__ part_o, const float* __restrict__ part_lse,
                 const int32_t* __restrict__ ids, int64_t rows, int32_t G, int32_t HG, int32_t d,
                 int32_t top_k, __nv_bfloat16* __restrict__ out) {
  const int64_t tg = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tg >= rows * G) return;
  const int lane = threadIdx.x & 31;
  const int32_t idv = lane < top_k ? __ldg(ids + tg * top_k + lane) : -1;
  const uint32_t valid = __ballot_sync(0xffffffffu, idv >= 0);  // bit r: slot r holds a block
  const int chunks = HG * d / 8;
  const int c0 = lane * CPL;
  if (c0 >= chunks) return;
  const int h = (c0 * 8) / d;
  const int64_t slot_elems = (int64_t)HG * d;
  const __half* o_tg = part_o + tg * top_k * slot_elems + (int64_t)c0 * 8;
  const float* l_tg = part_lse + tg * top_k * HG + h;

  float lse[KMAX];
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < KMAX; ++r) {
    lse[r] = (r < top_k && (valid >> r & 1u)) ? __ldg(l_tg + r * HG) : -INFINITY;
    m = fmaxf(m, lse[r]);
  }
  float acc[CPL * 8];
#pragma unroll
  for (int x = 0; x < CPL * 8; ++x) acc[x] = 0.f;
  float wsum = 0.f;
#pragma unroll
  for (int r = 0; r < KMAX; ++r) {
    if (r >= top_k || !(valid >> r & 1u)) continue;
    const float w = __expf(lse[r] - m);
    wsum += w;
    const uint4* src = reinterpret_cast<const uint4*>(o_tg + r * slot_elems);
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const uint4 v = __ldg(src + i);
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float2 f = __half22float2(hv[x]);
        acc[i * 8 + 2 * x] = fmaf(w, f.x, acc[i * 8 + 2 * x]);
        acc[i * 8 + 2 * x + 1] = fmaf(w, f.y, acc[i * 8 + 2 * x + 1]);
      }
    }
  }
  const float inv = 1.0f / wsum;
  uint4* dst = reinterpret_cast<uint4*>(out + tg * slot_elems + (int64_t)c0 * 8);
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    uint4 ov;
    ov.x = pack_bf16x2(acc[i * 8 + 0] * inv, acc[i * 8 + 1] * inv);
    ov.y = pack_bf16x2(acc[i * 8 + 2] * inv, acc[i * 8 + 3] * inv);
    ov.z = pack_bf16x2(acc[i * 8 + 4] * inv, acc[i * 8 + 5] * inv);
    ov.w = pack_bf16x2(acc[i * 8 + 6] * inv, acc[i * 8 + 7] * inv);
    dst[i] = ov;
  }
}

template <int KMAX>
cudaError_t launch_k(const MergeLaunch& p, cudaStream_t s, unsigned grid) {
  const int chunks = (p.H / p.G) * p.d / 8;  // 16-byte chunks per slot, a power of two >= 8
  auto* o = static_cast<__nv_bfloat16*>(p.out);
  const int HG = p.H / p.G;
  if (chunks >= 256) {
    merge_kernel<8, KMAX><<<grid, kWarps * 32, 0, s>>>(p.part_o, p.part_lse, p.ids, p.rows, p.G,
                                                        HG, p.d, p.top_k, o);
  } else if (chunks >= 128) {
    merge_kernel<4, KMAX><<<grid, kWarps * 32, 0, s>>>(p.part_o, p.part_lse, p.ids, p.rows, p.G,
                                                        HG, p.d, p.top_k, o);
  } else if (chunks >= 64) {
    merge_kernel<2, KMAX><<<grid, kWarps * 32, 0, s>>>(p.part_o, p.part_lse, p.ids, p.rows, p.G,
                                                        HG, p.d, p.top_k, o);
  } else {
    merge_kernel<1, KMAX><<<grid, kWarps * 32, 0, s>>>(p.part_o, p.part_lse, p.ids, p.rows, p.G,
                                                        HG, p.d, p.top_k, o);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeLaunch& p, cudaStream_t s) {
  const int64_t warps = p.rows * p.G;
  if (warps == 0) return cudaSuccess;
  const int chunks = (p.H / p.G) * p.d / 8;
  if (chunks > 32 * 8) return cudaErrorInvalidValue;  // H/G * d > 2048: not instantiated
  const unsigned grid = (unsigned)((warps + kWarps - 1) / kWarps);
  if (p.top_k <= 16) return launch_k<16>(p, s, grid);
  return launch_k<32>(p, s, grid);
}

}  // namespace msa
