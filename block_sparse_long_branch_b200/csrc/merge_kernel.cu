// merge_kernel.cu -- combines the per-block partial softmaxes of each query.
//
// The Main Branch is one exact softmax over all selected keys (ai-tool-zukan
// "MiniMax MSA guide", section "Index BranchとMain Branchの役割分担").  The
// key-block-outer kernel produces it in pieces, one per selected block r:
// o_r (normalised over block r) and lse_r = log sum_{s in r} exp(logit_s).
// The exact result is  out = sum_r exp(lse_r - L) o_r  with  L = log sum_r
// exp(lse_r),  i.e. the standard log-sum-exp split of a softmax.
//
// One warp per (query t, group g): the group's H/G heads x d values of one
// slot are contiguous (2 KiB for 8 heads of 128), so every slot is read with
// fully coalesced 16-byte loads.  HBM-bound.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32)
    merge_kernel(const __half* __restrict__ part_o, const float* __restrict__ part_lse,
                 const int32_t* __restrict__ ids, int64_t rows, int32_t G, int32_t HG, int32_t d,
                 int32_t top_k, __nv_bfloat16* __restrict__ out) {
  const int64_t tg = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tg >= rows * G) return;
  const int lane = threadIdx.x & 31;
  const int32_t* sel = ids + tg * top_k;
  uint32_t valid = 0;  // bit r: slot r holds a block
  for (int r = 0; r < top_k; ++r)
    if (__ldg(sel + r) >= 0) valid |= 1u << r;
  const int chunks = HG * d / 8;  // 16-byte chunks per slot
  const int64_t slot_elems = (int64_t)HG * d;
  const __half* o_tg = part_o + tg * top_k * slot_elems;
  const float* l_tg = part_lse + tg * top_k * HG;
  // output rows of group g: heads g*HG .. g*HG+HG-1 of query t -> contiguous
  __nv_bfloat16* o_out = out + tg * slot_elems;
  for (int c = lane; c < chunks; c += 32) {
    const int h = (c * 8) / d;
    float m = -INFINITY;
    for (int r = 0; r < top_k; ++r)
      if (valid >> r & 1u) m = fmaxf(m, __ldg(l_tg + r * HG + h));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float wsum = 0.f;
    for (int r = 0; r < top_k; ++r) {
      if (!(valid >> r & 1u)) continue;
      const float w = __expf(__ldg(l_tg + r * HG + h) - m);
      wsum += w;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(o_tg + r * slot_elems) + c);
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float2 f = __half22float2(hv[x]);
        acc[2 * x] = fmaf(w, f.x, acc[2 * x]);
        acc[2 * x + 1] = fmaf(w, f.y, acc[2 * x + 1]);
      }
    }
    const float inv = 1.0f / wsum;
    uint4 ov;
    ov.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    ov.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    ov.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    ov.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    reinterpret_cast<uint4*>(o_out)[c] = ov;
  }
}

}  // namespace

cudaError_t launch_merge(const MergeLaunch& p, cudaStream_t s) {
  const int64_t warps = p.rows * p.G;
  if (warps == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((warps + kWarps - 1) / kWarps);
  merge_kernel<<<grid, kWarps * 32, 0, s>>>(p.part_o, p.part_lse, p.ids, p.rows, p.G, p.H / p.G,
                                            p.d, p.top_k,
                                            static_cast<__nv_bfloat16*>(p.out));
  return cudaGetLastError();
}

}  // namespace msa
