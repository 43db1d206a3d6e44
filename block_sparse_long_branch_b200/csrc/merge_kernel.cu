// merge_kernel.cu -- combines the per-block partial softmaxes of each query.
//
// The Main Branch is one exact softmax over all selected keys (ai-tool-zukan
// "MiniMax MSA guide", section "Index BranchとMain Branchの役割分担").  The
// key-block-outer kernel produces it in pieces, one per selected block r: the
// unnormalised o'_r = sum_{s in r} exp(logit_s - m_r) v'_s, where v' is the
// value row scaled by 2^-e_r, with m~_r = m_r + e_r ln2 and l~_r = 2^-e_r
// sum_{s in r} exp(logit_s - m_r).  With M = max_r m~_r and w_r = exp(m~_r - M)
// the exact result is  out = sum_r w_r o'_r / sum_r w_r l~_r,  the standard
// max-shifted split of a softmax (the 2^e_r factors cancel).
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

// ALIGN: also the block-alignment outputs (see MergeLaunch): the attention
// mass of every slot, averaged over the group's heads, and the KL divergence
// of that mass from the softmax of the slots' pooled index scores.
template <int CPL, int KMAX, bool ALIGN>
__global__ void __launch_bounds__(kWarps * 32)
    merge_kernel(const __half* __restrict__ part_o, const float2* __restrict__ part_ml,
                 const int32_t* __restrict__ ids, int64_t rows, int32_t G, int32_t HG, int32_t d,
                 int32_t top_k, __nv_bfloat16* __restrict__ out, float* __restrict__ block_score,
                 float* __restrict__ block_mass, float* __restrict__ kl) {
  const int64_t tg = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tg >= rows * G) return;
  const int lane = threadIdx.x & 31;
  const int32_t idv = lane < top_k ? __ldg(ids + tg * top_k + lane) : -1;
  const uint32_t valid = __ballot_sync(0xffffffffu, idv >= 0);  // bit r: slot r holds a block
  const int chunks = HG * d / 8;
  const int c0 = lane * CPL;
  if (!ALIGN && c0 >= chunks) return;
  const bool active = c0 < chunks;
  const int h = active ? (c0 * 8) / d : 0;
  const int64_t slot_elems = (int64_t)HG * d;
  const __half* o_tg = part_o + tg * top_k * slot_elems + (int64_t)c0 * 8;
  const float2* l_tg = part_ml + tg * top_k * HG + h;

  // slot r's weight w_r = exp(m~_r - M) (in wt[r], 0 for empty slots) and the
  // normaliser sum_r w_r l~_r; l~ is not kept past this point
  float wt[KMAX], lt[KMAX];
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < KMAX; ++r) {
    const bool use = active && r < top_k && (valid >> r & 1u);
    const float2 ml = use ? __ldg(l_tg + r * HG) : make_float2(-INFINITY, 0.f);
    wt[r] = ml.x;
    lt[r] = ml.y;
    m = fmaxf(m, wt[r]);
  }
  float wsum = 0.f;
#pragma unroll
  for (int r = 0; r < KMAX; ++r) {
    wt[r] = (r < top_k && (valid >> r & 1u)) ? __expf(wt[r] - m) : 0.f;
    // explicit roundings: the same sum whether or not the products are kept
    // for the alignment outputs (no fused multiply-add in one variant only)
    lt[r] = __fmul_rn(lt[r], wt[r]);
    wsum = __fadd_rn(wsum, lt[r]);
  }
  if (ALIGN) {
    // per slot: this head's softmax weight; summed over the head leaders
    // (the first lane of each head) and divided by H/G
    const bool leader = active && (c0 * 8) % d == 0;
    float mass[KMAX];
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      float w = (leader && r < top_k && (valid >> r & 1u)) ? lt[r] / wsum : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
      mass[r] = w / (float)HG;
    }
    // KL(mass || softmax over the filled slots of their pooled index scores)
    float smax = -INFINITY;
    float sc[KMAX];
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      sc[r] = (r < top_k && (valid >> r & 1u)) ? block_score[tg * top_k + r] : -INFINITY;
      smax = fmaxf(smax, sc[r]);
    }
    float z = 0.f;
#pragma unroll
    for (int r = 0; r < KMAX; ++r)
      if (r < top_k && (valid >> r & 1u)) z += __expf(sc[r] - smax);
    const float logz = __logf(z) + smax;
    float div = 0.f;
#pragma unroll
    for (int r = 0; r < KMAX; ++r)
      if (r < top_k && (valid >> r & 1u) && mass[r] > 0.f)
        div += mass[r] * (__logf(mass[r]) - (sc[r] - logz));
    if (lane < top_k) {
      block_mass[tg * top_k + lane] = (valid >> lane & 1u) ? mass[lane] : 0.f;
      if (!(valid >> lane & 1u)) block_score[tg * top_k + lane] = -INFINITY;
    }
    if (lane == 0) kl[tg] = div;
    if (!active) return;
  }
  float acc[CPL * 8];
#pragma unroll
  for (int x = 0; x < CPL * 8; ++x) acc[x] = 0.f;
#pragma unroll
  for (int r = 0; r < KMAX; ++r) {
    if (r >= top_k || !(valid >> r & 1u)) continue;
    const float w = wt[r];
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

template <int KMAX, bool ALIGN>
cudaError_t launch_k(const MergeLaunch& p, cudaStream_t s, unsigned grid) {
  const int chunks = (p.H / p.G) * p.d / 8;  // 16-byte chunks per slot, a power of two >= 8
  auto* o = static_cast<__nv_bfloat16*>(p.out);
  const int HG = p.H / p.G;
#define MSA_MERGE(CPL)                                                                       \
  merge_kernel<CPL, KMAX, ALIGN><<<grid, kWarps * 32, 0, s>>>(                               \
      p.part_o, p.part_ml, p.ids, p.rows, p.G, HG, p.d, p.top_k, o, p.block_score,          \
      p.block_mass, p.kl)
  if (chunks >= 256)
    MSA_MERGE(8);
  else if (chunks >= 128)
    MSA_MERGE(4);
  else if (chunks >= 64)
    MSA_MERGE(2);
  else
    MSA_MERGE(1);
#undef MSA_MERGE
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeLaunch& p, cudaStream_t s) {
  const int64_t warps = p.rows * p.G;
  if (warps == 0) return cudaSuccess;
  const int chunks = (p.H / p.G) * p.d / 8;
  if (chunks > 32 * 8) return cudaErrorInvalidValue;  // H/G * d > 2048: not instantiated
  const unsigned grid = (unsigned)((warps + kWarps - 1) / kWarps);
  const bool align = p.block_mass != nullptr;
  if (align && (!p.block_score || !p.kl)) return cudaErrorInvalidValue;
  if (p.top_k <= 16) return align ? launch_k<16, true>(p, s, grid) : launch_k<16, false>(p, s, grid);
  return align ? launch_k<32, true>(p, s, grid) : launch_k<32, false>(p, s, grid);
}

}  // namespace msa
