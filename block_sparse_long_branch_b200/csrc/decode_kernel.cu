// decode_kernel.cu -- one decode step: the newest query of each sequence runs
// the same two branches over its cache.  The pages report decode speed-ups
// (zhaixingw "MiniMax M3 深度评测", section "这套注意力到底怎么省的") but describe
// no separate decode algorithm; the plainest reading is used: query position
// L_b - 1, its own key already in the cache.
//
//   1. decode_index_kernel : HBM-bound scan of the index-key cache.  Each warp
//      scores a 128-key block against the sequence's G index queries with
//      mma.sync m16n8k16 (keys as M, groups as N).  The reduction axis is
//      permuted identically for both operands so that every lane reads 16
//      contiguous bytes of a key row straight from global memory.
//      Writes the pooled (max) score of every non-local block.
//   2. decode_topk_kernel  : per (sequence, group), the best k-1 non-local
//      blocks under (score desc, id asc), plus the local block, ascending.
//   3. decode_attn_kernel  : per (sequence, group, slot), softmax of the
//      group's heads over the slot's block (causal on the local block), the
//      partial (o, lse) in the same layout as the prefill partials.
//   4. the prefill merge kernel combines the slots.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kBlock = 128;
constexpr int kIdxWarps = 8;
constexpr int kBlocksPerCta = 16;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int64_t pooled_offset(const int64_t* cu, int b) {
  return cu[b] / kBlock + b;
}

// DI: index dim.  Lane (g = lane/4, t = lane%4) owns physical dims
// [t*DI/4, (t+1)*DI/4) of key rows g and g+8 of each 16-key tile; in k-step kk
// its mma positions (2t,2t+1 | 2t+8,2t+9) hold physical dims t*DI/4 + 4kk +
// (0,1 | 2,3).  q_idx uses the same map, so the dot products are unchanged.
template <int DI>
__global__ void __launch_bounds__(kIdxWarps * 32)
    decode_index_kernel(const __nv_bfloat16* __restrict__ q_idx,
                        const __nv_bfloat16* __restrict__ k_idx, const int64_t* __restrict__ cu,
                        int32_t G, float* __restrict__ pooled, int64_t pooled_cap,
                        uint32_t* err) {
  constexpr int WPR = DI / 8;    // 32-bit words per lane per key row
  constexpr int STEPS = DI / 16;
  const int b = blockIdx.y;
  const int64_t s0 = cu[b];
  const int64_t L = cu[b + 1] - s0;
  const int64_t nb = (L + kBlock - 1) / kBlock;
  const int64_t j_lo = (int64_t)blockIdx.x * kBlocksPerCta;
  const int64_t j_hi = min64(j_lo + kBlocksPerCta, nb - 1);  // non-local blocks only
  if (j_lo >= j_hi) return;
  if (pooled_offset(cu, b) + nb > pooled_cap) {  // workspace sized for fewer cache rows
    if (threadIdx.x == 0) record_error(err, kDevBadIndex);
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int n_tiles = (G + 7) / 8;
  float* pout = pooled + pooled_offset(cu, b) * G;

  for (int nt = 0; nt < n_tiles; ++nt) {
    // B operand: index query of group (nt*8 + gq), this lane's dims
    uint32_t qw[WPR];
    const int grp = nt * 8 + gq;
    if (grp < G) {
      const uint4* src = reinterpret_cast<const uint4*>(q_idx + ((int64_t)b * G + grp) * DI +
                                                        tq * (DI / 4));
#pragma unroll
      for (int i = 0; i < WPR / 4; ++i) {
        const uint4 v = __ldg(src + i);
        qw[4 * i] = v.x, qw[4 * i + 1] = v.y, qw[4 * i + 2] = v.z, qw[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < WPR; ++i) qw[i] = 0;
    }
    for (int64_t j = j_lo + warp; j < j_hi; j += kIdxWarps) {
      const __nv_bfloat16* blk = k_idx + (s0 + j * kBlock) * DI;
      float m0 = -INFINITY, m1 = -INFINITY;  // groups nt*8 + 2tq, +1
#pragma unroll 2
      for (int mt = 0; mt < kBlock / 16; ++mt) {
        uint32_t w0[WPR], w1[WPR];
        const uint4* r0 = reinterpret_cast<const uint4*>(blk + (mt * 16 + gq) * DI + tq * (DI / 4));
        const uint4* r1 = reinterpret_cast<const uint4*>(blk + (mt * 16 + gq + 8) * DI + tq * (DI / 4));
#pragma unroll
        for (int i = 0; i < WPR / 4; ++i) {
          const uint4 a = __ldg(r0 + i), c = __ldg(r1 + i);
          w0[4 * i] = a.x, w0[4 * i + 1] = a.y, w0[4 * i + 2] = a.z, w0[4 * i + 3] = a.w;
          w1[4 * i] = c.x, w1[4 * i + 1] = c.y, w1[4 * i + 2] = c.z, w1[4 * i + 3] = c.w;
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < STEPS; ++kk)
          mma_bf16_16816(acc, w0[2 * kk], w1[2 * kk], w0[2 * kk + 1], w1[2 * kk + 1], qw[2 * kk],
                         qw[2 * kk + 1]);
        m0 = fmaxf(m0, fmaxf(acc[0], acc[2]));
        m1 = fmaxf(m1, fmaxf(acc[1], acc[3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      if (gq == 0) {
        const int g0 = nt * 8 + 2 * tq;
        if (g0 < G) pout[j * G + g0] = m0;
        if (g0 + 1 < G) pout[j * G + g0 + 1] = m1;
      }
    }
  }
}

// Sorted (desc score, asc id) list of the best KSEL candidates seen by a thread.
template <int KSEL>
struct TopList {
  float sc[KSEL];
  int32_t id[KSEL];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < KSEL; ++i) sc[i] = -INFINITY, id[i] = 0x7FFFFFFF;
  }
  // candidates must arrive in increasing id order
  __device__ __forceinline__ void insert(float s, int32_t j) {
    if (!(s > sc[KSEL - 1])) return;
    sc[KSEL - 1] = s;
    id[KSEL - 1] = j;
#pragma unroll
    for (int i = KSEL - 1; i > 0; --i)
      if (sc[i] > sc[i - 1] || (sc[i] == sc[i - 1] && id[i] < id[i - 1])) {
        const float ts = sc[i];
        sc[i] = sc[i - 1];
        sc[i - 1] = ts;
        const int32_t ti = id[i];
        id[i] = id[i - 1];
        id[i - 1] = ti;
      }
  }
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int i = 0; i + 1 < KSEL; ++i) sc[i] = sc[i + 1], id[i] = id[i + 1];
    sc[KSEL - 1] = -INFINITY;
    id[KSEL - 1] = 0x7FFFFFFF;
  }
};

__device__ __forceinline__ bool better(float sa, int32_t ia, float sb, int32_t ib) {
  return sa > sb || (sa == sb && ia < ib);
}

template <int KSEL>
__global__ void __launch_bounds__(256)
    decode_topk_kernel(const float* __restrict__ pooled, const int64_t* __restrict__ cu, int32_t G,
                       int32_t top_k, int64_t pooled_cap, int32_t* __restrict__ ids) {
  const int g = blockIdx.x, b = blockIdx.y;
  const int64_t L = cu[b + 1] - cu[b];
  const int64_t nb = (L + kBlock - 1) / kBlock;
  // no scores were written past the workspace: keep only the local block
  const int64_t n_cand = (pooled_offset(cu, b) + nb > pooled_cap) ? 0 : nb - 1;
  const float* ps = pooled + pooled_offset(cu, b) * G + g;
  TopList<KSEL> list;
  list.init();
  for (int64_t j = threadIdx.x; j < n_cand; j += blockDim.x) list.insert(ps[j * G], (int32_t)j);

  __shared__ float ws_s[8];
  __shared__ int32_t ws_i[8];
  __shared__ int32_t chosen[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int want = (int)min64(top_k - 1, n_cand);
  for (int round = 0; round < want; ++round) {
    float s = list.sc[0];
    int32_t i = list.id[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      const int32_t i2 = __shfl_xor_sync(0xffffffffu, i, o);
      if (better(s2, i2, s, i)) s = s2, i = i2;
    }
    if (lane == 0) ws_s[warp] = s, ws_i[warp] = i;
    __syncthreads();
    float bs = ws_s[0];
    int32_t bi = ws_i[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (better(ws_s[w], ws_i[w], bs, bi)) bs = ws_s[w], bi = ws_i[w];
    if (list.id[0] == bi) list.pop();  // ids are unique: exactly one owner pops
    if (threadIdx.x == 0) chosen[round] = bi;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int32_t o[33];
    int n = 0;
    o[n++] = (int32_t)(nb - 1);
    for (int r = 0; r < want; ++r) o[n++] = chosen[r];
    for (int x = 1; x < n; ++x)  // insertion sort, ascending
      for (int y = x; y > 0 && o[y - 1] > o[y]; --y) {
        const int32_t t = o[y];
        o[y] = o[y - 1];
        o[y - 1] = t;
      }
    int32_t* dst = ids + ((int64_t)b * G + g) * top_k;
    for (int r = 0; r < top_k; ++r) dst[r] = r < n ? o[r] : -1;
  }
}

// One CTA of 128 threads per (slot r, group g, sequence b).
template <int D>
__global__ void __launch_bounds__(128)
    decode_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                       const __nv_bfloat16* __restrict__ vc, const int64_t* __restrict__ cu,
                       const int32_t* __restrict__ ids, int32_t H, int32_t G, int32_t top_k,
                       float scale, __half* __restrict__ part_o, float* __restrict__ part_lse,
                       uint32_t* err) {
  constexpr int MAXHG = 8;
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int HG = H / G;
  const int tid = threadIdx.x;
  const int64_t slot = ((int64_t)b * G + g) * top_k + r;
  const int32_t j = ids[slot];
  const int64_t s0 = cu[b];
  const int64_t L = cu[b + 1] - s0;
  const int64_t nb = (L + kBlock - 1) / kBlock;
  if (j < 0 || j >= nb) {
    if (j >= nb) record_error(err, kDevBadIndex);
    for (int h = tid; h < HG; h += blockDim.x) part_lse[slot * HG + h] = -INFINITY;
    return;
  }
  __shared__ float q_s[MAXHG][D];
  __shared__ float p_s[MAXHG][kBlock];
  __shared__ __align__(16) __nv_bfloat16 v_s[kBlock][D];
  __shared__ float red[MAXHG][4];
  const int nkeys = (int)min64(kBlock, L - (int64_t)j * kBlock);  // keys s <= L-1

  for (int hb = 0; hb < HG; hb += MAXHG) {
    const int hn = min(MAXHG, HG - hb);
    for (int x = tid; x < hn * D; x += blockDim.x) {
      const int h = x / D, c = x % D;
      q_s[h][c] = __bfloat162float(q[((int64_t)b * H + g * HG + hb + h) * D + c]) * scale;
    }
    for (int x = tid; x < kBlock * D / 8; x += blockDim.x) {
      const int s = x / (D / 8), c8 = x % (D / 8);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (s < nkeys)
        val = __ldg(reinterpret_cast<const uint4*>(vc + ((s0 + (int64_t)j * kBlock + s) * G + g) * D) + c8);
      reinterpret_cast<uint4*>(&v_s[s][0])[c8] = val;
    }
    __syncthreads();
    // logits: thread = key
    float kreg[D];
    if (tid < nkeys) {
      const uint4* kr = reinterpret_cast<const uint4*>(kc + ((s0 + (int64_t)j * kBlock + tid) * G + g) * D);
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 val = __ldg(kr + c8);
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&val);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 f = __bfloat1622float2(hv[x]);
          kreg[c8 * 8 + 2 * x] = f.x;
          kreg[c8 * 8 + 2 * x + 1] = f.y;
        }
      }
    }
    const int lane = tid & 31, warp = tid >> 5;
    for (int h = 0; h < hn; ++h) {
      float sv = -INFINITY;
      if (tid < nkeys) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c = 0; c < D; c += 2) {
          a0 = fmaf(q_s[h][c], kreg[c], a0);
          a1 = fmaf(q_s[h][c + 1], kreg[c + 1], a1);
        }
        sv = a0 + a1;
      }
      float m = sv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[h][warp] = m;
      __syncthreads();
      m = fmaxf(fmaxf(red[h][0], red[h][1]), fmaxf(red[h][2], red[h][3]));
      const float p = tid < nkeys ? __expf(sv - m) : 0.f;
      float l = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      __syncthreads();
      if (lane == 0) red[h][warp] = l;
      __syncthreads();
      l = red[h][0] + red[h][1] + red[h][2] + red[h][3];
      p_s[h][tid] = p / l;
      if (tid == 0) part_lse[slot * HG + hb + h] = m + logf(l);
    }
    __syncthreads();
    // o[h][c] = sum_s p[h][s] v[s][c]
    for (int c = tid; c < D; c += blockDim.x) {
      float acc[MAXHG];
#pragma unroll
      for (int h = 0; h < MAXHG; ++h) acc[h] = 0.f;
      for (int s = 0; s < nkeys; ++s) {
        const float vv = __bfloat162float(v_s[s][c]);
#pragma unroll
        for (int h = 0; h < MAXHG; ++h)
          if (h < hn) acc[h] = fmaf(p_s[h][s], vv, acc[h]);
      }
      for (int h = 0; h < hn; ++h) part_o[(slot * HG + hb + h) * D + c] = __float2half_rn(acc[h]);
    }
    __syncthreads();
  }
}

}  // namespace

size_t decode_pooled_rows(int64_t total_len, int32_t B) {
  return (size_t)(total_len / kBlock + B + 1);
}

static void mark_ev(const DecodeLaunch& p, int i, cudaStream_t s) {
  if (p.events && i < p.n_events && p.events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(p.events[i]), s);
}

cudaError_t launch_decode(const DecodeLaunch& p, cudaStream_t s, int* launches) {
  mark_ev(p, 0, s);
  const int64_t max_nb = (p.max_seqlen + kBlock - 1) / kBlock;
  const int64_t chunks = (max_nb + kBlocksPerCta - 1) / kBlocksPerCta;
  dim3 gi((unsigned)(chunks > 0 ? chunks : 1), (unsigned)p.B);
  const auto* qi = static_cast<const __nv_bfloat16*>(p.q_idx);
  const auto* ki = static_cast<const __nv_bfloat16*>(p.k_idx_cache);
  if (p.d_idx == 128)
    decode_index_kernel<128><<<gi, kIdxWarps * 32, 0, s>>>(qi, ki, p.cu_seqlens, p.G, p.pooled,
                                                            p.pooled_cap, p.err);
  else
    decode_index_kernel<64><<<gi, kIdxWarps * 32, 0, s>>>(qi, ki, p.cu_seqlens, p.G, p.pooled,
                                                           p.pooled_cap, p.err);
  ++*launches;
  mark_ev(p, 1, s);
  dim3 gt((unsigned)p.G, (unsigned)p.B);
  if (p.top_k <= 16)
    decode_topk_kernel<15><<<gt, 256, 0, s>>>(p.pooled, p.cu_seqlens, p.G, p.top_k, p.pooled_cap,
                                              p.ids);
  else
    decode_topk_kernel<31><<<gt, 256, 0, s>>>(p.pooled, p.cu_seqlens, p.G, p.top_k, p.pooled_cap,
                                              p.ids);
  ++*launches;
  mark_ev(p, 2, s);
  dim3 ga((unsigned)p.top_k, (unsigned)p.G, (unsigned)p.B);
  const auto* q = static_cast<const __nv_bfloat16*>(p.q);
  const auto* kc = static_cast<const __nv_bfloat16*>(p.k_cache);
  const auto* vc = static_cast<const __nv_bfloat16*>(p.v_cache);
  if (p.d == 128)
    decode_attn_kernel<128><<<ga, 128, 0, s>>>(q, kc, vc, p.cu_seqlens, p.ids, p.H, p.G, p.top_k,
                                               p.scale, p.part_o, p.part_lse, p.err);
  else
    decode_attn_kernel<64><<<ga, 128, 0, s>>>(q, kc, vc, p.cu_seqlens, p.ids, p.H, p.G, p.top_k,
                                              p.scale, p.part_o, p.part_lse, p.err);
  ++*launches;
  mark_ev(p, 3, s);
  MergeLaunch m{};
  m.part_o = p.part_o;
  m.part_lse = p.part_lse;
  m.ids = p.ids;
  m.rows = p.B;
  m.H = p.H;
  m.G = p.G;
  m.d = p.d;
  m.top_k = p.top_k;
  m.out = p.out;
  cudaError_t e = launch_merge(m, s);
  ++*launches;
  mark_ev(p, 4, s);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace msa
