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
//      contiguous bytes of a key row straight from global memory.  With an
//      e4m3 cache (one fp32 scale per key row), decode_index_fp8_kernel does
//      the same on mma.sync m16n8k32 e4m3 over half the bytes.
//      Writes the pooled (max) score of every non-local block, [G][nb] per
//      sequence so that each group's scores are contiguous.
//   2. decode_attend_kernel : n_split CTAs per (sequence, group).  Each one
//      selects, exactly and identically to its siblings, the best k-1
//      non-local blocks under (score desc, id asc) plus the local block (a
//      threshold from per-warp bests, then an exact ranking of the candidates
//      by counting; sorted per-thread lists and warp tournaments when the
//      scores cluster), then attends over its share of them (selected blocks
//      z, z + n_split, ...) with an online softmax: S^T = K Q^T on mma.sync
//      with K rows loaded one block ahead, P carried as two bf16 parts (hi and
//      lo) into O^T += V^T P^T with V double-buffered by cp.async.  Split CTAs
//      leave (o, m, l) partials; the last to finish (a ticket per (sequence,
//      group)) merges them and writes the output.
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
        if (g0 < G) pout[(int64_t)g0 * nb + j] = m0;
        if (g0 + 1 < G) pout[(int64_t)(g0 + 1) * nb + j] = m1;
      }
    }
  }
}

__device__ __forceinline__ void mma_e4m3_16832(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same scan over an e4m3 index-key cache with one fp32 scale per cached
// key row (index dim 128): the score of key s is kscale[s] * <q8, k8[s]> (the
// query's own scale, a positive constant of the (sequence, group), is left
// out: it cannot change the ranking).  Lane (g = lane/4, t = lane%4) owns bytes
// [32t, 32t+32) of key rows g and g+8 of each 16-key tile; in k-step kk its mma
// positions (4t..4t+3 | 16+4t..16+4t+3) hold physical bytes 32t + 8kk + (0..3 |
// 4..7), and q8 uses the same map, so the dot products are unchanged.
__global__ void __launch_bounds__(kIdxWarps * 32)
    decode_index_fp8_kernel(const uint8_t* __restrict__ q_idx8, const uint8_t* __restrict__ k_idx8,
                            const float* __restrict__ kscale, const int64_t* __restrict__ cu,
                            int32_t G, float* __restrict__ pooled, int64_t pooled_cap,
                            uint32_t* err) {
  constexpr int DI = 128;
  constexpr int WPR = DI / 16;  // 32-bit words per lane per key row (32 bytes)
  constexpr int STEPS = DI / 32;
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
    uint32_t qw[WPR];
    const int grp = nt * 8 + gq;
    if (grp < G) {
      const uint4* src =
          reinterpret_cast<const uint4*>(q_idx8 + ((int64_t)b * G + grp) * DI + tq * (DI / 4));
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
      const int64_t row0 = s0 + j * kBlock;
      const uint8_t* blk = k_idx8 + row0 * DI;
      float m0 = -INFINITY, m1 = -INFINITY;  // groups nt*8 + 2tq, +1
#pragma unroll 2
      for (int mt = 0; mt < kBlock / 16; ++mt) {
        uint32_t w0[WPR], w1[WPR];
        const uint4* r0 = reinterpret_cast<const uint4*>(blk + (mt * 16 + gq) * DI + tq * (DI / 4));
        const uint4* r1 =
            reinterpret_cast<const uint4*>(blk + (mt * 16 + gq + 8) * DI + tq * (DI / 4));
#pragma unroll
        for (int i = 0; i < WPR / 4; ++i) {
          const uint4 a = __ldg(r0 + i), c = __ldg(r1 + i);
          w0[4 * i] = a.x, w0[4 * i + 1] = a.y, w0[4 * i + 2] = a.z, w0[4 * i + 3] = a.w;
          w1[4 * i] = c.x, w1[4 * i + 1] = c.y, w1[4 * i + 2] = c.z, w1[4 * i + 3] = c.w;
        }
        const float sc0 = __ldg(kscale + row0 + mt * 16 + gq);
        const float sc1 = __ldg(kscale + row0 + mt * 16 + gq + 8);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < STEPS; ++kk)
          mma_e4m3_16832(acc, w0[2 * kk], w1[2 * kk], w0[2 * kk + 1], w1[2 * kk + 1], qw[2 * kk],
                         qw[2 * kk + 1]);
        m0 = fmaxf(m0, fmaxf(acc[0] * sc0, acc[2] * sc1));
        m1 = fmaxf(m1, fmaxf(acc[1] * sc0, acc[3] * sc1));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      if (gq == 0) {
        const int g0 = nt * 8 + 2 * tq;
        if (g0 < G) pout[(int64_t)g0 * nb + j] = m0;
        if (g0 + 1 < G) pout[(int64_t)(g0 + 1) * nb + j] = m1;
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
  // candidates must arrive in increasing id order: a later equal score loses
  __device__ __forceinline__ void insert(float s, int32_t j) {
    if (!(s > sc[KSEL - 1])) return;
    sc[KSEL - 1] = s;
    id[KSEL - 1] = j;
#pragma unroll
    for (int i = KSEL - 1; i > 0; --i)
      if (sc[i] > sc[i - 1]) {
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

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kCandCap = 256;  // candidates kept for the exact ranking step

template <int KSEL>
struct SelScratch {
  float wl_s[kAttnWarps][KSEL];  // each warp's best candidates, best first
  int32_t wl_i[kAttnWarps][KSEL];
  float tm_s[kAttnThreads];      // each warp's best thread bests
  int32_t tm_i[kAttnThreads];
  float cand_s[kCandCap];        // candidates not worse than the threshold
  int32_t cand_i[kCandCap];
};

template <int D, int NT, int KSEL>
struct AttnSmem {
  // the sequence's pooled scores staged for the selection, in what is left
  // of the V tiles' space next to the selection scratch
  static constexpr int kStageCap =
      (int)((sizeof(__nv_bfloat16) * 2 * kBlock * D - sizeof(SelScratch<KSEL>)) / sizeof(float));
  union {
    __nv_bfloat16 v[2][kBlock * D];  // attention: V tiles, 16-byte chunks swizzled by key
    struct {                         // selection (done before the first V copy)
      SelScratch<KSEL> sel_scr;
      float stage[kStageCap];
    };
  };
  __nv_bfloat16 p[NT * 8][kBlock + 8];     // P (heads x keys), padded rows: bf16(p)
  __nv_bfloat16 p_lo[NT * 8][kBlock + 8];  // and the rest, bf16(p - bf16(p))
  float red_m[kAttnWarps][NT * 8];
  float red_l[kAttnWarps][NT * 8];
  float m_run[NT * 8], l_run[NT * 8], alpha[NT * 8];
  float o_t[NT * 8][D + 4];             // final O (heads x d) for coalesced stores
  int32_t pick[32];  // the best non-local blocks, best first
  int32_t sel[32];   // all selected blocks, ascending
  int32_t mine[32];  // the selected blocks this CTA attends to
  float thr_s;
  int32_t thr_i, ncand;
  int32_t nsel, nmine, last;
};

// smem offset (elements) of 16-byte chunk c of key row s in a swizzled V tile
template <int D>
__device__ __forceinline__ int v_off(int s, int c) {
  return s * D + ((c ^ (s & 7)) << 3);
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// n_split CTAs per (group g, sequence b), split z taking the selected blocks
// z, z + n_split, ...:
//   1. top-k over the pooled scores of the sequence's non-local blocks
//      (register lists per thread, then k-1 rounds of a block arg-max); every
//      split computes the same selection;
//   2. attention of the group's H/G heads over this split's blocks with an
//      online softmax across blocks;
//   3. with several splits, each writes its unnormalised O and (max, sum) to
//      the workspace and the last split to finish (a ticket per (b, g)) merges
//      them with log-sum-exp weights.  S^T = K Q^T on mma.sync (K rows read
//      straight from global memory with the permuted reduction axis, Q in
//      registers), P to shared memory, O^T += V^T P^T on mma.sync with V in a
//      swizzled shared tile (ldmatrix.trans).  The next block's V is copied in
//      (cp.async) while the current one is used.
template <int D, int NT, int KSEL>
__global__ void __launch_bounds__(kAttnThreads)
    decode_attend_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                         const __nv_bfloat16* __restrict__ vc, const int64_t* __restrict__ cu,
                         const float* __restrict__ pooled, int64_t pooled_cap, int32_t G,
                         int32_t HG, int32_t top_k, float scale_log2,
                         int32_t* __restrict__ ids_out, __nv_bfloat16* __restrict__ out,
                         int32_t n_split, float* __restrict__ part, int32_t* __restrict__ tickets) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  AttnSmem<D, NT, KSEL>& sm = *reinterpret_cast<AttnSmem<D, NT, KSEL>*>(smem_raw);
  const int g = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t s0 = cu[b];
  const int64_t L = cu[b + 1] - s0;
  const int64_t nb = (L + kBlock - 1) / kBlock;

  // ---------------- 1. selection ----------------
  // The best `want` non-local blocks under (score desc, id asc), a strict
  // total order:
  //  (a) each thread finds its best candidate (j = tid + 256 i);
  //  (b) each warp takes the best R = ceil(want/8) of its threads' bests
  //      (R rounds of a warp arg-max), and thr = the want-th best of those
  //      8R distinct candidates.  Every one of the best `want` is then not
  //      worse than thr;
  //  (c) every candidate not worse than thr is collected (usually a few more
  //      than `want`) and ranked exactly by counting.
  // If more than kCandCap candidates pass (heavy ties), per-thread lists and
  // warp tournaments are used instead.  Finally the picks and the local block
  // are put in ascending id order, again by counting.
  {
    const int64_t n_cand = (pooled_offset(cu, b) + nb > pooled_cap) ? 0 : nb - 1;
    const float* ps = pooled + pooled_offset(cu, b) * G + (int64_t)g * nb;  // [G][nb] per sequence
    const int want = (int)min64(top_k - 1, n_cand);
    // the scores are staged in shared memory when they fit (8,191 candidates of
    // a 1M-token sequence do at d = 128): their loads then go out 16 a thread at
    // a time, once, instead of once per pass below
    const bool staged = n_cand <= AttnSmem<D, NT, KSEL>::kStageCap;
    if (staged) {
      constexpr int kSB = 16;
      for (int64_t j0 = tid; j0 < n_cand; j0 += kSB * kAttnThreads) {
        float v[kSB];
#pragma unroll
        for (int c = 0; c < kSB; ++c) {
          const int64_t j = j0 + (int64_t)c * kAttnThreads;
          v[c] = j < n_cand ? __ldg(ps + j) : 0.f;
        }
#pragma unroll
        for (int c = 0; c < kSB; ++c) {
          const int64_t j = j0 + (int64_t)c * kAttnThreads;
          if (j < n_cand) sm.stage[j] = v[c];
        }
      }
      __syncthreads();
    }
    auto cand = [&](int64_t j) { return staged ? sm.stage[j] : __ldg(ps + j); };
    constexpr int kBatch = 8;
    float best_s = -INFINITY;
    int32_t best_i = 0x7FFFFFFF;
    for (int64_t j0 = tid; j0 < n_cand; j0 += kBatch * kAttnThreads) {
      float v[kBatch];
#pragma unroll
      for (int c = 0; c < kBatch; ++c) {
        const int64_t j = j0 + (int64_t)c * kAttnThreads;
        v[c] = j < n_cand ? cand(j) : -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < kBatch; ++c) {
        const int64_t j = j0 + (int64_t)c * kAttnThreads;
        if (j < n_cand && better(v[c], (int32_t)j, best_s, best_i)) best_s = v[c], best_i = (int32_t)j;
      }
    }
    // (b) per warp: its best R thread bests into tm[warp * R + round]
    const int R = (want + kAttnWarps - 1) / kAttnWarps;
    {
      float ms = best_s;
      int32_t mi = best_i;
      for (int round = 0; round < R; ++round) {
        float sc = ms;
        int32_t id = mi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float s2 = __shfl_xor_sync(0xffffffffu, sc, o);
          const int32_t i2 = __shfl_xor_sync(0xffffffffu, id, o);
          if (better(s2, i2, sc, id)) sc = s2, id = i2;
        }
        if (mi == id) ms = -INFINITY, mi = 0x7FFFFFFF;  // the owner drops it
        if (lane == 0) sm.sel_scr.tm_s[warp * R + round] = sc, sm.sel_scr.tm_i[warp * R + round] = id;
      }
    }
    if (tid == 0) {
      sm.ncand = 0;
      // the worst possible key: kept if fewer than `want` of the 8R are real
      // candidates, and then every candidate is collected
      sm.thr_s = -INFINITY;
      sm.thr_i = 0x7FFFFFFF;
    }
    __syncthreads();
    if (warp == 0 && want > 0) {
      // thr = the want-th best of the 8R collected (lane x ranks entry x)
      for (int x = lane; x < kAttnWarps * R; x += 32) {
        const float sx = sm.sel_scr.tm_s[x];
        const int32_t ix = sm.sel_scr.tm_i[x];
        int rank = 0;
        for (int y = 0; y < kAttnWarps * R; ++y) rank += better(sm.sel_scr.tm_s[y], sm.sel_scr.tm_i[y], sx, ix);
        if (rank == want - 1) sm.thr_s = sx, sm.thr_i = ix;
      }
    }
    __syncthreads();
    // (c) collect the candidates not worse than thr
    if (want > 0) {
      const float ts = sm.thr_s;
      const int32_t ti = sm.thr_i;
      for (int64_t j0 = tid; j0 < n_cand; j0 += kBatch * kAttnThreads) {
        float v[kBatch];
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
          const int64_t j = j0 + (int64_t)c * kAttnThreads;
          v[c] = j < n_cand ? cand(j) : -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < kBatch; ++c) {
          const int64_t j = j0 + (int64_t)c * kAttnThreads;
          if (j < n_cand && !better(ts, ti, v[c], (int32_t)j)) {
            const int x = atomicAdd(&sm.ncand, 1);
            if (x < kCandCap) sm.sel_scr.cand_s[x] = v[c], sm.sel_scr.cand_i[x] = (int32_t)j;
          }
        }
      }
    }
    __syncthreads();
    const int nc = sm.ncand;
    if (nc <= kCandCap) {
      // exact ranks among the collected: the best `want` go to pick[0..want)
      for (int x = tid; x < nc; x += kAttnThreads) {
        const float s_x = sm.sel_scr.cand_s[x];
        const int32_t i_x = sm.sel_scr.cand_i[x];
        int rank = 0;
        for (int y = 0; y < nc; ++y) rank += better(sm.sel_scr.cand_s[y], sm.sel_scr.cand_i[y], s_x, i_x);
        if (rank < want) sm.pick[rank] = i_x;
      }
    } else {
      // fallback: per-thread lists, then warp tournaments
      TopList<KSEL> list;
      list.init();
      for (int64_t j = tid; j < n_cand; j += kAttnThreads) list.insert(cand(j), (int32_t)j);
      for (int round = 0; round < want; ++round) {
        float sc = list.sc[0];
        int32_t id = list.id[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float s2 = __shfl_xor_sync(0xffffffffu, sc, o);
          const int32_t i2 = __shfl_xor_sync(0xffffffffu, id, o);
          if (better(s2, i2, sc, id)) sc = s2, id = i2;
        }
        if (list.id[0] == id) list.pop();  // real ids are unique; empty heads pop harmlessly
        if (lane == 0) sm.sel_scr.wl_s[warp][round] = sc, sm.sel_scr.wl_i[warp][round] = id;
      }
      __syncthreads();
      if (warp == 0) {
        TopList<KSEL> wl;
        wl.init();
#pragma unroll
        for (int i = 0; i < KSEL; ++i)
          if (lane < kAttnWarps && i < want) wl.sc[i] = sm.sel_scr.wl_s[lane][i], wl.id[i] = sm.sel_scr.wl_i[lane][i];
        for (int round = 0; round < want; ++round) {
          float sc = wl.sc[0];
          int32_t id = wl.id[0];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float s2 = __shfl_xor_sync(0xffffffffu, sc, o);
            const int32_t i2 = __shfl_xor_sync(0xffffffffu, id, o);
            if (better(s2, i2, sc, id)) sc = s2, id = i2;
          }
          if (wl.id[0] == id) wl.pop();
          if (lane == 0) sm.pick[round] = id;
        }
      }
    }
    __syncthreads();
    // ascending ids: the picks by counting, then the local block (the largest)
    const int n = want + 1;
    if (tid < want) {
      const int32_t my = sm.pick[tid];
      int pos = 0;
      for (int y = 0; y < want; ++y) pos += sm.pick[y] < my;
      sm.sel[pos] = my;
    } else if (tid == want) {
      sm.sel[want] = (int32_t)(nb - 1);
    }
    if (tid < NT * 8) sm.m_run[tid] = -INFINITY, sm.l_run[tid] = 0.f;
    __syncthreads();
    if (tid < n && tid % n_split == split) sm.mine[tid / n_split] = sm.sel[tid];
    if (split == 0 && tid < top_k)
      ids_out[((int64_t)b * G + g) * top_k + tid] = tid < n ? sm.sel[tid] : -1;
    if (tid == 0) {
      sm.nsel = n;
      sm.nmine = n > split ? (n - split - 1) / n_split + 1 : 0;
    }
    __syncthreads();
  }

  // ---------------- 2. attention ----------------
  constexpr int WPR = D / 8;  // 32-bit words per lane per row (permuted reduction axis)
  const int gq = lane >> 2, tq = lane & 3;
  const int nsel = sm.nmine;
  const __nv_bfloat16* kbase = kc + (s0 * G + g) * (int64_t)D;
  const __nv_bfloat16* vbase = vc + (s0 * G + g) * (int64_t)D;
  const int64_t row_pitch = (int64_t)G * D;

  // Q^T fragments: head nt*8+gq of this group, this lane's dims
  uint32_t qw[NT][WPR];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = nt * 8 + gq;
    if (h < HG) {
      const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)b * G * HG + g * HG + h) * D +
                                                        tq * (D / 4));
#pragma unroll
      for (int i = 0; i < WPR / 4; ++i) {
        const uint4 v = __ldg(src + i);
        qw[nt][4 * i] = v.x, qw[nt][4 * i + 1] = v.y, qw[nt][4 * i + 2] = v.z,
        qw[nt][4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < WPR; ++i) qw[nt][i] = 0;
    }
  }

  auto load_v = [&](int bi, int buf) {
    const int64_t j = sm.mine[bi];
    const int nk = (int)min64(kBlock, L - j * kBlock);
    for (int x = tid; x < kBlock * (D / 8); x += kAttnThreads) {
      const int s = x / (D / 8), c = x % (D / 8);
      const __nv_bfloat16* src = vbase + (j * kBlock + (s < nk ? s : 0)) * row_pitch + c * 8;
      cp_async_16_zfill(&sm.v[buf][v_off<D>(s, c)], src, s < nk);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float oacc[NT][4];  // O^T fragment: d rows 16*warp + gq (+8), heads nt*8 + 2tq (+1)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;

  // this warp's 16 key rows of a block, lanes reading 16 contiguous bytes each
  uint32_t w0[WPR], w1[WPR];
  auto load_k = [&](int bi) {
    const int64_t jj = sm.mine[bi];
    const int nkk = (int)min64(kBlock, L - jj * kBlock);
    const int r0i = warp * 16 + gq, r1i = r0i + 8;
    const uint4* r0 = reinterpret_cast<const uint4*>(
        kbase + (jj * kBlock + (r0i < nkk ? r0i : 0)) * row_pitch + tq * (D / 4));
    const uint4* r1 = reinterpret_cast<const uint4*>(
        kbase + (jj * kBlock + (r1i < nkk ? r1i : 0)) * row_pitch + tq * (D / 4));
#pragma unroll
    for (int i = 0; i < WPR / 4; ++i) {
      const uint4 a4 = __ldg(r0 + i), c4 = __ldg(r1 + i);
      w0[4 * i] = a4.x, w0[4 * i + 1] = a4.y, w0[4 * i + 2] = a4.z, w0[4 * i + 3] = a4.w;
      w1[4 * i] = c4.x, w1[4 * i + 1] = c4.y, w1[4 * i + 2] = c4.z, w1[4 * i + 3] = c4.w;
    }
  };

  if (nsel > 0) {
    load_v(0, 0);
    load_k(0);
  }
  for (int bi = 0; bi < nsel; ++bi) {
    const int buf = bi & 1;
    const int64_t j = sm.mine[bi];
    const int nk = (int)min64(kBlock, L - j * kBlock);
    if (bi + 1 < nsel) load_v(bi + 1, buf ^ 1);

    // ---- S^T (keys x heads) for this warp's 16 keys (K rows loaded one block ahead) ----
    const int k0 = warp * 16 + gq, k1 = k0 + 8;
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_bf16_16816(sacc[nt], w0[2 * kk], w1[2 * kk], w0[2 * kk + 1], w1[2 * kk + 1],
                       qw[nt][2 * kk], qw[nt][2 * kk + 1]);
      // log2-domain logits; keys past the end of the sequence are masked
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = (e < 2) ? k0 : k1;
        sacc[nt][e] = key < nk ? sacc[nt][e] * scale_log2 : -INFINITY;
      }
      // per-warp max of heads 2tq, 2tq+1 over its 16 keys
      float m0 = fmaxf(sacc[nt][0], sacc[nt][2]), m1 = fmaxf(sacc[nt][1], sacc[nt][3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      if (gq == 0) sm.red_m[warp][nt * 8 + 2 * tq] = m0, sm.red_m[warp][nt * 8 + 2 * tq + 1] = m1;
    }
    if (bi + 1 < nsel) load_k(bi + 1);  // in flight during the softmax and PV of this block
    __syncthreads();
    if (tid < NT * 8) {
      float bm = sm.red_m[0][tid];
#pragma unroll
      for (int w = 1; w < kAttnWarps; ++w) bm = fmaxf(bm, sm.red_m[w][tid]);
      const float mo = sm.m_run[tid];
      const float mn = fmaxf(mo, bm);
      sm.alpha[tid] = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
      sm.m_run[tid] = mn;
    }
    __syncthreads();
    // ---- P = exp2(S - m) (heads x keys) as two bf16 parts, hi = bf16(p) and
    // lo = bf16(p - hi), so that the PV product sees p to about 16 significant
    // bits (bf16 alone, 8 bits, is too coarse for a softmax over a handful of
    // keys); row sums of the unrounded values ----
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * tq, h1 = h0 + 1;
      const float mh0 = sm.m_run[h0], mh1 = sm.m_run[h1];
      const float e00 = fast_exp2(sacc[nt][0] - mh0), e01 = fast_exp2(sacc[nt][1] - mh1);
      const float e10 = fast_exp2(sacc[nt][2] - mh0), e11 = fast_exp2(sacc[nt][3] - mh1);
      const __nv_bfloat16 p00 = __float2bfloat16_rn(e00), p01 = __float2bfloat16_rn(e01);
      const __nv_bfloat16 p10 = __float2bfloat16_rn(e10), p11 = __float2bfloat16_rn(e11);
      sm.p[h0][k0] = p00;
      sm.p[h1][k0] = p01;
      sm.p[h0][k1] = p10;
      sm.p[h1][k1] = p11;
      sm.p_lo[h0][k0] = __float2bfloat16_rn(e00 - __bfloat162float(p00));
      sm.p_lo[h1][k0] = __float2bfloat16_rn(e01 - __bfloat162float(p01));
      sm.p_lo[h0][k1] = __float2bfloat16_rn(e10 - __bfloat162float(p10));
      sm.p_lo[h1][k1] = __float2bfloat16_rn(e11 - __bfloat162float(p11));
      float l0 = e00 + e10;
      float l1 = e01 + e11;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      if (gq == 0) sm.red_l[warp][h0] = l0, sm.red_l[warp][h1] = l1;
    }
    // this block's V tile has landed (the next one may still be in flight)
    if (bi + 1 < nsel)
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (tid < NT * 8) {
      float ls = 0.f;
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) ls += sm.red_l[w][tid];
      sm.l_run[tid] = sm.alpha[tid] * sm.l_run[tid] + ls;
    }
    // ---- O^T (d x heads) = alpha * O^T + V^T P^T : warp w owns d rows 16w..16w+15 ----
    if (warp < D / 16) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float a0 = sm.alpha[nt * 8 + 2 * tq], a1 = sm.alpha[nt * 8 + 2 * tq + 1];
        oacc[nt][0] *= a0;
        oacc[nt][1] *= a1;
        oacc[nt][2] *= a0;
        oacc[nt][3] *= a1;
      }
      const int dchunk = warp * 2 + ((lane >> 3) & 1);  // 16-byte chunk of d
#pragma unroll
      for (int kk = 0; kk < kBlock / 16; ++kk) {
        const int key = kk * 16 + (lane & 7) + ((lane >> 4) << 3);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(a0, a1, a2, a3, &sm.v[buf][v_off<D>(key, dchunk)]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const __nv_bfloat16* prow = &sm.p[nt * 8 + gq][kk * 16 + 2 * tq];
          const __nv_bfloat16* lrow = &sm.p_lo[nt * 8 + gq][kk * 16 + 2 * tq];
          mma_bf16_16816(oacc[nt], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(prow),
                         *reinterpret_cast<const uint32_t*>(prow + 8));
          mma_bf16_16816(oacc[nt], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(lrow),
                         *reinterpret_cast<const uint32_t*>(lrow + 8));
        }
      }
    }
    __syncthreads();  // p, red_*, alpha and this V buffer are reused next block
  }

  // ---------------- output ----------------
  if (warp < D / 16) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * tq;
      const int d0 = warp * 16 + gq;
      sm.o_t[h0][d0] = oacc[nt][0];
      sm.o_t[h0 + 1][d0] = oacc[nt][1];
      sm.o_t[h0][d0 + 8] = oacc[nt][2];
      sm.o_t[h0 + 1][d0 + 8] = oacc[nt][3];
    }
  }
  __syncthreads();
  __nv_bfloat16* orow = out + ((int64_t)b * G * HG + g * HG) * D;
  if (n_split == 1) {
    // O / l -> bf16 [heads][d]
    for (int x = tid; x < HG * (D / 8); x += kAttnThreads) {
      const int h = x / (D / 8), c = x % (D / 8);
      const float inv = sm.l_run[h] > 0.f ? 1.0f / sm.l_run[h] : 0.f;
      uint4 w;
      w.x = pack_bf16x2(sm.o_t[h][c * 8 + 0] * inv, sm.o_t[h][c * 8 + 1] * inv);
      w.y = pack_bf16x2(sm.o_t[h][c * 8 + 2] * inv, sm.o_t[h][c * 8 + 3] * inv);
      w.z = pack_bf16x2(sm.o_t[h][c * 8 + 4] * inv, sm.o_t[h][c * 8 + 5] * inv);
      w.w = pack_bf16x2(sm.o_t[h][c * 8 + 6] * inv, sm.o_t[h][c * 8 + 7] * inv);
      reinterpret_cast<uint4*>(orow + (int64_t)h * D)[c] = w;
    }
    return;
  }
  // this split's partial: O [NT*8][D] (unnormalised), then max and sum (log2 domain)
  constexpr int kPart = NT * 8 * (D + 2);
  const int64_t pg = (int64_t)b * G + g;
  float* mypart = part + (pg * n_split + split) * kPart;
  for (int x = tid; x < NT * 8 * (D / 4); x += kAttnThreads) {
    const int h = x / (D / 4), c = x % (D / 4);
    reinterpret_cast<float4*>(mypart + h * D)[c] =
        make_float4(sm.o_t[h][4 * c], sm.o_t[h][4 * c + 1], sm.o_t[h][4 * c + 2],
                    sm.o_t[h][4 * c + 3]);
  }
  if (tid < NT * 8) {
    mypart[NT * 8 * D + tid] = sm.m_run[tid];
    mypart[NT * 8 * D + NT * 8 + tid] = sm.l_run[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = atomicAdd(tickets + pg, 1) == n_split - 1;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  // last split: out = sum_z 2^(m_z - M) O_z / sum_z 2^(m_z - M) l_z
  const float* gpart = part + pg * n_split * kPart;
  for (int x = tid; x < HG * (D / 8); x += kAttnThreads) {
    const int h = x / (D / 8), c = x % (D / 8);
    float M = -INFINITY;
    for (int z = 0; z < n_split; ++z) M = fmaxf(M, __ldcg(gpart + z * kPart + NT * 8 * D + h));
    float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int z = 0; z < n_split; ++z) {
      const float* pz = gpart + z * kPart;
      const float mz = __ldcg(pz + NT * 8 * D + h);
      const float wz = mz == -INFINITY ? 0.f : fast_exp2(mz - M);
      L += wz * __ldcg(pz + NT * 8 * D + NT * 8 + h);
      const float4 a = __ldcg(reinterpret_cast<const float4*>(pz + h * D + c * 8));
      const float4 e = __ldcg(reinterpret_cast<const float4*>(pz + h * D + c * 8 + 4));
      acc[0] += wz * a.x, acc[1] += wz * a.y, acc[2] += wz * a.z, acc[3] += wz * a.w;
      acc[4] += wz * e.x, acc[5] += wz * e.y, acc[6] += wz * e.z, acc[7] += wz * e.w;
    }
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    uint4 w;
    w.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    w.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    w.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    w.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    reinterpret_cast<uint4*>(orow + (int64_t)h * D)[c] = w;
  }
}

template <int D, int NT, int KSEL>
cudaError_t launch_attend(const DecodeLaunch& p, cudaStream_t s) {
  auto kern = decode_attend_kernel<D, NT, KSEL>;
  const int smem = (int)sizeof(AttnSmem<D, NT, KSEL>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.G, (unsigned)p.B, (unsigned)p.n_split);
  kern<<<grid, kAttnThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(p.q), static_cast<const __nv_bfloat16*>(p.k_cache),
      static_cast<const __nv_bfloat16*>(p.v_cache), p.cu_seqlens, p.pooled, p.pooled_cap, p.G,
      p.H / p.G, p.top_k, p.scale * 1.4426950408889634f, p.ids,
      static_cast<__nv_bfloat16*>(p.out), p.n_split, p.part, p.tickets);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_attend_d(const DecodeLaunch& p, cudaStream_t s) {
  const int HG = p.H / p.G;
  if (HG <= 8) {
    if (p.top_k <= 16) return launch_attend<D, 1, 15>(p, s);
    return launch_attend<D, 1, 31>(p, s);
  }
  if (HG <= 16) {
    if (p.top_k <= 16) return launch_attend<D, 2, 15>(p, s);
    return launch_attend<D, 2, 31>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_partial_floats(int32_t H, int32_t G, int32_t d) {
  const int HG = H / G;
  const int heads = HG <= 8 ? 8 : 16;  // NT * 8
  return (size_t)heads * (d + 2);
}

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
  if (p.k_idx_scale) {
    if (p.d_idx != 128) return cudaErrorInvalidValue;
    decode_index_fp8_kernel<<<gi, kIdxWarps * 32, 0, s>>>(
        static_cast<const uint8_t*>(p.q_idx), static_cast<const uint8_t*>(p.k_idx_cache),
        p.k_idx_scale, p.cu_seqlens, p.G, p.pooled, p.pooled_cap, p.err);
  } else if (p.d_idx == 128)
    decode_index_kernel<128><<<gi, kIdxWarps * 32, 0, s>>>(qi, ki, p.cu_seqlens, p.G, p.pooled,
                                                            p.pooled_cap, p.err);
  else
    decode_index_kernel<64><<<gi, kIdxWarps * 32, 0, s>>>(qi, ki, p.cu_seqlens, p.G, p.pooled,
                                                           p.pooled_cap, p.err);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mark_ev(p, 1, s);
  e = p.d == 128 ? launch_attend_d<128>(p, s) : launch_attend_d<64>(p, s);
  ++*launches;
  mark_ev(p, 2, s);
  return e;
}

}  // namespace msa
