// align_kernel.cu -- index scores of the selected blocks, for the
// block-alignment diagnostic of msa_prefill_block_alignment.
//
// The Index Branch is trained by bringing its block-score distribution close
// to the distribution of where the Main Branch's exact attention actually
// went, with a KL divergence (ai-tool-zukan "MiniMax MSA guide", section
// "選択を学習可能にするKL損失").  This forward-only diagnostic emits the two:
// the pooled index score of every selected block (here) and the Main Branch
// attention mass of every selected block (merge kernel).
//
// block_score_kernel: one CTA per (group g, key block j) query list.  The
// block's index keys (128 x d_idx bf16) are loaded once into shared memory
// (16-byte chunks swizzled by row); each warp then scores 8 listed queries at
// a time with mma.sync m16n8k16 (keys as M, queries as N, index dims as K)
// and keeps, per query, the max over the block's visible keys (s <= t on the
// query's own block).  Not on the prefill hot path.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kScoreWarps = 8;
constexpr int kKeysPerBlock = 128;

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// byte offset of 16-byte chunk c of key row `row` (DI/8 chunks per row)
template <int DI>
__device__ __forceinline__ int key_off(int row, int c) {
  constexpr int CH = DI / 8;
  return row * (DI * 2) + ((c ^ (row & (CH - 1))) << 4);
}

template <int DI>
__global__ void __launch_bounds__(kScoreWarps * 32)
    block_score_kernel(const __nv_bfloat16* __restrict__ q_idx,
                       const __nv_bfloat16* __restrict__ k_idx, int64_t N, int32_t G,
                       int64_t nb, int64_t row_begin, int64_t rows, int32_t top_k,
                       const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ entries,
                       float* __restrict__ score, uint32_t* err) {
  __shared__ __align__(128) uint8_t sk[kKeysPerBlock * DI * 2];
  const int64_t x = blockIdx.x;
  const int g = (int)(x / nb), j = (int)(x - (int64_t)g * nb);
  const int32_t beg = row_ptr[x], end = row_ptr[x + 1];
  if (beg >= end) return;
  const int64_t key0 = (int64_t)j * kKeysPerBlock;
  const int nkeys = (int)min64(kKeysPerBlock, N - key0);
  constexpr int CH = DI / 8;
  for (int i = threadIdx.x; i < kKeysPerBlock * CH; i += blockDim.x) {
    const int row = i / CH, c = i % CH;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < nkeys) v = __ldg(reinterpret_cast<const uint4*>(k_idx + (key0 + row) * DI) + c);
    *reinterpret_cast<uint4*>(sk + key_off<DI>(row, c)) = v;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  // ldmatrix row and column chunk of this lane within a 16 x 16 A tile
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_chunk = lane >> 4;
  for (int32_t e0 = beg + warp * 8; e0 < end; e0 += kScoreWarps * 8) {
    // B operand: query n = gq of this batch, dims 16ks + 2tq (+1) and +8
    const int32_t ent_n = (e0 + gq < end) ? __ldg(entries + e0 + gq) : -1;
    int64_t t_n = ent_n >= 0 ? (int64_t)(ent_n >> 5) : row_begin;
    if (t_n < row_begin || t_n >= row_begin + rows || t_n >= N) {
      if (ent_n >= 0) record_error(err, kDevBadIndex);
      t_n = row_begin;
    }
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(q_idx + (t_n * G + g) * DI);
    uint32_t qb[DI / 16][2];
#pragma unroll
    for (int ks = 0; ks < DI / 16; ++ks) {
      qb[ks][0] = __ldg(qrow + ks * 8 + tq);
      qb[ks][1] = __ldg(qrow + ks * 8 + 4 + tq);
    }
    // the queries of this lane's two D columns (2tq, 2tq + 1)
    int64_t tc[2];
    bool vc[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int32_t en = (e0 + 2 * tq + h < end) ? __ldg(entries + e0 + 2 * tq + h) : -1;
      vc[h] = en >= 0;
      tc[h] = vc[h] ? (int64_t)(en >> 5) : -1;
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll 1
    for (int mt = 0; mt < kKeysPerBlock / 16; ++mt) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < DI / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, sk + key_off<DI>(mt * 16 + a_row, ks * 2 + a_chunk));
        mma16816(c, a, qb[ks][0], qb[ks][1]);
      }
      // D rows: keys mt*16 + gq (+8); columns: queries 2tq, 2tq + 1
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = mt * 16 + gq + ((e >> 1) << 3);
        const int h = e & 1;
        if (key < nkeys && key0 + key <= tc[h]) mx[h] = fmaxf(mx[h], c[e]);
      }
    }
    // max over the lanes holding the same columns (those with the same tq)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
    }
    if (gq == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int32_t e = e0 + 2 * tq + h;
        if (e < end && vc[h]) {
          const int32_t en = __ldg(entries + e);
          const int64_t t = en >> 5;
          const int r = en & 31;
          if (t >= row_begin && t < row_begin + rows && r < top_k)
            score[((t - row_begin) * G + g) * top_k + r] = mx[h];
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_block_scores(const BlockScoreLaunch& p, cudaStream_t s) {
  const int64_t lists = (int64_t)p.G * p.nb;
  if (lists == 0) return cudaSuccess;
  if (p.d_idx == 128)
    block_score_kernel<128><<<(unsigned)lists, kScoreWarps * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(p.q_idx), static_cast<const __nv_bfloat16*>(p.k_idx),
        p.N, p.G, p.nb, p.row_begin, p.rows, p.top_k, p.row_ptr, p.entries, p.score, p.err);
  else
    block_score_kernel<64><<<(unsigned)lists, kScoreWarps * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(p.q_idx), static_cast<const __nv_bfloat16*>(p.k_idx),
        p.N, p.G, p.nb, p.row_begin, p.rows, p.top_k, p.row_ptr, p.entries, p.score, p.err);
  return cudaGetLastError();
}

}  // namespace msa
