// index_kernel.cu -- Index Branch on the 5th-generation tensor cores.
//
// Computes, per (query t, group g), the token scores <q_idx[t,g], k_idx[s]>,
// their max over each 128-token key block, and the forced-local top-k block
// set (ai-tool-zukan "MiniMax MSA guide", sections "2段階構造の中身——ブロック
// 選択から厳密アテンションまで" and "クエリを含むローカルブロックの強制取り込み";
// one index-query head per group against one shared index-key head, section
// "Index BranchとMain Branchの役割分担").
//
// Tiling.  A tile is 128 index-query rows: T = 128/G consecutive tokens of one
// query block times all G groups, i.e. 128 contiguous rows of q_idx viewed as
// [N*G][d_idx].  Every key block j < blk(t) is fully visible to every token of
// the tile, so selection needs no causal mask: the local block is forced in
// and never scored.  One tcgen05.mma chain of M=128 x N=256 covers two key
// blocks (K=16 per bf16 instruction, K=32 per e4m3 one) and accumulates a
// 128x256 fp32 score tile in TMEM.  (N=128 per block would re-read the A
// tile from shared memory twice as often, which then runs at the tensor
// pipe's own rate.)
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0  TMA producer: q_idx tile once per tile, k_idx pairs into a ring
//           of shared-memory stages (128-byte swizzle, no multicast);
//   warp 1  MMA issuer: one elected thread, double-buffered TMEM accumulators
//           (2 x 256 columns), tcgen05.commit -> mbarriers;
//   warps 2-5  epilogue: thread <-> TMEM lane <-> tile row; tcgen05.ld the
//           row's 256 scores in 32-column chunks, each load in flight while
//           the previous chunk is folded into eight independent max chains;
//           max per block, then a one-step insert into a register-resident
//           sorted list of the best (k-1) blocks (an equal score keeps the
//           lower id, since blocks arrive in increasing id order).
//
// Tiles are ordered longest first (latest query block first) and dealt to
// the CTAs round-robin.
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace msa {
namespace {

constexpr int kRows = 128;      // UMMA M: index-query rows per tile
constexpr int kPairKeys = 256;  // UMMA N: two key blocks per MMA
constexpr int kBlock = 128;     // B_k

// FP8: e4m3 index queries and keys (kind::f8f6f4, 32 elements per MMA K
// step) with one fp32 scale per 128-key block; otherwise bf16 (kind::f16,
// 16 per step).  Either way a K step is 32 bytes of a 128-byte swizzled row.
template <int DI, bool FP8 = false>
struct IdxCfg {
  static constexpr int kElemBytes = FP8 ? 1 : 2;
  static constexpr int kRowBytes = DI * kElemBytes;
  static constexpr int kRegions = kRowBytes / 128;  // 128-byte swizzle spans per row
  static constexpr int kRegionElems = 128 / kElemBytes;
  static constexpr int kKSteps = kRowBytes / 32;
  static constexpr int kABytes = kRows * kRowBytes;
  static constexpr int kBBytes = kPairKeys * kRowBytes;
  static constexpr int kStages = kRowBytes == 256 ? 3 : 5;
  static constexpr int kSmem = kABytes + kStages * kBBytes + 1024;
};
constexpr int kThreads = 192;

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// instruction descriptor of kind::f8f6f4: D fp32, A and B e4m3 (format 0), K-major
__host__ __device__ constexpr uint32_t idesc_e4m3(uint32_t M, uint32_t N) {
  return (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

struct IdxArgs {
  int64_t N;
  int64_t row_begin, row_end;
  int32_t G, log2G, top_k;
  int32_t qb_lo, n_qblocks;
  int64_t nb;
  int32_t* ids;
  float* scores;
  const float* kscale;  // FP8 only: [nb] scale of each key block
  const int4* units;    // packed sequences: {first token, key row 0, local block, end}
  int32_t n_ublocks;    // entries of `units`
  uint32_t* err;
};

struct Unit {
  int32_t b;        // query block (local to its sequence)
  int64_t tok0;     // first token of the tile
  int64_t row0;     // first q_idx row ([N*G] view)
  int64_t key0;     // first row of the sequence's keys
  int64_t end;      // end of the sequence (one past its last token)
  int32_t nblk;     // key blocks scored
  int32_t pairs;    // MMAs of N=256
  bool valid;
};

// Tile v: query block v / G (latest first) and its sub-tile v % G.  With
// packed sequences the query blocks come from a table, ordered the same way
// across sequences, and every offset is relative to the sequence's first row.
template <bool SCORES>
__device__ __forceinline__ Unit make_unit(const IdxArgs& a, int v) {
  Unit u;
  const int T = kRows >> a.log2G;
  const int sub = v & (a.G - 1);
  if (a.units) {
    const int4 e = __ldg(a.units + (v >> a.log2G));
    u.b = e.z;
    u.tok0 = (int64_t)e.x + (int64_t)sub * T;
    u.key0 = e.y;
    u.end = e.w;
  } else {
    u.b = a.qb_lo + (a.n_qblocks - 1 - (v >> a.log2G));
    u.tok0 = (int64_t)u.b * kBlock + (int64_t)sub * T;
    u.key0 = 0;
    u.end = a.N;
  }
  u.row0 = u.tok0 * a.G;
  u.nblk = SCORES ? u.b + 1 : u.b;
  u.pairs = (u.nblk + 1) >> 1;
  u.valid = u.tok0 < u.end && u.tok0 < a.row_end && u.tok0 + T > a.row_begin;
  return u;
}


// folds 32 fp32 scores held as raw TMEM words into eight running max chains
// (three-input max; consecutive instructions are independent), in program
// order with the surrounding TMEM loads and waits
__device__ __forceinline__ void max_chains_ordered(float (&x)[8], const uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    x[i & 7] = max3f_ordered(x[i & 7], __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
}

template <int DI, int MAXSEL, bool SCORES, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    index_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const IdxArgs a) {
  using Cfg = IdxCfg<DI, FP8>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + Cfg::kABytes;

  __shared__ uint64_t bar_a_full, bar_a_empty;
  __shared__ uint64_t bar_b_full[S], bar_b_empty[S];
  __shared__ uint64_t bar_acc_full[2], bar_acc_empty[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&bar_a_full, 1);
    mbar_init(&bar_a_empty, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar_b_full[s], 1);
      mbar_init(&bar_b_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], 128);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;
  const int n_units = (a.units ? a.n_ublocks : a.n_qblocks) << a.log2G;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      int stage = 0;
      uint32_t sphase = 0, aphase = 0;
      bool a_issued = false;
      uint32_t a_last = 0;
      bool b_issued[S];
      uint32_t b_last[S];
      for (int s = 0; s < S; ++s) b_issued[s] = false, b_last[s] = 0;
      bool ok = true;
      for (int v = blockIdx.x; v < n_units && ok; v += gridDim.x) {
        const Unit u = make_unit<SCORES>(a, v);
        if (!u.valid) continue;
        if (!mbar_wait(&bar_a_empty, aphase ^ 1, abort_flag, a.err, kDevTimeoutMma)) break;
        mbar_arrive_expect_tx(&bar_a_full, Cfg::kABytes);
#pragma unroll
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d(sA + r * kRows * 128, &map_q, &bar_a_full, r * Cfg::kRegionElems,
                      (int32_t)u.row0);
        a_issued = true;
        a_last = aphase;
        aphase ^= 1;
        for (int p = 0; p < u.pairs; ++p) {
          if (!mbar_wait(&bar_b_empty[stage], sphase ^ 1, abort_flag, a.err, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_b_full[stage], Cfg::kBBytes);
#pragma unroll
          for (int r = 0; r < Cfg::kRegions; ++r)
            tma_load_2d(sB + stage * Cfg::kBBytes + r * kPairKeys * 128, &map_k, &bar_b_full[stage],
                        r * Cfg::kRegionElems, (int32_t)(u.key0 + p * kPairKeys));
          b_issued[stage] = true;
          b_last[stage] = sphase;
          if (++stage == S) stage = 0, sphase ^= 1;
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA exits
        volatile int no_abort = 0;
        if (a_issued) mbar_wait(&bar_a_full, a_last, &no_abort, nullptr, 0);
        for (int s = 0; s < S; ++s)
          if (b_issued[s]) mbar_wait(&bar_b_full[s], b_last[s], &no_abort, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc =
          FP8 ? idesc_e4m3(kRows, kPairKeys) : idesc_bf16(kRows, kPairKeys, false, false);
      int stage = 0, acc = 0;
      uint32_t sphase = 0, aphase = 0;
      uint32_t accphase[2] = {0, 0};
      bool committed = false;
      uint64_t* last_bar = nullptr;
      uint32_t last_par = 0;
      bool ok = true;
      const uint32_t a_base = smem_u32(sA);
      for (int v = blockIdx.x; v < n_units && ok; v += gridDim.x) {
        const Unit u = make_unit<SCORES>(a, v);
        if (!u.valid) continue;
        if (!mbar_wait(&bar_a_full, aphase, abort_flag, a.err, kDevTimeoutLoad)) break;
        for (int p = 0; p < u.pairs; ++p) {
          if (!mbar_wait(&bar_acc_empty[acc], accphase[acc] ^ 1, abort_flag, a.err,
                         kDevTimeoutConsumer) ||
              !mbar_wait(&bar_b_full[stage], sphase, abort_flag, a.err, kDevTimeoutLoad)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sB + stage * Cfg::kBBytes);
          const uint32_t d = tmem + acc * kPairKeys;
#pragma unroll
          for (int kk = 0; kk < Cfg::kKSteps; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_base + (kk >> 2) * kRows * 128 + (kk & 3) * 32,
                                                16, 1024);
            const uint64_t bd = smem_desc_sw128(
                b_base + (kk >> 2) * kPairKeys * 128 + (kk & 3) * 32, 16, 1024);
            if constexpr (FP8)
              umma_e4m3(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
            else
              umma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_b_empty[stage]);
          umma_commit(&bar_acc_full[acc]);
          committed = true;
          last_bar = &bar_acc_full[acc];
          last_par = accphase[acc];
          accphase[acc] ^= 1;
          acc ^= 1;
          if (++stage == S) stage = 0, sphase ^= 1;
        }
        if (!ok) break;
        umma_commit(&bar_a_empty);
        aphase ^= 1;
      }
      if (*abort_flag && committed) {
        volatile int no_abort = 0;
        mbar_wait(last_bar, last_par, &no_abort, nullptr, 0);  // MMAs done before TMEM is freed
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int g = row & (a.G - 1);
    const int tl = row >> a.log2G;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int acc = 0;
    uint32_t accphase[2] = {0, 0};
    bool ok = true;
    for (int v = blockIdx.x; v < n_units && ok; v += gridDim.x) {
      const Unit u = make_unit<SCORES>(a, v);
      if (!u.valid) continue;
      const int64_t t = u.tok0 + tl;
      const bool row_out = t >= a.row_begin && t < a.row_end && t < u.end;
      float sc[MAXSEL > 0 ? MAXSEL : 1];
      int32_t id[MAXSEL > 0 ? MAXSEL : 1];
#pragma unroll
      for (int i = 0; i < (MAXSEL > 0 ? MAXSEL : 1); ++i) sc[i] = -INFINITY, id[i] = -1;
      // local-block mask (scores mode only): keys s = 128*b + c with c <= lim
      const int lim = static_cast<int>(t - u.key0 - (int64_t)u.b * kBlock);
      float* srow = nullptr;
      if (SCORES && row_out) srow = a.scores + ((t - a.row_begin) * a.G + g) * a.nb;

      for (int p = 0; p < u.pairs; ++p) {
        if (!mbar_wait(&bar_acc_full[acc], accphase[acc], abort_flag, a.err, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = lane_addr + acc * kPairKeys;
        float m[2];
        if (SCORES) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(col + h * 128 + c * 32, r[c]);
            tmem_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) reg_fence(r[c]);
            const int j = 2 * p + h;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (j != u.b || c * 32 + i <= lim) mx = fmaxf(mx, __uint_as_float(r[c][i]));
            m[h] = mx;
          }
        } else {
          // eight 32-column chunks, double-buffered: the next chunk's TMEM load
          // is in flight while this one is folded into eight max chains
          uint32_t ra[32], rb[32];
          float x[8];
          tmem_ld_32x32b_x32(col, ra);
          tmem_wait();
          reg_fence(ra);
#pragma unroll
          for (int c = 0; c < 8; c += 2) {
            if ((c & 3) == 0) {
#pragma unroll
              for (int i = 0; i < 8; ++i) x[i] = -INFINITY;
            }
            tmem_ld_32x32b_x32(col + (c + 1) * 32, rb);
            max_chains_ordered(x, ra);
            tmem_wait();
            reg_fence(rb);
            if (c + 2 < 8) tmem_ld_32x32b_x32(col + (c + 2) * 32, ra);
            max_chains_ordered(x, rb);
            if ((c & 3) == 2)
              m[c >> 2] = max3f_ordered(max3f_ordered(x[0], x[1], x[2]),
                                        max3f_ordered(x[3], x[4], x[5]), fmaxf(x[6], x[7]));
            if (c + 2 < 8) {
              tmem_wait();
              reg_fence(ra);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar_acc_empty[acc]);
        accphase[acc] ^= 1;
        acc ^= 1;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 2 * p + h;
          if (j >= u.nblk) continue;
          // the keys of block j were quantised with the block's scale (> 0)
          const float mj = FP8 ? m[h] * __ldg(a.kscale + j) : m[h];
          if constexpr (SCORES) {
            if (row_out) srow[j] = mj;
          } else {
            if (mj > sc[MAXSEL - 1]) {
              // insert into the descending list in one step: slot i keeps its
              // entry when that entry is not below mj (an equal, earlier block
              // ranks higher), takes mj at the first slot below it, and takes
              // slot i-1's entry after that
#pragma unroll
              for (int i = MAXSEL - 1; i > 0; --i) {
                const bool keep = sc[i] >= mj;
                const bool here = sc[i - 1] >= mj;
                id[i] = keep ? id[i] : (here ? j : id[i - 1]);
                sc[i] = fmaxf(fminf(sc[i - 1], mj), sc[i]);
              }
              id[0] = sc[0] >= mj ? id[0] : j;
              sc[0] = fmaxf(sc[0], mj);
            }
          }
        }
      }
      if (!ok) break;
      if (!row_out) continue;
      if constexpr (SCORES) {
        for (int64_t j = u.nblk; j < a.nb; ++j) srow[j] = -INFINITY;
      } else {
        // selected = local block + best (top_k-1) earlier blocks, ascending
        constexpr int NOUT = MAXSEL + 1;
        int32_t o[NOUT];
        o[0] = u.b;
#pragma unroll
        for (int i = 0; i < MAXSEL; ++i)
          o[i + 1] = (i < a.top_k - 1 && id[i] >= 0) ? id[i] : 0x7FFFFFFF;
#pragma unroll
        for (int x = 0; x < NOUT; ++x)
#pragma unroll
          for (int y = 0; y + 1 < NOUT - x; ++y)
            if (o[y] > o[y + 1]) {
              const int32_t tmp = o[y];
              o[y] = o[y + 1];
              o[y + 1] = tmp;
            }
        int32_t* dst = a.ids + ((t - a.row_begin) * a.G + g) * a.top_k;
#pragma unroll
        for (int i = 0; i < NOUT; ++i)
          if (i < a.top_k) dst[i] = o[i] == 0x7FFFFFFF ? -1 : o[i];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DI, int MAXSEL, bool SCORES, bool FP8 = false>
cudaError_t launch_impl(const IndexLaunch& p, cudaStream_t s) {
  using Cfg = IdxCfg<DI, FP8>;
  CUtensorMap mq, mk;
  // rows of DI elements; make_tmap_2d counts the pitch in 2-byte units
  const CUtensorMapDataType type =
      FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_tmap_2d(&mq, type, p.q_idx, (uint64_t)p.N * p.G, DI, Cfg::kRowBytes / 2, kRows,
                    Cfg::kRegionElems, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&mk, type, p.k_idx, (uint64_t)p.N, DI, Cfg::kRowBytes / 2, kPairKeys,
                    Cfg::kRegionElems, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  IdxArgs a;
  a.N = p.N;
  a.row_begin = p.row_begin;
  a.row_end = p.row_end;
  a.G = p.G;
  a.log2G = 31 - __builtin_clz(p.G);
  a.top_k = p.top_k;
  a.qb_lo = static_cast<int32_t>(p.row_begin / kBlock);
  a.n_qblocks = static_cast<int32_t>((p.row_end - 1) / kBlock) - a.qb_lo + 1;
  a.nb = (p.N + kBlock - 1) / kBlock;
  a.ids = p.ids;
  a.scores = p.scores;
  a.kscale = p.kscale;
  a.units = p.units;
  a.n_ublocks = p.n_units;
  a.err = p.err;
  const int n_units = (p.units ? p.n_units : a.n_qblocks) * p.G;
  if (n_units < 1) return cudaSuccess;
  const int grid = n_units < p.num_sms ? n_units : p.num_sms;
  auto kern = index_kernel<DI, MAXSEL, SCORES, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, Cfg::kSmem, s>>>(mq, mk, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_select(const IndexLaunch& p, cudaStream_t s) {
  if (p.kscale) {  // e4m3 index tensors: d_idx = 128 only
    if (p.d_idx != 128) return cudaErrorInvalidValue;
    if (p.top_k <= 16) return launch_impl<128, 15, false, true>(p, s);
    return launch_impl<128, 31, false, true>(p, s);
  }
  if (p.d_idx == 128) {
    if (p.top_k <= 16) return launch_impl<128, 15, false>(p, s);
    return launch_impl<128, 31, false>(p, s);
  }
  if (p.top_k <= 16) return launch_impl<64, 15, false>(p, s);
  return launch_impl<64, 31, false>(p, s);
}

cudaError_t launch_index_scores(const IndexLaunch& p, cudaStream_t s) {
  if (p.d_idx == 128) return launch_impl<128, 0, true>(p, s);
  return launch_impl<64, 0, true>(p, s);
}

}  // namespace msa
