// main_kernel.cu -- Main Branch prefill, key-block outer loop, gathered queries.
//
// Exact softmax attention over the selected blocks only (ai-tool-zukan "MiniMax
// MSA guide", section "Index BranchとMain Branchの役割分担"), computed with the
// key/value block as the outer loop: each work unit is one (group g, key block
// j) and a run of the queries that selected it; K_j and V_j are loaded once per
// unit and the hitting queries' heads are gathered into 128-row tiles
// (tnkblog MiniMax M3 / MSA post, section "MSA の実装"; CSDN M3 write-up,
// section "MiniMax Sparse Attention（MSA）": KV outer, gather Q, each KV block
// read once).
//
// Per tile (128 rows = TT tokens x the H/G heads of group g):
//   S = Q_tile K_j^T            tcgen05.mma M=128 N=128 K=d   (TMEM, fp32)
//   P = exp(scale*(S - rowmax)) softmax warps, causal mask on the local block;
//                               fp16 P overwrites the S columns already read
//   O = P V_j                   tcgen05.mma M=128 N=d  K=128, A = P from TMEM,
//                               B = V_j (fp16) from shared memory (MN-major)
// and the row's partial (o = O / rowsum in fp16, lse = scale*rowmax +
// ln rowsum) goes to slot (t, g, r, head); the merge kernel combines the <= k
// slots of a query with log-sum-exp weights.
//
// Warp roles (640 threads, one CTA per SM, persistent over units):
//   warp 0     Q producer: a TMA gather of each hitting token's H/G
//              contiguous query rows into a 2-stage ring;
//   warp 18    K/V loader: TMA of K_j / V_j (3-D map: one group's rows) once
//              per unit, plus an L2 prefetch of the next unit's blocks;
//   warp 1     S issuer (one thread): S MMAs of all tiles in order;
//   warp 19    PV issuer (one thread): PV MMAs of all tiles in order.  Two
//              issuing threads on different schedulers keep the tensor pipe
//              fed: one thread issuing both would be busy most of the time;
//   warps 2-17 two softmax + epilogue groups of 8 warps taking alternate
//              tiles; a tile row is split between two warps of its group
//              (TMEM lane = row, 64 columns each).  The epilogue stages the
//              fp16 partials in the group's shared staging buffer and writes
//              each token's heads with a TMA store (2 KiB for 8 heads of 128).
// TMEM: two S/P buffers (2 x 128 columns) and two O buffers (2 x 128
// columns), buffer w belonging to softmax group w.  Keeping P in TMEM halves
// the shared-memory operand traffic of the PV product and leaves the P
// stores off the shared-memory pipe.
//
// Precision of the PV product.  P in [0, 1] goes to the tensor cores in fp16
// (11-bit significand) rather than bf16 (8 bits): with bf16 P a softmax over
// a handful of keys (the first tokens of a sequence) can be off by 2^-9 of
// |v| per weight, which together with the bf16 output rounding exceeds 1e-2
// on outputs of magnitude 2 to 4.  The two operands of one MMA share a type,
// so V is converted to fp16 once per call (v_to_fp16_kernel below).
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace msa {
namespace {

// Q producer, S issuer, 2 softmax groups of 8 warps, K/V loader, PV issuer
constexpr int kThreads = 640;
constexpr int kKVWarp = 18;
constexpr int kPVWarp = 19;
constexpr int kGroupThreads = 256;
constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kQStages = 2;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory tiles of 128 rows x D (Q, and the fp16 O staging) are kept as
// 16 groups of 8 rows; a group holds its D/64 column chunks one after the
// other, each chunk 8 rows x 128 bytes with the 128-byte swizzle.  The 8-row
// group of a token's heads is then 1-2 KiB of contiguous shared memory,
// moved by ONE 3-D TMA copy (x = 64 columns, y = rows, z = chunk; chunk
// stride 128 bytes in global memory), and the K-major MMA operand advances by
// D/64 KiB per 8 rows.
template <int D>
struct MainCfg {
  static constexpr int kRegions = D / 64;
  static constexpr int kGroupBytes = kRegions * 1024;  // one 8-row group
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKVBytes = kKeys * D * 2;
  static constexpr int kOBytes = kRows * D * 2;  // fp16 staging of one O tile
  static constexpr int kOffK = kQStages * kQBytes;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffO = kOffV + kKVBytes;
  static constexpr int kSmem = kOffO + 2 * kOBytes + 1024;
};

struct MainArgs {
  int64_t N, row_begin, rows;
  int32_t H, G, HG, log2slot, TT, top_k;
  float scale, scale_log2;
  int64_t nb;
  const int32_t* row_ptr;
  const int32_t* entries;
  const int32_t* unit_ptr;
  const int4* unit_desc;
  const int32_t* blk_row0;  // packed sequences: first K/V row of key block j (else j*128)
  __half* part_o;
  float* part_lse;
  uint32_t* err;
};

struct MUnit {
  int32_t g, j, e0, e1, ntiles;
  int32_t row0;  // first K/V row of the unit's key block
};

__device__ __forceinline__ MUnit decode_unit(const MainArgs& a, int u) {
  const int4 d = __ldg(a.unit_desc + u);  // {g, j, first entry, end entry}
  MUnit m;
  m.g = d.x;
  m.j = d.y;
  m.e0 = d.z;
  m.e1 = d.w;
  m.ntiles = (m.e1 - m.e0 + a.TT - 1) / a.TT;
  m.row0 = a.blk_row0 ? __ldg(a.blk_row0 + m.j) : m.j * kKeys;
  return m;
}

// position of a tile in this CTA's sequence of units
struct TilePos {
  int u, i;
  MUnit m;
  bool more;
};

__device__ __forceinline__ TilePos first_tile(const MainArgs& a, int n_units) {
  TilePos p;
  p.u = blockIdx.x;
  p.i = 0;
  p.more = p.u < n_units;
  if (p.more) p.m = decode_unit(a, p.u);
  return p;
}

__device__ __forceinline__ void next_tile(TilePos& p, const MainArgs& a, int n_units) {
  if (!p.more) return;
  if (++p.i >= p.m.ntiles) {
    p.i = 0;
    p.u += gridDim.x;
    p.more = p.u < n_units;
    if (p.more) p.m = decode_unit(a, p.u);
  }
}

// raw list entry of this thread's row in tile p (-1 for padding rows)
__device__ __forceinline__ int32_t prefetch_entry(const MainArgs& a, const TilePos& p, int ts,
                                                  int hh) {
  const int e = p.m.e0 + p.i * a.TT + ts;
  return (e < p.m.e1 && hh < a.HG) ? __ldg(a.entries + e) : -1;
}

// decoded list entry, validated against the lists' query range
__device__ __forceinline__ bool check_entry(const MainArgs& a, int32_t ent, int64_t& t, int& r) {
  t = (int64_t)(ent >> 5);
  r = ent & 31;
  const bool ok = ent >= 0 && t >= a.row_begin && t < a.row_begin + a.rows && t < a.N &&
                  r < a.top_k;
  if (!ok) {
    record_error(a.err, kDevBadIndex);
    t = a.row_begin;
    r = 0;
  }
  return ok;
}

__device__ __forceinline__ bool read_entry(const MainArgs& a, int e, int64_t& t, int& r) {
  const int32_t ent = __ldg(a.entries + e);
  t = (int64_t)(ent >> 5);
  r = ent & 31;
  const bool ok = ent >= 0 && t >= a.row_begin && t < a.row_begin + a.rows && t < a.N &&
                  r < a.top_k;
  if (!ok) {
    record_error(a.err, kDevBadIndex);
    t = a.row_begin;
    r = 0;
  }
  return ok;
}

// exp2 of 32 scores of a row, packed two fp16 per word (the even column in
// the lower half, the layout of an A operand in TMEM), and the fp32 sum of the
// rounded values.  MASK: keep columns <= lim (relative to the first of the 32).
// p <= 1, so the fp16 conversion never overflows.
template <bool MASK>
__device__ __forceinline__ void softmax32(const uint32_t (&sv)[32], uint64_t k2, uint64_t nm2,
                                          int lim, uint32_t taddr, uint64_t& acc_a,
                                          uint64_t& acc_b) {
  uint32_t w[16];
#pragma unroll
  for (int x2 = 0; x2 < 16; ++x2) {
    const int col = 2 * x2;
    const uint64_t s2 = f2_pack(__uint_as_float(sv[col]), __uint_as_float(sv[col + 1]));
    float a0, a1;
    f2_unpack(f2_fma(s2, k2, nm2), a0, a1);
    float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
    if (MASK) {
      p0 = col <= lim ? p0 : 0.f;
      p1 = col + 1 <= lim ? p1 : 0.f;
    }
    w[x2] = pack_half2(p0, p1);
    if (x2 & 1)
      acc_b = f2_add(acc_b, half2_as_f2(w[x2]));
    else
      acc_a = f2_add(acc_a, half2_as_f2(w[x2]));
    if ((x2 & 7) == 7) tmem_st_32x32b_x8(taddr + (x2 - 7), &w[x2 - 7]);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    main_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                const MainArgs a) {
  using Cfg = MainCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sO = smem + Cfg::kOffO;

  __shared__ uint64_t bar_q_full[kQStages], bar_q_empty[kQStages];
  __shared__ uint64_t bar_k_full, bar_k_empty, bar_v_full, bar_v_empty;
  __shared__ uint64_t bar_s_full[2], bar_s_empty[2];
  __shared__ uint64_t bar_p_full[2];
  __shared__ uint64_t bar_o_full[2], bar_o_empty[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ float xchg_max[2][2][kRows];  // [group][column half][row]
  __shared__ float xchg_sum[2][2][kRows];

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bar_q_full[s], 1);
      mbar_init(&bar_q_empty[s], 1);
    }
    mbar_init(&bar_k_full, 1);
    mbar_init(&bar_k_empty, 1);
    mbar_init(&bar_v_full, 1);
    mbar_init(&bar_v_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_s_empty[i], 1);  // committed by the PV that read P
      mbar_init(&bar_p_full[i], kGroupThreads);
      mbar_init(&bar_o_full[i], 1);
      mbar_init(&bar_o_empty[i], kGroupThreads);
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
  const int n_units = __ldg(a.unit_ptr + a.G * a.nb);
  const int slot = 1 << a.log2slot;

  if (warp == 0) {
    // ---------------- Q gather producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_o);
    }
    int qs = 0;
    uint32_t qph = 0;
    // last issued phase per stage, for draining after an abort
    uint32_t q_last[kQStages] = {};
    bool q_any[kQStages] = {};
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const MUnit m = decode_unit(a, u);
      for (int i = 0; i < m.ntiles && ok; ++i) {
        const int eb = m.e0 + i * a.TT;
        const int nt = min(a.TT, m.e1 - eb);
        // the entry loads overlap the wait for a free stage
        int64_t t = 0;
        int r = 0;
        if (lane < nt) read_entry(a, eb + lane, t, r);
        if (lane == 0) {
          ok = mbar_wait(&bar_q_empty[qs], qph ^ 1, abort_flag, a.err, kDevTimeoutMma);
          if (ok) {
            mbar_arrive_expect_tx(&bar_q_full[qs], (uint32_t)nt * slot * D * 2);
            q_any[qs] = true;
            q_last[qs] = qph;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane < nt) {
          // the token's slot rows, 8 at a time (rows past H/G are other
          // heads' queries, never used; past the tensor end they read zero)
          const int32_t qrow = (int32_t)(t * a.H + (int64_t)m.g * a.HG);
          uint8_t* dst = sQ + qs * Cfg::kQBytes + (lane * slot / 8) * Cfg::kGroupBytes;
          for (int k8 = 0; k8 < slot; k8 += 8)
            tma_load_3d(dst + (k8 / 8) * Cfg::kGroupBytes, &map_q, &bar_q_full[qs], 0,
                        qrow + k8, 0);
        }
        __syncwarp();
        if (++qs == kQStages) qs = 0, qph ^= 1;
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int no_abort = 0;
      for (int s = 0; s < kQStages; ++s)
        if (q_any[s]) mbar_wait(&bar_q_full[s], q_last[s], &no_abort, nullptr, 0);
    }
  } else if (warp == kKVWarp) {
    // ---------------- K/V loader ----------------
    // K_j and V_j of each unit into their single buffers, and an L2 prefetch
    // of the next unit's blocks so that those loads hit L2.
    if (lane == 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      uint32_t kph = 0, vph = 0;
      bool k_any = false, v_any = false;
      uint32_t k_last = 0, v_last = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const MUnit m = decode_unit(a, u);
        if (u + (int)gridDim.x < n_units) {
          const MUnit nx = decode_unit(a, u + gridDim.x);
#pragma unroll
          for (int ri = 0; ri < Cfg::kRegions; ++ri) {
            tma_prefetch_l2_3d(&map_k, ri * 64, nx.g, nx.row0);
            tma_prefetch_l2_3d(&map_v, ri * 64, nx.g, nx.row0);
          }
        }
        if (!mbar_wait(&bar_k_empty, kph ^ 1, abort_flag, a.err, kDevTimeoutMma)) break;
        mbar_arrive_expect_tx(&bar_k_full, Cfg::kKVBytes);
#pragma unroll
        for (int ri = 0; ri < Cfg::kRegions; ++ri)
          tma_load_3d(sK + ri * kKeys * 128, &map_k, &bar_k_full, ri * 64, m.g, m.row0);
        k_any = true;
        k_last = kph;
        kph ^= 1;
        if (!mbar_wait(&bar_v_empty, vph ^ 1, abort_flag, a.err, kDevTimeoutMma)) break;
        mbar_arrive_expect_tx(&bar_v_full, Cfg::kKVBytes);
#pragma unroll
        for (int ri = 0; ri < Cfg::kRegions; ++ri)
          tma_load_3d(sV + ri * kKeys * 128, &map_v, &bar_v_full, ri * 64, m.g, m.row0);
        v_any = true;
        v_last = vph;
        vph ^= 1;
      }
      if (*abort_flag) {
        volatile int no_abort = 0;
        if (k_any) mbar_wait(&bar_k_full, k_last, &no_abort, nullptr, 0);
        if (v_any) mbar_wait(&bar_v_full, v_last, &no_abort, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------- S issuer (one thread) ----------------
    // S = Q K^T for every tile in order, into S buffer n%2 once the PV of
    // tile n-2 has released it.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, false, false);
      TilePos sc = first_tile(a, n_units);
      int qs = 0, sb = 0;
      uint32_t qph = 0, kph = 0;
      uint32_t sph[2] = {0, 0};
      bool committed = false;
      uint64_t* last_bar = nullptr;
      uint32_t last_par = 0;
      const uint32_t k_base = smem_u32(sK);
      while (sc.more) {
        if (sc.i == 0) {
          if (!mbar_wait(&bar_k_full, kph, abort_flag, a.err, kDevTimeoutLoad)) break;
          kph ^= 1;
        }
        if (!mbar_wait(&bar_q_full[qs], qph, abort_flag, a.err, kDevTimeoutLoad)) break;
        if (!mbar_wait(&bar_s_empty[sb], sph[sb] ^ 1, abort_flag, a.err, kDevTimeoutMma)) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + qs * Cfg::kQBytes);
        const uint32_t d_tm = tmem + sb * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(q_base + (kk >> 2) * 1024 + (kk & 3) * 32, 16,
                                              Cfg::kGroupBytes);
          const uint64_t bd =
              smem_desc_sw128(k_base + (kk >> 2) * kKeys * 128 + (kk & 3) * 32, 16, 1024);
          umma_bf16(d_tm, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar_q_empty[qs]);
        umma_commit(&bar_s_full[sb]);
        if (sc.i == sc.m.ntiles - 1) umma_commit(&bar_k_empty);
        committed = true;
        last_bar = &bar_s_full[sb];
        last_par = sph[sb];
        sph[sb] ^= 1;
        sb ^= 1;
        if (++qs == kQStages) qs = 0, qph ^= 1;
        next_tile(sc, a, n_units);
      }
      if (*abort_flag && committed) {
        volatile int no_abort = 0;
        mbar_wait(last_bar, last_par, &no_abort, nullptr, 0);
      }
    }
  } else if (warp == kPVWarp) {
    // ---------------- PV issuer (one thread) ----------------
    // O = P V for every tile in order: A = P from the tile's S/P buffer in
    // TMEM, B = V_j from shared memory, into O buffer n%2 once the epilogue
    // of tile n-2 has read it.
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_f16(kRows, D, false, true);  // fp16 P and V
      TilePos pc = first_tile(a, n_units);
      int pb = 0;
      uint32_t vph = 0;
      uint32_t pph[2] = {0, 0};
      bool committed = false;
      uint64_t* last_bar = nullptr;
      uint32_t last_par = 0;
      const uint32_t v_base = smem_u32(sV);
      while (pc.more) {
        if (pc.i == 0) {
          if (!mbar_wait(&bar_v_full, vph, abort_flag, a.err, kDevTimeoutLoad)) break;
          vph ^= 1;
        }
        // S/P buffer pb and O buffer pb are used in lockstep: one phase each
        if (!mbar_wait(&bar_p_full[pb], pph[pb], abort_flag, a.err, kDevTimeoutConsumer)) break;
        if (!mbar_wait(&bar_o_empty[pb], pph[pb] ^ 1, abort_flag, a.err, kDevTimeoutConsumer))
          break;
        tc_fence_after();
        const uint32_t d_tm = tmem + 256 + pb * 128;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // keys 16kk..16kk+15: written by column half kk/4 as 8 packed
          // columns at offset 8*(kk%4) of that half's S columns
          const uint32_t a_tm = tmem + pb * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
          const uint64_t bd = smem_desc_sw128(v_base + kk * 16 * 128, kKeys * 128, 1024);
          umma_f16_ts(d_tm, a_tm, bd, idesc_o, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar_s_empty[pb]);  // P read: the S/P buffer is free
        umma_commit(&bar_o_full[pb]);
        if (pc.i == pc.m.ntiles - 1) umma_commit(&bar_v_empty);
        committed = true;
        last_bar = &bar_o_full[pb];
        last_par = pph[pb];
        pph[pb] ^= 1;
        pb ^= 1;
        next_tile(pc, a, n_units);
      }
      if (*abort_flag && committed) {
        volatile int no_abort = 0;
        mbar_wait(last_bar, last_par, &no_abort, nullptr, 0);
      }
    }
  } else {
    // ---------------- softmax + epilogue: two groups of 8 warps ----------------
    // Group grp (warps 2+8grp .. 9+8grp) owns the tiles of parity grp, with S/P
    // buffer grp and O buffer grp.  Each row of a tile is split between two
    // warps of the group (same TMEM lane quarter, column half hc), which
    // combine their row max and row sum through shared memory.  Warp w reaches
    // TMEM lane quarter w%4, so warps 2+8grp+i (hc = 0) and 6+8grp+i (hc = 1)
    // hold the same quarter (2+i)%4.
    //
    // The epilogue of a tile runs one group iteration late, after the softmax
    // of the group's next tile: its PV product then completes while the group
    // works on that softmax instead of being waited for.
    const int grp = (warp - 2) >> 3;
    const int hc = ((warp - 2) & 7) >> 2;  // column half: S/P columns 64hc..64hc+63
    const int quarter = warp & 3;
    // The two warps of a lane quarter (hc = 0, 1) share their 32 rows: the
    // max and sum exchanges and the staging of a row group's partials only
    // couple this pair, so they synchronise with a 64-thread named barrier.
    const uint32_t bar_id = 1 + grp * 4 + quarter;
    const int row = quarter * 32 + lane;
    const int ts = row >> a.log2slot;
    const int hh = row & (slot - 1);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = grp * 128 + hc * 64, o_col = 256 + grp * 128 + hc * 64;
    const bool has_o = hc * 64 < D;
    uint8_t* obuf = sO + grp * Cfg::kOBytes;
    // staging of this row: its 8-row group, chunk hc, line hc*rows + row%8
    // (rows = min(H/G, 8): the height of the TMA store box)
    const int box_rows = a.HG < 8 ? a.HG : 8;
    uint8_t* oblk = obuf + (row >> 3) * Cfg::kGroupBytes;
    const int oline = hc * box_rows + (row & 7);
    const bool stage_row = (row & 7) < box_rows;
    uint32_t sph = 0, oph = 0;
    bool ok = true;
    bool store_pending = false;  // this thread issued TMA stores from obuf

    // the tile whose epilogue is pending (this thread's row of it): first
    // partial row, lse and 1/rowsum
    bool pend = false, pend_valid = false;
    int64_t pend_slot = 0;
    float pend_lse = 0.f, pend_inv = 1.f;

    // O / l -> fp16 staged in obuf, then one TMA store per token and region
    auto epilogue = [&]() -> bool {
      if (!mbar_wait(&bar_o_full[grp], oph, abort_flag, a.err, kDevTimeoutMma)) return false;
      tc_fence_after();
      // 32 columns at a time; the O buffer is released after the last load
      const uint64_t inv2 = f2_pack(pend_inv, pend_inv);
#pragma unroll 1
      for (int oc = 0; oc < 2; ++oc) {
        uint32_t o[32];
        if (has_o) {
          tmem_ld_32x32b_x32(lane_addr + o_col + oc * 32, o);
          tmem_wait();
          reg_fence(o);
        }
        if (oc == 1) {
          tc_fence_before();
          mbar_arrive(&bar_o_empty[grp]);
          oph ^= 1;
        }
        if (has_o && stage_row) {
          // 128-byte-swizzled staging: conflict-free writes; the TMA store
          // below undoes the swizzle on its way to global memory
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint4 w;
#pragma unroll
            for (int x2 = 0; x2 < 4; ++x2) {
              float f0, f1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o[c4 * 8 + 2 * x2]),
                                       __uint_as_float(o[c4 * 8 + 2 * x2 + 1])),
                               inv2),
                        f0, f1);
              (&w.x)[x2] = pack_half2(f0, f1);
            }
            *reinterpret_cast<uint4*>(oblk + sw128_offset(oline, oc * 4 + c4)) = w;
          }
        }
      }
      fence_async_smem();
      named_barrier(bar_id, 64);
      if (pend_valid && hc == 0) {
        a.part_lse[pend_slot + hh] = pend_lse;
        if ((hh & 7) == 0) {
          // this row's 8-row group: all of its column chunks in one copy
          tma_store_3d(&map_o, oblk, 0, (int32_t)(pend_slot + hh), 0);
          bulk_commit();
          store_pending = true;
        }
      }
      return true;
    };

    TilePos cur = first_tile(a, n_units);
    if (grp == 1) next_tile(cur, a, n_units);
    int32_t cur_ent = cur.more ? prefetch_entry(a, cur, ts, hh) : -1;

    // one pass per tile of this group, plus a last one that only drains the
    // pending epilogue
    while (cur.more || pend) {
      if (!cur.more) {
        // staging must be free: wait for the last store's read
        if (store_pending) {
          bulk_wait_read<0>();
          store_pending = false;
        }
        named_barrier(bar_id, 64);
        if (!epilogue()) ok = false;
        break;
      }
      TilePos nxt = cur;
      next_tile(nxt, a, n_units);
      next_tile(nxt, a, n_units);
      const int32_t nxt_ent = nxt.more ? prefetch_entry(a, nxt, ts, hh) : -1;
      const MUnit& m = cur.m;
      const int e = m.e0 + cur.i * a.TT + ts;
      const bool row_valid = (e < m.e1) && (hh < a.HG);
      int64_t t = 0;
      int r = 0;
      bool good = false;
      if (row_valid) good = check_entry(a, cur_ent, t, r);
      // last visible column of this half (keys s <= t on the local block)
      const int lim = (row_valid ? (int)min64(t - (int64_t)m.row0, kKeys - 1) : kKeys - 1) -
                      hc * 64;
      const bool unmasked = __all_sync(0xffffffffu, lim >= 63);

      // ---- pass 1: max over this half's 64 scores ----
      if (!mbar_wait(&bar_s_full[grp], sph, abort_flag, a.err, kDevTimeoutMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float hmx = -INFINITY;
      {
        uint32_t sv[2][32];
        tmem_ld_32x32b_x32(lane_addr + s_col, sv[0]);
        tmem_ld_32x32b_x32(lane_addr + s_col + 32, sv[1]);
        tmem_wait();
        reg_fence(sv[0]);
        reg_fence(sv[1]);
        if (unmasked) {
          float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            x0 = max3f(x0, __uint_as_float(sv[0][x]), __uint_as_float(sv[0][x + 1]));
            x1 = max3f(x1, __uint_as_float(sv[1][x]), __uint_as_float(sv[1][x + 1]));
          }
          hmx = fmaxf(x0, x1);
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (c * 32 + x <= lim) hmx = fmaxf(hmx, __uint_as_float(sv[c][x]));
        }
      }
      xchg_max[grp][hc][row] = hmx;
      // the previous tile's partials must be out of the staging buffer before
      // the epilogue rewrites it; the barrier also publishes both maxima
      if (store_pending) {
        bulk_wait_read<0>();
        store_pending = false;
      }
      named_barrier(bar_id, 64);
      float mx = fmaxf(xchg_max[grp][0][row], xchg_max[grp][1][row]);
      if (!(row_valid && good) || !(mx > -INFINITY)) mx = 0.f;
      const float mxs = mx * a.scale_log2;

      // ---- pass 2: P = exp2(scale*log2e*(S - max)) in bf16, 32 columns at a time ----
      // chunk pc of this half's S columns becomes 16 packed P columns written
      // over S columns this thread has already read (s_col + 16pc ..)
      const uint64_t k2 = f2_pack(a.scale_log2, a.scale_log2);
      const uint64_t nm2 = f2_pack(-mxs, -mxs);
      uint64_t acc_a = f2_pack(0.f, 0.f), acc_b = acc_a;
#pragma unroll 1
      for (int pc = 0; pc < 2; ++pc) {
        uint32_t sv[32];
        tmem_ld_32x32b_x32(lane_addr + s_col + pc * 32, sv);
        tmem_wait();
        reg_fence(sv);
        const uint32_t p_addr = lane_addr + s_col + pc * 16;
        if (unmasked)
          softmax32<false>(sv, k2, nm2, 0, p_addr, acc_a, acc_b);
        else
          softmax32<true>(sv, k2, nm2, lim - pc * 32, p_addr, acc_a, acc_b);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full[grp]);
      sph ^= 1;
      float la0, la1, lb0, lb1;
      f2_unpack(acc_a, la0, la1);
      f2_unpack(acc_b, lb0, lb1);
      xchg_sum[grp][hc][row] = (la0 + la1) + (lb0 + lb1);
      named_barrier(bar_id, 64);
      const float l = xchg_sum[grp][0][row] + xchg_sum[grp][1][row];

      // ---- epilogue of the group's previous tile ----
      if (pend && !epilogue()) {
        ok = false;
        break;
      }
      pend = true;
      pend_valid = row_valid && good;
      pend_slot = (((t - a.row_begin) * a.G + m.g) * a.top_k + r) * a.HG;
      pend_lse = mx * a.scale + __logf(l);
      pend_inv = 1.0f / l;
      cur = nxt;
      cur_ent = nxt_ent;
    }
    if (store_pending) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// V (bf16) -> fp16, 16 bytes per thread and step; records kDevValueRange for
// a value beyond the fp16 range or NaN (saturated to +-65504 / kept NaN)
__global__ void __launch_bounds__(256) v_to_fp16_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, int64_t n8,
                                                        uint32_t* err) {
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * 256) {
    const uint4 w = __ldg(src + i);
    uint4 o;
    const uint32_t* wi = &w.x;
    uint32_t* oi = &o.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float lo = __uint_as_float(wi[c] << 16), hi = __uint_as_float(wi[c] & 0xFFFF0000u);
      bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
      oi[c] = pack_half2_satfinite(lo, hi);
    }
    dst[i] = o;
  }
  if (bad) record_error(err, kDevValueRange);
}

template <int D>
cudaError_t launch_main_impl(const MainLaunch& p, cudaStream_t s) {
  using Cfg = MainCfg<D>;
  const int HG = p.H / p.G;
  const int slot = HG < 8 ? 8 : HG;
  CUtensorMap mq, mk, mv, mo;
  const uint64_t part_rows = (uint64_t)p.rows * p.G * p.top_k * HG;
  const uint32_t box_rows = HG < 8 ? HG : 8;
  // [rows][D] viewed as (64 columns, rows, D/64 chunks)
  if (!make_tmap_bf16_3d(&mq, p.q, 64, (uint64_t)p.N * p.H, D / 64, D, 64, 64, 8, D / 64,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_3d(&mo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.part_o, 64, part_rows, D / 64, D, 64,
                    64, box_rows, D / 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bf16_3d(&mk, p.k, D, p.G, p.N, D, (uint64_t)p.G * D, 64, 1, kKeys,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_3d(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.v, D, p.G, p.N, D,
                    (uint64_t)p.G * D, 64, 1, kKeys, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  MainArgs a;
  a.N = p.N;
  a.row_begin = p.row_begin;
  a.rows = p.rows;
  a.H = p.H;
  a.G = p.G;
  a.HG = HG;
  a.log2slot = 31 - __builtin_clz(slot);
  a.TT = kRows / slot;
  a.top_k = p.top_k;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.nb = p.nb;
  a.row_ptr = p.row_ptr;
  a.entries = p.entries;
  a.unit_ptr = p.unit_ptr;
  a.unit_desc = p.unit_desc;
  a.blk_row0 = p.blk_row0;
  a.part_o = p.part_o;
  a.part_lse = p.part_lse;
  a.err = p.err;
  auto kern = main_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<p.grid, kThreads, Cfg::kSmem, s>>>(mq, mk, mv, mo, a);
  return cudaGetLastError();
}

}  // namespace

int main_tile_tokens(int H, int G) {
  const int HG = H / G;
  return kRows / (HG < 8 ? 8 : HG);
}

cudaError_t launch_v_to_fp16(const void* src, void* dst, int64_t n, uint32_t* err, int sms,
                             cudaStream_t s) {
  if (n % 8 != 0 || (reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15)
    return cudaErrorInvalidValue;
  const int64_t n8 = n / 8;
  const int64_t want = (n8 + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
  v_to_fp16_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                        n8, err);
  return cudaGetLastError();
}

cudaError_t launch_main(const MainLaunch& p, cudaStream_t s) {
  if (p.d == 128) return launch_main_impl<128>(p, s);
  return launch_main_impl<64>(p, s);
}

}  // namespace msa
