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
//   P = exp(scale*(S - rowmax)) softmax warpgroup, one thread per row, the
//                               whole row of S in registers; causal mask on
//                               the local block; P in fp16 into TMEM
//   O = P V'_j                  tcgen05.mma M=128 N=d  K=128, A = P from TMEM,
//                               B = V'_j (fp16) from shared memory (MN-major)
// The row's partial is stored unnormalised: o' = O in fp16 at slot (t, g, r,
// head), with m~ = scale*rowmax + e_j*ln2 and l~ = rowsum * 2^-e_j, where V'_j
// = V_j * 2^-e_j is block j's value tile scaled into fp16 by a power of two
// (v_to_fp16_kernel below).  The merge kernel combines the <= k slots of a
// query: out = sum_r exp(m~_r - M) o'_r / sum_r exp(m~_r - M) l~_r.
//
// Warp roles (512 threads = 4 warpgroups, one CTA per SM, persistent):
//   WG0, WG1   softmax of the even / odd tiles (176 registers a thread);
//   WG2        epilogue of every tile: O from TMEM -> fp16, staged in shared
//              memory, one TMA store per token (2 KiB for 8 heads of 128);
//   WG3        warp 12 Q producer (a TMA gather of each hitting token's H/G
//              contiguous query rows into a 3-stage ring), warp 13 K/V loader
//              (once per unit, plus an L2 prefetch of the next unit's blocks),
//              warp 14 S issuer, warp 15 PV issuer (one thread each).
// TMEM (512 columns): one S buffer (0-127), two P buffers (128-191, 192-255)
// and two O buffers (256-383, 384-511).  A softmax thread copies its row of S
// into registers and releases the S buffer at once, so the next tile's S
// product runs while this tile's exponentials are computed; P and O are
// double-buffered between the two softmax warpgroups.
//
// Precision of the PV product.  P in [0, 1] goes to the tensor cores in fp16
// (11-bit significand) rather than bf16 (8 bits): with bf16 P a softmax over
// a handful of keys (the first tokens of a sequence) can be off by 2^-9 of
// |v| per weight, which together with the bf16 output rounding exceeds 1e-2
// on outputs of magnitude 2 to 4.  The two operands of one MMA share a type,
// so V is converted to fp16 once per call, block by block, each key block
// (and group) with its own power-of-two scale so that any finite bf16 value
// fits and the unnormalised o' (at most 128 * max|V'|) cannot overflow.
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"

namespace msa {
namespace {

constexpr int kThreads = 512;
constexpr int kQWarp = 12, kKVWarp = 13, kSWarp = 14;  // warp 15: PV issuer
constexpr int kGroupThreads = 128;  // one warpgroup
// registers per thread after the split; launched with 128 each, and
// 2*128*176 + 128*112 + 128*48 = 512*128
constexpr uint32_t kRegSoftmax = 176, kRegEpi = 112, kRegProd = 48;
constexpr int kLaunchRegs = 128;
constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kQStages = 3;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// largest |V'| after scaling: 128 * 511.75 = 65504, the fp16 maximum, bounds
// the unnormalised PV sum of one block
constexpr float kVMax = 511.75f;

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
  static constexpr int kSmem = kOffO + kOBytes + 1024;
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
  const int32_t* vexp;      // [j][G]: V'_j = V_j * 2^-vexp
  __half* part_o;
  float2* part_ml;
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

// The row of tile p that this thread owns: whether it is a real (query, head)
// row, its first partial row (slot of head 0 of its token) and its last
// visible key (relative to the block's first row; >= 127: all visible).
struct RowInfo {
  bool valid;
  int64_t slot;
  int lim;
};

__device__ __forceinline__ RowInfo row_info(const MainArgs& a, const TilePos& p, int32_t ent,
                                            int ts, int hh) {
  RowInfo ri;
  const int e = p.m.e0 + p.i * a.TT + ts;
  const bool row_valid = (e < p.m.e1) && (hh < a.HG);
  int64_t t = a.row_begin;
  int r = 0;
  bool good = false;
  if (row_valid) good = check_entry(a, ent, t, r);
  ri.valid = row_valid && good;
  ri.slot = (((t - a.row_begin) * a.G + p.m.g) * a.top_k + r) * a.HG;
  ri.lim = ri.valid ? (int)min64(t - (int64_t)p.m.row0, kKeys - 1) : kKeys - 1;
  return ri;
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
  __shared__ uint64_t bar_s_full[2], bar_s_empty;
  __shared__ uint64_t bar_p_full[2], bar_p_empty[2];
  __shared__ uint64_t bar_o_full[2], bar_o_empty[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

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
    mbar_init(&bar_s_empty, kGroupThreads);  // the softmax warpgroup has read S
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_full[i], kGroupThreads);
      mbar_init(&bar_p_empty[i], 1);  // committed by the PV that read P
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
  const int wg = warp >> 2;

  if (wg == 3) {
    regs_decrease<kRegProd>();
    if (warp == kQWarp) {
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
          if (lane < nt) check_entry(a, __ldg(a.entries + eb + lane), t, r);
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
    } else if (warp == kSWarp) {
      // ---------------- S issuer (one thread) ----------------
      // S = Q K^T for every tile in order, into the S buffer once the softmax
      // of the previous tile has copied it out.
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16(kRows, kKeys, false, false);
        TilePos sc = first_tile(a, n_units);
        int qs = 0, n = 0;
        uint32_t qph = 0, kph = 0, sph = 0;
        bool committed = false;
        uint64_t* last_bar = nullptr;
        uint32_t last_par = 0;
        uint32_t sfull_ph[2] = {0, 0};
        const uint32_t k_base = smem_u32(sK);
        while (sc.more) {
          if (sc.i == 0) {
            if (!mbar_wait(&bar_k_full, kph, abort_flag, a.err, kDevTimeoutLoad)) break;
            kph ^= 1;
          }
          if (!mbar_wait(&bar_q_full[qs], qph, abort_flag, a.err, kDevTimeoutLoad)) break;
          if (!mbar_wait(&bar_s_empty, sph ^ 1, abort_flag, a.err, kDevTimeoutConsumer)) break;
          sph ^= 1;
          tc_fence_after();
          const uint32_t q_base = smem_u32(sQ + qs * Cfg::kQBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(q_base + (kk >> 2) * 1024 + (kk & 3) * 32, 16,
                                                Cfg::kGroupBytes);
            const uint64_t bd =
                smem_desc_sw128(k_base + (kk >> 2) * kKeys * 128 + (kk & 3) * 32, 16, 1024);
            umma_bf16(tmem + kColS, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_q_empty[qs]);
          umma_commit(&bar_s_full[n & 1]);
          if (sc.i == sc.m.ntiles - 1) umma_commit(&bar_k_empty);
          committed = true;
          last_bar = &bar_s_full[n & 1];
          last_par = sfull_ph[n & 1];
          sfull_ph[n & 1] ^= 1;
          ++n;
          if (++qs == kQStages) qs = 0, qph ^= 1;
          next_tile(sc, a, n_units);
        }
        if (*abort_flag && committed) {
          volatile int no_abort = 0;
          mbar_wait(last_bar, last_par, &no_abort, nullptr, 0);
        }
      }
    } else {
      // ---------------- PV issuer (one thread) ----------------
      // O = P V' for every tile in order: A = P from P buffer n%2 in TMEM,
      // B = V'_j from shared memory, into O buffer n%2 once the epilogue of
      // tile n-2 has read it.
      if (lane == 0) {
        constexpr uint32_t idesc_o = idesc_f16(kRows, D, false, true);  // fp16 P and V'
        TilePos pc = first_tile(a, n_units);
        int b = 0;
        uint32_t vph = 0;
        uint32_t pph[2] = {0, 0}, oph[2] = {0, 0};
        bool committed = false;
        uint64_t* last_bar = nullptr;
        uint32_t last_par = 0;
        const uint32_t v_base = smem_u32(sV);
        while (pc.more) {
          if (pc.i == 0) {
            if (!mbar_wait(&bar_v_full, vph, abort_flag, a.err, kDevTimeoutLoad)) break;
            vph ^= 1;
          }
          if (!mbar_wait(&bar_p_full[b], pph[b], abort_flag, a.err, kDevTimeoutConsumer)) break;
          if (!mbar_wait(&bar_o_empty[b], oph[b] ^ 1, abort_flag, a.err, kDevTimeoutConsumer))
            break;
          tc_fence_after();
          const uint32_t d_tm = tmem + kColO + b * 128;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            // keys 16kk..16kk+15: 8 packed columns of the P buffer
            const uint32_t a_tm = tmem + kColP + b * 64 + kk * 8;
            const uint64_t bd = smem_desc_sw128(v_base + kk * 16 * 128, kKeys * 128, 1024);
            umma_f16_ts(d_tm, a_tm, bd, idesc_o, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_p_empty[b]);  // P read: the P buffer is free
          umma_commit(&bar_o_full[b]);
          if (pc.i == pc.m.ntiles - 1) umma_commit(&bar_v_empty);
          committed = true;
          last_bar = &bar_o_full[b];
          last_par = oph[b];
          pph[b] ^= 1;
          oph[b] ^= 1;
          b ^= 1;
          next_tile(pc, a, n_units);
        }
        if (*abort_flag && committed) {
          volatile int no_abort = 0;
          mbar_wait(last_bar, last_par, &no_abort, nullptr, 0);
        }
      }
    }
  } else if (wg == 2) {
    regs_decrease<kRegEpi>();
    // ---------------- epilogue: O -> fp16 partials ----------------
    // Tile n's O is in buffer n%2.  Each thread owns one row (TMEM lane); the
    // warp stages its 32 rows (128-byte swizzled) and one lane per 8-row group
    // writes the group's heads with a TMA store.
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int ts = row >> a.log2slot;
    const int hh = row & (slot - 1);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int box_rows = a.HG < 8 ? a.HG : 8;
    uint8_t* oblk = sO + (row >> 3) * Cfg::kGroupBytes;
    const bool stage_row = (row & 7) < box_rows;
    uint32_t oph[2] = {0, 0};
    int ob = 0;
    bool store_pending = false;  // this thread issued TMA stores from the staging
    TilePos cur = first_tile(a, n_units);
    int32_t cur_ent = cur.more ? prefetch_entry(a, cur, ts, hh) : -1;
    while (cur.more) {
      TilePos nxt = cur;
      next_tile(nxt, a, n_units);
      const int32_t nxt_ent = nxt.more ? prefetch_entry(a, nxt, ts, hh) : -1;
      const RowInfo ri = row_info(a, cur, cur_ent, ts, hh);
      if (!mbar_wait(&bar_o_full[ob], oph[ob], abort_flag, a.err, kDevTimeoutMma)) break;
      oph[ob] ^= 1;
      tc_fence_after();
      // the previous tile's stores must have read the staging
      if (store_pending) {
        bulk_wait_read<0>();
        store_pending = false;
      }
      __syncwarp();
      const uint32_t o_col = kColO + ob * 128;
#pragma unroll
      for (int rg = 0; rg < Cfg::kRegions; ++rg) {
        uint32_t o0[32], o1[32];
        tmem_ld_32x32b_x32(lane_addr + o_col + rg * 64, o0);
        tmem_ld_32x32b_x32(lane_addr + o_col + rg * 64 + 32, o1);
        tmem_wait();
        reg_fence(o0);
        reg_fence(o1);
        if (rg == Cfg::kRegions - 1) {
          tc_fence_before();
          mbar_arrive(&bar_o_empty[ob]);
        }
        if (stage_row) {
          const int line = rg * box_rows + (row & 7);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const uint32_t* src = c4 < 4 ? &o0[c4 * 8] : &o1[(c4 - 4) * 8];
            uint4 w;
            w.x = pack_half2_satfinite(__uint_as_float(src[0]), __uint_as_float(src[1]));
            w.y = pack_half2_satfinite(__uint_as_float(src[2]), __uint_as_float(src[3]));
            w.z = pack_half2_satfinite(__uint_as_float(src[4]), __uint_as_float(src[5]));
            w.w = pack_half2_satfinite(__uint_as_float(src[6]), __uint_as_float(src[7]));
            *reinterpret_cast<uint4*>(oblk + sw128_offset(line, c4)) = w;
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (ri.valid && (row & 7) == 0) {
        // this row's 8-row group: all of its column chunks in one copy
        tma_store_3d(&map_o, oblk, 0, (int32_t)(ri.slot + hh), 0);
        bulk_commit();
        store_pending = true;
      }
      ob ^= 1;
      cur = nxt;
      cur_ent = nxt_ent;
    }
    if (store_pending) bulk_wait<0>();
  } else {
    regs_increase<kRegSoftmax>();
    // ---------------- softmax: one warpgroup per tile parity ----------------
    const int grp = wg;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int ts = row >> a.log2slot;
    const int hh = row & (slot - 1);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t p_col = kColP + grp * 64;
    const uint64_t k2 = f2_pack(a.scale_log2, a.scale_log2);
    uint32_t sph = 0, pph = 0;
    int unit_seen = -1;
    float e_ln2 = 0.f, e_inv = 1.f;
    TilePos cur = first_tile(a, n_units);
    if (grp == 1) next_tile(cur, a, n_units);
    int32_t cur_ent = cur.more ? prefetch_entry(a, cur, ts, hh) : -1;
    while (cur.more) {
      TilePos nxt = cur;
      next_tile(nxt, a, n_units);
      next_tile(nxt, a, n_units);
      const int32_t nxt_ent = nxt.more ? prefetch_entry(a, nxt, ts, hh) : -1;
      const RowInfo ri = row_info(a, cur, cur_ent, ts, hh);
      if (cur.u != unit_seen) {
        unit_seen = cur.u;
        const int ev = __ldg(a.vexp + (int64_t)cur.m.j * a.G + cur.m.g);
        e_ln2 = (float)ev * kLn2;
        e_inv = __int_as_float((127 - ev) << 23);  // 2^-ev, 0 <= ev <= 126
      }
      const bool masked = __any_sync(0xffffffffu, ri.lim < kKeys - 1);

      // ---- S row -> registers; the S buffer is free again ----
      if (!mbar_wait(&bar_s_full[grp], sph, abort_flag, a.err, kDevTimeoutMma)) break;
      sph ^= 1;
      tc_fence_after();
      uint32_t s[kKeys];
      tmem_ld_32x32b_x32_at<0>(lane_addr + kColS, s);
      tmem_ld_32x32b_x32_at<32>(lane_addr + kColS + 32, s);
      tmem_ld_32x32b_x32_at<64>(lane_addr + kColS + 64, s);
      tmem_ld_32x32b_x32_at<96>(lane_addr + kColS + 96, s);
      tmem_wait();
      reg_fence(s);
      tc_fence_before();
      mbar_arrive(&bar_s_empty);

      // ---- row max (keys s <= t only, on the local block) ----
      if (masked) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (c > ri.lim) s[c] = 0xFF800000u;  // -inf: exp gives 0
      }
      float mx;
      {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kKeys; c += 8) {
          m0 = max3f(m0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          m1 = max3f(m1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
          m2 = max3f(m2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
          m3 = max3f(m3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
        }
        mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      }
      if (!ri.valid || !(mx > -INFINITY)) mx = 0.f;
      const float mxs = mx * a.scale_log2;
      const uint64_t nm2 = f2_pack(-mxs, -mxs);

      // ---- P = exp2(scale*log2e*(S - max)) in fp16 -> P buffer ----
      // the PV product of this warpgroup's previous tile must have read it
      if (!mbar_wait(&bar_p_empty[grp], pph ^ 1, abort_flag, a.err, kDevTimeoutMma)) break;
      pph ^= 1;
      tc_fence_after();
      uint64_t acc_a = f2_pack(0.f, 0.f), acc_b = acc_a;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t w[16];
#pragma unroll
        for (int x2 = 0; x2 < 16; ++x2) {
          const int col = 32 * q4 + 2 * x2;
          const uint64_t s2 = f2_pack(__uint_as_float(s[col]), __uint_as_float(s[col + 1]));
          float a0, a1;
          f2_unpack(f2_fma(s2, k2, nm2), a0, a1);
          const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
          w[x2] = pack_half2(p0, p1);
          if (x2 & 1)
            acc_b = f2_add(acc_b, f2_pack(p0, p1));
          else
            acc_a = f2_add(acc_a, f2_pack(p0, p1));
        }
        tmem_st_32x32b_x16(lane_addr + p_col + 16 * q4, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full[grp]);
      float la0, la1, lb0, lb1;
      f2_unpack(acc_a, la0, la1);
      f2_unpack(acc_b, lb0, lb1);
      const float l = (la0 + la1) + (lb0 + lb1);
      if (ri.valid) a.part_ml[ri.slot + hh] = make_float2(mx * a.scale + e_ln2, l * e_inv);
      cur = nxt;
      cur_ent = nxt_ent;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// V (bf16) -> V' = fp16(V * 2^-e) for each key block j and group g, with the
// smallest e >= 0 that brings the block's largest finite |v| to at most 511.75;
// e is written to vexp[j][g].  Block j covers rows [row0_j, row0_{j+1}) (at
// most 128; row0_j = blk_row0[j], or 128 j).  One CTA per block.  A NaN or
// infinite value records kDevValueRange and is stored as 0 or +-65504: finite,
// so that it adds nothing to the queries that do not see its key (a masked key
// meets V' with a zero probability on the tensor cores, and 0 * NaN = NaN).
__global__ void __launch_bounds__(256) v_to_fp16_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst,
                                                        int32_t* __restrict__ vexp, int64_t N,
                                                        int32_t G, int32_t d, int64_t nb,
                                                        const int32_t* __restrict__ blk_row0,
                                                        uint32_t* err) {
  __shared__ uint32_t gmax[128];  // |v| maxima as float bits (non-negative: ordered as integers)
  __shared__ float gscale[128];
  const int64_t row_chunks = (int64_t)G * d / 8;
  const int cpg = d / 8;  // 16-byte chunks per (row, group)
  for (int64_t j = blockIdx.x; j < nb; j += gridDim.x) {
    const int64_t r0 = blk_row0 ? blk_row0[j] : j * kKeys;
    int64_t r1 = j + 1 < nb ? (blk_row0 ? blk_row0[j + 1] : (j + 1) * kKeys) : N;
    r1 = min64(min64(r1, r0 + kKeys), N);
    const int64_t n = (r1 > r0 ? r1 - r0 : 0) * row_chunks;
    const uint4* s = src + r0 * row_chunks;
    uint4* o = dst + r0 * row_chunks;
    for (int g = threadIdx.x; g < G; g += blockDim.x) gmax[g] = 0u;
    __syncthreads();
    bool bad = false;
    int cur_g = -1;
    uint32_t cur_m = 0;
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
      const uint4 w = __ldg(s + c);
      const uint32_t* wi = &w.x;
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = fabsf(__uint_as_float(wi[i] << 16));
        const float hi = fabsf(__uint_as_float(wi[i] & 0xFFFF0000u));
        const bool lo_ok = lo <= 3.4e38f, hi_ok = hi <= 3.4e38f;  // false for NaN and inf
        mx = fmaxf(mx, fmaxf(lo_ok ? lo : 0.f, hi_ok ? hi : 0.f));
        bad |= !lo_ok || !hi_ok;
      }
      const int g = (int)((c / cpg) % G);
      if (g != cur_g) {
        if (cur_g >= 0) atomicMax(&gmax[cur_g], cur_m);
        cur_g = g;
        cur_m = 0u;
      }
      cur_m = max(cur_m, __float_as_uint(mx));
    }
    if (cur_g >= 0) atomicMax(&gmax[cur_g], cur_m);
    if (bad) record_error(err, kDevValueRange);
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
      float m = __uint_as_float(gmax[g]);
      int e = 0;
      while (e < 126 && m > kVMax) {  // exact halvings
        m *= 0.5f;
        ++e;
      }
      vexp[j * G + g] = e;
      gscale[g] = __int_as_float((127 - e) << 23);
    }
    __syncthreads();
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
      const uint4 w = __ldg(s + c);
      const float sc = gscale[(c / cpg) % G];
      uint4 out;
      const uint32_t* wi = &w.x;
      uint32_t* oi = &out.x;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float lo = __uint_as_float(wi[i] << 16), hi = __uint_as_float(wi[i] & 0xFFFF0000u);
        lo = lo == lo ? lo : 0.f;  // NaN -> 0; infinities saturate below
        hi = hi == hi ? hi : 0.f;
        oi[i] = pack_half2_satfinite(lo * sc, hi * sc);
      }
      o[c] = out;
    }
    __syncthreads();
  }
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
  a.vexp = p.vexp;
  a.part_o = p.part_o;
  a.part_ml = p.part_ml;
  a.err = p.err;
  auto kern = main_kernel<D>;
  // The warpgroups' register budgets are carved out of the registers the CTA is
  // launched with; the kernel must be compiled to exactly that many a thread,
  // or the budget increase would wait forever.
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  static_assert(2 * 128 * kRegSoftmax + 128 * kRegEpi + 128 * kRegProd ==
                    (uint32_t)kThreads * kLaunchRegs,
                "register split must add up to the launch budget");
  if (attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<p.grid, kThreads, Cfg::kSmem, s>>>(mq, mk, mv, mo, a);
  return cudaGetLastError();
}

}  // namespace

int main_tile_tokens(int H, int G) {
  const int HG = H / G;
  return kRows / (HG < 8 ? 8 : HG);
}

cudaError_t launch_v_to_fp16(const void* src, void* dst, int32_t* vexp, int64_t N, int32_t G,
                             int32_t d, int64_t nb, const int32_t* blk_row0, uint32_t* err,
                             int sms, cudaStream_t s) {
  if ((d % 8) != 0 || G > 128 || ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15))
    return cudaErrorInvalidValue;
  if (nb == 0) return cudaSuccess;
  const int64_t cap = (int64_t)sms * 8;
  const unsigned grid = (unsigned)(nb < cap ? nb : cap);
  v_to_fp16_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                        vexp, N, G, d, nb, blk_row0, err);
  return cudaGetLastError();
}

cudaError_t launch_main(const MainLaunch& p, cudaStream_t s) {
  if (p.d == 128) return launch_main_impl<128>(p, s);
  return launch_main_impl<64>(p, s);
}

}  // namespace msa
