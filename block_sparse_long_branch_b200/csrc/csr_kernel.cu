// csr_kernel.cu -- inversion of the block selection into per-(group, key block)
// query lists: the schedule of the KV-block-outer Main Branch (tnkblog MiniMax
// M3 / MSA post, section "MSA の実装": key blocks are the outer loop and the
// queries that hit a block are gathered; CSDN M3 write-up, section "MiniMax
// Sparse Attention（MSA）").
//
// Deterministic stable counting sort on the key (g, j), in t order, over
// parts of R query rows (R grows with nb so that the (part, list) count table
// stays at most half the size of the ids):
//   1. count   : per part and set of groups (all whose bins fit shared
//                memory), a histogram over the key blocks -> cnt[part][g*nb +
//                j] (coalesced) and the list totals (atomics); the last CTA
//                scans the totals into row_ptr and cuts the lists into Main
//                Branch work units
//   2. colscan : the table scanned in (list, part) order, in place, from
//                row_ptr: where each part's hits on each list start
//   3. scatter : one warp per (part, set of groups) loads its part's start
//                offsets, then walks the rows in t order, one row of every
//                group of the set per step; the hits of one step never share
//                a key, so each advances its key's offset by one
// Integer work: each id is read twice and each entry written once.  At the
// sizes measured it is bound by latency and by the scatter's stores (one
// row step writes 32 entries of 32 different lists), not by HBM bandwidth.
//
// For a batch of packed sequences the ids are local to each sequence; the key
// is row_base[row] + id, a global block number.  The plan kernels at the end
// of the anonymous namespace build row_base and the other tables of that
// schedule (the Index Branch's tiles, each block's first K/V row) on the
// device.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kBinSlice = 16384;  // shared-memory bins per pass (64 KiB)
constexpr int kCountThreads = 512;
constexpr int kScanWarps = 32;    // column scan: 32 warps over the parts of 32 lists
constexpr int kKeyRows = 64;      // rows of keys a scatter warp stages at a time

// Packed sequences: ids are local to each sequence and row_base[row] (the
// global number of the row's sequence's first block) turns them into the list
// key; without it the id is the key.
__device__ __forceinline__ int32_t list_key(const int32_t* row_base, int64_t row, int32_t j) {
  return (row_base && j >= 0) ? __ldg(row_base + row) + j : j;
}

__device__ __forceinline__ int32_t warp_incl_scan(int32_t x) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) >= o) x += y;
  }
  return x;
}

struct ListTail {
  int32_t* row_ptr;    // [n_lists + 1]
  int32_t per_unit;    // entries per Main Branch work unit
  int32_t* unit_ptr;   // optional: [n_lists + 1] exclusive prefix of the unit counts
  int4* unit_desc;     // {g, j, first entry, end entry} of every unit
};

// row_ptr = the exclusive prefix of the per-list totals and, optionally, the
// Main Branch work units (each list cut into runs of at most per_unit
// entries).  One CTA: each thread takes a contiguous range of lists, the CTA
// scans the per-thread sums, and each thread fills its range.
__device__ void list_prefix(const int32_t* tot, int64_t n_lists, int64_t nb, const ListTail& t) {
  __shared__ int32_t wt_e[32], wt_u[32];
  const int nt = blockDim.x, tid = threadIdx.x, w = tid >> 5, l = tid & 31, nw = nt >> 5;
  const int64_t per = (n_lists + nt - 1) / nt;
  const int64_t x0 = min64((int64_t)tid * per, n_lists), x1 = min64(x0 + per, n_lists);
  const int32_t pu = t.per_unit;
  int32_t se = 0, su = 0;
  for (int64_t x = x0; x < x1; ++x) {
    const int32_t c = __ldcg(tot + x);
    se += c;
    su += (c + pu - 1) / pu;
  }
  const int32_t ie = warp_incl_scan(se), iu = warp_incl_scan(su);
  if (l == 31) wt_e[w] = ie, wt_u[w] = iu;
  __syncthreads();
  if (w == 0) {
    const int32_t te = l < nw ? wt_e[l] : 0, tu = l < nw ? wt_u[l] : 0;
    const int32_t je = warp_incl_scan(te), ju = warp_incl_scan(tu);
    if (l < nw) wt_e[l] = je - te, wt_u[l] = ju - tu;
  }
  __syncthreads();
  int32_t e = wt_e[w] + ie - se, u = wt_u[w] + iu - su;
  for (int64_t x = x0; x < x1; ++x) {
    const int32_t c = __ldcg(tot + x);
    t.row_ptr[x] = e;
    if (t.unit_ptr) {
      t.unit_ptr[x] = u;
      const int g = (int)(x / nb), j = (int)(x - (int64_t)g * nb);
      for (int32_t e0 = e; e0 < e + c; e0 += pu, ++u)
        t.unit_desc[u] = make_int4(g, j, e0, min(e + c, e0 + pu));
    }
    e += c;
  }
  if (tid == nt - 1) {  // its range is the last (possibly empty): e and u are the totals
    t.row_ptr[n_lists] = e;
    if (t.unit_ptr) t.unit_ptr[n_lists] = u;
  }
}

// 1. Per part of R query rows and per set of gpc groups (all of them when
// their gpc * nb bins fit kBinSlice): a shared-memory histogram of the part's
// hits over the set's keys, written as cnt[part][g*nb + j] (contiguous per
// part) and added to the list totals tot[g*nb + j].  Thread t owns column
// t % (gpc * top_k) of every row it visits (one row's ids of the set are
// contiguous).  The last CTA to finish (a ticket) computes row_ptr and the
// work units from the totals.
__global__ void __launch_bounds__(kCountThreads)
    csr_count_kernel(const int32_t* __restrict__ ids, int64_t rows, int32_t G, int32_t top_k,
                     int64_t nb, int32_t R, int32_t gpc, int32_t* __restrict__ cnt,
                     int32_t* __restrict__ tot, int32_t* __restrict__ ticket,
                     const int32_t* __restrict__ row_base, uint32_t* err, ListTail tail) {
  extern __shared__ int32_t bins[];  // [gpc][width]
  __shared__ int last;
  const int part = blockIdx.x, g0 = blockIdx.y * gpc;
  const int ng = min(gpc, G - g0);
  const int64_t K = (int64_t)G * nb;
  const int64_t r0 = (int64_t)part * R;
  const int nrows = (int)(min64(rows, r0 + R) - r0);
  const int per_row = ng * top_k;
  const int col = threadIdx.x % per_row, rstep = blockDim.x / per_row;
  const int rsub = threadIdx.x / per_row;
  const int gk = col / top_k;  // group of this column within the set
  const bool on = rsub < rstep;
  int32_t* crow = cnt + (int64_t)part * K + (int64_t)g0 * nb;
  const int32_t* idrow = ids + (r0 * G + g0) * top_k + col;
  const int64_t id_pitch = (int64_t)G * top_k;
  const int slice_w = kBinSlice / ng;  // one pass whenever ng > 1 (gpc * nb <= kBinSlice)
  for (int64_t s0 = 0; s0 < nb; s0 += slice_w) {
    const int width = (int)min64(slice_w, nb - s0);
    for (int i = threadIdx.x; i < ng * width; i += blockDim.x) bins[i] = 0;
    __syncthreads();
    if (on) {
      constexpr int kB = 16;
      for (int rr0 = rsub; rr0 < nrows; rr0 += rstep * kB) {
        int32_t v[kB];
#pragma unroll
        for (int q = 0; q < kB; ++q) {
          const int rr = rr0 + q * rstep;
          v[q] = rr < nrows ? __ldg(idrow + rr * id_pitch) : -1;
        }
#pragma unroll
        for (int q = 0; q < kB; ++q) {
          const int rr = rr0 + q * rstep;
          if (rr >= nrows) continue;
          const int32_t j = list_key(row_base, r0 + rr, v[q]);
          if (j < -1 || j >= nb) {
            if (s0 == 0) record_error(err, kDevBadIndex);
            continue;
          }
          if (j >= s0 && j < s0 + width) atomicAdd(&bins[gk * width + (int)(j - s0)], 1);
        }
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ng * width; i += blockDim.x) {
      const int gg = i / width, x = i - gg * width;
      const int32_t c = bins[i];
      crow[(int64_t)gg * nb + s0 + x] = c;
      if (c) atomicAdd(tot + (int64_t)(g0 + gg) * nb + s0 + x, c);
    }
    __syncthreads();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(ticket, 1) == (int)(gridDim.x * gridDim.y) - 1;
    __threadfence();
  }
  __syncthreads();
  if (!last) return;
  list_prefix(tot, K, nb, tail);
}

// 2. The count table in (list, part) order, scanned in place: cnt[part][x]
// becomes row_ptr[x] + the hits of list x in earlier parts, where this part's
// hits on x start.  One CTA per 32 lists: lane = list (coalesced rows of the
// table), warp w walks a contiguous run of parts.
__global__ void __launch_bounds__(kScanWarps * 32)
    csr_colscan_kernel(int32_t* __restrict__ cnt, int64_t K, int64_t nparts,
                       const int32_t* __restrict__ row_ptr) {
  __shared__ int32_t part_sum[kScanWarps][33];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int64_t x = (int64_t)blockIdx.x * 32 + l;
  const int64_t per = (nparts + kScanWarps - 1) / kScanWarps;
  const int64_t p0 = min64((int64_t)w * per, nparts), p1 = min64(p0 + per, nparts);
  constexpr int kB = 8;  // parts loaded at once
  int32_t s = 0;
  if (x < K) {
    for (int64_t pb = p0; pb < p1; pb += kB) {
      int32_t c[kB];
#pragma unroll
      for (int q = 0; q < kB; ++q) c[q] = pb + q < p1 ? cnt[(pb + q) * K + x] : 0;
#pragma unroll
      for (int q = 0; q < kB; ++q) s += c[q];
    }
  }
  part_sum[w][l] = s;
  __syncthreads();
  if (x >= K) return;
  int32_t base = __ldg(row_ptr + x);
  for (int v = 0; v < w; ++v) base += part_sum[v][l];
  for (int64_t pb = p0; pb < p1; pb += kB) {
    int32_t c[kB];
#pragma unroll
    for (int q = 0; q < kB; ++q) c[q] = pb + q < p1 ? cnt[(pb + q) * K + x] : 0;
#pragma unroll
    for (int q = 0; q < kB; ++q)
      if (pb + q < p1) {
        cnt[(pb + q) * K + x] = base;
        base += c[q];
      }
  }
}

// 3. One warp per (part, group set): the set is gpw = 32 / top_k groups (one
// when top_k > 16).  A row's ids are distinct within a group and different
// groups key different lists, so the gpw * top_k hits of one row never share
// a key: each lane reads its key's next free entry, writes there and advances
// it, with no ranking among the lanes; rows are walked in order, so every
// list stays in t order.  The part's start offsets of every key of the set's
// groups (the slice of nb keys given by s0) are loaded once, contiguously;
// keys are staged kKeyRows rows at a time with independent loads.
__global__ void __launch_bounds__(32)
    csr_scatter_kernel(const int32_t* __restrict__ ids, int64_t row_begin, int64_t rows,
                       int32_t G, int32_t top_k, int64_t nb, int32_t R, int32_t bins, int32_t gpw,
                       const int32_t* __restrict__ start, const int32_t* __restrict__ row_base,
                       int32_t* __restrict__ entries) {
  extern __shared__ int32_t sm[];
  int32_t* run = sm;                // [gpw][bins]: next free entry of each key of the slice
  int32_t* keys = sm + gpw * bins;  // [kKeyRows][gpw * top_k]: keys of the staged rows
  const int part = blockIdx.x, g0 = blockIdx.y * gpw;
  const int lane = threadIdx.x;
  const int64_t K = (int64_t)G * nb;
  const int64_t r0 = (int64_t)part * R;
  const int nrows = (int)(min64(rows, r0 + R) - r0);
  const int per_row = gpw * top_k;  // hits of one row handled by one lane each (<= 32)
  const int ngrp = min(gpw, G - g0);
  const bool active = lane < per_row;
  const int gi = active ? lane / top_k : 0;
  const int r = active ? lane - gi * top_k : 0;
  const int32_t* srow = start + (int64_t)part * K + (int64_t)g0 * nb;
  const int32_t* idcol = ids + (r0 * G + g0) * top_k + lane;  // this lane's column
  const int64_t id_pitch = (int64_t)G * top_k;
  const bool col_on = lane < ngrp * top_k;
  constexpr int kB = 8;  // loads in flight per lane
  for (int64_t s0 = 0; s0 < nb; s0 += kBinSlice) {
    const int width = (int)min64(kBinSlice, nb - s0);
    for (int gg = 0; gg < ngrp; ++gg)
      for (int x0 = lane; x0 < width; x0 += 32 * kB) {
        int32_t v[kB];
#pragma unroll
        for (int q = 0; q < kB; ++q)
          v[q] = x0 + 32 * q < width ? __ldg(srow + (int64_t)gg * nb + s0 + x0 + 32 * q) : 0;
#pragma unroll
        for (int q = 0; q < kB; ++q)
          if (x0 + 32 * q < width) run[gg * bins + x0 + 32 * q] = v[q];
      }
    for (int rb = 0; rb < nrows; rb += kKeyRows) {
      const int nr = min(kKeyRows, nrows - rb);
      __syncwarp();
      if (active) {
        for (int rr0 = 0; rr0 < nr; rr0 += kB) {
          int32_t v[kB];
#pragma unroll
          for (int q = 0; q < kB; ++q)
            v[q] = (col_on && rr0 + q < nr) ? __ldg(idcol + (int64_t)(rb + rr0 + q) * id_pitch) : -1;
#pragma unroll
          for (int q = 0; q < kB; ++q)
            if (rr0 + q < nr)
              keys[(rr0 + q) * per_row + lane] = list_key(row_base, r0 + rb + rr0 + q, v[q]);
        }
      }
      __syncwarp();
      for (int rr = 0; rr < nr; ++rr) {
        const int32_t j = active ? keys[rr * per_row + lane] : -1;
        if (j >= s0 && j < s0 + width) {
          int32_t* slot = run + gi * bins + (int)(j - s0);
          const int32_t pos = *slot;
          entries[pos] = (int32_t)(((row_begin + r0 + rb + rr) << 5) | r);
          *slot = pos + 1;
        }
        __syncwarp();
      }
    }
  }
}

// ---- schedule of a batch of packed sequences --------------------------------
// One CTA: blocks per sequence, their exclusive prefix (blk_base), and the
// first unit of every local block level b when the units are ordered by b
// descending (the longest rows of the Index Branch first), then by sequence.
__global__ void __launch_bounds__(1024) varlen_levels_kernel(const VarlenOffsets off,
                                                             int32_t max_nb,
                                                             int32_t* __restrict__ nbs,
                                                             int32_t* __restrict__ blk_base,
                                                             int32_t* __restrict__ level) {
  __shared__ int32_t sh_nb[kVarlenMaxSeqs];
  __shared__ int32_t sh_scan[1024];
  const int tid = threadIdx.x, B = off.B;
  for (int b = tid; b < B; b += 1024) {
    const int32_t n = (int32_t)((off.cu[b + 1] - off.cu[b] + 127) / 128);
    sh_nb[b] = n;
    nbs[b] = n;
  }
  __syncthreads();
  if (tid == 0) {  // B <= 1024: a serial prefix is cheap next to the kernels it plans
    int32_t acc = 0;
    for (int b = 0; b < B; ++b) {
      blk_base[b] = acc;
      acc += sh_nb[b];
    }
    blk_base[B] = acc;
  }
  // units of level b: the sequences with more than b blocks; levels from the
  // top down, scanned in chunks of 1024 with a carry
  int32_t carry = 0;
  for (int32_t c0 = 0; c0 < max_nb; c0 += 1024) {
    const int32_t b = max_nb - 1 - (c0 + tid);  // descending
    int32_t cnt = 0;
    if (b >= 0)
      for (int x = 0; x < B; ++x) cnt += sh_nb[x] > b;
    sh_scan[tid] = cnt;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan
      const int32_t v = tid >= o ? sh_scan[tid - o] : 0;
      __syncthreads();
      sh_scan[tid] += v;
      __syncthreads();
    }
    if (b >= 0) level[b] = carry + sh_scan[tid] - cnt;
    carry += sh_scan[1023];
    __syncthreads();
  }
  if (tid == 0) level[max_nb] = carry;
}

// largest s < B with key[s] <= x (key non-decreasing): the owner of x
template <typename T>
__device__ __forceinline__ int owner_of(const T* key, int B, int64_t x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)key[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Grid-stride: the unit table and first K/V row of every global block, and
// the block base of every packed row.
__global__ void __launch_bounds__(256) varlen_tables_kernel(const VarlenOffsets off, int32_t NB,
                                                            int64_t N,
                                                            const int32_t* __restrict__ nbs,
                                                            const int32_t* __restrict__ blk_base,
                                                            const int32_t* __restrict__ level,
                                                            int4* __restrict__ units,
                                                            int32_t* __restrict__ blk_row0,
                                                            int32_t* __restrict__ row_base) {
  const int B = off.B;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t J = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; J < NB; J += stride) {
    const int s = owner_of(blk_base, B, J);
    const int32_t b = (int32_t)(J - blk_base[s]);
    int32_t rank = 0;  // earlier sequences on the same level
    for (int x = 0; x < s; ++x) rank += __ldg(nbs + x) > b;
    const int64_t r0 = off.cu[s] + (int64_t)b * 128;
    units[level[b] + rank] = make_int4((int32_t)r0, (int32_t)off.cu[s], b, (int32_t)off.cu[s + 1]);
    blk_row0[J] = (int32_t)r0;
  }
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < N; t += stride)
    row_base[t] = __ldg(blk_base + owner_of(off.cu, B, t));
}

}  // namespace

// Query rows per part: the (part, list) count table stays at most half the
// size of the ids (nb / R <= top_k / 2 for top_k = 16), and parts stay short
// enough for many scatter warps.
static int64_t part_rows(int64_t nb) {
  int64_t R = 64;
  while (R < 2048 && nb > 8 * R) R *= 2;
  return R;
}

size_t csr_scratch_bytes(int64_t rows, int32_t G, int32_t top_k, int64_t nb) {
  (void)top_k;
  const int64_t nparts = (rows + part_rows(nb) - 1) / part_rows(nb);
  const int64_t K = (int64_t)G * nb;
  const size_t elems = (size_t)(nparts * K) + (size_t)K + 1;  // table, totals, ticket
  return (elems * sizeof(int32_t) + 255) & ~(size_t)255;
}

cudaError_t launch_csr(const CsrLaunch& p, cudaStream_t s, int* launches) {
  const int64_t R = part_rows(p.nb);
  const int64_t nparts = (p.rows + R - 1) / R;
  const int64_t K = (int64_t)p.G * p.nb;
  int32_t* cnt = static_cast<int32_t*>(p.scratch);
  int32_t* tot = cnt + nparts * K;
  int32_t* ticket = tot + K;
  cudaError_t e;
  if (nparts == 0) {
    if ((e = cudaMemsetAsync(p.row_ptr, 0, (size_t)(K + 1) * sizeof(int32_t), s)) != cudaSuccess)
      return e;
    if (p.unit_ptr)
      return cudaMemsetAsync(p.unit_ptr, 0, (size_t)(K + 1) * sizeof(int32_t), s);
    return cudaSuccess;
  }
  if ((e = cudaMemsetAsync(tot, 0, (size_t)(K + 1) * sizeof(int32_t), s)) != cudaSuccess) return e;
  const int bins = (int)(p.nb < kBinSlice ? p.nb : kBinSlice);
  const size_t bin_bytes = (size_t)bins * sizeof(int32_t);
  // groups per count CTA: all whose bins fit one pass of kBinSlice, and whose
  // ids of one row fit the CTA's threads
  const int gpc = (int)min64(min64(p.G, p.nb <= kBinSlice ? kBinSlice / p.nb : 1),
                             kCountThreads / p.top_k);
  const size_t count_bytes = (size_t)min64((int64_t)gpc * p.nb, kBinSlice) * sizeof(int32_t);
  // groups per scatter warp: one row's hits of gpw groups fill at most 32 lanes,
  // and their offsets and staged keys fit 200 KiB of shared memory
  int gpw = p.top_k <= 16 ? (int)min64(32 / p.top_k, p.G) : 1;
  auto scatter_smem = [&](int w) {
    return (size_t)w * bin_bytes + (size_t)kKeyRows * w * p.top_k * sizeof(int32_t);
  };
  while (gpw > 1 && scatter_smem(gpw) > 200 * 1024) --gpw;
  const size_t scatter_bytes = scatter_smem(gpw);
  if (count_bytes > 48 * 1024 &&
      (e = cudaFuncSetAttribute(csr_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)count_bytes)) != cudaSuccess)
    return e;
  if (scatter_bytes > 48 * 1024 &&
      (e = cudaFuncSetAttribute(csr_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)scatter_bytes)) != cudaSuccess)
    return e;
  ListTail tail;
  tail.row_ptr = p.row_ptr;
  tail.per_unit = p.unit_ptr ? p.tile_tokens * p.unit_tiles : 1;
  tail.unit_ptr = p.unit_ptr;
  tail.unit_desc = p.unit_desc;
  csr_count_kernel<<<dim3((unsigned)nparts, (unsigned)((p.G + gpc - 1) / gpc)), kCountThreads,
                     count_bytes, s>>>(p.ids, p.rows, p.G, p.top_k, p.nb, (int32_t)R, gpc, cnt,
                                       tot, ticket, p.row_base, p.err, tail);
  ++*launches;
  csr_colscan_kernel<<<(unsigned)((K + 31) / 32), kScanWarps * 32, 0, s>>>(cnt, K, nparts,
                                                                            p.row_ptr);
  ++*launches;
  dim3 sgrid((unsigned)nparts, (unsigned)((p.G + gpw - 1) / gpw));
  csr_scatter_kernel<<<sgrid, 32, scatter_bytes, s>>>(p.ids, p.row_begin, p.rows, p.G, p.top_k,
                                                      p.nb, (int32_t)R, bins, gpw, cnt,
                                                      p.row_base, p.entries);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_varlen_plan(const VarlenOffsets& off, const VarlenPlan& p, cudaStream_t s,
                               int* launches) {
  if (off.B < 1 || off.B > kVarlenMaxSeqs || p.max_nb < 1) return cudaErrorInvalidValue;
  varlen_levels_kernel<<<1, 1024, 0, s>>>(off, p.max_nb, p.nbs, p.blk_base, p.level);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t work = p.N > p.NB ? p.N : p.NB;
  const unsigned grid = (unsigned)((work + 255) / 256 < 1184 ? (work + 255) / 256 : 1184);
  varlen_tables_kernel<<<grid, 256, 0, s>>>(off, p.NB, p.N, p.nbs, p.blk_base, p.level, p.units,
                                             p.blk_row0, p.row_base);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace msa
