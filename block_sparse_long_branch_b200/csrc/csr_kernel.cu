// csr_kernel.cu -- inversion of the block selection into per-(group, key block)
// query lists: the schedule of the KV-block-outer Main Branch (tnkblog MiniMax
// M3 / MSA post, section "MSA の実装": key blocks are the outer loop and the
// queries that hit a block are gathered; CSDN M3 write-up, section "MiniMax
// Sparse Attention（MSA）").
//
// Deterministic stable counting sort on the key (g, j), in t order:
//   1. hist    : per tile of kTileTok query rows and per group, a shared-memory
//                histogram over the key blocks -> cnt[(g*nb + j)*ntiles + tile]
//   2. scan    : exclusive prefix over that table (flattened g, j, tile), so
//                the entry gives where tile `tile`'s hits on (g, j) start
//   3. row_ptr : row_ptr[g*nb+j] = scanned[(g*nb+j)*ntiles]
//   4. scatter : one warp per (tile, set of groups) copies its tile's keys and
//                their start offsets into shared memory, then walks the rows
//                in t order, one row of every group of the set per step; the
//                hits of one step never share a key, so each advances its
//                key's offset by one
//   5. units   : one CTA: per list, the number of Main Branch work units, their
//                exclusive prefix and the unit table
// HBM-bound integer work: each id is read twice, each entry written once.
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

constexpr int kTileTok = 256;      // query rows per histogram tile
constexpr int kBinSlice = 16384;   // shared-memory bins per pass (64 KiB)
constexpr int kScanThreads = 1024;
constexpr int kScanPer = 4;
constexpr int kScanChunk = kScanThreads * kScanPer;

// Packed sequences: ids are local to each sequence and row_base[row] (the
// global number of the row's sequence's first block) turns them into the list
// key; without it the id is the key.
__device__ __forceinline__ int32_t list_key(const int32_t* row_base, int64_t row, int32_t j) {
  return (row_base && j >= 0) ? __ldg(row_base + row) + j : j;
}

__global__ void __launch_bounds__(256) csr_hist_kernel(const int32_t* __restrict__ ids, int64_t rows,
                                                       int32_t G, int32_t top_k, int64_t nb,
                                                       int32_t ntiles, int32_t* __restrict__ cnt,
                                                       const int32_t* __restrict__ row_base,
                                                       uint32_t* err) {
  extern __shared__ int32_t bins[];
  const int tile = blockIdx.x, g = blockIdx.y;
  const int64_t r0 = (int64_t)tile * kTileTok;
  const int64_t r1 = min(rows, r0 + kTileTok);
  const int64_t n_el = (r1 - r0) * top_k;
  for (int64_t s0 = 0; s0 < nb; s0 += kBinSlice) {
    const int width = (int)min64(kBinSlice, nb - s0);
    for (int i = threadIdx.x; i < width; i += blockDim.x) bins[i] = 0;
    __syncthreads();
    for (int64_t e = threadIdx.x; e < n_el; e += blockDim.x) {
      const int64_t row = r0 + e / top_k;
      const int r = (int)(e % top_k);
      const int32_t j = list_key(row_base, row, ids[(row * G + g) * top_k + r]);
      if (j < -1 || j >= nb) {
        if (s0 == 0) record_error(err, kDevBadIndex);
        continue;
      }
      if (j >= s0 && j < s0 + width) atomicAdd(&bins[j - s0], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < width; i += blockDim.x)
      cnt[((int64_t)g * nb + s0 + i) * ntiles + tile] = bins[i];
    __syncthreads();
  }
}

// ---- exclusive scan (int32), chunk of 4096 per CTA --------------------------
__device__ __forceinline__ int32_t warp_incl_scan(int32_t x) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) >= o) x += y;
  }
  return x;
}

__global__ void __launch_bounds__(kScanThreads) scan_chunks_kernel(int32_t* __restrict__ data,
                                                                   int64_t n,
                                                                   int32_t* __restrict__ sums) {
  __shared__ int32_t warp_tot[32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanPer;
  int32_t v[kScanPer];
  int32_t local = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    v[i] = (base + i < n) ? data[base + i] : 0;
    local += v[i];
  }
  const int32_t incl = warp_incl_scan(local);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int32_t t = warp_tot[l];
    const int32_t ti = warp_incl_scan(t);
    warp_tot[l] = ti - t;
    if (l == 31 && sums) sums[blockIdx.x] = ti;
  }
  __syncthreads();
  int32_t run = warp_tot[w] + incl - local;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    if (base + i < n) data[base + i] = run;
    run += v[i];
  }
}

__global__ void add_offsets_kernel(int32_t* __restrict__ data, int64_t n,
                                   const int32_t* __restrict__ offs) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) data[i] += offs[i / kScanChunk];
}

size_t scan_scratch_elems(int64_t n) {
  size_t s = 0;
  while (n > kScanChunk) {
    n = (n + kScanChunk - 1) / kScanChunk;
    s += (size_t)n;
  }
  return s + 1;
}

// In-place exclusive scan of data[0..n); `tmp` holds scan_scratch_elems(n).
cudaError_t exclusive_scan(int32_t* data, int64_t n, int32_t* tmp, cudaStream_t s, int* launches) {
  if (n <= 0) return cudaSuccess;
  const int64_t nch = (n + kScanChunk - 1) / kScanChunk;
  scan_chunks_kernel<<<(unsigned)nch, kScanThreads, 0, s>>>(data, n, nch > 1 ? tmp : nullptr);
  ++*launches;
  if (nch > 1) {
    cudaError_t e = exclusive_scan(tmp, nch, tmp + nch, s, launches);
    if (e != cudaSuccess) return e;
    add_offsets_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(data, n, tmp);
    ++*launches;
  }
  return cudaGetLastError();
}

// row_ptr[x] = scanned[x * ntiles]; the end, row_ptr[n_lists], is the last
// exclusive value plus the last count (saved before the in-place scan)
__global__ void csr_rowptr_kernel(const int32_t* __restrict__ scanned, int64_t n_lists,
                                  int32_t ntiles, const int32_t* __restrict__ last_count,
                                  int32_t* __restrict__ row_ptr) {
  const int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x < n_lists) row_ptr[x] = scanned[x * ntiles];
  if (x == n_lists) row_ptr[x] = scanned[n_lists * ntiles - 1] + *last_count;
}

// One warp per (tile, group set): the set is GPW = 32 / top_k groups (one when
// top_k > 16).  A row's ids are distinct within a group and different groups
// key different lists, so the GPW * top_k hits of one row never share a key:
// each lane reads its key's next free entry, writes there and advances it,
// with no ranking among the lanes; rows are walked in order, so every list
// stays in t order.  The tile's keys are first copied to shared memory with
// independent loads, and so are the start offsets of every key of the set's
// groups (the slice of nb keys given by s0).
__global__ void __launch_bounds__(32) csr_scatter_kernel(const int32_t* __restrict__ ids,
                                                         int64_t row_begin, int64_t rows,
                                                         int32_t G, int32_t top_k, int64_t nb,
                                                         int32_t ntiles, int32_t bins,
                                                         int32_t gpw,
                                                         const int32_t* __restrict__ scanned,
                                                         const int32_t* __restrict__ row_base,
                                                         int32_t* __restrict__ entries) {
  extern __shared__ int32_t sm[];
  int32_t* run = sm;                 // [gpw][bins]: next free entry of each key of the slice
  int32_t* keys = sm + gpw * bins;   // [kTileTok][gpw * top_k]: the tile's keys, by row
  const int tile = blockIdx.x, g0 = blockIdx.y * gpw;
  const int lane = threadIdx.x;
  const int64_t r0 = (int64_t)tile * kTileTok;
  const int64_t r1 = min(rows, r0 + kTileTok);
  const int nrows = (int)(r1 - r0);
  const int per_row = gpw * top_k;  // hits of one row handled by one lane each (<= 32)
  const int ngrp = min(gpw, G - g0);
  for (int e = lane; e < nrows * per_row; e += 32) {
    const int rr = e / per_row, c = e - rr * per_row;
    const int gi = c / top_k, r = c - gi * top_k;
    const int64_t row = r0 + rr;
    keys[e] = gi < ngrp ? list_key(row_base, row, __ldg(ids + (row * G + g0 + gi) * top_k + r))
                        : -1;
  }
  const bool active = lane < per_row;
  const int gi = active ? lane / top_k : 0;
  const int r = active ? lane - gi * top_k : 0;
  for (int64_t s0 = 0; s0 < nb; s0 += kBinSlice) {
    const int width = (int)min64(kBinSlice, nb - s0);
    // where this tile's hits on each key of the slice start, per group of the set
    for (int i = lane; i < ngrp * width; i += 32) {
      const int gg = i / width, x = i - gg * width;
      run[gg * bins + x] = __ldg(scanned + ((int64_t)(g0 + gg) * nb + s0 + x) * ntiles + tile);
    }
    __syncwarp();
    for (int rr = 0; rr < nrows; ++rr) {
      const int32_t j = active ? keys[rr * per_row + lane] : -1;
      if (j >= s0 && j < s0 + width) {
        int32_t* slot = run + gi * bins + (int)(j - s0);
        const int32_t pos = *slot;
        entries[pos] = (int32_t)(((row_begin + r0 + rr) << 5) | r);
        *slot = pos + 1;
      }
      __syncwarp();
    }
  }
}

// Work units of the Main Branch: list x = g*nb + j is cut into runs of at
// most `per_unit` entries; unit_ptr[x] is the exclusive prefix of the unit
// counts (unit_ptr[n_lists] the total) and unit u gets {g, j, first entry,
// end entry}.  One CTA: each thread counts a contiguous range of lists, the
// CTA scans the per-thread sums, and each thread fills its range.
constexpr int kUnitThreads = 1024;
__global__ void __launch_bounds__(kUnitThreads)
    units_kernel(const int32_t* __restrict__ row_ptr, int64_t n_lists, int64_t nb,
                 int32_t per_unit, int32_t* __restrict__ unit_ptr, int4* __restrict__ unit_desc) {
  __shared__ int32_t warp_tot[32];
  const int64_t per = (n_lists + kUnitThreads - 1) / kUnitThreads;
  const int64_t x0 = min64((int64_t)threadIdx.x * per, n_lists);
  const int64_t x1 = min64(x0 + per, n_lists);
  int32_t mine = 0;
  for (int64_t x = x0; x < x1; ++x) mine += (row_ptr[x + 1] - row_ptr[x] + per_unit - 1) / per_unit;
  const int32_t incl = warp_incl_scan(mine);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int32_t t = warp_tot[l];
    warp_tot[l] = warp_incl_scan(t) - t;
  }
  __syncthreads();
  int32_t u = warp_tot[w] + incl - mine;
  for (int64_t x = x0; x < x1; ++x) {
    unit_ptr[x] = u;
    const int32_t beg = row_ptr[x], end = row_ptr[x + 1];
    const int g = (int)(x / nb), j = (int)(x - (int64_t)g * nb);
    for (int32_t e0 = beg; e0 < end; e0 += per_unit, ++u)
      unit_desc[u] = make_int4(g, j, e0, min(end, e0 + per_unit));
  }
  if (threadIdx.x == kUnitThreads - 1) unit_ptr[n_lists] = u;
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

size_t csr_scratch_bytes(int64_t rows, int32_t G, int32_t top_k, int64_t nb) {
  (void)top_k;
  const int64_t ntiles = (rows + kTileTok - 1) / kTileTok;
  const int64_t table = (int64_t)G * nb * ntiles;
  const int64_t lists = (int64_t)G * nb + 1;
  size_t elems = (size_t)table + scan_scratch_elems(table) + 2 + scan_scratch_elems(lists) + 2;
  return (elems * sizeof(int32_t) + 255) & ~(size_t)255;
}

cudaError_t launch_csr(const CsrLaunch& p, cudaStream_t s, int* launches) {
  const int64_t ntiles = (p.rows + kTileTok - 1) / kTileTok;
  const int64_t n_lists = (int64_t)p.G * p.nb;
  const int64_t table = n_lists * ntiles;
  int32_t* cnt = static_cast<int32_t*>(p.scratch);
  int32_t* scan_tmp = cnt + table;
  int32_t* last = scan_tmp + scan_scratch_elems(table) + 1;  // the table's last count
  const int bins = (int)(p.nb < kBinSlice ? p.nb : kBinSlice);
  cudaError_t e;

  dim3 grid((unsigned)ntiles, (unsigned)p.G);
  const size_t bin_bytes = (size_t)bins * sizeof(int32_t);
  // groups per scatter warp: one row's hits of gpw groups fill at most 32 lanes,
  // and their offsets and keys fit 200 KiB of shared memory
  int gpw = p.top_k <= 16 ? (int)min64(32 / p.top_k, p.G) : 1;
  auto scatter_smem = [&](int w) {
    return (size_t)w * bin_bytes + (size_t)kTileTok * w * p.top_k * sizeof(int32_t);
  };
  while (gpw > 1 && scatter_smem(gpw) > 200 * 1024) --gpw;
  const size_t scatter_bytes = scatter_smem(gpw);
  if (bin_bytes > 48 * 1024 &&
      (e = cudaFuncSetAttribute(csr_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)bin_bytes)) != cudaSuccess)
    return e;
  if (scatter_bytes > 48 * 1024 &&
      (e = cudaFuncSetAttribute(csr_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)scatter_bytes)) != cudaSuccess)
    return e;
  csr_hist_kernel<<<grid, 256, bin_bytes, s>>>(p.ids, p.rows, p.G, p.top_k, p.nb,
                                               (int32_t)ntiles, cnt, p.row_base, p.err);
  ++*launches;
  if ((e = cudaMemcpyAsync(last, cnt + table - 1, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) !=
      cudaSuccess)
    return e;
  if ((e = exclusive_scan(cnt, table, scan_tmp, s, launches)) != cudaSuccess) return e;
  csr_rowptr_kernel<<<(unsigned)((n_lists + 1 + 255) / 256), 256, 0, s>>>(
      cnt, n_lists, (int32_t)ntiles, last, p.row_ptr);
  ++*launches;
  dim3 sgrid((unsigned)ntiles, (unsigned)((p.G + gpw - 1) / gpw));
  csr_scatter_kernel<<<sgrid, 32, scatter_bytes, s>>>(p.ids, p.row_begin, p.rows, p.G,
                                                      p.top_k, p.nb, (int32_t)ntiles, bins, gpw,
                                                      cnt, p.row_base, p.entries);
  ++*launches;
  if (p.unit_ptr) {
    units_kernel<<<1, kUnitThreads, 0, s>>>(p.row_ptr, n_lists, p.nb,
                                            p.tile_tokens * p.unit_tiles, p.unit_ptr,
                                            p.unit_desc);
    ++*launches;
  }
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
