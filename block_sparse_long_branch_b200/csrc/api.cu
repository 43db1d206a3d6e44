// api.cu -- the C ABI (include/msa.h): argument validation, workspace layout,
// and the order of launches on the caller's stream.  No device memory is
// allocated here and the stream is never synchronised (except in
// msa_get_device_error).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/msa.h"
#include "kernels.h"

namespace msa {
namespace {

constexpr int kBlock = 128;
constexpr size_t kHeader = 256;  // device error word + reserved
constexpr int kUnitTiles = 16;   // Main Branch tiles per work unit

thread_local int g_launches = 0;
thread_local void* const* g_events = nullptr;
thread_local int g_n_events = 0;

void mark(int i, cudaStream_t s) {
  if (g_events && i < g_n_events && g_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(g_events[i]), s);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

msa_status_t check_cfg(const msa_config_t* c) {
  if (!c) return MSA_ERR_INVALID_ARG;
  if (c->num_heads <= 0 || c->num_groups <= 0 || c->head_dim <= 0 || c->index_dim <= 0 ||
      c->top_k <= 0 || c->block_size <= 0)
    return MSA_ERR_INVALID_ARG;
  if (c->num_heads % c->num_groups != 0) return MSA_ERR_INVALID_ARG;
  if (!(c->softmax_scale > 0.f) || !isfinite(c->softmax_scale)) return MSA_ERR_INVALID_ARG;
  if (c->block_size != kBlock) return MSA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (c->index_dim != 64 && c->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (c->top_k > 32) return MSA_ERR_UNSUPPORTED;
  if (!pow2(c->num_groups) || c->num_groups > 128) return MSA_ERR_UNSUPPORTED;
  const int hg = c->num_heads / c->num_groups;
  if (!pow2(hg) || hg > 128) return MSA_ERR_UNSUPPORTED;
  if (hg * c->head_dim > 2048) return MSA_ERR_UNSUPPORTED;  // one group's heads: <= 4 KiB bf16
  return MSA_OK;
}

msa_status_t check_tokens(const msa_config_t* c, int64_t n) {
  if (n < 1) return MSA_ERR_INVALID_ARG;
  if (n >= (int64_t(1) << 26)) return MSA_ERR_UNSUPPORTED;
  if (n * c->num_heads >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  if (n * c->num_groups * c->top_k >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// decode attention tiles a group's heads in 8s, at most two tiles
constexpr int kDecodeMaxHeadsPerGroup = 16;

int64_t n_blocks(int64_t n) { return (n + kBlock - 1) / kBlock; }

// the dequantised q, k, v (bf16) of msa_prefill_q8kv4
size_t mx_dequant_bytes(const msa_config_t* c, int64_t N) {
  return align256((size_t)N * c->num_heads * c->head_dim * 2) +
         2 * align256((size_t)N * c->num_groups * c->head_dim * 2);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// ---- prefill workspace: the fp16 copy of V for all N tokens, then the
// scratch of one chunk of `rows` query rows ---------------------------------
struct PrefillLayout {
  size_t v16, vexp, ids, row_ptr, entries, unit_ptr, unit_list, csr, part_o, part_ml, total;
};

PrefillLayout prefill_layout(const msa_config_t* c, int64_t N, int64_t rows, int64_t nb,
                             bool own_ids) {
  const int64_t G = c->num_groups, k = c->top_k, HG = c->num_heads / c->num_groups;
  const int64_t slots = rows * G * k;
  const int64_t lists = G * nb;
  const int64_t per_unit = (int64_t)main_tile_tokens(c->num_heads, c->num_groups) * kUnitTiles;
  const int64_t max_units = (slots + per_unit - 1) / per_unit + lists;
  PrefillLayout L;
  size_t off = kHeader;
  // at a fixed offset for every chunk of the call: converted once, read by all
  // (the scale exponents cover every key block: nb is the call's block count
  // for a packed batch, at most n_blocks(N) for a chunk of one sequence)
  const int64_t nb_all = nb > n_blocks(N) ? nb : n_blocks(N);
  L.v16 = off;
  off += align256(N * G * c->head_dim * 2);
  L.vexp = off;
  off += align256(nb_all * G * 4);
  L.ids = off;
  off += own_ids ? align256(slots * 4) : 0;
  L.row_ptr = off;
  off += align256((lists + 1) * 4);
  L.entries = off;
  off += align256(slots * 4);
  L.unit_ptr = off;
  off += align256((lists + 1) * 4);
  L.unit_list = off;
  off += align256(max_units * 16);
  L.csr = off;
  off += csr_scratch_bytes(rows, (int32_t)G, (int32_t)k, nb);
  L.part_o = off;
  off += align256(slots * HG * c->head_dim * 2);
  L.part_ml = off;
  off += align256(slots * HG * 8);
  L.total = off;
  return L;
}

// Query rows per chunk that msa_prefill processes with `ws_bytes` of workspace:
// all of N if it fits, else the largest multiple of 128 rows that fits; 0 if
// not even 128 rows fit.
int64_t prefill_chunk(const msa_config_t* cfg, int64_t N, size_t ws_bytes, bool own_ids) {
  const int64_t nb = n_blocks(N);
  if (prefill_layout(cfg, N, N, nb, own_ids).total <= ws_bytes) return N;
  if (prefill_layout(cfg, N, kBlock, nb, own_ids).total > ws_bytes) return 0;
  int64_t lo = 1, hi = nb;  // in blocks
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (prefill_layout(cfg, N, mid * kBlock, nb, own_ids).total <= ws_bytes)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo * kBlock;
}

// decode workspace: header | split tickets | ids | split partials | pooled
// block scores (the rest).  The header and the tickets are zeroed by one
// memset per call.
struct DecodeLayout {
  size_t tickets, ids, part, fixed;
};
DecodeLayout decode_layout(const msa_config_t* c, int32_t B) {
  const int64_t G = c->num_groups, k = c->top_k;
  DecodeLayout l;
  size_t off = kHeader;
  l.tickets = off;
  off += align256((size_t)B * G * 4);
  l.ids = off;
  off += align256((size_t)B * G * k * 4);
  l.part = off;
  off += align256((size_t)B * G * kDecodeMaxSplit *
                  decode_partial_floats(c->num_heads, c->num_groups, c->head_dim) * 4);
  l.fixed = off;
  return l;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// A failed launch is reported through the status; the runtime's last-error
// slot is cleared so that the caller's next, unrelated CUDA call does not
// see it again (a sticky error stays sticky regardless).
msa_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MSA_OK;
  (void)cudaGetLastError();
  return MSA_ERR_CUDA;
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

const char* msa_status_string(msa_status_t s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case MSA_ERR_WORKSPACE: return "workspace missing or too small";
    case MSA_ERR_CUDA: return "CUDA runtime or launch error";
    case MSA_ERR_DEVICE_TIMEOUT: return "a device-side wait ran out";
    case MSA_ERR_DEVICE_INDEX: return "a device-side index was out of range";
    case MSA_ERR_DEVICE_RANGE: return "an input value was outside the range it is computed in";
  }
  return "unknown status";
}

int32_t msa_last_launch_count(void) { return g_launches; }

msa_status_t msa_set_phase_events(void* const* events, int32_t count) {
  if (events && count < 0) return MSA_ERR_INVALID_ARG;
  g_events = events;
  g_n_events = events ? count : 0;
  return MSA_OK;
}

msa_status_t msa_workspace_size(const msa_config_t* cfg, msa_op_t op, int64_t n_tokens,
                                int32_t batch, size_t* bytes) {
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (!bytes) return MSA_ERR_INVALID_ARG;
  if (op == MSA_OP_DECODE) {
    if (cfg->num_heads / cfg->num_groups > kDecodeMaxHeadsPerGroup) return MSA_ERR_UNSUPPORTED;
    // total cache rows over all sequences; only per-sequence lengths are bounded
    if (n_tokens < 1 || batch < 1 || batch > n_tokens || n_tokens >= (int64_t(1) << 40))
      return MSA_ERR_INVALID_ARG;
    *bytes = decode_layout(cfg, batch).fixed +
             decode_pooled_rows(n_tokens, batch) * cfg->num_groups * sizeof(float);
    return MSA_OK;
  }
  if ((st = check_tokens(cfg, n_tokens)) != MSA_OK) return st;
  const int64_t nb = n_blocks(n_tokens);
  switch (op) {
    case MSA_OP_SELECT_TOPK:
      *bytes = kHeader;
      return MSA_OK;
    case MSA_OP_BLOCK_QUERY_LISTS:
      *bytes = kHeader + csr_scratch_bytes(n_tokens, cfg->num_groups, cfg->top_k, nb);
      return MSA_OK;
    case MSA_OP_PREFILL:
      *bytes = prefill_layout(cfg, n_tokens, n_tokens, nb, true).total;
      return MSA_OK;
    case MSA_OP_PREFILL_Q8KV4:
      *bytes = prefill_layout(cfg, n_tokens, n_tokens, nb, true).total +
               mx_dequant_bytes(cfg, n_tokens);
      return MSA_OK;
    case MSA_OP_DECODE:
      break;
  }
  return MSA_ERR_INVALID_ARG;
}

msa_status_t msa_prefill_min_workspace(const msa_config_t* cfg, int64_t N, size_t* bytes) {
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (!bytes) return MSA_ERR_INVALID_ARG;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  const int64_t rows = N < kBlock ? N : kBlock;
  *bytes = prefill_layout(cfg, N, rows, n_blocks(N), true).total;
  return MSA_OK;
}

msa_status_t msa_prefill_chunk_tokens(const msa_config_t* cfg, int64_t N, size_t ws_bytes,
                                      int32_t ids_returned, int64_t* chunk) {
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (!chunk) return MSA_ERR_INVALID_ARG;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  *chunk = prefill_chunk(cfg, N, ws_bytes, ids_returned == 0);
  return *chunk == 0 ? MSA_ERR_WORKSPACE : MSA_OK;
}

msa_status_t msa_index_scores(const msa_config_t* cfg, const void* q_idx, const void* k_idx,
                              int64_t N, int64_t row_begin, int64_t row_count, float* scores,
                              msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (!q_idx || !k_idx || !scores) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(scores)) return MSA_ERR_INVALID_ARG;
  if (row_begin < 0 || row_count < 1 || row_begin + row_count > N) return MSA_ERR_INVALID_ARG;
  IndexLaunch p{};
  p.q_idx = q_idx;
  p.k_idx = k_idx;
  p.N = N;
  p.G = cfg->num_groups;
  p.d_idx = cfg->index_dim;
  p.top_k = cfg->top_k;
  p.row_begin = row_begin;
  p.row_end = row_begin + row_count;
  p.scores = scores;
  p.err = nullptr;
  p.num_sms = sm_count();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = cuda_status(launch_index_scores(p, s));
  g_launches = 1;
  return st;
}

msa_status_t msa_select_topk(const msa_config_t* cfg, const void* q_idx, const void* k_idx,
                             int64_t N, int32_t* ids, void* ws, size_t ws_bytes,
                             msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (!q_idx || !k_idx || !ids) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(ids)) return MSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kHeader || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  IndexLaunch p{};
  p.q_idx = q_idx;
  p.k_idx = k_idx;
  p.N = N;
  p.G = cfg->num_groups;
  p.d_idx = cfg->index_dim;
  p.top_k = cfg->top_k;
  p.row_begin = 0;
  p.row_end = N;
  p.ids = ids;
  p.err = at<uint32_t>(ws, 0);
  p.num_sms = sm_count();
  st = cuda_status(launch_index_select(p, s));
  g_launches = 1;
  return st;
}

msa_status_t msa_quantize_index_fp8(const msa_config_t* cfg, const void* q_idx, const void* k_idx,
                                    int64_t N, void* q_idx8, void* k_idx8, float* k_scale,
                                    msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (cfg->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (!q_idx || !k_idx || !q_idx8 || !k_idx8 || !k_scale) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(q_idx8) || !aligned16(k_idx8) ||
      !aligned16(k_scale))
    return MSA_ERR_INVALID_ARG;
  QuantLaunch p{};
  p.q_idx = q_idx;
  p.k_idx = k_idx;
  p.N = N;
  p.G = cfg->num_groups;
  p.d_idx = cfg->index_dim;
  p.q_idx8 = q_idx8;
  p.k_idx8 = k_idx8;
  p.kscale = k_scale;
  st = cuda_status(launch_quantize_index(p, reinterpret_cast<cudaStream_t>(stream)));
  g_launches = 2;
  return st;
}

msa_status_t msa_select_topk_fp8(const msa_config_t* cfg, const void* q_idx8, const void* k_idx8,
                                 const float* k_scale, int64_t N, int32_t* ids, void* ws,
                                 size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (cfg->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (!q_idx8 || !k_idx8 || !k_scale || !ids) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx8) || !aligned16(k_idx8) || !aligned16(ids)) return MSA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kHeader || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  IndexLaunch p{};
  p.q_idx = q_idx8;
  p.k_idx = k_idx8;
  p.kscale = k_scale;
  p.N = N;
  p.G = cfg->num_groups;
  p.d_idx = cfg->index_dim;
  p.top_k = cfg->top_k;
  p.row_begin = 0;
  p.row_end = N;
  p.ids = ids;
  p.err = at<uint32_t>(ws, 0);
  p.num_sms = sm_count();
  st = cuda_status(launch_index_select(p, s));
  g_launches = 1;
  return st;
}

msa_status_t msa_build_block_query_lists(const msa_config_t* cfg, const int32_t* ids, int64_t N,
                                         int32_t* row_ptr, int32_t* entries, void* ws,
                                         size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (!ids || !row_ptr || !entries) return MSA_ERR_INVALID_ARG;
  const int64_t nb = n_blocks(N);
  const size_t need = kHeader + csr_scratch_bytes(N, cfg->num_groups, cfg->top_k, nb);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  CsrLaunch p{};
  p.ids = ids;
  p.row_begin = 0;
  p.rows = N;
  p.G = cfg->num_groups;
  p.top_k = cfg->top_k;
  p.nb = nb;
  p.row_ptr = row_ptr;
  p.entries = entries;
  p.scratch = at<void>(ws, kHeader);
  p.err = at<uint32_t>(ws, 0);
  p.unit_ptr = nullptr;
  p.unit_desc = nullptr;
  int launches = 0;
  st = cuda_status(launch_csr(p, s, &launches));
  g_launches = launches;
  return st;
}

}  // extern "C"

namespace {

// One causal prefill of N tokens whose arguments were validated: index ->
// lists -> Main Branch -> merge per chunk of the query axis.  The workspace's
// error word is not cleared here.  Phase events are recorded when `events`.
// With block_mass non-null, also the block-alignment outputs (all three).
msa_status_t prefill_run(const msa_config_t* cfg, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, int64_t N, void* out,
                         int32_t* ids_out, void* ws, size_t ws_bytes, cudaStream_t s,
                         bool events, int* launches_out, float* block_score = nullptr,
                         float* block_mass = nullptr, float* kl = nullptr,
                         const float* k_scale = nullptr) {
  // k_scale set: q_idx / k_idx are e4m3 bytes and the selection is the
  // quantised one (d_idx 128); no alignment outputs in that case
  const int64_t nb = n_blocks(N);
  const bool own_ids = ids_out == nullptr;
  const int64_t chunk = prefill_chunk(cfg, N, ws_bytes, own_ids);
  if (chunk == 0) return MSA_ERR_WORKSPACE;
  auto mark = [&](int i, cudaStream_t st) {
    if (events) ::mark(i, st);
  };
  const int G = cfg->num_groups, H = cfg->num_heads, d = cfg->head_dim, kk = cfg->top_k;
  const int sms = sm_count();
  uint32_t* err = at<uint32_t>(ws, 0);
  int launches = 0;
  // V' in fp16 for the PV product (its offset is the same for every chunk)
  const PrefillLayout L0 = prefill_layout(cfg, N, chunk, nb, own_ids);
  void* v16 = at<void>(ws, L0.v16);
  int32_t* vexp = at<int32_t>(ws, L0.vexp);
  for (int64_t t0 = 0, c = 0; t0 < N; t0 += chunk, ++c) {
    const int64_t t1 = t0 + chunk < N ? t0 + chunk : N;
    const int ev = (int)(5 * c);
    mark(ev, s);
    const int64_t rows = t1 - t0;
    const int64_t nbc = n_blocks(t1);
    const PrefillLayout L = prefill_layout(cfg, N, rows, nbc, own_ids);
    int32_t* ids = own_ids ? at<int32_t>(ws, L.ids) : ids_out + t0 * G * kk;

    IndexLaunch ip{};
    ip.q_idx = q_idx;
    ip.k_idx = k_idx;
    ip.N = N;
    ip.G = G;
    ip.d_idx = cfg->index_dim;
    ip.top_k = kk;
    ip.row_begin = t0;
    ip.row_end = t1;
    ip.ids = ids;
    ip.kscale = k_scale;
    ip.err = err;
    ip.num_sms = sms;
    if (launch_index_select(ip, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
    ++launches;
    mark(ev + 1, s);

    CsrLaunch cp{};
    cp.ids = ids;
    cp.row_begin = t0;
    cp.rows = rows;
    cp.G = G;
    cp.top_k = kk;
    cp.nb = nbc;
    cp.row_ptr = at<int32_t>(ws, L.row_ptr);
    cp.entries = at<int32_t>(ws, L.entries);
    cp.scratch = at<void>(ws, L.csr);
    cp.err = err;
    cp.unit_ptr = at<int32_t>(ws, L.unit_ptr);
    cp.unit_desc = at<int4>(ws, L.unit_list);
    cp.tile_tokens = main_tile_tokens(H, G);
    cp.unit_tiles = kUnitTiles;
    if (launch_csr(cp, s, &launches) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
    if (block_mass) {
      BlockScoreLaunch bp{};
      bp.q_idx = q_idx;
      bp.k_idx = k_idx;
      bp.N = N;
      bp.G = G;
      bp.d_idx = cfg->index_dim;
      bp.top_k = kk;
      bp.nb = nbc;
      bp.row_begin = t0;
      bp.rows = rows;
      bp.row_ptr = cp.row_ptr;
      bp.entries = cp.entries;
      bp.score = block_score + t0 * G * kk;
      bp.err = err;
      if (launch_block_scores(bp, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
      ++launches;
    }
    mark(ev + 2, s);

    if (c == 0) {  // converted once, before the first Main Branch launch
      if (launch_v_to_fp16(v, v16, vexp, N, G, d, nb, nullptr, err, sms, s) != cudaSuccess)
        return cuda_status(cudaErrorLaunchFailure);
      ++launches;
    }
    MainLaunch mp{};
    mp.q = q;
    mp.k = k;
    mp.v = v16;
    mp.N = N;
    mp.H = H;
    mp.G = G;
    mp.d = d;
    mp.top_k = kk;
    mp.scale = cfg->softmax_scale;
    mp.row_begin = t0;
    mp.rows = rows;
    mp.nb = nbc;
    mp.row_ptr = cp.row_ptr;
    mp.entries = cp.entries;
    mp.unit_ptr = cp.unit_ptr;
    mp.unit_desc = cp.unit_desc;
    mp.vexp = vexp;
    mp.part_o = at<__half>(ws, L.part_o);
    mp.part_ml = at<float2>(ws, L.part_ml);
    mp.err = err;
    mp.grid = sms;
    if (launch_main(mp, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
    ++launches;
    mark(ev + 3, s);

    MergeLaunch gp{};
    gp.part_o = mp.part_o;
    gp.part_ml = mp.part_ml;
    gp.ids = ids;
    gp.rows = rows;
    gp.H = H;
    gp.G = G;
    gp.d = d;
    gp.top_k = kk;
    gp.out = static_cast<uint8_t*>(out) + (size_t)t0 * H * d * 2;
    if (block_mass) {
      gp.block_score = block_score + t0 * G * kk;
      gp.block_mass = block_mass + t0 * G * kk;
      gp.kl = kl + t0 * G;
    }
    if (launch_merge(gp, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
    ++launches;
    mark(ev + 4, s);
  }
  *launches_out += launches;
  return MSA_OK;
}

// ---- a batch of packed sequences in one pass --------------------------------
// Every kernel runs once over the whole batch: the Index Branch walks a table
// of (sequence, query block) tiles with keys offset to the sequence's first
// row, the query lists number key blocks globally (blk_base[b] + local id), and
// the Main Branch reads each block's K/V from its sequence's rows.  A
// sequence's last block may be partial; it is only ever its own tokens' local
// block, so the causal mask already hides the next sequence's rows behind it.
struct PackedLayout {
  PrefillLayout base;
  size_t nbs, blk_base, level, units, blk_row0, row_base, total;
};

PackedLayout packed_layout(const msa_config_t* c, int64_t N, int32_t B, int32_t NB,
                           int32_t max_nb, bool own_ids) {
  PackedLayout P;
  P.base = prefill_layout(c, N, N, NB, own_ids);
  size_t off = P.base.total;
  P.nbs = off;
  off += align256((size_t)B * 4);
  P.blk_base = off;
  off += align256((size_t)(B + 1) * 4);
  P.level = off;
  off += align256((size_t)(max_nb + 1) * 4);
  P.units = off;
  off += align256((size_t)NB * 16);
  P.blk_row0 = off;
  off += align256((size_t)NB * 4);
  P.row_base = off;
  off += align256((size_t)N * 4);
  P.total = off;
  return P;
}

// Runs the batch in one pass if it fits `ws_bytes` (and has at most
// kVarlenMaxSeqs sequences); *ran = false leaves it to the per-sequence path.
msa_status_t prefill_packed(const msa_config_t* cfg, const void* q, const void* k, const void* v,
                            const void* q_idx, const void* k_idx, const int64_t* cu, int32_t B,
                            void* out, int32_t* ids_out, void* ws, size_t ws_bytes,
                            cudaStream_t s, int* launches_out, bool* ran) {
  *ran = false;
  if (B > kVarlenMaxSeqs) return MSA_OK;
  const int64_t N = cu[B];
  int64_t NB = 0, max_nb = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int64_t nb = (cu[b + 1] - cu[b] + kBlock - 1) / kBlock;
    NB += nb;
    if (nb > max_nb) max_nb = nb;
  }
  if (check_tokens(cfg, N) != MSA_OK || NB >= (int64_t(1) << 30)) return MSA_OK;
  const bool own_ids = ids_out == nullptr;
  const PackedLayout P = packed_layout(cfg, N, B, (int32_t)NB, (int32_t)max_nb, own_ids);
  if (P.total > ws_bytes) return MSA_OK;
  *ran = true;
  const PrefillLayout& L = P.base;
  const int G = cfg->num_groups, H = cfg->num_heads, d = cfg->head_dim, kk = cfg->top_k;
  const int sms = sm_count();
  uint32_t* err = at<uint32_t>(ws, 0);
  int launches = 0;

  VarlenOffsets offs;
  offs.B = B;
  for (int32_t b = 0; b <= B; ++b) offs.cu[b] = cu[b];
  VarlenPlan pl{};
  pl.N = N;
  pl.NB = (int32_t)NB;
  pl.max_nb = (int32_t)max_nb;
  pl.nbs = at<int32_t>(ws, P.nbs);
  pl.blk_base = at<int32_t>(ws, P.blk_base);
  pl.level = at<int32_t>(ws, P.level);
  pl.units = at<int4>(ws, P.units);
  pl.blk_row0 = at<int32_t>(ws, P.blk_row0);
  pl.row_base = at<int32_t>(ws, P.row_base);
  if (launch_varlen_plan(offs, pl, s, &launches) != cudaSuccess)
    return cuda_status(cudaErrorLaunchFailure);

  int32_t* ids = own_ids ? at<int32_t>(ws, L.ids) : ids_out;
  IndexLaunch ip{};
  ip.q_idx = q_idx;
  ip.k_idx = k_idx;
  ip.N = N;
  ip.G = G;
  ip.d_idx = cfg->index_dim;
  ip.top_k = kk;
  ip.row_begin = 0;
  ip.row_end = N;
  ip.ids = ids;
  ip.units = pl.units;
  ip.n_units = (int32_t)NB;
  ip.err = err;
  ip.num_sms = sms;
  if (launch_index_select(ip, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
  ++launches;

  CsrLaunch cp{};
  cp.ids = ids;
  cp.row_begin = 0;
  cp.rows = N;
  cp.G = G;
  cp.top_k = kk;
  cp.nb = NB;
  cp.row_base = pl.row_base;
  cp.row_ptr = at<int32_t>(ws, L.row_ptr);
  cp.entries = at<int32_t>(ws, L.entries);
  cp.scratch = at<void>(ws, L.csr);
  cp.err = err;
  cp.unit_ptr = at<int32_t>(ws, L.unit_ptr);
  cp.unit_desc = at<int4>(ws, L.unit_list);
  cp.tile_tokens = main_tile_tokens(H, G);
  cp.unit_tiles = kUnitTiles;
  if (launch_csr(cp, s, &launches) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);

  void* v16 = at<void>(ws, L.v16);
  int32_t* vexp = at<int32_t>(ws, L.vexp);
  if (launch_v_to_fp16(v, v16, vexp, N, G, d, NB, pl.blk_row0, err, sms, s) != cudaSuccess)
    return cuda_status(cudaErrorLaunchFailure);
  ++launches;
  MainLaunch mp{};
  mp.q = q;
  mp.k = k;
  mp.v = v16;
  mp.N = N;
  mp.H = H;
  mp.G = G;
  mp.d = d;
  mp.top_k = kk;
  mp.scale = cfg->softmax_scale;
  mp.row_begin = 0;
  mp.rows = N;
  mp.nb = NB;
  mp.row_ptr = cp.row_ptr;
  mp.entries = cp.entries;
  mp.unit_ptr = cp.unit_ptr;
  mp.unit_desc = cp.unit_desc;
  mp.blk_row0 = pl.blk_row0;
  mp.vexp = vexp;
  mp.part_o = at<__half>(ws, L.part_o);
  mp.part_ml = at<float2>(ws, L.part_ml);
  mp.err = err;
  mp.grid = sms;
  if (launch_main(mp, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
  ++launches;

  MergeLaunch gp{};
  gp.part_o = mp.part_o;
  gp.part_ml = mp.part_ml;
  gp.ids = ids;
  gp.rows = N;
  gp.H = H;
  gp.G = G;
  gp.d = d;
  gp.top_k = kk;
  gp.out = out;
  if (launch_merge(gp, s) != cudaSuccess) return cuda_status(cudaErrorLaunchFailure);
  ++launches;
  *launches_out += launches;
  return MSA_OK;
}

msa_status_t check_prefill_ptrs(const void* q, const void* k, const void* v, const void* q_idx,
                                const void* k_idx, const void* out, const int32_t* ids_out,
                                const void* ws) {
  if (!q || !k || !v || !q_idx || !k_idx || !out) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) || !aligned16(k_idx) ||
      !aligned16(out) || (ids_out && !aligned16(ids_out)))
    return MSA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

}  // namespace

extern "C" {

msa_status_t msa_prefill(const msa_config_t* cfg, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, int64_t N, void* out,
                         int32_t* ids_out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, q_idx, k_idx, out, ids_out, ws)) != MSA_OK) return st;
  if (prefill_chunk(cfg, N, ws_bytes, ids_out == nullptr) == 0) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  int launches = 0;
  st = prefill_run(cfg, q, k, v, q_idx, k_idx, N, out, ids_out, ws, ws_bytes, s, true, &launches);
  g_launches = launches;
  return st;
}

msa_status_t msa_prefill_fp8_index(const msa_config_t* cfg, const void* q, const void* k,
                                   const void* v, const void* q_idx8, const void* k_idx8,
                                   const float* k_scale, int64_t N, void* out, int32_t* ids_out,
                                   void* ws, size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if (cfg->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if ((st = check_prefill_ptrs(q, k, v, q_idx8, k_idx8, out, ids_out, ws)) != MSA_OK) return st;
  if (!k_scale) return MSA_ERR_INVALID_ARG;
  if (prefill_chunk(cfg, N, ws_bytes, ids_out == nullptr) == 0) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  int launches = 0;
  st = prefill_run(cfg, q, k, v, q_idx8, k_idx8, N, out, ids_out, ws, ws_bytes, s, true,
                   &launches, nullptr, nullptr, nullptr, k_scale);
  g_launches = launches;
  return st;
}

msa_status_t msa_quantize_mx(const void* x, int64_t rows, int32_t d, int32_t fmt, void* codes,
                             uint8_t* scales, msa_stream_t stream) {
  g_launches = 0;
  if (rows < 0 || d <= 0 || d % 32 != 0 || (fmt != MSA_MX_E4M3 && fmt != MSA_MX_E2M1))
    return MSA_ERR_INVALID_ARG;
  if (rows == 0) return MSA_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)) return MSA_ERR_INVALID_ARG;
  const msa_status_t st =
      cuda_status(launch_mx_quantize(x, rows * (d / 32), fmt == MSA_MX_E4M3 ? kMxE4m3 : kMxE2m1,
                                     codes, scales, sm_count(),
                                     reinterpret_cast<cudaStream_t>(stream)));
  if (st == MSA_OK) g_launches = 1;
  return st;
}

msa_status_t msa_prefill_q8kv4(const msa_config_t* cfg, const void* q8, const uint8_t* q_scale,
                               const void* k4, const uint8_t* k_scale, const void* v4,
                               const uint8_t* v_scale, const void* q_idx, const void* k_idx,
                               int64_t N, void* out, int32_t* ids_out, void* ws, size_t ws_bytes,
                               msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if ((st = check_prefill_ptrs(q8, k4, v4, q_idx, k_idx, out, ids_out, ws)) != MSA_OK) return st;
  if (!q_scale || !k_scale || !v_scale) return MSA_ERR_INVALID_ARG;
  const size_t dq = mx_dequant_bytes(cfg, N);
  if (ws_bytes < dq) return MSA_ERR_WORKSPACE;
  const size_t pws = (ws_bytes - dq) & ~(size_t)255;  // the prefill's part, at the front
  if (prefill_chunk(cfg, N, pws, ids_out == nullptr) == 0) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  const int64_t H = cfg->num_heads, G = cfg->num_groups, d = cfg->head_dim;
  uint8_t* qd = static_cast<uint8_t*>(ws) + pws;
  uint8_t* kd = qd + align256((size_t)N * H * d * 2);
  uint8_t* vd = kd + align256((size_t)N * G * d * 2);
  const int sms = sm_count();
  cudaError_t e = launch_mx_dequantize(q8, q_scale, N * H * d / 32, kMxE4m3, qd, sms, s);
  if (e == cudaSuccess) e = launch_mx_dequantize(k4, k_scale, N * G * d / 32, kMxE2m1, kd, sms, s);
  if (e == cudaSuccess) e = launch_mx_dequantize(v4, v_scale, N * G * d / 32, kMxE2m1, vd, sms, s);
  if (e != cudaSuccess) return cuda_status(e);
  int launches = 3;
  st = prefill_run(cfg, qd, kd, vd, q_idx, k_idx, N, out, ids_out, ws, pws, s, true, &launches);
  g_launches = launches;
  return st;
}

msa_status_t msa_prefill_block_alignment(const msa_config_t* cfg, const void* q, const void* k,
                                         const void* v, const void* q_idx, const void* k_idx,
                                         int64_t N, void* out, int32_t* ids_out,
                                         float* block_score, float* block_mass, float* kl,
                                         void* ws, size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if ((st = check_tokens(cfg, N)) != MSA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, q_idx, k_idx, out, ids_out, ws)) != MSA_OK) return st;
  if (!block_score || !block_mass || !kl || !aligned16(block_score) || !aligned16(block_mass) ||
      !aligned16(kl))
    return MSA_ERR_INVALID_ARG;
  if (prefill_chunk(cfg, N, ws_bytes, ids_out == nullptr) == 0) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  int launches = 0;
  st = prefill_run(cfg, q, k, v, q_idx, k_idx, N, out, ids_out, ws, ws_bytes, s, true, &launches,
                   block_score, block_mass, kl);
  g_launches = launches;
  return st;
}

msa_status_t msa_prefill_varlen_workspace_size(const msa_config_t* cfg, const int64_t* cu_seqlens,
                                               int32_t B, size_t* bytes) {
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (!bytes || !cu_seqlens || B < 1 || cu_seqlens[0] != 0) return MSA_ERR_INVALID_ARG;
  int64_t max_len = 0, NB = 0, max_nb = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int64_t L = cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return MSA_ERR_INVALID_ARG;
    if (L > max_len) max_len = L;
    const int64_t nb = (L + kBlock - 1) / kBlock;
    NB += nb;
    if (nb > max_nb) max_nb = nb;
  }
  if (max_len == 0) return MSA_ERR_INVALID_ARG;
  if ((st = check_tokens(cfg, max_len)) != MSA_OK) return st;
  const int64_t N = cu_seqlens[B];
  if (B <= kVarlenMaxSeqs && check_tokens(cfg, N) == MSA_OK && NB < (int64_t(1) << 30))
    *bytes = packed_layout(cfg, N, B, (int32_t)NB, (int32_t)max_nb, true).total;
  else  // one sequence after another
    *bytes = prefill_layout(cfg, max_len, max_len, n_blocks(max_len), true).total;
  return MSA_OK;
}

msa_status_t msa_prefill_varlen(const msa_config_t* cfg, const void* q, const void* k,
                                const void* v, const void* q_idx, const void* k_idx,
                                const int64_t* cu_seqlens, int32_t B, void* out,
                                int32_t* ids_out, void* ws, size_t ws_bytes,
                                msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (!cu_seqlens || B < 1 || cu_seqlens[0] != 0) return MSA_ERR_INVALID_ARG;
  int64_t max_len = 0;
  const int64_t ids_row_bytes = (int64_t)cfg->num_groups * cfg->top_k * 4;
  for (int32_t b = 0; b < B; ++b) {
    const int64_t L = cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return MSA_ERR_INVALID_ARG;
    if (L > max_len) max_len = L;
    // every sequence's rows of ids_out must start 16-byte aligned
    if (ids_out && L > 0 && (cu_seqlens[b] * ids_row_bytes) % 16 != 0)
      return MSA_ERR_UNSUPPORTED;
  }
  if (max_len == 0) return MSA_ERR_INVALID_ARG;
  if ((st = check_tokens(cfg, max_len)) != MSA_OK) return st;
  if ((st = check_prefill_ptrs(q, k, v, q_idx, k_idx, out, ids_out, ws)) != MSA_OK) return st;
  // every sequence fits the workspace if the longest does
  if (prefill_chunk(cfg, max_len, ws_bytes, ids_out == nullptr) == 0) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MSA_ERR_CUDA;
  const int64_t H = cfg->num_heads, G = cfg->num_groups, d = cfg->head_dim;
  const int64_t di = cfg->index_dim, kk = cfg->top_k;
  int launches = 0;
  bool ran = false;
  st = prefill_packed(cfg, q, k, v, q_idx, k_idx, cu_seqlens, B, out, ids_out, ws, ws_bytes, s,
                      &launches, &ran);
  if (st != MSA_OK || ran) {
    g_launches = launches;
    return st;
  }
  // too large for one pass: one sequence after another, each chunked to fit
  for (int32_t b = 0; b < B; ++b) {
    const int64_t r0 = cu_seqlens[b], L = cu_seqlens[b + 1] - r0;
    if (L == 0) continue;
    // the sequence's rows of every packed tensor (16-byte aligned: rows are
    // whole multiples of 16 bytes for the supported shapes)
    const auto* qb = static_cast<const uint8_t*>(q) + r0 * H * d * 2;
    const auto* kb = static_cast<const uint8_t*>(k) + r0 * G * d * 2;
    const auto* vb = static_cast<const uint8_t*>(v) + r0 * G * d * 2;
    const auto* qib = static_cast<const uint8_t*>(q_idx) + r0 * G * di * 2;
    const auto* kib = static_cast<const uint8_t*>(k_idx) + r0 * di * 2;
    auto* ob = static_cast<uint8_t*>(out) + r0 * H * d * 2;
    int32_t* idb = ids_out ? ids_out + r0 * G * kk : nullptr;
    st = prefill_run(cfg, qb, kb, vb, qib, kib, L, ob, idb, ws, ws_bytes, s, false, &launches);
    if (st != MSA_OK) return st;
  }
  g_launches = launches;
  return MSA_OK;
}

namespace {
// msa_decode, or with k_idx_scale set its e4m3-index variant
msa_status_t decode_run(const msa_config_t* cfg, const void* q, const void* q_idx,
                        const void* k_cache, const void* v_cache, const void* k_idx_cache,
                        const float* k_idx_scale, const int64_t* cu_seqlens, int32_t B,
                        int64_t max_seqlen, void* out, int32_t* ids_out, void* ws,
                        size_t ws_bytes, msa_stream_t stream) {
  g_launches = 0;
  msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (cfg->num_heads / cfg->num_groups > kDecodeMaxHeadsPerGroup) return MSA_ERR_UNSUPPORTED;
  if (!q || !q_idx || !k_cache || !v_cache || !k_idx_cache || !cu_seqlens || !out)
    return MSA_ERR_INVALID_ARG;
  if (B < 1 || max_seqlen < 1) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(q_idx) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(k_idx_cache) || !aligned16(out) || (ids_out && !aligned16(ids_out)))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_tokens(cfg, max_seqlen)) != MSA_OK) return st;
  if (!ws || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  const DecodeLayout lay = decode_layout(cfg, B);
  const size_t fixed = lay.fixed;
  const size_t row_bytes = (size_t)cfg->num_groups * sizeof(float);
  if (ws_bytes < fixed + row_bytes * (size_t)(B + 1)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // error word and split tickets
  if (cudaMemsetAsync(ws, 0, lay.ids, s) != cudaSuccess) return MSA_ERR_CUDA;
  DecodeLaunch p{};
  p.q = q;
  p.q_idx = q_idx;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.k_idx_cache = k_idx_cache;
  p.k_idx_scale = k_idx_scale;
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.H = cfg->num_heads;
  p.G = cfg->num_groups;
  p.d = cfg->head_dim;
  p.d_idx = cfg->index_dim;
  p.top_k = cfg->top_k;
  p.max_seqlen = max_seqlen;
  p.scale = cfg->softmax_scale;
  p.out = out;
  p.ids = ids_out ? ids_out : at<int32_t>(ws, lay.ids);
  p.pooled = at<float>(ws, fixed);
  p.pooled_cap = (int64_t)((ws_bytes - fixed) / row_bytes);
  p.err = at<uint32_t>(ws, 0);
  p.num_sms = sm_count();
  // enough CTAs for about three per SM, at most kDecodeMaxSplit per (b, g)
  {
    const int64_t pairs = (int64_t)B * cfg->num_groups;
    const int64_t want = (3 * (int64_t)p.num_sms) / pairs;
    p.n_split = (int32_t)(want < 1 ? 1 : (want > kDecodeMaxSplit ? kDecodeMaxSplit : want));
  }
  p.part = at<float>(ws, lay.part);
  p.tickets = at<int32_t>(ws, lay.tickets);
  p.events = g_events;
  p.n_events = g_n_events;
  int launches = 0;
  st = cuda_status(launch_decode(p, s, &launches));
  g_launches = launches;
  return st;
}
}  // namespace

msa_status_t msa_decode(const msa_config_t* cfg, const void* q, const void* q_idx,
                        const void* k_cache, const void* v_cache, const void* k_idx_cache,
                        const int64_t* cu_seqlens, int32_t B, int64_t max_seqlen, void* out,
                        int32_t* ids_out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  return decode_run(cfg, q, q_idx, k_cache, v_cache, k_idx_cache, nullptr, cu_seqlens, B,
                    max_seqlen, out, ids_out, ws, ws_bytes, stream);
}

msa_status_t msa_decode_fp8_index(const msa_config_t* cfg, const void* q, const void* q_idx8,
                                  const void* k_cache, const void* v_cache,
                                  const void* k_idx8_cache, const float* k_idx_scale,
                                  const int64_t* cu_seqlens, int32_t B, int64_t max_seqlen,
                                  void* out, int32_t* ids_out, void* ws, size_t ws_bytes,
                                  msa_stream_t stream) {
  g_launches = 0;
  const msa_status_t st = check_cfg(cfg);
  if (st != MSA_OK) return st;
  if (cfg->index_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (!k_idx_scale || !aligned16(k_idx_scale)) return MSA_ERR_INVALID_ARG;
  return decode_run(cfg, q, q_idx8, k_cache, v_cache, k_idx8_cache, k_idx_scale, cu_seqlens, B,
                    max_seqlen, out, ids_out, ws, ws_bytes, stream);
}

msa_status_t msa_quantize_rows_fp8(const void* x, int64_t rows, void* x8, float* scale,
                                   msa_stream_t stream) {
  g_launches = 0;
  if (rows < 0) return MSA_ERR_INVALID_ARG;
  if (rows == 0) return MSA_OK;
  if (!x || !x8 || !scale || !aligned16(x) || !aligned16(x8) || !aligned16(scale))
    return MSA_ERR_INVALID_ARG;
  const msa_status_t st = cuda_status(
      launch_quantize_rows(x, rows, x8, scale, reinterpret_cast<cudaStream_t>(stream)));
  if (st == MSA_OK) g_launches = 1;
  return st;
}

msa_status_t msa_get_device_error(void* ws, msa_stream_t stream, uint32_t* code) {
  if (!ws || !code) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MSA_ERR_CUDA;
  uint32_t c = 0;
  if (cudaMemcpy(&c, ws, sizeof c, cudaMemcpyDeviceToHost) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof c) != cudaSuccess) return MSA_ERR_CUDA;
  *code = c;
  if (c == 0) return MSA_OK;
  if ((c & 0xF00u) == 0x100u) return MSA_ERR_DEVICE_TIMEOUT;
  if ((c & 0xF00u) == 0x300u) return MSA_ERR_DEVICE_RANGE;
  return MSA_ERR_DEVICE_INDEX;
}

}  // extern "C"
