// decode_static.cu -- msa_decode_static: the decode step with its scratch in
// a fixed device array that is part of this library, for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is unavailable or forbidden --
// a serving loop whose memory is fully reserved up front by another runtime,
// a host thread that must not take the allocator's locks while other work is
// in flight, or an embedding that only hands this library raw input/output
// pointers.  msa_decode needs a caller-provided workspace; this variant uses
// g_decode_scratch instead and allocates nothing.
//
// The array occupies kStaticScratchBytes on every GPU that loads this library
// (when the module is loaded) until the process exits.  Its device address is
// looked up with cudaGetSymbolAddress on every call, with the caller's device
// current: the first call on a device may load the module there, so make it
// before any stream capture; later calls only look the address up, which also
// stays right after a cudaDeviceReset recreates the context.  All calls share
// the array and it keeps the previous call's contents: the decode path clears
// its error word at the start of every call and writes every other scratch
// value before reading it.  Calls whose work overlaps on the GPU (different
// streams, or different host threads) race on the array and must be
// serialised by the caller.
#include "../../include/msa.h"
#include "kernels.h"

namespace msa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device.
cudaError_t static_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_decode_static(const msa_config_t* cfg, const void* q,
                                          const void* q_idx, const void* k_cache,
                                          const void* v_cache, const void* k_idx_cache,
                                          const int64_t* cu_seqlens, int32_t B,
                                          int64_t max_seqlen, int64_t total_len, void* out,
                                          int32_t* ids_out, int32_t check_device_error,
                                          msa_stream_t stream) {
  if (total_len < 1 || max_seqlen > total_len || B < 1 || B > total_len)
    return MSA_ERR_INVALID_ARG;  // total_len must be the sum of the sequence lengths
  size_t need = 0;
  msa_status_t st = msa_workspace_size(cfg, MSA_OP_DECODE, total_len, B, &need);
  if (st != MSA_OK) return st;
  if (need > msa::kStaticScratchBytes) return MSA_ERR_WORKSPACE;  // beyond the fixed array
  void* scratch = nullptr;
  if (msa::static_scratch(&scratch) != cudaSuccess) return MSA_ERR_CUDA;
  st = msa_decode(cfg, q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens, B, max_seqlen, out,
                  ids_out, scratch, msa::kStaticScratchBytes, stream);
  if (st != MSA_OK || !check_device_error) return st;
  uint32_t code = 0;
  return msa_get_device_error(scratch, stream, &code);
}
