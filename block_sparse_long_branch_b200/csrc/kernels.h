// kernels.h -- launchers shared between the kernel translation units and the
// C-ABI layer.  Host-side declarations only.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msa {

// ---- Index Branch (index_kernel.cu) ---------------------------------------
struct IndexLaunch {
  const void* q_idx;  // [N][G][d_idx] bf16, or e4m3 when kscale is set
  const void* k_idx;  // [N][d_idx] bf16, or e4m3 when kscale is set
  // optional, packed sequences (selection only): one entry per (sequence, query
  // block) {first token, first row of the sequence, local block, end of the
  // sequence}, longest first; ids are then local to each sequence
  const int4* units;
  int32_t n_units;
  int64_t N;
  int32_t G, d_idx, top_k;
  int64_t row_begin, row_end;  // query rows processed: [row_begin, row_end)
  int32_t* ids;                // selection mode: [row_end-row_begin][G][top_k]
  float* scores;               // scores mode: [row_end-row_begin][G][nb]
  const float* kscale;         // e4m3 selection only: [nb] scale of each key block
  uint32_t* err;
  int num_sms;
};
cudaError_t launch_index_select(const IndexLaunch& p, cudaStream_t s);
cudaError_t launch_index_scores(const IndexLaunch& p, cudaStream_t s);

// ---- query-list inversion (csr_kernel.cu) ---------------------------------
struct CsrLaunch {
  const int32_t* ids;  // [rows][G][top_k], query t = row_begin + row
  int64_t row_begin, rows;
  int32_t G, top_k;
  int64_t nb;          // key blocks (lists per group)
  // optional, packed sequences: per query row, the global number of its
  // sequence's first key block (ids are local: list = row_base[row] + id)
  const int32_t* row_base;
  int32_t* row_ptr;    // [G*nb+1]
  int32_t* entries;    // [rows*G*top_k]
  void* scratch;       // csr_scratch_bytes()
  uint32_t* err;
  // optional: main-branch work units (tiles of `tile_tokens` queries, at most
  // `unit_tiles` tiles per unit) per list, exclusive prefix in unit_ptr[G*nb+1]
  int32_t* unit_ptr;
  int4* unit_desc;  // [max units]: {g, j, first entry, end entry} of every unit
  int32_t tile_tokens, unit_tiles;
};
size_t csr_scratch_bytes(int64_t rows, int32_t G, int32_t top_k, int64_t nb);
cudaError_t launch_csr(const CsrLaunch& p, cudaStream_t s, int* launches);

// ---- schedule of a batch of packed sequences (csr_kernel.cu) ---------------
// Sequence b owns packed rows cu[b] .. cu[b+1]-1 and key blocks blk_base[b] ..
// blk_base[b+1]-1 of the global numbering (nb_b = ceil(L_b / 128) each).
constexpr int kVarlenMaxSeqs = 1024;  // sequences whose offsets travel as a kernel parameter
struct VarlenOffsets {
  int32_t B;
  int64_t cu[kVarlenMaxSeqs + 1];
};
struct VarlenPlan {
  int64_t N;         // packed rows (cu[B])
  int32_t NB;        // global key blocks
  int32_t max_nb;    // blocks of the longest sequence
  // workspace outputs
  int32_t* nbs;      // [B] blocks per sequence
  int32_t* blk_base; // [B+1]
  int32_t* level;    // [max_nb + 1]: first unit of local block b (longest first)
  int4* units;       // [NB] {first token, first row of the sequence, local block, end}
  int32_t* blk_row0; // [NB] first K/V row of each global block
  int32_t* row_base; // [N] blk_base of each row's sequence
};
cudaError_t launch_varlen_plan(const VarlenOffsets& off, const VarlenPlan& p, cudaStream_t s,
                               int* launches);

// ---- Main Branch (main_kernel.cu) -----------------------------------------
struct MainLaunch {
  const void* q;  // [N][H][d] bf16
  const void* k;  // [N][G][d] bf16
  const void* v;  // [N][G][d] fp16: V converted by launch_v_to_fp16
  int64_t N;
  int32_t H, G, d, top_k;
  float scale;
  int64_t row_begin, rows;  // query rows covered by the lists
  int64_t nb;
  const int32_t* row_ptr;   // [G*nb+1]
  const int32_t* entries;
  const int32_t* unit_ptr;   // [G*nb+1]
  const int4* unit_desc;     // [units] {g, j, first entry, end entry}
  const int32_t* blk_row0;   // optional, packed sequences: first K/V row of key block j
  const int32_t* vexp;       // [nb][G] from launch_v_to_fp16
  __half* part_o;   // [rows][G][top_k][H/G][d] fp16, unnormalised o'
  float2* part_ml;  // [rows][G][top_k][H/G] (m~, l~)
  uint32_t* err;
  int grid;
};
// query tokens per 128-row Main Branch tile
int main_tile_tokens(int H, int G);
// V' = fp16(V * 2^-e) for the PV product of the Main Branch: V [N][G][d] bf16,
// V' the same layout (both 16-byte aligned, d a multiple of 8, G <= 128).  Key
// block j (rows blk_row0[j] .. blk_row0[j+1]-1, or 128j .. 128j+127) and group
// g take the smallest e >= 0 with max|v| * 2^-e <= 511.75, written to
// vexp[j*G + g].  A NaN or infinite value records kDevValueRange.
cudaError_t launch_v_to_fp16(const void* src, void* dst, int32_t* vexp, int64_t N, int32_t G,
                             int32_t d, int64_t nb, const int32_t* blk_row0, uint32_t* err,
                             int sms, cudaStream_t s);
cudaError_t launch_main(const MainLaunch& p, cudaStream_t s);

// ---- merge (merge_kernel.cu) ----------------------------------------------
struct MergeLaunch {
  const __half* part_o;
  const float2* part_ml;
  const int32_t* ids;  // [rows][G][top_k]
  int64_t rows;
  int32_t H, G, d, top_k;
  void* out;  // [rows][H][d] bf16 (already offset to row_begin)
  // optional block-alignment outputs (all three or none; offset to row_begin):
  float* block_score;        // in:  [rows][G][top_k] pooled index scores (empty slots
                             //      are set to -inf here)
  float* block_mass;         // out: [rows][G][top_k] attention mass, mean over the group's heads
  float* kl;                 // out: [rows][G] KL(mass || softmax of the scores over the slots)
};
cudaError_t launch_merge(const MergeLaunch& p, cudaStream_t s);

// e4m3 index tensors (quant_kernel.cu): q_idx8 [N][G][d_idx], k_idx8 [N][d_idx],
// kscale [ceil(N/128)] (one scale per 128-key block); d_idx = 128.
struct QuantLaunch {
  const void* q_idx;  // bf16
  const void* k_idx;  // bf16
  int64_t N;
  int32_t G, d_idx;
  void* q_idx8;
  void* k_idx8;
  float* kscale;
};
cudaError_t launch_quantize_index(const QuantLaunch& p, cudaStream_t s);
// rows x 128 bf16 -> e4m3 with one fp32 scale per row (the same rule as the
// index-query rows above): x8 [rows][128], scale [rows]
cudaError_t launch_quantize_rows(const void* x, int64_t rows, void* x8, float* scale,
                                 cudaStream_t s);

// Block-alignment diagnostic: pooled index score of every listed (t, r).
struct BlockScoreLaunch {
  const void* q_idx;  // [N][G][d_idx] bf16
  const void* k_idx;  // [N][d_idx] bf16
  int64_t N;
  int32_t G, d_idx, top_k;
  int64_t nb, row_begin, rows;
  const int32_t* row_ptr;  // [G*nb+1] lists of the query chunk
  const int32_t* entries;
  float* score;  // [rows][G][top_k]; slots without a list entry are not written
  uint32_t* err;
};
cudaError_t launch_block_scores(const BlockScoreLaunch& p, cudaStream_t s);

// ---- decode (decode_kernel.cu) --------------------------------------------
struct DecodeLaunch {
  const void* q;            // [B][H][d]
  const void* q_idx;        // [B][G][d_idx]
  const void* k_cache;      // [sumL][G][d]
  const void* v_cache;      // [sumL][G][d]
  const void* k_idx_cache;  // [sumL][d_idx] bf16, or e4m3 when k_idx_scale is set
  // optional: e4m3 index cache -- q_idx [B][G][128] and k_idx_cache [sumL][128]
  // are e4m3 bytes and key row s scores k_idx_scale[s] * <q8, k8[s]>
  const float* k_idx_scale;
  const int64_t* cu_seqlens;
  int32_t B, H, G, d, d_idx, top_k;
  int64_t max_seqlen;
  float scale;
  void* out;       // [B][H][d] bf16
  int32_t* ids;    // [B][G][top_k]
  float* pooled;   // pooled_cap rows of G: sequence b owns rows from cu[b]/128 + b, as [G][nb_b]
  int64_t pooled_cap;
  int32_t n_split;   // CTAs per (sequence, group) in the attention step
  float* part;       // [B][G][n_split][partial]: split partials (n_split > 1)
  int32_t* tickets;  // [B][G], zero at launch: arrivals of the splits
  uint32_t* err;
  int num_sms;
  void* const* events;  // optional phase events (msa_set_phase_events)
  int n_events;
};
size_t decode_pooled_rows(int64_t total_len, int32_t B);

// ---- MX block formats of the quantised Main Branch (mx_kernel.cu) ----------
// x [n_blocks * 32] bf16 <-> codes (e4m3: one byte per value; e2m1: two values
// per byte, element 2i in the low nibble) and one E8M0 scale byte per block.
constexpr int kMxE4m3 = 0, kMxE2m1 = 1;
cudaError_t launch_mx_quantize(const void* x, int64_t n_blocks, int fmt, void* codes,
                               uint8_t* scales, int sms, cudaStream_t s);
cudaError_t launch_mx_dequantize(const void* codes, const uint8_t* scales, int64_t n_blocks,
                                 int fmt, void* out, int sms, cudaStream_t s);
// floats of one split partial of the decode attention: [heads][d] + max + sum
size_t decode_partial_floats(int32_t H, int32_t G, int32_t d);
constexpr int kDecodeMaxSplit = 4;
cudaError_t launch_decode(const DecodeLaunch& p, cudaStream_t s, int* launches);

}  // namespace msa
