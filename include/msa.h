/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention hot path.
 *
 * MSA is two-branch block-sparse attention on top of GQA (ai-tool-zukan
 * "MiniMax MSA guide", section "MiniMax MSAとは何か"):
 *   Index Branch: every causally visible key token is scored with one
 *     index-query head per GQA group against one shared index-key head; the
 *     token scores are max-pooled per 128-token key block; a top-k operator
 *     keeps k blocks per (query, group), and the block holding the query is
 *     always kept (guide, sections "2段階構造の中身——ブロック選択から厳密アテンション
 *     まで" and "クエリを含むローカルブロックの強制取り込み").  All heads of a group
 *     share its block set (section "GQAグループ単位の選択共有とは").
 *   Main Branch: exact causal softmax attention over the selected blocks
 *     only (section "Index BranchとMain Branchの役割分担"), organised with key
 *     blocks as the outer loop and the hitting queries gathered per block
 *     (tnkblog MiniMax M3 / MSA post, section "MSA の実装").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers unless stated otherwise, to
 *    contiguous row-major data, 16-byte aligned.  bf16 tensors are passed as
 *    `const void*` (IEEE bfloat16 bit patterns).
 *  - Shapes use N tokens, H query heads, G groups (KV heads; head h belongs to
 *    group h / (H/G)), d head dim, d_idx index dim, nb = ceil(N/128) blocks,
 *    k = top_k.
 *  - Ownership: the caller allocates and owns every buffer, the workspace
 *    included.  The library never allocates device memory and never
 *    synchronises the stream (except msa_get_device_error).  Every call is
 *    asynchronous and ordered on `stream`.
 *  - Errors: arguments are validated on the host before any launch; an
 *    invalid call returns a status and launches nothing.  A failed launch
 *    returns MSA_ERR_CUDA.  Kernels never trap: a wait that runs out, a bad
 *    index or an input value out of range is recorded in a device error word
 *    inside the workspace and read back with msa_get_device_error.
 *  - Supported shapes: block_size 128; head_dim and index_dim 64 or 128;
 *    1 <= top_k <= 32; G divides 128; H/G is a power of two with
 *    (H/G) * head_dim <= 2048; 1 <= N < 2^26.  Others return
 *    MSA_ERR_UNSUPPORTED.
 *  - Readings where the pages are silent: the token score is the raw dot
 *    product (no scale); "visible" means key s <= query t; k includes the
 *    local block; equal pooled scores go to the lower block id; ids are
 *    written ascending with -1 padding; logits are softmax_scale * <q, k>.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* msa_stream_t;

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer */
  MSA_ERR_UNSUPPORTED = 2,    /* shape outside the supported set above */
  MSA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
  MSA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  MSA_ERR_DEVICE_TIMEOUT = 5, /* a kernel wait ran out (reported by msa_get_device_error) */
  MSA_ERR_DEVICE_INDEX = 6,   /* a kernel met an out-of-range id (msa_get_device_error) */
  MSA_ERR_DEVICE_RANGE = 7    /* an input value outside the range it is computed in
                                 (msa_get_device_error) */
} msa_status_t;

typedef struct {
  int32_t num_heads;   /* H */
  int32_t num_groups;  /* G: GQA groups = KV heads = index-query heads */
  int32_t head_dim;    /* d */
  int32_t index_dim;   /* d_idx */
  int32_t block_size;  /* B_k, must be 128 (guide, table "既定ブロックサイズ") */
  int32_t top_k;       /* k blocks per (query, group), counting the local block */
  float softmax_scale; /* logits = softmax_scale * <q, k>, usually 1/sqrt(d) */
} msa_config_t;

typedef enum {
  MSA_OP_SELECT_TOPK = 0,
  MSA_OP_BLOCK_QUERY_LISTS = 1,
  MSA_OP_PREFILL = 2,
  MSA_OP_DECODE = 3,
  MSA_OP_PREFILL_Q8KV4 = 4
} msa_op_t;

/*
 * Workspace bytes needed by `op`.
 *   SELECT_TOPK, BLOCK_QUERY_LISTS, PREFILL: n_tokens = N, batch ignored.
 *     For PREFILL this is the size that processes all N queries in one pass;
 *     msa_prefill also accepts less (down to msa_prefill_min_workspace) and
 *     then walks the query axis in chunks (msa_prefill_chunk_tokens).
 *   DECODE: n_tokens = total cache rows (sum of sequence lengths), batch = B.
 *   PREFILL_Q8KV4: n_tokens = N; the PREFILL size plus the dequantised
 *     q, k, v (bf16) that msa_prefill_q8kv4 keeps at the end of its workspace.
 * Host-only; returns MSA_ERR_INVALID_ARG / MSA_ERR_UNSUPPORTED like the op.
 */
MSA_API msa_status_t msa_workspace_size(const msa_config_t* cfg, msa_op_t op, int64_t n_tokens,
                                int32_t batch, size_t* bytes);

/* Smallest workspace msa_prefill accepts for N tokens (it then processes the
 * query axis in chunks of at least 128 tokens).  Host-only. */
MSA_API msa_status_t msa_prefill_min_workspace(const msa_config_t* cfg, int64_t N, size_t* bytes);

/* Query rows per chunk msa_prefill uses with ws_bytes of workspace: N when
 * the whole axis fits, else the largest multiple of 128 that fits.
 * ids_returned: non-zero when msa_prefill is given ids_out (the workspace then
 * holds no ids).  MSA_ERR_WORKSPACE if not even 128 rows fit.  Host-only. */
MSA_API msa_status_t msa_prefill_chunk_tokens(const msa_config_t* cfg, int64_t N,
                                              size_t ws_bytes, int32_t ids_returned,
                                              int64_t* chunk);

/*
 * Index Branch scores, pooled per block (guide, section "2段階構造の中身": token
 * scores max-pooled to the block level).
 *   q_idx  [N][G][d_idx] bf16, k_idx [N][d_idx] bf16.
 *   scores [row_count][G][nb] fp32 out: for query row t = row_begin + i,
 *          scores[i][g][j] = max over keys s in block j with s <= t of
 *          <q_idx[t][g], k_idx[s]> (fp32 accumulation of bf16 products);
 *          -inf for blocks with no visible key (j > t/128).
 *   0 <= row_begin, row_begin + row_count <= N, row_count >= 1.
 * Needs no workspace.  Meant for inspection and tests; msa_select_topk does
 * not materialise these scores.
 */
MSA_API msa_status_t msa_index_scores(const msa_config_t* cfg, const void* q_idx, const void* k_idx,
                              int64_t N, int64_t row_begin, int64_t row_count, float* scores,
                              msa_stream_t stream);

/*
 * Index Branch selection: ids[t][g] = the local block t/128 plus the
 * min(k-1, t/128) earlier blocks with the highest pooled scores (ties -> lower
 * block id), ascending, padded with -1 (guide, sections "2段階構造の中身" and
 * "クエリを含むローカルブロックの強制取り込み"; budget k*128 keys per query,
 * table in "ブロック単位選択の数値設計").
 *   q_idx [N][G][d_idx] bf16, k_idx [N][d_idx] bf16 -> ids [N][G][k] int32.
 *   ws: at least msa_workspace_size(cfg, MSA_OP_SELECT_TOPK, N, 0).
 * Scores are fp32 on the tensor cores; two blocks whose scores differ by less
 * than the fp32 rounding of a d_idx-term dot product may rank differently than
 * in exact arithmetic.
 */
MSA_API msa_status_t msa_select_topk(const msa_config_t* cfg, const void* q_idx, const void* k_idx,
                             int64_t N, int32_t* ids, void* ws, size_t ws_bytes,
                             msa_stream_t stream);

/*
 * Inversion of the selection map into per-(group, key block) query lists, the
 * schedule of the KV-block-outer Main Branch (tnkblog MiniMax M3 / MSA post,
 * section "MSA の実装"; CSDN M3 write-up, section "MiniMax Sparse Attention
 * （MSA）": key blocks as the outer loop, the queries that hit a block gathered).
 *   ids     [N][G][k] int32 (as written by msa_select_topk; -1 = empty)
 *   row_ptr [G*nb + 1] int32 out: list of (g, j) is entries[row_ptr[g*nb+j] ..
 *           row_ptr[g*nb+j+1]).
 *   entries [N*G*k] int32 out (capacity): each entry is (t << 5) | r, the
 *           query t and the slot r with ids[t][g][r] == j; ascending t.
 *   ws: at least msa_workspace_size(cfg, MSA_OP_BLOCK_QUERY_LISTS, N, 0).
 * Deterministic; an id outside [-1, nb) raises MSA_ERR_DEVICE_INDEX in the
 * device error word and is skipped.
 */
MSA_API msa_status_t msa_build_block_query_lists(const msa_config_t* cfg, const int32_t* ids, int64_t N,
                                         int32_t* row_ptr, int32_t* entries, void* ws,
                                         size_t ws_bytes, msa_stream_t stream);

/*
 * Whole prefill: Index Branch selection, query lists, Main Branch over the
 * selected blocks, merge of the per-block partial softmaxes.
 *   q [N][H][d], k/v [N][G][d], q_idx [N][G][d_idx], k_idx [N][d_idx] bf16.
 *   out [N][H][d] bf16 out: softmax over the keys s <= t of the selected
 *       blocks of softmax_scale*<q[t][h], k[s][g]>, times v[s][g]; fp32
 *       accumulation, rounded to bf16 (nearest even).  The probabilities
 *       and v meet on the tensor cores in fp16: each key block's v (per
 *       group) is first scaled by the power of two 2^-e that brings its
 *       largest |v| to at most 511.75 (e = 0 when it already is), so any
 *       finite bf16 v is accepted; within a block scaled this way, values
 *       below 2^(e-14) are held to an absolute 2^(e-25).  A NaN or infinite
 *       v is recorded as 0x301 (MSA_ERR_DEVICE_RANGE) in the device error
 *       word.
 *   ids_out [N][G][k] int32 out, nullable: the selection used.
 *   ws: at least msa_prefill_min_workspace(); with less than
 *       msa_workspace_size(PREFILL, N) the query axis is processed in chunks.
 */
MSA_API msa_status_t msa_prefill(const msa_config_t* cfg, const void* q, const void* k, const void* v,
                         const void* q_idx, const void* k_idx, int64_t N, void* out,
                         int32_t* ids_out, void* ws, size_t ws_bytes, msa_stream_t stream);

/*
 * Quantised Index Branch (e4m3).  The pages report the sparse attention's
 * indexer and main branch moving from Q8KV8 to Q8KV4 in a later model
 * (dot-ai "MiniMax M3.1 Flashとは？428BのMoEモデルがウェイト公開", the passage on
 * the ModelScope model card's quantisation) but give no number format; the
 * reading used here, for the indexer only, with d_idx = 128:
 *   per index-query row (t, g) and per 128-key block j of the index keys,
 *   s = max|x| / 448 (fp32, nearest; 1 when the max is 0), x8 = e4m3(x / s)
 *   (fp32 division, nearest even, saturating at +-448).
 * msa_quantize_index_fp8: q_idx [N][G][128], k_idx [N][128] bf16 ->
 *   q_idx8 [N][G][128], k_idx8 [N][128] e4m3 bytes, k_scale [ceil(N/128)] fp32
 *   (the query rows' scales are not kept: see below).
 * msa_select_topk_fp8: as msa_select_topk, ranking block j of a query row by
 *   k_scale[j] * max over its keys of <q_idx8[t][g], k_idx8[s]> (fp32
 *   accumulation on kind::f8f6f4 tensor cores).  A row's own scale is a
 *   positive factor of all its scores and cannot change its ranking.
 *   k_scale: device, [ceil(N/128)] fp32, every entry finite and > 0 (the
 *   quantiser writes 1 for an all-zero block); not checked on the device.
 *   ws: at least msa_workspace_size(cfg, MSA_OP_SELECT_TOPK, N, 0).
 * d_idx other than 128 -> MSA_ERR_UNSUPPORTED.
 */
MSA_API msa_status_t msa_quantize_index_fp8(const msa_config_t* cfg, const void* q_idx,
                                            const void* k_idx, int64_t N, void* q_idx8,
                                            void* k_idx8, float* k_scale, msa_stream_t stream);
MSA_API msa_status_t msa_select_topk_fp8(const msa_config_t* cfg, const void* q_idx8,
                                         const void* k_idx8, const float* k_scale, int64_t N,
                                         int32_t* ids, void* ws, size_t ws_bytes,
                                         msa_stream_t stream);

/*
 * msa_prefill with the quantised Index Branch: the selection of
 * msa_select_topk_fp8 on e4m3 index tensors (as msa_quantize_index_fp8
 * writes them), then the same query lists, Main Branch and merge.
 *   q [N][H][d], k/v [N][G][d] bf16; q_idx8 [N][G][128], k_idx8 [N][128] e4m3
 *   bytes; k_scale [ceil(N/128)] fp32 (device, every entry finite and > 0).
 *   Other arguments, the workspace and the chunking as for msa_prefill.
 * d_idx other than 128 -> MSA_ERR_UNSUPPORTED.
 */
MSA_API msa_status_t msa_prefill_fp8_index(const msa_config_t* cfg, const void* q, const void* k,
                                           const void* v, const void* q_idx8, const void* k_idx8,
                                           const float* k_scale, int64_t N, void* out,
                                           int32_t* ids_out, void* ws, size_t ws_bytes,
                                           msa_stream_t stream);

/*
 * Quantised Main Branch inputs ("Q8KV4"; same passage as above: the sparse
 * attention moving from Q8KV8 to Q8KV4).  The pages name no format; the
 * reading used is the OCP Microscaling (MX) formats, version 1.0: every 32
 * consecutive values along a row share one power-of-two scale 2^X stored as
 * an E8M0 byte (X + 127), X = floor(log2(max|x|)) - emax (emax 8 for e4m3, 2
 * for e2m1; -127 for an all-zero block; clamped to [-127, 127]), and each
 * element is the nearest value of its format to x / 2^X, ties to even,
 * saturating at 448 (e4m3) or 6 (e2m1).  Q is MXFP8 (e4m3), K and V MXFP4
 * (e2m1, two per byte, element 2i in the low nibble).
 *
 * msa_quantize_mx: x [rows][d] bf16 (d a multiple of 32) -> codes and scales.
 *   fmt 0 (MSA_MX_E4M3): codes [rows][d] bytes; fmt 1 (MSA_MX_E2M1): codes
 *   [rows][d/2] bytes.  scales [rows][d/32] bytes.  x and codes 16-byte
 *   aligned; device pointers; rows = 0 is a no-op.  Inputs must be finite.
 */
#define MSA_MX_E4M3 0
#define MSA_MX_E2M1 1
MSA_API msa_status_t msa_quantize_mx(const void* x, int64_t rows, int32_t d, int32_t fmt,
                                     void* codes, uint8_t* scales, msa_stream_t stream);

/*
 * msa_prefill on MX inputs: q8 [N][H][d] e4m3 with q_scale [N][H][d/32];
 * k4, v4 [N][G][d/2] packed e2m1 with k_scale, v_scale [N][G][d/32] (as
 * msa_quantize_mx writes them); q_idx, k_idx bf16 as for msa_prefill.  The
 * three are dequantised exactly to bf16 (at most 4 significant bits times a
 * power of two) in the last msa_workspace_size(PREFILL_Q8KV4) -
 * msa_workspace_size(PREFILL) bytes of the workspace, and msa_prefill runs
 * on them with the rest: the output is the bf16 prefill of the dequantised
 * tensors.  ws: at least msa_prefill_min_workspace() plus those bytes (the
 * query axis is then chunked as in msa_prefill).  Phase events
 * (msa_set_phase_events) start at the index kernel, after the dequantisation.
 */
MSA_API msa_status_t msa_prefill_q8kv4(const msa_config_t* cfg, const void* q8,
                                       const uint8_t* q_scale, const void* k4,
                                       const uint8_t* k_scale, const void* v4,
                                       const uint8_t* v_scale, const void* q_idx,
                                       const void* k_idx, int64_t N, void* out, int32_t* ids_out,
                                       void* ws, size_t ws_bytes, msa_stream_t stream);

/*
 * msa_prefill plus the data of the Index Branch's KL alignment, forward only:
 * the Index Branch is trained to bring its distribution of block scores
 * close to the distribution of where the Main Branch's exact attention went
 * (ai-tool-zukan "MiniMax MSA guide", section "選択を学習可能にするKL損失").
 * The pages do not define the two distributions; the readings used are, per
 * (token t, group g, slot r) of the selection ids[t][g][r]:
 *   block_score [N][G][k] fp32 out: the pooled index score of block
 *     ids[t][g][r] (max over its visible keys of <q_idx[t][g], k_idx[s]>,
 *     the score the selection ranks by; the forced local block included);
 *     -inf for an empty slot.
 *   block_mass  [N][G][k] fp32 out: the share of the Main Branch softmax of
 *     token t that falls on the keys of that block, averaged over the H/G
 *     heads of group g (sums to 1 over the slots); 0 for an empty slot.
 *   kl [N][G] fp32 out: KL(block_mass || softmax over the filled slots of
 *     block_score), in nats.
 * Other arguments and the workspace as for msa_prefill.  The default
 * msa_prefill path does none of this extra work.
 */
MSA_API msa_status_t msa_prefill_block_alignment(const msa_config_t* cfg, const void* q,
                                                 const void* k, const void* v, const void* q_idx,
                                                 const void* k_idx, int64_t N, void* out,
                                                 int32_t* ids_out, float* block_score,
                                                 float* block_mass, float* kl, void* ws,
                                                 size_t ws_bytes, msa_stream_t stream);

/*
 * Prefill of B independent sequences packed along the token axis (no
 * attention across sequences); each is the causal prefill msa_prefill
 * computes.  The pages serve MSA to batched requests but describe no batched
 * kernel.  When the workspace holds the whole batch (at least
 * msa_prefill_varlen_workspace_size()) and B <= 1024, the batch runs in one
 * pass: every kernel runs once, over tiles of all sequences, with key blocks
 * numbered across the batch.  Otherwise the sequences run one after another,
 * each as msa_prefill, on `stream` and `ws`.
 *   q [T][H][d], k/v [T][G][d], q_idx [T][G][d_idx], k_idx [T][d_idx] bf16,
 *     T = cu_seqlens[B]; sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 *     and its token i is position i of that sequence.
 *   cu_seqlens [B+1] int64, HOST pointer: cu_seqlens[0] = 0, non-decreasing,
 *     at least one non-empty sequence; empty sequences are skipped.
 *   out [T][H][d] bf16 out; ids_out [T][G][k] int32 out, nullable (ids are
 *     block numbers within the token's own sequence; every sequence's rows
 *     must start 16-byte aligned, else MSA_ERR_UNSUPPORTED).
 *   ws: at least msa_prefill_min_workspace() for the longest sequence; with
 *     less than msa_prefill_varlen_workspace_size() every sequence runs in
 *     query chunks that fit, as in msa_prefill.
 * Phase events (msa_set_phase_events) are not recorded by this call.
 */
MSA_API msa_status_t msa_prefill_varlen_workspace_size(const msa_config_t* cfg,
                                                       const int64_t* cu_seqlens, int32_t B,
                                                       size_t* bytes);
MSA_API msa_status_t msa_prefill_varlen(const msa_config_t* cfg, const void* q, const void* k,
                                        const void* v, const void* q_idx, const void* k_idx,
                                        const int64_t* cu_seqlens, int32_t B, void* out,
                                        int32_t* ids_out, void* ws, size_t ws_bytes,
                                        msa_stream_t stream);

/*
 * One decode step for B sequences.  The pages give decode speed-ups only
 * (zhaixingw M3 review, section "这套注意力到底怎么省的"); the plainest reading,
 * used here, is the same two branches for the newest query row, which sits at
 * position L_b - 1 of its sequence (its own key/value rows are already in the
 * caches).
 *   q [B][H][d], q_idx [B][G][d_idx] bf16;
 *   k_cache, v_cache [sum L][G][d], k_idx_cache [sum L][d_idx] bf16, packed:
 *     sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1;
 *   cu_seqlens [B+1] int64, DEVICE pointer, cu_seqlens[0] = 0, every L_b >= 1;
 *   max_seqlen: host value >= every L_b (sizes the grid);
 *   out [B][H][d] bf16 out; ids_out [B][G][k] int32 out, nullable.
 *   ws: at least msa_workspace_size(cfg, MSA_OP_DECODE, sum L, B).
 * H/G above 16 -> MSA_ERR_UNSUPPORTED (here and in the decode workspace size).
 */
MSA_API msa_status_t msa_decode(const msa_config_t* cfg, const void* q, const void* q_idx,
                        const void* k_cache, const void* v_cache, const void* k_idx_cache,
                        const int64_t* cu_seqlens, int32_t B, int64_t max_seqlen, void* out,
                        int32_t* ids_out, void* ws, size_t ws_bytes, msa_stream_t stream);

/*
 * msa_decode with the quantised (e4m3) Index Branch over an e4m3 index-key
 * cache: the "Q8" indexer of the model card's Q8KV8 -> Q8KV4 move (dot-ai
 * "MiniMax M3.1 Flashとは？428BのMoEモデルがウェイト公開", the passage on the
 * ModelScope model card's quantisation), read as e4m3 with one fp32 scale per
 * index-key row: a decode cache grows by one token at a time, and a per-row
 * scale lets each token be quantised once, when it is appended.
 *   q_idx8 [B][G][128] e4m3 bytes (per-row scales, as msa_quantize_rows_fp8
 *     writes them; the query scales are not needed: a positive constant of a
 *     (sequence, group) cannot change its ranking);
 *   k_idx8_cache [sum L][128] e4m3 bytes, k_idx_scale [sum L] fp32 (device,
 *     every entry finite and > 0; not checked on the device): key row s
 *     scores k_idx_scale[s] * <q_idx8[b][g], k_idx8_cache[s]> (fp32
 *     accumulation of exact e4m3 products), max-pooled per block.
 *   Everything else (q, k/v caches, cu_seqlens, outputs, workspace, H/G
 *   limit) as for msa_decode.  d_idx other than 128 -> MSA_ERR_UNSUPPORTED.
 */
MSA_API msa_status_t msa_decode_fp8_index(const msa_config_t* cfg, const void* q,
                                          const void* q_idx8, const void* k_cache,
                                          const void* v_cache, const void* k_idx8_cache,
                                          const float* k_idx_scale, const int64_t* cu_seqlens,
                                          int32_t B, int64_t max_seqlen, void* out,
                                          int32_t* ids_out, void* ws, size_t ws_bytes,
                                          msa_stream_t stream);

/*
 * Per-row e4m3 quantiser for the decode index tensors (same passage and
 * reading as above): x [rows][128] bf16 -> x8 [rows][128] e4m3 bytes and
 * scale [rows] fp32, s = max|x| / 448 (fp32, nearest; 1 for an all-zero row),
 * x8 = e4m3(x / s) (fp32 division, nearest even, saturating at +-448).  All
 * pointers device, 16-byte aligned.  rows = 0 is a no-op.
 */
MSA_API msa_status_t msa_quantize_rows_fp8(const void* x, int64_t rows, void* x8, float* scale,
                                           msa_stream_t stream);

/*
 * msa_decode without a workspace argument, for callers that cannot allocate
 * device memory (a serving loop whose memory another runtime reserved up
 * front, a thread that must not enter the allocator, an embedding that only
 * passes raw input/output pointers).  The pages have no counterpart: this is
 * a deployment convenience around msa_decode, whose arguments it shares.
 *   total_len: host value, the sum of the sequence lengths (cu_seqlens[B]).
 *   check_device_error: non-zero -> synchronise `stream` after the launches
 *     and return the device error status (as msa_get_device_error would).
 * Scratch lives in a 16 MiB array compiled into this library, held on every
 * GPU that loads the library until the process exits.  A call that needs more
 * (msa_workspace_size(cfg, MSA_OP_DECODE, total_len, B) > 16 MiB; with G=8
 * that is about 64M cached tokens in total) returns MSA_ERR_WORKSPACE and
 * launches nothing.  The first call on a device looks
 * up the array's address (cudaGetSymbolAddress): make it before any stream
 * capture.  All calls share the array, so calls that overlap on the GPU race;
 * the caller serialises them.  Allocates nothing: no cudaMalloc / cudaFree.
 */
MSA_API msa_status_t msa_decode_static(const msa_config_t* cfg, const void* q, const void* q_idx,
                                       const void* k_cache, const void* v_cache,
                                       const void* k_idx_cache, const int64_t* cu_seqlens,
                                       int32_t B, int64_t max_seqlen, int64_t total_len,
                                       void* out, int32_t* ids_out, int32_t check_device_error,
                                       msa_stream_t stream);

/*
 * Reads and clears the device error word of a workspace used by the calls
 * above.  Synchronises `stream` first.  *code = 0 when no kernel reported a
 * problem; otherwise the first code recorded (0x1xx: a wait ran out ->
 * returns MSA_ERR_DEVICE_TIMEOUT; 0x2xx: an out-of-range id ->
 * MSA_ERR_DEVICE_INDEX; 0x301: a prefill V value that is NaN or infinite ->
 * MSA_ERR_DEVICE_RANGE).
 */
MSA_API msa_status_t msa_get_device_error(void* ws, msa_stream_t stream, uint32_t* code);

/*
 * Self-test of the kernels' failure path; the pages have no counterpart.
 * Launches one CTA that waits, with the same bounded mbarrier wait every
 * kernel of this library uses, on a barrier that nothing ever arrives on.
 * After `limit_ns` (device %globaltimer; 1000 .. 10^9) the wait gives up,
 * records 0x1FE in the device error word of `ws` and the kernel returns, so
 * the context stays usable.  Read the result with msa_get_device_error, which
 * then returns MSA_ERR_DEVICE_TIMEOUT with *code = 0x1FE.
 *   ws: device workspace of at least 256 bytes (its error word is cleared
 *       first).  Returns MSA_ERR_INVALID_ARG for a null/misaligned ws or a
 *       limit out of range, MSA_ERR_CUDA if the launch fails.
 */
MSA_API msa_status_t msa_selftest_wait_timeout(void* ws, uint64_t limit_ns, msa_stream_t stream);

/* Static description of a status code. */
MSA_API const char* msa_status_string(msa_status_t status);

/* Number of kernel launches the last successful call on this host thread
 * issued (for accounting in benchmarks). */
MSA_API int32_t msa_last_launch_count(void);

/*
 * Measurement hook (host thread local).  When `events` is non-NULL, later
 * msa_prefill and msa_decode calls on this thread record CUDA events (type
 * cudaEvent_t, created by the caller) on their stream at phase boundaries:
 *   prefill chunk c: events[5c+0] before the index kernel, [5c+1] after it,
 *     [5c+2] after the query-list kernels, [5c+3] after the Main Branch
 *     kernel, [5c+4] after the merge kernel (only while 5c+4 < count);
 *   decode: [0] before the index scan, [1] after it, [2] after the fused
 *     top-k + attention kernel.
 * Pass NULL to stop recording.  The events are not owned by the library.
 */
MSA_API msa_status_t msa_set_phase_events(void* const* events, int32_t count);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
