/*
 * msa_oracle.c -- plain, slow, fp64 CPU reference for the MSA hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes (MiniMax Sparse Attention, two-branch block-sparse
 * attention on top of GQA):
 *
 *   Index Branch  -- ai-tool-zukan "MiniMax MSA guide", section
 *     "2段階構造の中身——ブロック選択から厳密アテンションまで": every causally
 *     visible key token is scored against the query's index head, the token
 *     scores are max-pooled per key block, and a top-k operator keeps the best
 *     blocks per (query, GQA group); the block holding the query is always
 *     kept (same guide, section "クエリを含むローカルブロックの強制取り込み";
 *     zhaixingw "MiniMax M3 深度评测", section "这套注意力到底怎么省的").
 *     One index-query head per group against one shared index-key head
 *     (guide, section "Index BranchとMain Branchの役割分担").  Selection is
 *     shared by the heads of a group and independent across groups (guide,
 *     section "GQAグループ単位の選択共有とは").  Block size 128 and k = 16
 *     blocks, a 2,048-token budget (guide, table in section
 *     "ブロック単位選択の数値設計（128トークン×16ブロック=2048）").
 *
 *   Main Branch  -- same guide, section "Index BranchとMain Branchの役割分担":
 *     ordinary exact softmax attention, restricted to the selected blocks.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - token score = raw dot product <q_idx[t,g], k_idx[s]>, no scale, no
 *     activation;
 *   - visible means s <= t (self included); the pooled score of a block is the
 *     max over its visible tokens;
 *   - k counts the forced local block: local + the best (k-1) earlier blocks;
 *     with fewer than k visible blocks every visible block is taken;
 *   - ranking is (pooled score descending, block id ascending) -- equal scores
 *     go to the lower block id;
 *   - ids are written ascending, padded with -1;
 *   - logits are scale * <q, k>; head h belongs to group h / (H/G).
 *
 * All arithmetic is fp64; bf16 inputs are widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

static double bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void widen(const uint16_t* src, double* dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_to_f64(src[i]);
}

/*
 * Index Branch, scoring + block max-pooling.
 *
 * qi_rows : [n][G][di] bf16 -- the index-query vectors of the n query rows
 * pos     : [n]             -- causal position t of each query row
 * k_idx   : [T][di] bf16    -- shared index-key head, T > max(pos)
 * pooled  : [n][G][nb_out]  -- out: max over visible tokens of each block,
 *                              -inf for blocks with no visible token.
 */
ORACLE_API void msa_oracle_pooled_scores(const uint16_t* qi_rows, const int64_t* pos,
                                         int64_t n, const uint16_t* k_idx, int32_t G,
                                         int32_t di, int32_t block, int64_t nb_out,
                                         double* pooled)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t t = pos[i];
        double* qv = (double*)malloc(sizeof(double) * (size_t)di);
        double* kv = (double*)malloc(sizeof(double) * (size_t)di);
        for (int32_t g = 0; g < G; ++g) {
            widen(qi_rows + ((size_t)i * G + g) * di, qv, di);
            double* out = pooled + ((size_t)i * G + g) * nb_out;
            for (int64_t j = 0; j < nb_out; ++j) out[j] = -INFINITY;
            for (int64_t s = 0; s <= t; ++s) {
                const int64_t j = s / block;
                if (j >= nb_out) break;
                widen(k_idx + (size_t)s * di, kv, di);
                double dot = 0.0;
                for (int32_t c = 0; c < di; ++c) dot += qv[c] * kv[c];
                if (dot > out[j]) out[j] = dot;
            }
        }
        free(qv);
        free(kv);
    }
}

/*
 * The same pooled scores for inputs given in fp64 (the quantised Index
 * Branch: dequantised e4m3 values times their scales).
 *
 * qi_rows : [n][G][di] fp64, k_rows : [T][di] fp64; other arguments and
 * pooled as msa_oracle_pooled_scores.
 */
ORACLE_API void msa_oracle_pooled_scores_f64(const double* qi_rows, const int64_t* pos,
                                             int64_t n, const double* k_rows, int32_t G,
                                             int32_t di, int32_t block, int64_t nb_out,
                                             double* pooled)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t t = pos[i];
        for (int32_t g = 0; g < G; ++g) {
            const double* qv = qi_rows + ((size_t)i * G + g) * di;
            double* out = pooled + ((size_t)i * G + g) * nb_out;
            for (int64_t j = 0; j < nb_out; ++j) out[j] = -INFINITY;
            for (int64_t s = 0; s <= t; ++s) {
                const int64_t j = s / block;
                if (j >= nb_out) break;
                const double* kv = k_rows + (size_t)s * di;
                double dot = 0.0;
                for (int32_t c = 0; c < di; ++c) dot += qv[c] * kv[c];
                if (dot > out[j]) out[j] = dot;
            }
        }
    }
}

typedef struct {
    double score;
    int64_t id;
} cand_t;

/* Order of the top-k operator: higher pooled score first, lower id on ties. */
static int cand_cmp(const void* a, const void* b)
{
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

static int id_cmp(const void* a, const void* b)
{
    const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Index Branch, selection: the forced local block blk(t) = t / block plus the
 * best min(top_k - 1, blk(t)) earlier blocks under (score desc, id asc).
 * Output ids ascending, padded with -1.
 *
 * pooled : [n][G][nb_in] (from msa_oracle_pooled_scores; entries j < blk(t)
 *          are read, nb_in must exceed blk(t) of every row)
 * ids    : [n][G][top_k] int32, out
 */
ORACLE_API void msa_oracle_select_blocks(const double* pooled, const int64_t* pos, int64_t n,
                                         int32_t G, int64_t nb_in, int32_t block,
                                         int32_t top_k, int32_t* ids)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t local = pos[i] / block;
        cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(local > 0 ? local : 1));
        int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)top_k);
        for (int32_t g = 0; g < G; ++g) {
            const double* row = pooled + ((size_t)i * G + g) * nb_in;
            for (int64_t j = 0; j < local; ++j) {
                cand[j].score = row[j];
                cand[j].id = j;
            }
            qsort(cand, (size_t)local, sizeof(cand_t), cand_cmp);
            int64_t take = local < (int64_t)(top_k - 1) ? local : (int64_t)(top_k - 1);
            int32_t cnt = 0;
            sel[cnt++] = (int32_t)local;
            for (int64_t r = 0; r < take; ++r) sel[cnt++] = (int32_t)cand[r].id;
            qsort(sel, (size_t)cnt, sizeof(int32_t), id_cmp);
            int32_t* out = ids + ((size_t)i * G + g) * top_k;
            for (int32_t r = 0; r < top_k; ++r) out[r] = r < cnt ? sel[r] : -1;
        }
        free(cand);
        free(sel);
    }
}

/*
 * Main Branch: exact causal softmax attention of every query head over the
 * keys of its group's selected blocks (keys s <= t only).
 *
 * q_rows : [n][H][d] bf16, pos : [n], k/v : [T][G][d] bf16 (T > max pos)
 * ids    : [n][G][top_k] (ascending, -1 padded)
 * out    : [n][H][d] fp64
 * part_lse (nullable) : [n][H][top_k]     per-block log-sum-exp of the logits
 * part_o   (nullable) : [n][H][top_k][d]  per-block softmax-weighted values
 *   (slot r describes block ids[r]; empty slots get lse = -inf and o = 0)
 */
ORACLE_API void msa_oracle_block_attention(const uint16_t* q_rows, const int64_t* pos, int64_t n,
                                           const uint16_t* k, const uint16_t* v, int32_t H,
                                           int32_t G, int32_t d, int32_t block, int32_t top_k,
                                           double scale, const int32_t* ids, double* out,
                                           double* part_lse, double* part_o)
{
    const int32_t hpg = H / G;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t t = pos[i];
        const int64_t cap = (int64_t)top_k * block;
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
        int32_t* slot = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
        double* logit = (double*)malloc(sizeof(double) * (size_t)cap);
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
        double* kv = (double*)malloc(sizeof(double) * (size_t)d);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        for (int32_t h = 0; h < H; ++h) {
            const int32_t g = h / hpg;
            const int32_t* sel = ids + ((size_t)i * G + g) * top_k;
            int64_t nk = 0;
            for (int32_t r = 0; r < top_k; ++r) {
                if (sel[r] < 0) continue;
                const int64_t s0 = (int64_t)sel[r] * block;
                for (int64_t s = s0; s < s0 + block && s <= t; ++s) {
                    keys[nk] = s;
                    slot[nk] = r;
                    ++nk;
                }
            }
            widen(q_rows + ((size_t)i * H + h) * d, qv, d);
            for (int64_t e = 0; e < nk; ++e) {
                widen(k + ((size_t)keys[e] * G + g) * d, kv, d);
                double dot = 0.0;
                for (int32_t c = 0; c < d; ++c) dot += qv[c] * kv[c];
                logit[e] = scale * dot;
            }
            /* single softmax over all selected keys */
            double m = -INFINITY;
            for (int64_t e = 0; e < nk; ++e)
                if (logit[e] > m) m = logit[e];
            double l = 0.0;
            for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
            for (int64_t e = 0; e < nk; ++e) {
                const double p = exp(logit[e] - m);
                l += p;
                widen(v + ((size_t)keys[e] * G + g) * d, kv, d);
                for (int32_t c = 0; c < d; ++c) acc[c] += p * kv[c];
            }
            double* o = out + ((size_t)i * H + h) * d;
            for (int32_t c = 0; c < d; ++c) o[c] = acc[c] / l;

            /* per-block pieces of the same softmax, for per-kernel parity */
            if (part_lse || part_o) {
                for (int32_t r = 0; r < top_k; ++r) {
                    double mr = -INFINITY, lr = 0.0;
                    for (int64_t e = 0; e < nk; ++e)
                        if (slot[e] == r && logit[e] > mr) mr = logit[e];
                    for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
                    for (int64_t e = 0; e < nk; ++e) {
                        if (slot[e] != r) continue;
                        const double p = exp(logit[e] - mr);
                        lr += p;
                        widen(v + ((size_t)keys[e] * G + g) * d, kv, d);
                        for (int32_t c = 0; c < d; ++c) acc[c] += p * kv[c];
                    }
                    const size_t ps = ((size_t)i * H + h) * top_k + r;
                    if (part_lse) part_lse[ps] = lr > 0.0 ? mr + log(lr) : -INFINITY;
                    if (part_o)
                        for (int32_t c = 0; c < d; ++c)
                            part_o[ps * d + c] = lr > 0.0 ? acc[c] / lr : 0.0;
                }
            }
        }
        free(keys);
        free(slot);
        free(logit);
        free(qv);
        free(kv);
        free(acc);
    }
}

/*
 * Inversion of the selection map into per-(group, key block) lists of the
 * query rows that selected the block: the "KV block outer, gather the queries
 * that hit it" access pattern (tnkblog MiniMax M3 / MSA post, section
 * "MSA の実装"; CSDN M3 write-up, section "MiniMax Sparse Attention（MSA）",
 * hardware-friendly operator).
 *
 * ids     : [N][G][top_k], -1 = empty
 * row_ptr : [G*nb + 1] out, list of (g, j) is entries[row_ptr[g*nb+j] ..)
 * entries : out, each entry (t << 5) | r  (query t, slot r), ascending t
 * returns the number of entries, or -1 if an id is out of range.
 */
ORACLE_API int64_t msa_oracle_block_query_lists(const int32_t* ids, int64_t N, int32_t G,
                                                int64_t nb, int32_t top_k, int32_t* row_ptr,
                                                int32_t* entries)
{
    const int64_t nrows = (int64_t)G * nb;
    int64_t* cursor = (int64_t*)calloc((size_t)nrows + 1, sizeof(int64_t));
    for (int64_t t = 0; t < N; ++t)
        for (int32_t g = 0; g < G; ++g)
            for (int32_t r = 0; r < top_k; ++r) {
                const int32_t j = ids[((size_t)t * G + g) * top_k + r];
                if (j < 0) continue;
                if (j >= nb) {
                    free(cursor);
                    return -1;
                }
                cursor[(int64_t)g * nb + j + 1] += 1;
            }
    for (int64_t x = 0; x < nrows; ++x) cursor[x + 1] += cursor[x];
    for (int64_t x = 0; x <= nrows; ++x) row_ptr[x] = (int32_t)cursor[x];
    for (int64_t t = 0; t < N; ++t)
        for (int32_t g = 0; g < G; ++g)
            for (int32_t r = 0; r < top_k; ++r) {
                const int32_t j = ids[((size_t)t * G + g) * top_k + r];
                if (j < 0) continue;
                entries[cursor[(int64_t)g * nb + j]++] = (int32_t)((t << 5) | r);
            }
    const int64_t total = row_ptr[nrows];
    free(cursor);
    return total;
}
