/*
 * msa_oracle.c -- plain, slow, obviously correct CPU oracle for the hot path
 * of MiniMax Sparse Attention (MSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link, load or call this file.  Only
 * the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *   [P2] "MiniMax M3模型算力成本大幅降低原因深度解析", sections
 *        "索引分支（Index Branch）" and "稀疏分支（Sparse Branch）":
 *        a single-head index key with block max-pooling ranks the KV blocks,
 *        the top-K blocks are kept, and standard GQA runs on raw KV over the
 *        kept blocks only.
 *   [P4] "MiniMax M3 深度实战 ...", section 2.3 "MSA 算法实现":
 *        `_select_blocks` always keeps the local (own) block; `forward`
 *        step 3 pads the ragged last block; step 5 is softmax(Q K^T /
 *        sqrt(d_head)) V over the gathered keys.
 *        Section 2.2 "KV Outer Gather Q": the per-block list of hit queries
 *        (the inversion of the per-query selection).
 *        Section 3.3: decode = one query, the newest position.
 *
 * Readings taken where the pages are silent:
 *   - K counts the own block; ties in the index score go to the lower block
 *     index; ids are emitted ascending and padded with -1.
 *   - The own block is forced, the other candidates are blocks j < own(t).
 *   - Query i of n_q sits at position t = T - n_q + i.
 *   - Index scores are not scaled (ranking is scale invariant).
 *   - GQA: query head h reads kv head h / (Hq / Hkv).
 *   - lse is the natural log of sum_i exp(q.k_i / sqrt(d)).
 *
 * Precision: bf16 inputs are widened exactly to double; every dot product,
 * exponential and sum is evaluated in double.  For the integer-valued index
 * keys the pages' workloads use, the double dot products are exact.
 *
 * Parallelism: OpenMP over independent query rows (the loop body is the
 * plain definition; threads only split the rows).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Status codes of this file (not shared with the CUDA library). */
#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_NO_MEM 2

/* Exact widening of a bf16 bit pattern: bf16 is the top 16 bits of fp32. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Row r of the flattened (Bt, n_q) query grid -> (sequence b, position t). */
static void row_to_bt(int64_t r, int n_q, int T, int *b, int64_t *t)
{
    *b = (int)(r / n_q);
    *t = (int64_t)T - n_q + (r % n_q);
}

/* ------------------------------------------------------------------------ */
/* Index branch [P2 "索引分支"]:                                             */
/*   s(t, j) = max over keys i in block j with i <= t of q_idx[t] . k_idx[i] */
/* ------------------------------------------------------------------------ */
static double index_block_score(const uint16_t *q_idx_row, const uint16_t *k_idx_seq,
                                int64_t t, int T, int d_idx, int block, int j)
{
    int64_t lo = (int64_t)j * block;
    int64_t hi = lo + block;
    if (hi > T) hi = T;          /* ragged last block: padded keys do not exist */
    if (hi > t + 1) hi = t + 1;  /* causal: i <= t */
    double best = -INFINITY;
    for (int64_t i = lo; i < hi; ++i) {
        const uint16_t *krow = k_idx_seq + i * d_idx;
        double dot = 0.0;
        for (int c = 0; c < d_idx; ++c)
            dot += bf16_bits_to_double(q_idx_row[c]) * bf16_bits_to_double(krow[c]);
        if (dot > best) best = dot;
    }
    return best;
}

/* Ranking key: higher score first, then lower block index. */
static int ranks_before(double s_a, int j_a, double s_b, int j_b)
{
    if (s_a != s_b) return s_a > s_b;
    return j_a < j_b;
}

/*
 * Top-K block selection for one query (own block forced, K counts it).
 * Writes K ids ascending, -1 padded.  `scores` is scratch of length own.
 */
static void select_row(const uint16_t *q_idx_row, const uint16_t *k_idx_seq, int64_t t,
                       int T, int d_idx, int block, int K, double *scores,
                       unsigned char *taken, int32_t *ids_row)
{
    int own = (int)(t / block);
    for (int j = 0; j < own; ++j) {
        scores[j] = index_block_score(q_idx_row, k_idx_seq, t, T, d_idx, block, j);
        taken[j] = 0;
    }
    int eligible = own + 1;                      /* blocks 0..own */
    int m = (K < eligible ? K : eligible) - 1;   /* ranked picks besides own */
    int n_sel = 0;
    int32_t sel[1024 + 1];
    for (int p = 0; p < m; ++p) {
        int best = -1;
        for (int j = 0; j < own; ++j) {
            if (taken[j]) continue;
            if (best < 0 || ranks_before(scores[j], j, scores[best], best)) best = j;
        }
        taken[best] = 1;
        sel[n_sel++] = best;
    }
    sel[n_sel++] = own;
    /* ascending order (insertion sort, n_sel <= K) */
    for (int a = 1; a < n_sel; ++a) {
        int32_t x = sel[a];
        int b = a - 1;
        while (b >= 0 && sel[b] > x) { sel[b + 1] = sel[b]; --b; }
        sel[b + 1] = x;
    }
    for (int s = 0; s < K; ++s) ids_row[s] = (s < n_sel) ? sel[s] : -1;
}

/*
 * q_idx: [Bt][n_q][d_idx] bf16 bits; k_idx: [Bt][T][d_idx] bf16 bits.
 * rows: flattened query rows r = b*n_q + i to evaluate (NULL = all Bt*n_q).
 * ids_out: [n_rows][K] int32.
 */
int oracle_index_topk(const uint16_t *q_idx, const uint16_t *k_idx, int Bt, int n_q, int T,
                      int d_idx, int block, int K, const int64_t *rows, int64_t n_rows,
                      int32_t *ids_out)
{
    if (!q_idx || !k_idx || !ids_out || Bt < 1 || n_q < 1 || n_q > T || d_idx < 1 ||
        block < 1 || K < 1 || K > 1024)
        return ORC_BAD_ARG;
    if (!rows) n_rows = (int64_t)Bt * n_q;
    int n_blocks = (T + block - 1) / block;
    int bad = 0;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)n_blocks);
        unsigned char *taken = (unsigned char *)malloc((size_t)n_blocks);
        if (!scores || !taken) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < n_rows; ++n) {
            if (!scores || !taken) continue;
            int64_t r = rows ? rows[n] : n;
            int b;
            int64_t t;
            row_to_bt(r, n_q, T, &b, &t);
            select_row(q_idx + r * d_idx, k_idx + (int64_t)b * T * d_idx, t, T, d_idx,
                       block, K, scores, taken, ids_out + n * K);
        }
        free(scores);
        free(taken);
    }
    return bad ? ORC_NO_MEM : ORC_OK;
}

/*
 * Per-query index scores for inspection: scores_out[n][j] = s(t, j) for
 * j < own(t) and NaN elsewhere.  [n_rows][n_blocks] doubles.
 */
int oracle_index_scores(const uint16_t *q_idx, const uint16_t *k_idx, int Bt, int n_q, int T,
                        int d_idx, int block, const int64_t *rows, int64_t n_rows,
                        double *scores_out)
{
    if (!q_idx || !k_idx || !scores_out || Bt < 1 || n_q < 1 || n_q > T || block < 1)
        return ORC_BAD_ARG;
    if (!rows) n_rows = (int64_t)Bt * n_q;
    int n_blocks = (T + block - 1) / block;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_rows; ++n) {
        int64_t r = rows ? rows[n] : n;
        int b;
        int64_t t;
        row_to_bt(r, n_q, T, &b, &t);
        int own = (int)(t / block);
        for (int j = 0; j < n_blocks; ++j)
            scores_out[n * n_blocks + j] =
                (j < own) ? index_block_score(q_idx + r * d_idx, k_idx + (int64_t)b * T * d_idx,
                                              t, T, d_idx, block, j)
                          : NAN;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Inversion [P4 section 2.2]: per KV block, the list of hit queries.        */
/* ------------------------------------------------------------------------ */
/*
 * ids: [Bt][n_q][K] (ascending, -1 padded).  Output CSR over the Bt*N
 * (sequence, block) pairs: row_ptr[Bt*N + 1]; entries[row_ptr[-1]] where each
 * entry is (b*n_q + i)*K + slot, listed in ascending query order within a
 * block.
 */
int oracle_select_invert(const int32_t *ids, int Bt, int n_q, int T, int block, int K,
                         int32_t *row_ptr, int32_t *entries)
{
    if (!ids || !row_ptr || !entries || Bt < 1 || n_q < 1 || block < 1 || K < 1)
        return ORC_BAD_ARG;
    int n_blocks = (T + block - 1) / block;
    int64_t n_lists = (int64_t)Bt * n_blocks;
    int64_t *cursor = (int64_t *)calloc((size_t)n_lists + 1, sizeof(int64_t));
    if (!cursor) return ORC_NO_MEM;
    /* count */
    for (int b = 0; b < Bt; ++b)
        for (int i = 0; i < n_q; ++i)
            for (int s = 0; s < K; ++s) {
                int32_t j = ids[((int64_t)b * n_q + i) * K + s];
                if (j >= 0) cursor[(int64_t)b * n_blocks + j + 1] += 1;
            }
    /* exclusive prefix */
    for (int64_t l = 0; l < n_lists; ++l) cursor[l + 1] += cursor[l];
    for (int64_t l = 0; l <= n_lists; ++l) row_ptr[l] = (int32_t)cursor[l];
    /* fill in query order: lists come out sorted by query */
    for (int b = 0; b < Bt; ++b)
        for (int i = 0; i < n_q; ++i)
            for (int s = 0; s < K; ++s) {
                int64_t r = (int64_t)b * n_q + i;
                int32_t j = ids[r * K + s];
                if (j >= 0) entries[cursor[(int64_t)b * n_blocks + j]++] = (int32_t)(r * K + s);
            }
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Sparse branch [P2 "稀疏分支"; P4 section 2.3, forward step 5]:            */
/*   softmax(q_h . k_i / sqrt(d)) over the keys of the selected blocks with */
/*   i <= t, output = sum p_i v_i with kv head h / G.                        */
/* ------------------------------------------------------------------------ */
static double attn_logit(const uint16_t *qrow, const uint16_t *krow, int d)
{
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += bf16_bits_to_double(qrow[c]) * bf16_bits_to_double(krow[c]);
    return dot / sqrt((double)d);
}

/*
 * Attention of one (query, head) over the keys of the listed blocks.
 * n_blocks_listed entries of `blocks` (entries < 0 are skipped).  Writes
 * out_row[d] and *lse.  If no key qualifies, writes NaN out and -inf lse.
 * `x` is scratch for the logits.
 */
static void attend(const uint16_t *qrow, const uint16_t *k_seq, const uint16_t *v_seq,
                   int64_t t, int T, int Hkv, int d, int kvh, int block,
                   const int32_t *blocks, int n_blocks_listed, double *x,
                   double *out_row, double *lse)
{
    /* gather the key set U(t) in ascending key order */
    int64_t n = 0;
    double mx = -INFINITY;
    for (int s = 0; s < n_blocks_listed; ++s) {
        int32_t j = blocks[s];
        if (j < 0) continue;
        int64_t lo = (int64_t)j * block, hi = lo + block;
        if (hi > T) hi = T;
        if (hi > t + 1) hi = t + 1;
        for (int64_t i = lo; i < hi; ++i) {
            double xi = attn_logit(qrow, k_seq + (i * Hkv + kvh) * d, d);
            x[n++] = xi;
            if (xi > mx) mx = xi;
        }
    }
    if (n == 0) {
        for (int c = 0; c < d; ++c) out_row[c] = NAN;
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int64_t a = 0; a < n; ++a) sum += exp(x[a] - mx);
    double l = mx + log(sum);
    *lse = l;
    for (int c = 0; c < d; ++c) out_row[c] = 0.0;
    n = 0;
    for (int s = 0; s < n_blocks_listed; ++s) {
        int32_t j = blocks[s];
        if (j < 0) continue;
        int64_t lo = (int64_t)j * block, hi = lo + block;
        if (hi > T) hi = T;
        if (hi > t + 1) hi = t + 1;
        for (int64_t i = lo; i < hi; ++i) {
            double p = exp(x[n++] - l);
            const uint16_t *vrow = v_seq + (i * Hkv + kvh) * d;
            for (int c = 0; c < d; ++c) out_row[c] += p * bf16_bits_to_double(vrow[c]);
        }
    }
}

static int check_attn_args(const void *q, const void *k, const void *v, const void *ids, int Bt,
                           int n_q, int T, int Hq, int Hkv, int d, int block, int K)
{
    return !q || !k || !v || !ids || Bt < 1 || n_q < 1 || n_q > T || Hq < 1 || Hkv < 1 ||
           Hq % Hkv != 0 || d < 1 || block < 1 || K < 1;
}

/*
 * q: [Bt][n_q][Hq][d]; k, v: [Bt][T][Hkv][d] (bf16 bits).
 * ids: [n_rows][K], the selection of each listed row (aligned with `rows`).
 * out: [n_rows][Hq][d] double; lse: [n_rows][Hq] double.
 * Duplicate ids in a row are treated as a set (each key counted once).
 */
int oracle_sparse_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *ids, int Bt, int n_q, int T, int Hq, int Hkv, int d,
                       int block, int K, const int64_t *rows, int64_t n_rows, double *out,
                       double *lse)
{
    if (check_attn_args(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K) || !out || !lse)
        return ORC_BAD_ARG;
    if (!rows) n_rows = (int64_t)Bt * n_q;
    int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)K * (size_t)block);
        int32_t *uniq = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
        if (!x || !uniq) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < n_rows; ++n) {
            if (!x || !uniq) continue;
            int64_t r = rows ? rows[n] : n;
            int b;
            int64_t t;
            row_to_bt(r, n_q, T, &b, &t);
            /* the key set is a union: drop repeated block ids */
            int nu = 0;
            for (int s = 0; s < K; ++s) {
                int32_t j = ids[n * K + s];
                int dup = 0;
                for (int u = 0; u < nu; ++u) dup |= (uniq[u] == j);
                if (!dup) uniq[nu++] = j;
            }
            for (int h = 0; h < Hq; ++h)
                attend(q + (r * Hq + h) * d, k + (int64_t)b * T * Hkv * d,
                       v + (int64_t)b * T * Hkv * d, t, T, Hkv, d, h / G, block, uniq, nu, x,
                       out + (n * Hq + h) * d, lse + n * Hq + h);
        }
        free(x);
        free(uniq);
    }
    return bad ? ORC_NO_MEM : ORC_OK;
}

/*
 * Per-slot partial attention: for each listed row, slot s and head h, the
 * attention restricted to block ids[s] alone.  part_out: [n_rows][K][Hq][d],
 * part_lse: [n_rows][K][Hq]; a padded slot (-1) gives NaN / -inf.
 */
int oracle_sparse_attn_partials(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const int32_t *ids, int Bt, int n_q, int T, int Hq, int Hkv,
                                int d, int block, int K, const int64_t *rows, int64_t n_rows,
                                double *part_out, double *part_lse)
{
    if (check_attn_args(q, k, v, ids, Bt, n_q, T, Hq, Hkv, d, block, K) || !part_out ||
        !part_lse)
        return ORC_BAD_ARG;
    if (!rows) n_rows = (int64_t)Bt * n_q;
    int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)block);
        if (!x) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < n_rows; ++n) {
            if (!x) continue;
            int64_t r = rows ? rows[n] : n;
            int b;
            int64_t t;
            row_to_bt(r, n_q, T, &b, &t);
            for (int s = 0; s < K; ++s)
                for (int h = 0; h < Hq; ++h)
                    attend(q + (r * Hq + h) * d, k + (int64_t)b * T * Hkv * d,
                           v + (int64_t)b * T * Hkv * d, t, T, Hkv, d, h / G, block,
                           ids + n * K + s, 1, x, part_out + ((n * K + s) * Hq + h) * d,
                           part_lse + (n * K + s) * Hq + h);
        }
        free(x);
    }
    return bad ? ORC_NO_MEM : ORC_OK;
}

/*
 * Log-sum-exp combine of per-slot partials (the merge of normalised partial
 * softmax results): LSE = log sum_s exp(lse_s);  out = sum_s exp(lse_s - LSE) o_s.
 * Slots with lse_s = -inf contribute nothing.  part_out: [n][K][H][d],
 * part_lse: [n][K][H]; out: [n][H][d], lse: [n][H].
 */
int oracle_lse_combine(const double *part_out, const double *part_lse, int64_t n, int K, int H,
                       int d, double *out, double *lse)
{
    if (!part_out || !part_lse || !out || !lse || K < 1 || H < 1 || d < 1) return ORC_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        for (int h = 0; h < H; ++h) {
            double mx = -INFINITY;
            for (int s = 0; s < K; ++s) {
                double l = part_lse[(r * K + s) * H + h];
                if (l > mx) mx = l;
            }
            double *o = out + (r * H + h) * d;
            if (mx == -INFINITY) {
                for (int c = 0; c < d; ++c) o[c] = NAN;
                lse[r * H + h] = -INFINITY;
                continue;
            }
            double sum = 0.0;
            for (int s = 0; s < K; ++s) {
                double l = part_lse[(r * K + s) * H + h];
                if (l != -INFINITY) sum += exp(l - mx);
            }
            double L = mx + log(sum);
            lse[r * H + h] = L;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int s = 0; s < K; ++s) {
                double l = part_lse[(r * K + s) * H + h];
                if (l == -INFINITY) continue;
                double w = exp(l - L);
                const double *os = part_out + ((r * K + s) * H + h) * d;
                for (int c = 0; c < d; ++c) o[c] += w * os[c];
            }
        }
    return ORC_OK;
}
