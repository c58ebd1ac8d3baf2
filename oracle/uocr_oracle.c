/*
 * uocr_oracle.c -- TEST INFRASTRUCTURE, not product code.
 *
 * A plain, slow, fp64 CPU restatement of the SR-SWA / DASH block-sparse
 * attention step (Unlimited-OCR-2).  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline leg may load or call it.  It shares no source,
 * header, table or helper with the CUDA library; it reads the same bf16 bit
 * patterns and widens them to double before any arithmetic.
 *
 * Sources (web pages, cited by site and section):
 *   [rkmt]  Unlimited-OCR-2 architecture walk-through, news.rkmt.cn/news/25027
 *           section "五、SR-SWA：块级稀疏注意力如何落地" (steps 1-4) and
 *           section "三" (MHA: 10 attention heads = 10 KV heads, head dim 128,
 *           an embedded 1-head x 128-dim Lightning Indexer).
 *   [lqnn]  Unlimited-OCR-2-8bit (MLX) page, www.lqnn.cn/news/271890, section
 *           "128K 上下文的显存账本" (16 blocks x 32 tokens = 512 tokens,
 *           4 local + 12 remote).
 *   [chenxutan] Unlimited OCR v1 article, chenxutan.com/d/4261.html, section
 *           2.3.2: the standard scaled-dot-product helper (softmax(qk^T/sqrt(d)) v).
 *
 * Every size (block size, number of local / remote blocks, heads, dims) is a
 * runtime argument so that tiny cases can be brute-forced in the tests.
 *
 * Cache layouts (the same bytes the library reads):
 *   indexer keys  idx_k_pool [num_pages][blk][d_idx]          bf16 bits
 *   attention K/V k_pool/v_pool [num_pages][H][blk][D]         bf16 bits
 *   block table   bt_row[j] = physical page of logical block j
 * A query of a sequence sits at token position p (0-based) and sees tokens
 * 0..p.  Block j covers tokens blk*j .. blk*j+blk-1.
 *
 * Parity status: every function here is pinned by tests/test_oracle_pins.py
 * (closed forms, brute force, invariants, a library attention routine).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of causal blocks for a query at position p: blocks 0..floor(p/blk). */
int uocr_oracle_num_causal_blocks(int p, int blk)
{
    if (p < 0) return 0;
    return p / blk + 1;
}

/*
 * [rkmt 五 step 1-2] Block score of every causal block j < nb:
 *   s[j] = max over tokens t of block j with t <= p of  sum_d qi[d] * ki[t][d]
 * (the indexer is one head of d_idx dims; the score is the raw dot product,
 * taken as a maximum over the block's tokens).
 * Returns nb.  s must hold nb doubles.
 */
int uocr_oracle_block_scores(const uint16_t *idx_q, const uint16_t *idx_k_pool,
                             const int32_t *bt_row, int p, int blk, int d_idx,
                             double *s)
{
    int nb = uocr_oracle_num_causal_blocks(p, blk);
    for (int j = 0; j < nb; ++j) {
        const uint16_t *page = idx_k_pool + (size_t)bt_row[j] * blk * d_idx;
        double best = -INFINITY;
        for (int r = 0; r < blk; ++r) {
            int t = j * blk + r;
            if (t > p) break;
            double dot = 0.0;
            for (int d = 0; d < d_idx; ++d)
                dot += bf16_bits_to_double(idx_q[d]) *
                       bf16_bits_to_double(page[(size_t)r * d_idx + d]);
            if (dot > best) best = dot;
        }
        s[j] = best;
    }
    return nb;
}

/* Ranking order used for the remote top-k: higher score first, then the lower
 * block id (the pages leave ties open; this is the deterministic choice). */
typedef struct { double s; int j; } ranked_t;

static int rank_cmp(const void *a, const void *b)
{
    const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int int_cmp(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/*
 * [rkmt 五 step 3], [lqnn 显存账本] Block selection.
 *   local  = the n_local most recent causal blocks  {nb-n_local, ..., nb-1} (clipped at 0)
 *   remote = the n_remote highest-scoring blocks among the remaining candidates
 *            [0, nb-n_local), ranked by (score desc, block id asc); all of them
 *            when there are no more than n_remote.
 * sel (n_local + n_remote ints) receives the union in ascending order, padded
 * with -1.  Returns the number of selected blocks.
 * near_tie (may be NULL) is set when more than n_remote candidates exist and the
 * n_remote-th and (n_remote+1)-th ranked scores differ by less than tie_eps.
 */
int uocr_oracle_select(const double *s, int nb, int n_local, int n_remote,
                       double tie_eps, int32_t *sel, int *near_tie)
{
    int n_sel = n_local + n_remote;
    int n_cand = nb - n_local;
    if (n_cand < 0) n_cand = 0;
    int n_take = n_cand < n_remote ? n_cand : n_remote;
    int *chosen = (int *)malloc(sizeof(int) * (size_t)(n_sel > 0 ? n_sel : 1));
    int count = 0;

    if (near_tie) *near_tie = 0;
    if (n_cand > 0) {
        ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)n_cand);
        for (int j = 0; j < n_cand; ++j) { r[j].s = s[j]; r[j].j = j; }
        qsort(r, (size_t)n_cand, sizeof(ranked_t), rank_cmp);
        for (int k = 0; k < n_take; ++k) chosen[count++] = r[k].j;
        if (near_tie && n_cand > n_remote && n_remote > 0)
            *near_tie = (r[n_remote - 1].s - r[n_remote].s) < tie_eps;
        free(r);
    }
    for (int j = (nb - n_local > 0 ? nb - n_local : 0); j < nb; ++j)
        chosen[count++] = j;
    qsort(chosen, (size_t)count, sizeof(int), int_cmp);
    for (int k = 0; k < n_sel; ++k) sel[k] = (k < count) ? chosen[k] : -1;
    free(chosen);
    return count;
}

/*
 * [rkmt 五 step 4], [chenxutan 2.3.2 scaled dot product] Exact attention of one
 * query over the tokens of the selected blocks (t <= p only), per head h:
 *   z_t   = scale * sum_d q[h][d] * k[h][t][d]
 *   out_h = sum_t exp(z_t - max z) v[h][t] / sum_t exp(z_t - max z)
 * sel holds n_sel logical block ids; entries < 0 are ignored.  Only the pages
 * of the selected blocks are read.  With no visible token the output is 0.
 */
void uocr_oracle_attend(const uint16_t *q, const uint16_t *k_pool,
                        const uint16_t *v_pool, const int32_t *bt_row,
                        const int32_t *sel, int n_sel, int p, int H, int D,
                        int blk, double scale, double *out)
{
    int max_tok = n_sel * blk;
    double *z = (double *)malloc(sizeof(double) * (size_t)(max_tok > 0 ? max_tok : 1));
    const uint16_t **vrow = (const uint16_t **)malloc(sizeof(void *) * (size_t)(max_tok > 0 ? max_tok : 1));

    for (int h = 0; h < H; ++h) {
        int n = 0;
        for (int k = 0; k < n_sel; ++k) {
            int j = sel[k];
            if (j < 0) continue;
            size_t tile = ((size_t)bt_row[j] * H + h) * blk * D;
            for (int r = 0; r < blk; ++r) {
                int t = j * blk + r;
                if (t > p) break;
                const uint16_t *krow = k_pool + tile + (size_t)r * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += bf16_bits_to_double(q[(size_t)h * D + d]) * bf16_bits_to_double(krow[d]);
                z[n] = scale * dot;
                vrow[n] = v_pool + tile + (size_t)r * D;
                ++n;
            }
        }
        double *o = out + (size_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (n == 0) continue;
        double m = -INFINITY;
        for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
        double denom = 0.0;
        for (int i = 0; i < n; ++i) {
            double w = exp(z[i] - m);
            denom += w;
            for (int d = 0; d < D; ++d) o[d] += w * bf16_bits_to_double(vrow[i][d]);
        }
        for (int d = 0; d < D; ++d) o[d] /= denom;
    }
    free(vrow);
    free(z);
}

/*
 * The whole step for a batch of queries, one query after another (OpenMP over
 * queries when compiled with -fopenmp; each query is independent).
 *   q_seq[i]  sequence of query i;  q_pos[i]  its token position p.
 *   scores    [n_q][max_blocks] doubles; entries j >= nb are set to -inf.
 *   sel       [n_q][n_local+n_remote]; near_tie [n_q].
 *   out       [n_q][H][D] doubles.
 * If sel_in is not NULL the selection step is skipped and attention runs over
 * sel_in (used to check an output computed over another valid selection).
 * Any of scores / sel / near_tie / out may be NULL when not wanted (scores and
 * sel are then kept in scratch).  threads <= 0 keeps the OpenMP default.
 * Returns the number of threads used.
 */
int uocr_oracle_run(int n_q, const int32_t *q_seq, const int32_t *q_pos,
                    const uint16_t *q, const uint16_t *idx_q,
                    const uint16_t *k_pool, const uint16_t *v_pool,
                    const uint16_t *idx_k_pool, const int32_t *block_table,
                    int max_blocks, int H, int D, int d_idx, int blk,
                    int n_local, int n_remote, double scale, double tie_eps,
                    const int32_t *sel_in, double *scores, int32_t *sel,
                    int *near_tie, double *out, int threads)
{
    int n_sel = n_local + n_remote;
    int used = 1;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
    }
#else
    (void)threads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_q; ++i) {
        const int32_t *bt_row = block_table + (size_t)q_seq[i] * max_blocks;
        int p = q_pos[i];
        int32_t *my_sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_sel);
        if (sel_in) {
            memcpy(my_sel, sel_in + (size_t)i * n_sel, sizeof(int32_t) * (size_t)n_sel);
        } else {
            double *s = (double *)malloc(sizeof(double) * (size_t)max_blocks);
            int nb = uocr_oracle_block_scores(idx_q + (size_t)i * d_idx, idx_k_pool,
                                              bt_row, p, blk, d_idx, s);
            int tie = 0;
            uocr_oracle_select(s, nb, n_local, n_remote, tie_eps, my_sel, &tie);
            if (scores) {
                for (int j = 0; j < max_blocks; ++j)
                    scores[(size_t)i * max_blocks + j] = (j < nb) ? s[j] : -INFINITY;
            }
            if (near_tie) near_tie[i] = tie;
            free(s);
        }
        if (sel) memcpy(sel + (size_t)i * n_sel, my_sel, sizeof(int32_t) * (size_t)n_sel);
        if (out)
            uocr_oracle_attend(q + (size_t)i * H * D, k_pool, v_pool, bt_row, my_sel,
                               n_sel, p, H, D, blk, scale, out + (size_t)i * H * D);
        free(my_sel);
    }
    return used;
}

/*
 * [rkmt 四 (page2d), 六] page2d rotary position embedding of one head vector
 * (dim = 2 * n_pairs, rotate-half layout: pair i = dims i and i + n_pairs).
 * The n_pairs frequency pairs are split between two axes: the first
 * n_pairs - page_pairs pairs rotate by the in-page token offset `tok`, the
 * last page_pairs pairs by the page coordinate (page mod page_mod):
 *   angle_i = tok  * theta_tok ^ (-i / n_tok)          i <  n_tok = n_pairs - page_pairs
 *   angle_i = pg   * theta_page^(-(i - n_tok) / page_pairs)   i >= n_tok, pg = page mod page_mod
 *   out[i]           = x[i] cos(angle_i) - x[i + n_pairs] sin(angle_i)
 *   out[i + n_pairs] = x[i + n_pairs] cos(angle_i) + x[i] sin(angle_i)
 * ("resample": the n_tok token frequencies are spread over the whole spectrum
 * of a standard rotary table of n_tok pairs.)
 */
void uocr_oracle_rope_page2d(const uint16_t *x, int n_pairs, int page_pairs, double theta_tok,
                             double theta_page, int page_mod, long long tok, long long page, double *out)
{
    int n_tok = n_pairs - page_pairs;
    long long pg = page_mod > 0 ? ((page % page_mod) + page_mod) % page_mod : page;
    for (int i = 0; i < n_pairs; ++i) {
        double angle;
        if (i < n_tok)
            angle = (double)tok * pow(theta_tok, -(double)i / (double)n_tok);
        else
            angle = (double)pg * pow(theta_page, -(double)(i - n_tok) / (double)page_pairs);
        double c = cos(angle), s = sin(angle);
        double a = bf16_bits_to_double(x[i]), b = bf16_bits_to_double(x[i + n_pairs]);
        out[i] = a * c - b * s;
        out[i + n_pairs] = b * c + a * s;
    }
}

/*
 * [lqnn 显存账本], [leheaven 二 Token Sieve] Block-summary scoring: each KV block
 * carries one summary vector ("learnable summary vectors" / a block's "brief
 * representation"); the score of causal block j < nb is the raw dot product
 *   s[j] = sum_d idx_q[d] * summary[bt_row[j]][d]
 * (one vector per block instead of the maximum over its tokens).  Returns nb.
 */
int uocr_oracle_summary_scores(const uint16_t *idx_q, const uint16_t *summary_pool, const int32_t *bt_row,
                               int p, int blk, int d_idx, double *s)
{
    int nb = uocr_oracle_num_causal_blocks(p, blk);
    for (int j = 0; j < nb; ++j) {
        const uint16_t *v = summary_pool + (size_t)bt_row[j] * d_idx;
        double dot = 0.0;
        for (int d = 0; d < d_idx; ++d) dot += bf16_bits_to_double(idx_q[d]) * bf16_bits_to_double(v[d]);
        s[j] = dot;
    }
    return nb;
}

/* The mean of a page's blk indexer keys (one summary vector that needs no training). */
void uocr_oracle_block_mean(const uint16_t *idx_k_pool, int page, int blk, int d_idx, double *out)
{
    for (int d = 0; d < d_idx; ++d) {
        double acc = 0.0;
        for (int r = 0; r < blk; ++r) acc += bf16_bits_to_double(idx_k_pool[((size_t)page * blk + r) * d_idx + d]);
        out[d] = acc / blk;
    }
}

/*
 * [rkmt 五 page-aware candidates, image_bucket_constraint] Selection with a
 * candidate constraint: only remote candidates j in [0, nb - n_local) whose bit
 * (mask[j / 32] >> (j % 32)) & 1 is set may be picked; the local window is kept
 * unconditionally.  Otherwise as uocr_oracle_select (score desc, id asc; all
 * allowed candidates when there are no more than n_remote).
 */
int uocr_oracle_select_masked(const double *s, int nb, int n_local, int n_remote, const uint32_t *mask,
                              double tie_eps, int32_t *sel, int *near_tie)
{
    int n_sel = n_local + n_remote;
    int n_cand = nb - n_local > 0 ? nb - n_local : 0;
    ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(n_cand > 0 ? n_cand : 1));
    int m = 0;
    for (int j = 0; j < n_cand; ++j)
        if ((mask[j / 32] >> (j % 32)) & 1u) { r[m].s = s[j]; r[m].j = j; ++m; }
    qsort(r, (size_t)m, sizeof(ranked_t), rank_cmp);
    int n_take = m < n_remote ? m : n_remote;
    int *chosen = (int *)malloc(sizeof(int) * (size_t)(n_sel > 0 ? n_sel : 1));
    int count = 0;
    for (int k = 0; k < n_take; ++k) chosen[count++] = r[k].j;
    if (near_tie) *near_tie = (m > n_remote && n_remote > 0) ? (r[n_remote - 1].s - r[n_remote].s) < tie_eps : 0;
    for (int j = (nb - n_local > 0 ? nb - n_local : 0); j < nb; ++j) chosen[count++] = j;
    qsort(chosen, (size_t)count, sizeof(int), int_cmp);
    for (int k = 0; k < n_sel; ++k) sel[k] = (k < count) ? chosen[k] : -1;
    free(chosen);
    free(r);
    return count;
}
