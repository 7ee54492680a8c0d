/*
 * dsa_oracle.c -- plain, slow, obviously-correct CPU statement of the sparse
 * attention's key selection (the "lightning indexer" and its top-k).  TEST
 * INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
 * CPU-baseline leg may call it; the product path (the CUDA library) never
 * links, loads or calls it, and it shares no code, header or table with that
 * path.
 *
 * Everything is computed in double precision from the exact values of the
 * inputs (bf16 and fp32 widen to double without rounding), with no blocking,
 * fusion or reordering beyond what the definition states.
 *
 * Source of the definition: "GLM-5 . MoE transformer block" (open model atlas,
 * glm-5 / blocks / moe-blocks), section "All 43 steps", the indexer equations:
 *     w = x W_w                                     (one weight per index head)
 *     S_I[t,s] = 1 / (sqrt(32) sqrt(128)) * sum_{h=1..32} w[t,h] ReLU(q~[h,t] . k~[s])
 *     S~ = S_I + M                                  (M: the causal mask)
 *     M_sel[t,s] = M[t,s] if s in top_2048(S~[t]), -inf otherwise
 * and the nnterp encyclopedia page glm_moe_dsa, section "Up to 2048 tokens the
 * sparse attention is plain causal attention": the selection holds
 * min(index_topk, seq) int32 key indices per query; on a prompt of at most
 * index_topk tokens it lists every key and the causal mask removes the future
 * ones (row t keeps t + 1 keys).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - index heads NH and head width D are parameters; the scale is
 *     1 / (sqrt(NH) sqrt(D)) (1/64 at the pages' 32 x 128);
 *   - the queries of a sequence are its last T positions: query t sits at
 *     position S - T + t and sees keys s <= S - T + t (a prefill has T == S);
 *   - a masked key scores -infinity; the order is descending score, equal
 *     scores (the masked keys among them) by ascending key index; the
 *     selection is the first min(topk, S) keys of that order;
 *   - the selection is a set; it is listed in ascending key index.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t v)
{
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* scores[b][t][s] = S~ of one query and key: the indexer score where key s is
 * visible to query t, -infinity where the causal mask hides it.
 * q bf16 [B][T][NH][D], k bf16 [B][S][D], w fp32 [B][T][NH]. */
int oracle_dsa_scores(int64_t B, int64_t T, int64_t S, int64_t NH, int64_t D, const uint16_t *q,
                      const uint16_t *k, const float *w, double *scores)
{
    if (B < 0 || T < 0 || S < T || NH < 1 || D < 1 || !q || !k || !w || !scores)
        return 1;
    /* 1/(sqrt(NH) sqrt(D)) written as 1/sqrt(NH*D): the same number, and exact
     * when NH*D is a square (32*128 = 64^2) */
    const double scale = 1.0 / sqrt((double)(NH * D));
    int64_t row;
#pragma omp parallel for schedule(dynamic, 4)
    for (row = 0; row < B * T; ++row) {
        const int64_t b = row / T, t = row % T;
        const int64_t pos = S - T + t;
        for (int64_t s = 0; s < S; ++s) {
            double *out = scores + row * S + s;
            if (s > pos) {
                *out = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int64_t h = 0; h < NH; ++h) {
                const uint16_t *qv = q + (row * NH + h) * D;
                const uint16_t *kv = k + (b * S + s) * D;
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d)
                    dot += bf16_to_double(qv[d]) * bf16_to_double(kv[d]);
                const double relu = dot > 0.0 ? dot : 0.0;
                acc += (double)w[row * NH + h] * relu;
            }
            *out = scale * acc;
        }
    }
    return 0;
}

typedef struct {
    double score;
    int64_t idx;
} cand_t;

/* descending score, equal scores by ascending index */
static int cand_order(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->score > b->score)
        return -1;
    if (a->score < b->score)
        return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

static int idx_order(const void *pa, const void *pb)
{
    const int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* The top-min(topk, S) keys of every row of scores [R][S], listed in ascending
 * key index (sel [R][n_sel]).  kth[r] = the score of the last key taken in
 * the order, next[r] = the score of the first key left out (-infinity when
 * every key is taken): their gap tells how close the row is to a tie. */
int oracle_dsa_select(int64_t R, int64_t S, int64_t topk, const double *scores, int32_t *sel,
                      double *kth, double *next)
{
    if (R < 0 || S < 1 || topk < 1 || !scores || !sel)
        return 1;
    const int64_t n_sel = topk < S ? topk : S;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 4)
    for (r = 0; r < R; ++r) {
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)S);
        for (int64_t s = 0; s < S; ++s) {
            c[s].score = scores[r * S + s];
            c[s].idx = s;
        }
        qsort(c, (size_t)S, sizeof(cand_t), cand_order);
        int32_t *out = sel + r * n_sel;
        for (int64_t j = 0; j < n_sel; ++j)
            out[j] = (int32_t)c[j].idx;
        qsort(out, (size_t)n_sel, sizeof(int32_t), idx_order);
        if (kth)
            kth[r] = c[n_sel - 1].score;
        if (next)
            next[r] = n_sel < S ? c[n_sel].score : -INFINITY;
        free(c);
    }
    return 0;
}
