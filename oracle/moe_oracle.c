/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU statement of the
 * sigmoid-routed mixture-of-experts FFN.  TEST INFRASTRUCTURE ONLY: the
 * tests, the smoke check and the benchmark's CPU-baseline leg may call it;
 * the product path (the CUDA library) never links, loads or calls it, and it
 * shares no code, header or table with that path.
 *
 * Everything is computed in double precision from the exact values of the
 * inputs (bf16 and fp32 both widen to double without rounding).  There is no
 * blocking, fusion or reordering beyond what the definition states.
 *
 * Source of the definition: "GLM-5 . MoE transformer block" (open model atlas,
 * glm-5 / blocks / moe-blocks), section "All 43 steps", the "Mixture of
 * experts" equations:
 *     z = x W_r                          (router logits)
 *     s = sigmoid(z)
 *     E_sel_i = [ i in top_8(s + b) ]
 *     G_i = 2.5 * s_i E_sel_i / sum_j s_j E_sel_j
 *     g = x W1, u = x W3, a = g sigmoid(g), h = a (.) u, E_i = h W2
 *     y_routed = sum_i G_i E_i
 *     y_shared = the same SwiGLU with the shared expert's weights
 *     delta_ffn = y_routed + y_shared
 * and the nnterp encyclopedia pages for GLM-4.7-Flash and GLM-5, note
 * "The mixture: sigmoid scores, a selection bias, renormalized weights"
 * (bias used only to choose; weights are the un-biased sigmoids renormalised
 * and multiplied by routed_scaling_factor; the shared expert is added after
 * the routed sum).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - top-k ties: the lower expert index wins;
 *   - slot order: descending s + b, ties by ascending expert index;
 *   - margin of a token = key of the K-th selected minus key of the (K+1)-th
 *     candidate in that order (+infinity when K == E);
 *   - expert-sorted permutation (not on the pages): groups in expert order,
 *     the shared expert last as group E; inside a group rows are ordered by
 *     ascending token; a routed row is identified by a = t*K + slot, a shared
 *     row by a = T*K + t.
 *
 * Weight layouts are the module's [out, in] (lm_head page: "weight output by
 * input"): W1_e, W3_e are [I][H]; W2_e is [H][I]; W_r is [E][H].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* bf16 bit pattern -> exact double (bf16 is the top half of an IEEE fp32). */
static double bf16_to_double(uint16_t v)
{
    uint32_t bits = ((uint32_t)v) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Pre-FFN RMSNorm of the decoder block ("GLM-5 . MoE transformer block",
 * "All 43 steps": x_ffn = RMSNorm(x'_n); rms_norm_eps from the config):
 *   out[t,h] = x[t,h] * gamma[h] / sqrt(mean_h x[t,h]^2 + eps)
 * in double from the exact bf16 inputs (x and gamma bf16 bit patterns). */
int oracle_rmsnorm(int64_t T, int64_t H, const uint16_t *x, const uint16_t *gamma, double eps,
                   double *out)
{
    if (T < 0 || H <= 0 || eps < 0 || (T > 0 && (!x || !gamma || !out))) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double v = bf16_to_double(x[t * H + h]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t h = 0; h < H; ++h)
            out[t * H + h] = bf16_to_double(x[t * H + h]) * inv * bf16_to_double(gamma[h]);
    }
    return ORACLE_OK;
}

/* Parameter count of one MoE block: router matrix E*H, selection bias E,
 * and (E + n_shared) SwiGLU experts of three H*I matrices each.
 * ("Parameters" table of the GLM-5 MoE transformer block page.) */
int64_t oracle_param_count(int64_t H, int64_t I, int64_t E, int64_t n_shared)
{
    return E * H + E + (E + n_shared) * 3 * H * I;
}

/* Router logits z[t,e] = sum_h x[t,h] * W_r[e,h]  (equation z = x W_r). */
int oracle_logits(int64_t T, int64_t H, int64_t E, const uint16_t *x, const float *w_r,
                  double *z)
{
    if (T < 0 || H <= 0 || E <= 0 || (T > 0 && (!x || !w_r || !z))) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                acc += bf16_to_double(x[t * H + h]) * (double)w_r[e * H + h];
            z[t * E + e] = acc;
        }
    }
    return ORACLE_OK;
}

typedef struct {
    double key;
    int32_t e;
} cand_t;

/* Order for the selection: larger s + b first; equal keys -> smaller index. */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->e > b->e) - (a->e < b->e);
}

/* Selection and gates from given logits.
 *   s = sigmoid(z);  key = s + b;  the K largest keys are selected, in slot
 *   order (descending key, ascending index on ties);
 *   G_slot = scale * s_sel / sum over the selection of s  (un-biased s).
 * idx [T,K], gate [T,K], margin [T] (may be NULL). */
int oracle_select(int64_t T, int64_t E, int64_t K, double scale, const double *z,
                  const float *bias, int32_t *idx, double *gate, double *margin)
{
    if (T < 0 || E <= 0 || K <= 0 || K > E || (T > 0 && (!z || !bias || !idx || !gate)))
        return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        cand_t *c = (cand_t *)malloc((size_t)E * sizeof(cand_t));
        if (!c) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                for (int64_t e = 0; e < E; ++e) {
                    c[e].key = sigmoid(z[t * E + e]) + (double)bias[e];
                    c[e].e = (int32_t)e;
                }
                qsort(c, (size_t)E, sizeof(cand_t), cand_cmp);
                double denom = 0.0;
                for (int64_t k = 0; k < K; ++k) denom += sigmoid(z[t * E + c[k].e]);
                for (int64_t k = 0; k < K; ++k) {
                    idx[t * K + k] = c[k].e;
                    gate[t * K + k] = scale * sigmoid(z[t * E + c[k].e]) / denom;
                }
                if (margin) margin[t] = (K < E) ? c[K - 1].key - c[K].key : INFINITY;
            }
            free(c);
        }
    }
    return err;
}

/* Gates for a GIVEN selection (e.g. one produced elsewhere):
 * G_slot = scale * s_idx[slot] / sum_slots s, s = sigmoid(z). */
int oracle_gates_for(int64_t T, int64_t E, int64_t K, double scale, const double *z,
                     const int32_t *idx, double *gate)
{
    if (T < 0 || E <= 0 || K <= 0 || (T > 0 && (!z || !idx || !gate))) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= E) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double denom = 0.0;
        for (int64_t k = 0; k < K; ++k) denom += sigmoid(z[t * E + idx[t * K + k]]);
        for (int64_t k = 0; k < K; ++k)
            gate[t * K + k] = scale * sigmoid(z[t * E + idx[t * K + k]]) / denom;
    }
    return ORACLE_OK;
}

/* Expert-sorted permutation by counting:
 *   counts[g]  = rows of group g (g < E: assignments to expert g; g == E:
 *                the shared expert, T rows when has_shared, else 0);
 *   offsets[0] = 0, offsets[g+1] = offsets[g] + counts[g]   (E+2 entries);
 *   sorted[offsets[g] + r] = row id of the r-th row of group g, rows in
 *   ascending token order (routed row id t*K+slot, shared row id T*K+t). */
int oracle_permute(int64_t T, int64_t E, int64_t K, int has_shared, const int32_t *idx,
                   int32_t *counts, int32_t *offsets, int32_t *sorted)
{
    if (T < 0 || E <= 0 || K <= 0 || !counts || !offsets || (T > 0 && (!idx || !sorted)))
        return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= E) return ORACLE_ERR_ARG;
    for (int64_t g = 0; g <= E; ++g) counts[g] = 0;
    for (int64_t i = 0; i < T * K; ++i) counts[idx[i]] += 1;
    counts[E] = has_shared ? (int32_t)T : 0;
    offsets[0] = 0;
    for (int64_t g = 0; g <= E; ++g) offsets[g + 1] = offsets[g] + counts[g];
    int32_t *fill = (int32_t *)calloc((size_t)(E + 1), sizeof(int32_t));
    if (!fill) return ORACLE_ERR_NOMEM;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k) {
            int32_t g = idx[t * K + k];
            sorted[offsets[g] + fill[g]++] = (int32_t)(t * K + k);
        }
    if (has_shared)
        for (int64_t t = 0; t < T; ++t) sorted[offsets[E] + t] = (int32_t)(T * K + t);
    free(fill);
    return ORACLE_OK;
}

/* One SwiGLU expert applied to one token row, into out[H]:
 *   g_j = sum_h x_h W1[j,h],  u_j = sum_h x_h W3[j,h],
 *   h_j = g_j sigmoid(g_j) u_j,  out_c = sum_j h_j W2[c,j].
 * hbuf is caller scratch of I doubles. */
static void swiglu_row(int64_t H, int64_t I, const uint16_t *xrow, const uint16_t *w1,
                       const uint16_t *w3, const uint16_t *w2, double *hbuf, double *out)
{
    for (int64_t j = 0; j < I; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            double xv = bf16_to_double(xrow[h]);
            g += xv * bf16_to_double(w1[j * H + h]);
            u += xv * bf16_to_double(w3[j * H + h]);
        }
        hbuf[j] = g * sigmoid(g) * u;
    }
    for (int64_t c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < I; ++j) acc += hbuf[j] * bf16_to_double(w2[c * I + j]);
        out[c] = acc;
    }
}

/* MoE output for the tokens in tok_list (all T tokens when tok_list is NULL):
 *   y_slot[n,k,:] = gate[t,k] * E_{idx[t,k]}(x_t)           (if y_slot)
 *   y_routed[n,:] = sum over k = 0..K-1, in slot order, of y_slot[n,k,:]
 *   y_shared[n,:] = shared expert applied to x_t (zero if !has_shared)
 *   y[n,:]        = y_routed[n,:] + y_shared[n,:]
 * w1/w3/w2 are tables of E pointers (an expert that no listed token uses may
 * be NULL).  Gates are taken as given (no renormalisation), which is what an
 * ablation that zeroes some slots needs. */
int oracle_forward(int64_t T, int64_t H, int64_t I, int64_t E, int64_t K, int has_shared,
                   const uint16_t *x, const uint16_t *const *w1, const uint16_t *const *w3,
                   const uint16_t *const *w2, const uint16_t *ws1, const uint16_t *ws3,
                   const uint16_t *ws2, const int32_t *idx, const double *gate, int64_t n_tok,
                   const int64_t *tok_list, double *y, double *y_routed, double *y_shared,
                   double *y_slot)
{
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || K <= 0 || n_tok < 0 || !y) return ORACLE_ERR_ARG;
    if (n_tok > 0 && (!x || !w1 || !w3 || !w2 || !idx || !gate)) return ORACLE_ERR_ARG;
    if (has_shared && (!ws1 || !ws3 || !ws2)) return ORACLE_ERR_ARG;
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tok_list ? tok_list[n] : n;
        if (t < 0 || t >= T) return ORACLE_ERR_ARG;
        for (int64_t k = 0; k < K; ++k) {
            int32_t e = idx[t * K + k];
            if (e < 0 || e >= E || !w1[e] || !w3[e] || !w2[e]) return ORACLE_ERR_ARG;
        }
    }
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *hbuf = (double *)malloc((size_t)I * sizeof(double));
        double *eo = (double *)malloc((size_t)H * sizeof(double));
        double *routed = (double *)malloc((size_t)H * sizeof(double));
        double *shared = (double *)malloc((size_t)H * sizeof(double));
        if (!hbuf || !eo || !routed || !shared) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t n = 0; n < n_tok; ++n) {
                int64_t t = tok_list ? tok_list[n] : n;
                const uint16_t *xrow = x + t * H;
                for (int64_t c = 0; c < H; ++c) routed[c] = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    int32_t e = idx[t * K + k];
                    double gk = gate[t * K + k];
                    swiglu_row(H, I, xrow, w1[e], w3[e], w2[e], hbuf, eo);
                    for (int64_t c = 0; c < H; ++c) {
                        double v = gk * eo[c];
                        if (y_slot) y_slot[(n * K + k) * H + c] = v;
                        routed[c] += v;
                    }
                }
                if (has_shared)
                    swiglu_row(H, I, xrow, ws1, ws3, ws2, hbuf, shared);
                else
                    for (int64_t c = 0; c < H; ++c) shared[c] = 0.0;
                for (int64_t c = 0; c < H; ++c) {
                    y[n * H + c] = routed[c] + shared[c];
                    if (y_routed) y_routed[n * H + c] = routed[c];
                    if (y_shared) y_shared[n * H + c] = shared[c];
                }
            }
        }
        free(hbuf);
        free(eo);
        free(routed);
        free(shared);
    }
    return err;
}
