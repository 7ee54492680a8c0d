/*
 * srm_dsa.h -- C ABI of the sparse attention's key selection (the "lightning
 * indexer" scores and their top-k) for NVIDIA B200 (sm_100a).  Same library
 * as srm_moe.h (libsrm_moe.so); status codes and the device error word are
 * the ones srm_moe.h defines.
 *
 * Per query t of a sequence and key s it may see (causal), the indexer score is
 *     S[t,s] = 1 / (sqrt(NH) sqrt(D)) * sum_{h < NH} w[t,h] * ReLU(q[t,h,:] . k[s,:])
 * and the selection of query t is the min(topk, S) keys of highest score.
 * Definition: "GLM-5 . MoE transformer block" (open model atlas), section
 * "All 43 steps", the indexer equations (S_I with 32 heads of width 128, the
 * causal mask M, top_2048); the selection's shape and the short-prompt rule:
 * nnterp encyclopedia page glm_moe_dsa, section "Up to 2048 tokens the sparse
 * attention is plain causal attention" (int32 key indices [batch, query,
 * min(index_topk, seq)]; up to index_topk keys every key is listed).
 *
 * Readings fixed by this library where the pages are silent:
 *   - A call handles B independent sequences of S keys each; the T queries of
 *     a sequence are its last T positions: query t sits at position
 *     S - T + t and sees keys 0 .. S - T + t (a prefill has T == S).
 *   - Order of keys: descending score; equal scores by ascending key index;
 *     keys a query cannot see come after every key it can see, by ascending
 *     index (they score -infinity).  The selection is the first min(topk, S)
 *     keys of that order, listed in ASCENDING key index.  So a query that sees
 *     n <= topk keys selects keys 0 .. min(topk, S) - 1.
 *   - Arithmetic: q and k bf16, w fp32; each head's dot product accumulates
 *     in fp32 on the tensor cores, the head sum in fp32.
 *
 * Conventions: as in srm_moe.h -- DEVICE pointers owned by the caller, no
 * allocation, asynchronous on `stream` (a cudaStream_t as void*), host-side
 * validation returns a status before any launch, device-side problems (a
 * pipeline wait that ran out) go to the workspace's error word, read with
 * moe_get_device_error(ws, ...).
 *
 * Supported shapes: NH in {32, 64, 128}, D in {64, 128}, 1 <= topk <= 65536,
 * 1 <= T <= S <= 32768 (the top-k holds a row's keys in registers),
 * B >= 0 (B == 0 is a no-op), B*T*NH < 2^31, B*S < 2^31, B*T*S < 2^40.
 * q, k, w and the workspace must be 16-byte aligned (w is read by a bulk
 * copy); scores and sel 4-byte aligned.  Anything else returns
 * MOE_ERR_UNSUPPORTED (shape), MOE_ERR_ARG (T < 1, S < T, topk < 1, B < 0)
 * or MOE_ERR_ALIGN before any launch.
 */
#ifndef SRM_DSA_H
#define SRM_DSA_H

#include <stddef.h>
#include <stdint.h>

#include "srm_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One call's shape.  B sequences; T queries and S keys per sequence; NH index
 * heads of width D (GLM-5: 32 x 128); topk keys per query (GLM-5: 2048). */
typedef struct {
    int64_t B;
    int32_t T, S, n_heads, head_dim, topk;
} dsa_cfg_t;

/* Bytes of device workspace dsa_scores / dsa_topk / dsa_select need for this
 * shape (including room for the scores when dsa_select is given no scores
 * buffer); 0 for an unsupported shape.  Alignment: 256 bytes. */
size_t dsa_workspace_size(const dsa_cfg_t *cfg);

/* Indexer scores.
 *   q       bf16 [B][T][NH][D]   index queries (after their rotary step)
 *   k       bf16 [B][S][D]       index keys (after their norm and rotary step)
 *   w       fp32 [B][T][NH]      per-head weights (x W_w), 16-byte aligned
 *   scores  fp32 [B][T][S]       out: S[t,s] for every key query t sees; the
 *                                entries s > S - T + t are not written
 * Errors: MOE_ERR_ARG (NULL pointer), MOE_ERR_UNSUPPORTED, MOE_ERR_ALIGN,
 * MOE_ERR_WORKSPACE, MOE_ERR_CUDA; device: MOE_ERR_TIMEOUT.
 * Test-only switch: SRM_MOE_INJECT_STALL=1 in the environment makes the
 * score kernel issue no key copies, so its bounded waits run out and the
 * call reports MOE_ERR_TIMEOUT (failure-detection tests; leave it unset). */
moe_status_t dsa_scores(const dsa_cfg_t *cfg, const void *q, const void *k, const float *w,
                        float *scores, void *ws, size_t ws_bytes, void *stream);

/* Top-k key selection from scores as dsa_scores writes them (only the visible
 * entries are read).
 *   sel  int32 [B][T][min(topk, S)]  out: the selected key indices of each
 *                                    query, ascending
 * Errors: as dsa_scores. */
moe_status_t dsa_topk(const dsa_cfg_t *cfg, const float *scores, int32_t *sel, void *ws,
                      size_t ws_bytes, void *stream);

/* Both steps: dsa_scores then dsa_topk.  scores may be NULL (the workspace
 * then holds them); when given, it receives the scores as dsa_scores writes
 * them. */
moe_status_t dsa_select(const dsa_cfg_t *cfg, const void *q, const void *k, const float *w,
                        int32_t *sel, float *scores, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SRM_DSA_H */
