/*
 * srm_moe.h -- C ABI of the sigmoid-routed mixture-of-experts FFN for NVIDIA
 * B200 (sm_100a).  Library: libsrm_moe.so.
 *
 * The layer (GLM-4.7-Flash / GLM-5 decoder blocks) computes, per token row x:
 *     z = x W_r,  s = sigmoid(z),  selection = top_K(s + b),
 *     G_i = scale * s_i / sum over the selection of s_j   (un-biased s),
 *     y = sum over the selection of G_i * W2_i (silu(W1_i x) (.) W3_i x)
 *         + the shared expert's SwiGLU at weight 1.
 * Definition: "GLM-5 . MoE transformer block" (open model atlas), section
 * "All 43 steps", the Mixture-of-experts equations; selection-bias and
 * renormalisation rules: nnterp encyclopedia pages GLM-4.7-Flash and GLM-5,
 * section 03, note "The mixture: sigmoid scores, a selection bias,
 * renormalized weights".
 *
 * Conventions for every call:
 *   - All array arguments are DEVICE pointers unless stated otherwise, owned by
 *     the caller; the library never allocates, frees or keeps them.
 *   - Matrices are row-major and stored [out, in] (the module's weight layout,
 *     "GLM-5 . Vocabulary projection" page: weight held output by input), so the
 *     reduction dimension is contiguous.
 *   - bf16 means IEEE bfloat16 bit patterns (2 bytes).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and stream-ordered; nothing synchronises
 *     except moe_get_device_error.
 *   - Host-side validation happens before any launch and returns a status;
 *     on a non-OK status nothing was launched.  Problems only the device can
 *     see (a corrupt expert id, a pipeline wait that ran out) are recorded in
 *     the workspace's error word and read by moe_get_device_error; outputs of
 *     such a call are unspecified.  The first error is kept until read, so one
 *     read after a step covers all of its calls.  No kernel traps or asserts.
 *   - Supported shapes: 1 <= K <= E <= 256, K <= 16, H % 256 == 0,
 *     I % 128 == 0, T >= 0 (T == 0 is a no-op), T * (K + 1) < 2^31.
 *     Pointers that feed the tensor-memory-access engine (x, packed weights,
 *     workspace) must be 16-byte aligned; every pointer must be 4-byte aligned.
 */
#ifndef SRM_MOE_H
#define SRM_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_ARG = 1,          /* NULL pointer where one is required, negative size, K > E */
    MOE_ERR_UNSUPPORTED = 2,  /* shape outside the supported set listed above */
    MOE_ERR_ALIGN = 3,        /* pointer misaligned (see above) */
    MOE_ERR_WORKSPACE = 4,    /* ws_bytes < moe_workspace_size(cfg) */
    MOE_ERR_BAD_INDEX = 5,    /* device: an expert id outside [0, E) in topk_idx, a row id
                                 outside the rows in sorted, or a group range in offsets
                                 that is not 0 = offsets[0] <= o_g <= o_g+1 <= rows */
    MOE_ERR_TIMEOUT = 6,      /* device: a pipeline wait exceeded its time limit */
    MOE_ERR_CUDA = 7,         /* a CUDA runtime or driver call failed */
    MOE_ERR_RANGE = 8         /* device: an fp16 intermediate (h or a slot output) exceeded
                                 +-65504 and was saturated; the result is inexact */
} moe_status_t;

/* Shape and constants of one MoE block.
 *   T  tokens in this call, H hidden size, I expert intermediate size (the
 *   shared expert has the same width), E routed experts, K experts per token,
 *   routed_scale = routed_scaling_factor (2.5 on GLM-5, 1.8 on GLM-4.7-Flash;
 *   nnterp Config sections), has_shared = 1 to add the always-on shared
 *   expert (n_shared_experts = 1), 0 to leave it out. */
typedef struct {
    int64_t T;
    int32_t H, I, E, K;
    float routed_scale;
    int32_t has_shared;
} moe_cfg_t;

/* Expert weights after moe_pack_weights (device, bf16):
 *   w13: [(E+1) * 2I][H]  per group g (g = E is the shared expert), rows in
 *        units of 32: unit j holds rows 16j..16j+15 of W1_g (gate projection)
 *        followed by rows 16j..16j+15 of W3_g (up projection); the
 *        gate-then-up order is the fused gate_up_proj order of the nnterp
 *        GLM-4 page (section 03, "The MLP is GLM's fused one").
 *   w2:  [(E+1) * H][I]  W2_g (down projection) for g = 0..E, shared last,
 *        stored as IEEE fp16 (see moe_pack_weights). */
typedef struct {
    const void *w13;
    const void *w2;
} moe_weights_t;

/* Bytes of device workspace moe_route, moe_permute and moe_forward need for
 * `cfg` (one buffer serves all three).  Returns 0 for an invalid cfg.
 * The first 256 bytes of a workspace hold the device error word and other
 * control words: zero them once when the workspace is allocated (e.g.
 * cudaMemset); from then on the library keeps them (a device-side error stays
 * recorded until moe_get_device_error reads and clears it). */
size_t moe_workspace_size(const moe_cfg_t *cfg);

/* Staging buffers inside a workspace, for moe_workspace_offset. */
typedef enum {
    MOE_WS_TOKEN_ROWS = 0,   /* bf16 [T*K + T*has_shared][H]: token rows in expert-sorted
                                order (moe_gather_tokens writes, moe_expert_up reads) */
    MOE_WS_SLOT_OUTPUTS = 1  /* fp16 [T*K + T*has_shared][H]: weighted per-slot outputs,
                                row t*K + slot, shared rows T*K + t (moe_expert_down
                                writes, moe_combine reads) */
} moe_ws_region_t;

/* Byte offset of a staging buffer in a workspace laid out for cfg (16-byte
 * aligned when the workspace is); (size_t)-1 for an invalid cfg or region.
 * Lets a caller fill or read those buffers directly (the expert-parallel
 * calls of srm_ep.h do). */
size_t moe_workspace_offset(const moe_cfg_t *cfg, int32_t region);

/* Pack per-expert weights into the moe_weights_t layout.
 *   w1, w3: bf16 [E][I][H];  w2: bf16 [E][H][I];
 *   ws1, ws3: bf16 [I][H];  ws2: bf16 [H][I] (shared expert; ignored and may
 *   be NULL when has_shared == 0, in which case group E is zero-filled);
 *   w13_out: bf16 [(E+1)*2I][H];  w2_out: fp16 [(E+1)*H][I].
 * A re-layout; W2 is also converted from bf16 to fp16, which is exact for
 * magnitudes in [2^-17, 65504] (smaller ones keep fp16's subnormal spacing of
 * 2^-24, larger ones saturate).  The down projection multiplies fp16 h by
 * fp16 W2: fp16 holds h with three more mantissa bits than bf16 at the same
 * tensor-core rate.
 *   w2_inexact: int32 [1] device counter or NULL; out: the number of W2
 *   values (routed and shared) whose fp16 copy differs from the bf16 value
 *   (beyond +-65504, saturated; or too small for fp16's 2^-24 spacing,
 *   rounded).  0 means the packed W2 is exact.  The call zeroes it first.
 * cfg->T is not used. */
moe_status_t moe_pack_weights(const moe_cfg_t *cfg, const void *w1, const void *w3, const void *w2,
                              const void *ws1, const void *ws3, const void *ws2, void *w13_out,
                              void *w2_out, int32_t *w2_inexact, void *stream);

/* Router ("Mixture of experts" equations z = x W_r, s = sigmoid(z),
 * E_sel = top_K(s + b), G = scale * s E_sel / sum s E_sel).
 *   x:         bf16 [T][H]
 *   w_router:  fp32 [E][H]   (W_r stored [out, in])
 *   bias:      fp32 [E]      (e_score_correction_bias; used only to choose)
 *   topk_idx:  int32 [T][K]  out: selected experts, slot order = descending
 *              s + b, equal keys in ascending expert index
 *   topk_gate: fp32 [T][K]   out: G per slot (sums to routed_scale)
 *   margin:    fp32 [T] or NULL; out: (K-th key) - ((K+1)-th key) in the
 *              same order, +inf when K == E.
 *   logits:    fp32 [T][E] or NULL; out: z, the router logits before the
 *              sigmoid and the bias (the pages' router_logits value).
 *   ws, ws_bytes: workspace of at least moe_workspace_size(cfg) bytes (holds
 *              the bf16 split of W_r and, for small T, the partial logits).
 * z is computed on the tensor cores from an exact three-part bf16 split of
 * W_r (each product exact, fp32 accumulation): fp32-accurate logits.  This
 * call makes the split into the workspace every time (one small extra
 * kernel); moe_pack_router + moe_route_packed make it once. */
moe_status_t moe_route(const moe_cfg_t *cfg, const void *x, const float *w_router, const float *bias,
                       int32_t *topk_idx, float *topk_gate, float *margin, float *logits, void *ws,
                       size_t ws_bytes, void *stream);

/* Bytes of the packed router weights for cfg (2 * 3 * E_pad * H, E_pad = E
 * rounded up to 64).  0 for an invalid cfg. */
size_t moe_router_packed_size(const moe_cfg_t *cfg);

/* The exact three-part bf16 split of the router weights, made once:
 *   w_router_packed: [3][E_pad][H] bf16, part p row e = the p-th bf16 term of
 *   W_r[e] (hi = bf16(W), mid = bf16(W - hi), lo = bf16(W - hi - mid); the
 *   remainder is below 2^-24 |W|), rows E..E_pad-1 zero.  16-byte aligned,
 *   moe_router_packed_size(cfg) bytes.  cfg->T is not used. */
moe_status_t moe_pack_router(const moe_cfg_t *cfg, const float *w_router, void *w_router_packed,
                             void *stream);

/* moe_route with pre-packed router weights: logits, scores, biased top-K,
 * margin and gates in ONE kernel (for large T one CTA per 128 tokens selects
 * from the logits it holds, which reach global memory only if `logits` is
 * given; for small T the H range is split over several CTAs that meet at a
 * grid barrier bounded in time, MOE_ERR_TIMEOUT if it runs out, and sum their
 * partials in a fixed order).  Arguments as moe_route, with w_router_packed
 * from moe_pack_router in place of w_router.  Deterministic. */
moe_status_t moe_route_packed(const moe_cfg_t *cfg, const void *x, const void *w_router_packed,
                              const float *bias, int32_t *topk_idx, float *topk_gate, float *margin,
                              float *logits, void *ws, size_t ws_bytes, void *stream);

/* Expert-sorted permutation of the T*K assignments (deterministic).
 *   topk_idx: int32 [T][K] (as written by moe_route, or by the caller)
 *   counts:   int32 [E+1]  out: rows per group; counts[E] = T if has_shared
 *   offsets:  int32 [E+2]  out: exclusive prefix sum of counts
 *   sorted:   int32 [T*K + T*has_shared] out: sorted[offsets[g] + r] = row id
 *             of the r-th row of group g in ascending token order; a routed
 *             row id is t*K + slot, a shared row id is T*K + t.
 *   ws, ws_bytes: workspace of at least moe_workspace_size(cfg) bytes.
 * An id outside [0, E) is skipped and flagged MOE_ERR_BAD_INDEX on the device.
 * Up to 151552 assignments (at most one 1024-assignment chunk per SM) this is
 * one launch whose CTAs meet at a grid barrier bounded in time: MOE_ERR_TIMEOUT
 * on the device if they cannot all be resident at once (e.g. another stream's
 * kernels hold the SMs), the outputs then undefined. */
moe_status_t moe_permute(const moe_cfg_t *cfg, const int32_t *topk_idx, int32_t *counts,
                         int32_t *offsets, int32_t *sorted, void *ws, size_t ws_bytes, void *stream);

/* Expert FFNs and combine:
 *   y[t] = sum over slots k = 0..K-1 (in order) of topk_gate[t][k] * E_{idx}(x_t)
 *          + shared(x_t)   (fp16 per-slot outputs summed in fp32, one final
 *          rounding to bf16; an intermediate beyond the fp16 range saturates
 *          and is flagged MOE_ERR_RANGE on the device).
 * Gates are used AS GIVEN (no renormalisation), so a caller may zero or edit
 * them (expert ablation).  Inputs: x bf16 [T][H]; topk_gate fp32 [T][K];
 * offsets, sorted from moe_permute.  Output y: bf16 [T][H].
 * The intermediate activations live in the workspace. */
moe_status_t moe_forward(const moe_cfg_t *cfg, const moe_weights_t *weights, const void *x,
                         const float *topk_gate, const int32_t *offsets, const int32_t *sorted,
                         void *y, void *ws, size_t ws_bytes, void *stream);

/* The four stages moe_forward runs, in this order, exposed separately so a
 * caller can time or overlap them.  They communicate through the workspace
 * (token rows in expert-sorted order, the intermediate h and the per-slot
 * outputs), so the same ws, cfg, offsets and sorted must be used for all four.
 * offsets and sorted are checked on the device as they are read: a group whose
 * range is malformed (first offset not 0, an end before its start or past the
 * T*K + T*has_shared rows) is skipped and a row id outside the rows is ignored,
 * both flagged MOE_ERR_BAD_INDEX; nothing outside the buffers is accessed.
 *
 * Test-only switch: with the environment variable SRM_MOE_INJECT_STALL=1 at
 * the time of the call, moe_expert_up (and dsa_scores) issue no operand loads,
 * so their bounded pipeline waits run out and the call reports MOE_ERR_TIMEOUT
 * through the error word.  It exists for failure-detection tests; leave it
 * unset in production.
 *
 * moe_gather_tokens: copies the token rows of x into expert-sorted order in
 *   the workspace (row p = x of the token of sorted[p]; each row of x is read
 *   once and written to its K + 1 positions).  x: bf16 [T][H]. */
moe_status_t moe_gather_tokens(const moe_cfg_t *cfg, const void *x, const int32_t *sorted, void *ws,
                               size_t ws_bytes, void *stream);

/* moe_expert_up: for every group g and its rows (the gathered token rows),
 *   h = silu(x W1_g) (.) (x W3_g)  ("GLM-5 . MoE transformer block", Mixture
 *   of experts: g = x W1, u = x W3, a = g sigmoid(g), h = a (.) u); h is kept
 *   in fp16 in the workspace (magnitudes above 65504 saturate and are flagged
 *   MOE_ERR_RANGE).  Needs moe_gather_tokens first. */
moe_status_t moe_expert_up(const moe_cfg_t *cfg, const moe_weights_t *weights,
                           const int32_t *offsets, const int32_t *sorted, void *ws, size_t ws_bytes,
                           void *stream);

/* moe_expert_down: per row, E_g = h W2_g multiplied by that row's gate
 *   (topk_gate[t][slot]; 1 for the shared expert), written in fp16 to the
 *   row's (token, slot) position in the workspace ("expert_outputs: each
 *   routing slot's weighted expert output", nnterp GLM-5 page, The API). */
moe_status_t moe_expert_down(const moe_cfg_t *cfg, const moe_weights_t *weights,
                             const float *topk_gate, const int32_t *offsets, const int32_t *sorted,
                             void *ws, size_t ws_bytes, void *stream);

/* moe_combine: y[t] = (sum of the K slot outputs of token t, slots in order)
 *   + the shared expert's output, in fp32, rounded once to bf16 [T][H]
 *   (Delta_ffn = y_routed + y_shared). */
moe_status_t moe_combine(const moe_cfg_t *cfg, void *y, void *ws, size_t ws_bytes, void *stream);

/* moe_permute for callers that cannot allocate device memory (the pages have
 * no counterpart of this entry point; it exists for embedding).  Some hosts
 * cannot call cudaMalloc for a workspace: an engine that has reserved all
 * device memory for its own pool, a serving loop where cudaMalloc's implicit
 * device-wide synchronisation is not allowed, or a plugin that only receives
 * the tensors it works on.  This variant computes exactly what moe_permute
 * computes (same counts, offsets and sorted, bit for bit) with its scratch in
 * a static device array inside the library instead of a workspace.
 *   Limit: T * K <= 262144 (e.g. 32768 tokens at top-8), E <= 256; larger
 *   calls return MOE_ERR_UNSUPPORTED before any launch.
 *   Memory: every GPU that loads the library holds the array (about 256 KB)
 *   until the process exits.
 *   Set-up: the first call on each device looks up the array's device address
 *   (with that device current) and keeps it until the process exits; make that
 *   first call before any stream capture.  Resetting the device
 *   (cudaDeviceReset) after that is not supported.  Device ordinals 0-63 are
 *   supported (MOE_ERR_UNSUPPORTED otherwise).
 *   Sharing: all calls use the same array and it keeps the last call's
 *   contents (each call clears its error word first); calls that overlap on
 *   the GPU (unordered streams) race on it.
 *   Errors: an expert id outside [0, E) is skipped and reported in-band by
 *   setting offsets[0] = -1 (always 0 otherwise); the outputs are then not
 *   usable. */
moe_status_t moe_permute_noalloc(const moe_cfg_t *cfg, const int32_t *topk_idx, int32_t *counts,
                                 int32_t *offsets, int32_t *sorted, void *stream);

/* moe_combine followed by the block's residual add in the same pass
 * ("GLM-5 . MoE transformer block", All 43 steps: x_{n+1} = x'_n + Delta_ffn):
 *   y[t] = residual[t] + (sum of the K slot outputs, in order) + shared output,
 * in fp32, rounded once to bf16.  residual: bf16 [T][H] (x'_n, the stream the
 * pre-FFN RMSNorm read); NULL gives moe_combine. */
moe_status_t moe_combine_residual(const moe_cfg_t *cfg, const void *residual, void *y, void *ws,
                                  size_t ws_bytes, void *stream);

/* The decoder block's pre-FFN RMSNorm (All 43 steps: x_ffn = RMSNorm(x'_n)):
 *   x_ffn[t][h] = x[t][h] * gamma[h] / sqrt(mean_h x[t][h]^2 + eps)
 * in fp32, rounded once to bf16.  x, x_ffn: bf16 [T][H]; gamma: bf16 [H] (the
 * norm's weight); eps = rms_norm_eps (1e-5 in the GLM configs).  Only cfg->T
 * and cfg->H are used (cfg must still be valid). */
moe_status_t moe_rmsnorm(const moe_cfg_t *cfg, const void *x, const void *gamma, float eps,
                         void *x_ffn, void *stream);

/* The dense SwiGLU MLP of the first decoder blocks (GLM-5: blocks 0-2, 6144 ->
 * intermediate_size 12288; GLM-4.7-Flash: block 0, 2048 -> 10240; nnterp
 * Config sections and printouts), run through the same tensor-core kernels as
 * one group: y[t] = (residual[t] +) W2 (silu(W1 x_t) (.) W3 x_t).
 *   cfg:      E = 0, K = 0, has_shared = 1, I = the MLP's intermediate size
 *             (moe_workspace_size and moe_pack_weights accept this form; pack
 *             the MLP's gate/up/down weights as the shared expert ws1/ws3/ws2,
 *             w1/w3/w2 may be NULL)
 *   x:        bf16 [T][H];  residual: bf16 [T][H] or NULL;  y: bf16 [T][H]. */
moe_status_t moe_dense_mlp(const moe_cfg_t *cfg, const moe_weights_t *weights, const void *x,
                           const void *residual, void *y, void *ws, size_t ws_bytes, void *stream);

/* Read (and clear) the device error word of a workspace.  Synchronises
 * `stream`.  *device_status receives MOE_OK or the first device-side error
 * recorded since the last read.  Returns MOE_ERR_CUDA if the copy fails. */
moe_status_t moe_get_device_error(void *ws, moe_status_t *device_status, void *stream);

/* Static English description of a status code (never NULL). */
const char *moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SRM_MOE_H */
