/*
 * srm_ep.h -- C ABI of the expert-parallel form of the sigmoid-routed
 * mixture-of-experts FFN (one process per GPU, the routed experts split over
 * the GPUs of one NVSwitch node).  Same library as srm_moe.h
 * (libsrm_moe.so); status codes and the device error word are srm_moe.h's.
 *
 * The method is the one srm_moe.h computes ("GLM-5 . MoE transformer block",
 * "All 43 steps", Mixture-of-experts equations); the pages run it with one
 * expert-parallel group (GLM-5 config.json on the "Vocabulary projection"
 * page: "ep_size": 1).  Nothing couples two tokens, so the layer can also be
 * split by expert: rank r of R owns the routed experts
 * [expert_first[r], expert_first[r+1]) (contiguous ranges, every rank at least
 * one expert); the shared expert runs on every rank for that rank's own tokens.
 * One step, on every rank (each with its own T tokens):
 *   1. moe_route, moe_permute on the rank's tokens (srm_moe.h);
 *   2. every rank learns every rank's per-expert counts (an all-gather of
 *      counts[0..E), e.g. NCCL; the caller's job) and calls moe_ep_plan;
 *   3. moe_ep_dispatch: each routed assignment's token row and gate go to the
 *      owner of its expert (stores into the owner's buffers: peer memory on
 *      NVLink, no staging copy, no TMA multicast);
 *   4. after a barrier: each owner runs moe_expert_up and moe_expert_down
 *      (srm_moe.h) on what it received, as a block of its own ("owner cfg":
 *      T = rows received, K = 1, E = its expert count, has_shared = 0, the
 *      offsets and row list from moe_ep_plan);
 *   5. moe_ep_return: each owner stores every row's fp16 weighted output into
 *      the per-slot output buffer of the rank the row came from, at the row
 *      the single-GPU path uses (t*K + slot);
 *   6. after a barrier: each rank runs moe_ep_shared (its shared expert) and
 *      moe_combine (srm_moe.h).
 * The per-row arithmetic and the fixed-order combine are those of the
 * single-GPU path, so y equals moe_forward's on the same tokens, bit for bit.
 * Received rows are ordered by expert, then source rank, then token: the
 * layout does not depend on timing.
 *
 * Peer buffers: the arrays of device pointers below (one per rank, at most
 * MOE_EP_MAX_RANKS) must be usable from the calling GPU (the caller maps its
 * peers' buffers, e.g. through CUDA IPC or symmetric memory, and enables peer
 * access); on one GPU they may all be local ("virtual ranks").  The library
 * never waits for another rank: ordering between ranks (the barriers of steps
 * 4 and 6) is the caller's.
 */
#ifndef SRM_EP_H
#define SRM_EP_H

#include <stddef.h>
#include <stdint.h>

#include "srm_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_EP_MAX_RANKS 8

/* One device pointer per rank (entries past n_ranks are ignored). */
typedef struct {
    void *ptr[MOE_EP_MAX_RANKS];
} moe_ep_peers_t;

/* Receive layout of one step, from every rank's per-expert counts.
 *   cfg:          the SOURCE shape (H, I, E, K; T is not used)
 *   n_ranks, rank: 1 <= n_ranks <= MOE_EP_MAX_RANKS, 0 <= rank < n_ranks
 *   expert_first: HOST int32 [n_ranks + 1], 0 = expert_first[0] <
 *                 expert_first[1] < ... < expert_first[n_ranks] = E
 *   counts_all:   device int32 [n_ranks][E]: counts_all[s][e] = assignments of
 *                 rank s's tokens to expert e (moe_permute's counts[0..E))
 *   dst_row:      device int32 [E] out: row, in the buffers of the owner of
 *                 expert e, of this rank's first assignment to e (the rest
 *                 follow in this rank's token order)
 *   recv_offsets: device int32 [E_r + 2] out (E_r = this rank's expert count):
 *                 moe_permute-style offsets of the rows this rank receives
 *                 (its experts in order; the last two entries both equal the
 *                 total, an empty shared group)
 *   recv_sorted:  device int32 [max_rows] out: the row list of the owner cfg,
 *                 recv_sorted[i] = i for i below the total
 *   max_rows:     capacity of recv_sorted; a total above it is flagged
 *                 MOE_ERR_WORKSPACE in the error word of ws and nothing past
 *                 max_rows is written
 *   ws:           any workspace of this library (its error word is used)
 * The owner needs the total on the host to build its cfg: it is
 * recv_offsets[E_r] (or the sum of counts_all over its experts). */
moe_status_t moe_ep_plan(const moe_cfg_t *cfg, int32_t n_ranks, int32_t rank,
                         const int32_t *expert_first, const int32_t *counts_all, int32_t *dst_row,
                         int32_t *recv_offsets, int32_t *recv_sorted, int64_t max_rows, void *ws,
                         void *stream);

/* Step 3: send this rank's routed assignments to their owners.
 *   cfg:       the source shape (this rank's T)
 *   expert_first: HOST int32 [n_ranks + 1] as in moe_ep_plan
 *   dst_row:   from moe_ep_plan (this rank's)
 *   x:         bf16 [T][H]; topk_gate: fp32 [T][K]; offsets, sorted: this
 *              rank's moe_permute output
 *   recv_x:    per owner o, its token-row buffer: bf16 [rows_o][H], the
 *              MOE_WS_TOKEN_ROWS region of o's owner-cfg workspace
 *              (moe_workspace_offset), 16-byte aligned
 *   recv_gate: per owner, fp32 [rows_o] (the owner's topk_gate, K = 1)
 *   recv_src:  per owner, int32 [rows_o][2] = (source rank, source row id
 *              t*K + slot), 8-byte aligned
 *   recv_capacity: HOST int64 [n_ranks]: rows each owner's three buffers
 *              hold; a row at or past it is skipped and flagged
 *              MOE_ERR_WORKSPACE
 *   ws:        this rank's workspace (error word)
 * Row i of owner o receives x[t], G[t][slot] and (rank, t*K + slot). */
moe_status_t moe_ep_dispatch(const moe_cfg_t *cfg, int32_t n_ranks, int32_t rank,
                             const int32_t *expert_first, const int32_t *dst_row, const void *x,
                             const float *topk_gate, const int32_t *offsets, const int32_t *sorted,
                             const moe_ep_peers_t *recv_x, const moe_ep_peers_t *recv_gate,
                             const moe_ep_peers_t *recv_src, const int64_t *recv_capacity, void *ws,
                             void *stream);

/* Step 5: after moe_expert_down on the owner cfg (T = rows received, K = 1),
 * store each received row's fp16 output into the per-slot output buffer of
 * its source rank.
 *   owner_cfg: the owner cfg; owner_ws its workspace (holds the outputs)
 *   recv_src:  int32 [T][2] as written by moe_ep_dispatch
 *   dst_y:     per source rank s, the MOE_WS_SLOT_OUTPUTS region of s's
 *              workspace (moe_workspace_offset with s's own cfg)
 *   dst_rows:  HOST int32 [n_ranks]: T_s * K of each source (a row id at or
 *              above it is flagged MOE_ERR_BAD_INDEX and not stored) */
moe_status_t moe_ep_return(const moe_cfg_t *owner_cfg, int32_t n_ranks, const int32_t *recv_src,
                           const moe_ep_peers_t *dst_y, const int32_t *dst_rows, void *owner_ws,
                           size_t owner_ws_bytes, void *stream);

/* Step 6: the shared expert on this rank's own tokens, written where the
 * single-GPU path writes it (the per-slot output buffer's rows T*K + t), so
 * moe_combine can follow.
 *   cfg:    this rank's source cfg (has_shared = 1)
 *   shared: the shared expert's packed block (w13: bf16 [2I][H] in the
 *           moe_pack_weights layout of one group; w2: fp16 [H][I])
 *   x:      bf16 [T][H];  ws: this rank's workspace. */
moe_status_t moe_ep_shared(const moe_cfg_t *cfg, const moe_weights_t *shared, const void *x, void *ws,
                           size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SRM_EP_H */
