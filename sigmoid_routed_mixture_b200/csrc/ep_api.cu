// ep_api.cu -- host side of the expert-parallel calls declared in
// include/srm_ep.h: argument validation and the launches of ep.cu's kernels,
// asynchronous on the caller's stream.  (moe_ep_shared, which runs the grouped
// GEMMs, lives in api.cu with the other GEMM launches.)
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/srm_ep.h"
#include "../../include/srm_moe.h"
#include "host_util.h"
#include "kernels.h"

namespace {

using namespace srm::host;

// The error word is the first int of every workspace of this library.
int *error_word(void *ws) { return static_cast<int *>(ws); }

bool valid_cfg(const moe_cfg_t *cfg) { return cfg && moe_workspace_size(cfg) != 0; }

// expert_first: 0 = f[0] < f[1] < ... < f[R] = E
bool valid_partition(const int32_t *first, int n_ranks, int E, srm::EpInts *out) {
  if (!first || first[0] != 0 || first[n_ranks] != E) return false;
  for (int r = 0; r < n_ranks; ++r)
    if (first[r + 1] <= first[r]) return false;
  for (int r = 0; r <= srm::kEpMaxRanks; ++r) out->v[r] = r <= n_ranks ? first[r] : E;
  return true;
}

}  // namespace

extern "C" {

moe_status_t moe_ep_plan(const moe_cfg_t *cfg, int32_t n_ranks, int32_t rank,
                         const int32_t *expert_first, const int32_t *counts_all, int32_t *dst_row,
                         int32_t *recv_offsets, int32_t *recv_sorted, int64_t max_rows, void *ws,
                         void *stream) {
  if (!valid_cfg(cfg)) return MOE_ERR_ARG;
  if (n_ranks < 1 || n_ranks > MOE_EP_MAX_RANKS || rank < 0 || rank >= n_ranks || max_rows < 0)
    return MOE_ERR_ARG;
  srm::EpInts first;
  if (!valid_partition(expert_first, n_ranks, cfg->E, &first)) return MOE_ERR_ARG;
  if (!counts_all || !dst_row || !recv_offsets || !ws || (max_rows > 0 && !recv_sorted))
    return MOE_ERR_ARG;
  if (!aligned(counts_all, 4) || !aligned(dst_row, 4) || !aligned(recv_offsets, 4) ||
      (recv_sorted && !aligned(recv_sorted, 4)) || !aligned(ws, 256))
    return MOE_ERR_ALIGN;
  return cuda_status(srm::launch_ep_plan(n_ranks, rank, cfg->E, first, counts_all, dst_row,
                                         recv_offsets, recv_sorted, max_rows, error_word(ws),
                                         num_sms(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_dispatch(const moe_cfg_t *cfg, int32_t n_ranks, int32_t rank,
                             const int32_t *expert_first, const int32_t *dst_row, const void *x,
                             const float *topk_gate, const int32_t *offsets, const int32_t *sorted,
                             const moe_ep_peers_t *recv_x, const moe_ep_peers_t *recv_gate,
                             const moe_ep_peers_t *recv_src, const int64_t *recv_capacity, void *ws,
                             void *stream) {
  if (!valid_cfg(cfg)) return MOE_ERR_ARG;
  if (n_ranks < 1 || n_ranks > MOE_EP_MAX_RANKS || rank < 0 || rank >= n_ranks) return MOE_ERR_ARG;
  srm::EpInts first;
  if (!valid_partition(expert_first, n_ranks, cfg->E, &first)) return MOE_ERR_ARG;
  if (cfg->T == 0) return MOE_OK;
  if (!dst_row || !x || !topk_gate || !offsets || !sorted || !recv_x || !recv_gate || !recv_src ||
      !recv_capacity || !ws)
    return MOE_ERR_ARG;
  if (!aligned(x, 16) || !aligned(topk_gate, 4) || !aligned(offsets, 4) || !aligned(sorted, 4) ||
      !aligned(dst_row, 4) || !aligned(ws, 256))
    return MOE_ERR_ALIGN;
  srm::EpPtrs px = {}, pg = {}, ps = {};
  srm::EpI64 cap = {};
  for (int r = 0; r < n_ranks; ++r) {
    if (recv_capacity[r] < 0) return MOE_ERR_ARG;
    if (recv_capacity[r] > 0 && (!recv_x->ptr[r] || !recv_gate->ptr[r] || !recv_src->ptr[r]))
      return MOE_ERR_ARG;
    if (!aligned(recv_x->ptr[r], 16) || !aligned(recv_gate->ptr[r], 4) || !aligned(recv_src->ptr[r], 8))
      return MOE_ERR_ALIGN;
    px.p[r] = recv_x->ptr[r];
    pg.p[r] = recv_gate->ptr[r];
    ps.p[r] = recv_src->ptr[r];
    cap.v[r] = recv_capacity[r];
  }
  return cuda_status(srm::launch_ep_dispatch(
      n_ranks, rank, static_cast<int>(cfg->T), cfg->H, cfg->E, cfg->K, first, cap, dst_row,
      static_cast<const uint16_t *>(x), topk_gate, offsets, sorted, px, pg, ps, error_word(ws),
      num_sms(), static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_return(const moe_cfg_t *owner_cfg, int32_t n_ranks, const int32_t *recv_src,
                           const moe_ep_peers_t *dst_y, const int32_t *dst_rows, void *owner_ws,
                           size_t owner_ws_bytes, void *stream) {
  if (!valid_cfg(owner_cfg) || owner_cfg->K != 1 || owner_cfg->has_shared != 0) return MOE_ERR_ARG;
  if (n_ranks < 1 || n_ranks > MOE_EP_MAX_RANKS) return MOE_ERR_ARG;
  if (owner_cfg->T == 0) return MOE_OK;
  if (!recv_src || !dst_y || !dst_rows || !owner_ws) return MOE_ERR_ARG;
  if (!aligned(recv_src, 8) || !aligned(owner_ws, 256)) return MOE_ERR_ALIGN;
  if (owner_ws_bytes < moe_workspace_size(owner_cfg)) return MOE_ERR_WORKSPACE;
  srm::EpPtrs py = {};
  srm::EpInts rows = {};
  for (int r = 0; r < n_ranks; ++r) {
    if (dst_rows[r] < 0) return MOE_ERR_ARG;
    if (dst_rows[r] > 0 && !dst_y->ptr[r]) return MOE_ERR_ARG;
    if (!aligned(dst_y->ptr[r], 16)) return MOE_ERR_ALIGN;
    py.p[r] = dst_y->ptr[r];
    rows.v[r] = dst_rows[r];
  }
  const uint8_t *wsb = static_cast<const uint8_t *>(owner_ws);
  const uint16_t *y_local =
      reinterpret_cast<const uint16_t *>(wsb + moe_workspace_offset(owner_cfg, MOE_WS_SLOT_OUTPUTS));
  return cuda_status(srm::launch_ep_return(n_ranks, static_cast<int>(owner_cfg->T), owner_cfg->H,
                                           recv_src, y_local, py, rows, error_word(owner_ws),
                                           num_sms(), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
