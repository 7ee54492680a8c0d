// dsa_api.cu -- host side of the C ABI declared in include/srm_dsa.h:
// validation, workspace layout, tensor maps and the launches of the
// sparse-attention key selection (dsa.cu), asynchronous on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "../../include/srm_dsa.h"
#include "host_util.h"
#include "kernels.h"

namespace {

using namespace srm::host;

// Workspace: [0, 256) control words (+0 the device error word read by
// moe_get_device_error, +128 the unit counter, +132 the number of planned
// units), then the unit list (int2 per entry), then room for the scores.
struct DsaLayout {
  size_t ctl, units, scores, total;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

moe_status_t check(const dsa_cfg_t *c) {
  if (!c) return MOE_ERR_ARG;
  if (c->B < 0 || c->T < 1 || c->S < c->T || c->topk < 1) return MOE_ERR_ARG;
  if (c->n_heads != 32 && c->n_heads != 64 && c->n_heads != 128) return MOE_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return MOE_ERR_UNSUPPORTED;
  if (c->topk > 65536 || c->S > srm::kDsaMaxKeys) return MOE_ERR_UNSUPPORTED;
  if (c->B * c->T * static_cast<int64_t>(c->n_heads) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->B * static_cast<int64_t>(c->S) >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->B * c->T * static_cast<int64_t>(c->S) >= (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(srm::dsa_units_bound(c->T, c->S, c->n_heads)) * c->B >=
      (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

DsaLayout layout(const dsa_cfg_t &c) {
  DsaLayout L;
  size_t off = 0;
  L.ctl = off;
  off += 256;
  L.units = off;
  off = align_up(off + sizeof(int2) * static_cast<size_t>(srm::dsa_units_bound(c.T, c.S, c.n_heads)),
                 256);
  L.scores = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(c.B) * c.T * c.S, 256);
  L.total = off;
  return L;
}

moe_status_t check_ws(const dsa_cfg_t *cfg, const void *ws, size_t ws_bytes, DsaLayout *L) {
  moe_status_t st = check(cfg);
  if (st != MOE_OK) return st;
  if (!ws) return MOE_ERR_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  *L = layout(*cfg);
  if (ws_bytes < L->total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status_t run_scores(const dsa_cfg_t *cfg, const void *q, const void *k, const float *w,
                        float *scores, uint8_t *wsb, const DsaLayout &L, cudaStream_t s) {
  const int64_t B = cfg->B;
  const int T = cfg->T, S = cfg->S, NH = cfg->n_heads, D = cfg->head_dim;
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, q, static_cast<uint64_t>(D), static_cast<uint64_t>(B) * T * NH, 64,
                 static_cast<uint32_t>(srm::dsa_query_rows_per_tile(T, NH))) ||
      !make_tmap(&tk, k, static_cast<uint64_t>(D), static_cast<uint64_t>(B) * S, 64, 128))
    return MOE_ERR_CUDA;
  const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(NH) * D));
  // failure-detection tests only: SRM_MOE_INJECT_STALL=1 makes the producer
  // arm no key copy, so the call ends with MOE_ERR_TIMEOUT after the wait limit
  const char *inject = getenv("SRM_MOE_INJECT_STALL");
  const int stall = (inject && inject[0] == '1') ? 1 : 0;
  return cuda_status(srm::launch_dsa_scores(
      tq, tk, w, scores, reinterpret_cast<int2 *>(wsb + L.units),
      reinterpret_cast<int *>(wsb + L.ctl + 128), B, T, S, NH, D, scale,
      reinterpret_cast<int *>(wsb + L.ctl), stall, num_sms(), s));
}

}  // namespace

extern "C" {

size_t dsa_workspace_size(const dsa_cfg_t *cfg) {
  if (check(cfg) != MOE_OK) return 0;
  return layout(*cfg).total;
}

moe_status_t dsa_scores(const dsa_cfg_t *cfg, const void *q, const void *k, const float *w,
                        float *scores, void *ws, size_t ws_bytes, void *stream) {
  if (check(cfg) == MOE_OK && cfg->B == 0) return MOE_OK;  // nothing to do
  DsaLayout L;
  moe_status_t st = check_ws(cfg, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (!q || !k || !w || !scores) return MOE_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(scores, 4))
    return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  if (cudaMemsetAsync(wsb + L.ctl, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  return run_scores(cfg, q, k, w, scores, wsb, L, s);
}

moe_status_t dsa_topk(const dsa_cfg_t *cfg, const float *scores, int32_t *sel, void *ws,
                      size_t ws_bytes, void *stream) {
  if (check(cfg) == MOE_OK && cfg->B == 0) return MOE_OK;  // nothing to do
  DsaLayout L;
  moe_status_t st = check_ws(cfg, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (!scores || !sel) return MOE_ERR_ARG;
  if (!aligned(scores, 4) || !aligned(sel, 4)) return MOE_ERR_ALIGN;
  return cuda_status(srm::launch_dsa_topk(scores, cfg->B, cfg->T, cfg->S, cfg->topk, sel,
                                          static_cast<cudaStream_t>(stream)));
}

moe_status_t dsa_select(const dsa_cfg_t *cfg, const void *q, const void *k, const float *w,
                        int32_t *sel, float *scores, void *ws, size_t ws_bytes, void *stream) {
  if (check(cfg) == MOE_OK && cfg->B == 0) return MOE_OK;  // nothing to do
  DsaLayout L;
  moe_status_t st = check_ws(cfg, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (!q || !k || !w || !sel) return MOE_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(sel, 4) ||
      (scores && !aligned(scores, 4)))
    return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  float *sc = scores ? scores : reinterpret_cast<float *>(wsb + L.scores);
  if (cudaMemsetAsync(wsb + L.ctl, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  st = run_scores(cfg, q, k, w, sc, wsb, L, s);
  if (st != MOE_OK) return st;
  return cuda_status(srm::launch_dsa_topk(sc, cfg->B, cfg->T, cfg->S, cfg->topk, sel, s));
}

}  // extern "C"
