// kernels.h -- internal launch interface between the C-ABI host layer
// (api.cu) and the CUDA kernels of libsrm_moe.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace srm {

constexpr int kUp = 0;    // W1|W3 contraction + SwiGLU epilogue
constexpr int kDown = 1;  // W2 contraction + gate epilogue

struct GemmArgs {
  const int32_t *offsets;  // [groups + 1] first expert-sorted row of each group
  const int32_t *sorted;   // expert-sorted row ids (t*K + slot, or T*K + t for the shared expert)
  const float *gate;       // [T*K] routing gates (kDown)
  void *out;               // kUp: h fp16 [rows][I];  kDown: Y fp16 [n_rows_y][H]
  int *err;                // device error word
  int T;
  int K;
  int tk;                  // T * K
  int n_rows_y;            // T*K + T*has_shared: valid row ids are [0, n_rows_y)
  int groups;              // E + has_shared
  int n_total;             // output columns per group (2I for kUp, H for kDown)
  int k_total;             // reduction length (H for kUp, I for kDown)
  int out_ld;              // elements per output row (I for kUp, H for kDown)
  int *tile_counter;       // zeroed before the launch; units take their next tile from it
  int stall;               // failure-detection tests only: the producer issues no loads, so
                           // the MMA warp's bounded wait runs out (MOE_ERR_TIMEOUT)
};

// Tile shape of the grouped GEMMs: the weights are the MMA's M side (256 rows
// per CTA pair, 128 per single CTA), the tokens its N side (up to 256 per
// tile, rounded up to 16).  CTA pairs unless the experts average fewer than 8
// rows each.  Tensor maps: tokens [rows][K] (TokMaps), weights [rows][K] with
// boxes of gemm_w_box_rows() rows, 64 K-elements wide, 128-byte swizzle.
bool gemm_use_pairs(int64_t T, int K, int E);
int gemm_tok_box_rows();
int gemm_tok_big_box_rows();
int gemm_w_box_rows();
// the token rows as two tensor maps over the same memory: boxes of
// gemm_tok_box_rows() rows (tail tiles) and gemm_tok_big_box_rows() rows (full tiles)
struct TokMaps {
  CUtensorMap small, big;
};
cudaError_t launch_grouped_gemm(int mode, bool pair, const TokMaps &tok, const CUtensorMap &tmap_w,
                                const GemmArgs &p, int num_sms, cudaStream_t stream);

// router: W_r split into bf16 parts [3][e_pad][H] (wsplit), fp32 partial logits
// zp [splits][T][e_pad] (split-K only); tmap_x: x [T][H] box 64 x 128,
// tmap_w: wsplit [3*e_pad][H] box 64 x router_w_box_rows; grid_counter: an int zeroed
// before the launch (split-K grid barrier)
int router_e_pad(int E);
int router_splits(int T, int H);  // upper bound of the split count (workspace sizing)
int router_grid_splits(int T, int H, int num_sms);
// without a split, CTA pairs: tmap_w's box is then e_pad / 2 rows (router_w_box_rows)
bool router_use_pairs(int T, int H, int num_sms);
int router_w_box_rows(int E, bool pair);
cudaError_t launch_router_split(const float *w_r, int E, int H, uint16_t *wsplit, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_route(const CUtensorMap &tmap_x, const CUtensorMap &tmap_w, const float *bias, int T,
                         int H, int E, int K, float scale, float *zp, int *grid_counter,
                         int32_t *idx, float *gate, float *margin, float *logits, int *err,
                         int num_sms, cudaStream_t stream);

// chunk scratch: int32 [E * nchunks]; with a grid counter (one int, zeroed
// here) and at most num_sms chunks, one fused launch instead of three
int permute_num_chunks(int64_t n_assign);
cudaError_t launch_permute(const int32_t *idx, int T, int E, int K, int has_shared, int32_t *counts,
                           int32_t *offsets, int32_t *sorted, int32_t *chunk_scratch, int *err,
                           cudaStream_t stream, int *grid_counter = nullptr, int num_sms = 0);

// token rows in expert-sorted order: xs[p] = x[token of sorted[p]]; pos is
// int32 scratch [rows] (row id -> sorted position)
cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *sorted, int T, int H, int K,
                               int has_shared, int32_t *pos, uint16_t *xs, int *err, int num_sms,
                               cudaStream_t stream);

// y = (residual +) sum of slot outputs + shared output; residual may be NULL
cudaError_t launch_combine(const uint16_t *Y, const uint16_t *residual, uint16_t *y, int T, int H,
                           int K, int has_shared, int num_sms, cudaStream_t stream);

// offsets = {0, T}, sorted[t] = base + t: every token in one group, in order
cudaError_t launch_identity_rows(int32_t *offsets, int32_t *sorted, int T, int num_sms,
                                 cudaStream_t stream, int base = 0);

// expert-parallel dispatch / return (ep.cu); peers: one device pointer per rank
constexpr int kEpMaxRanks = 8;
struct EpPtrs {
  void *p[kEpMaxRanks];
};
struct EpInts {
  int v[kEpMaxRanks + 1];
};
struct EpI64 {
  int64_t v[kEpMaxRanks];
};
cudaError_t launch_ep_plan(int n_ranks, int rank, int E, const EpInts &expert_first,
                           const int32_t *counts_all, int32_t *dst_row, int32_t *recv_offsets,
                           int32_t *recv_sorted, int64_t max_rows, int *err, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_ep_dispatch(int n_ranks, int rank, int T, int H, int E, int K,
                               const EpInts &expert_first, const EpI64 &capacity,
                               const int32_t *dst_row, const uint16_t *x, const float *gate,
                               const int32_t *offsets, const int32_t *sorted, const EpPtrs &recv_x,
                               const EpPtrs &recv_gate, const EpPtrs &recv_src, int *err,
                               int num_sms, cudaStream_t stream);
cudaError_t launch_ep_return(int n_ranks, int rows, int H, const int32_t *recv_src,
                             const uint16_t *y_local, const EpPtrs &dst_y, const EpInts &dst_rows,
                             int *err, int num_sms, cudaStream_t stream);

cudaError_t launch_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int T, int H,
                           uint16_t *out, int num_sms, cudaStream_t stream);

cudaError_t launch_pack(const uint16_t *w1, const uint16_t *w3, const uint16_t *w2,
                        const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2, int H, int I,
                        int E, int has_shared, uint16_t *w13_out, uint16_t *w2_out,
                        int32_t *w2_inexact, int num_sms, cudaStream_t stream);

// ---- sparse-attention key selection (dsa.cu)
constexpr int kDsaMaxKeys = 32768;  // keys per sequence the top-k kernel holds in registers
int dsa_units_bound(int T, int S, int n_heads);
int dsa_query_rows_per_tile(int T, int n_heads);
cudaError_t launch_dsa_scores(const CUtensorMap &tq, const CUtensorMap &tk, const float *w,
                              float *scores, int2 *units, int *ctl, int64_t B, int T, int S,
                              int n_heads, int head_dim, float scale, int *err, int stall,
                              int num_sms, cudaStream_t stream);
cudaError_t launch_dsa_topk(const float *scores, int64_t B, int T, int S, int topk, int32_t *sel,
                            cudaStream_t stream);

}  // namespace srm
