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

// Tile shape of the grouped GEMMs: CTA pairs with 256-row tiles when the
// experts get many rows each (T*K >= 512*E), single CTAs with 128-row tiles
// otherwise (less padding of each expert's last tile, more weight bytes in
// flight per SM for small batches).  A tiles are 128 rows; the B box has
// gemm_b_box_rows(pair) rows.
bool gemm_use_pairs(int64_t T, int K, int E);
int gemm_b_box_rows(bool pair);
cudaError_t launch_grouped_gemm(int mode, bool pair, const CUtensorMap &ta, const CUtensorMap &tb,
                                const GemmArgs &p, int num_sms, cudaStream_t stream);

// router: W_r split into bf16 parts [3][e_pad][H] (wsplit), fp32 partial logits
// zp [splits][T][e_pad]; tmap_x: x [T][H] box 64 x 128, tmap_w: wsplit [3*e_pad][H]
// box 64 x e_pad
int router_e_pad(int E);
int router_splits(int T, int H);
cudaError_t launch_route(const CUtensorMap &tmap_x, const CUtensorMap &tmap_w, const float *w_r,
                         const float *bias, int T, int H, int E, int K, float scale,
                         uint16_t *wsplit, float *zp, int32_t *idx, float *gate, float *margin,
                         float *logits, int *err, int num_sms, cudaStream_t stream);

// chunk scratch: int32 [E * nchunks]
int permute_num_chunks(int64_t n_assign);
cudaError_t launch_permute(const int32_t *idx, int T, int E, int K, int has_shared, int32_t *counts,
                           int32_t *offsets, int32_t *sorted, int32_t *chunk_scratch, int *err,
                           cudaStream_t stream);

// token rows in expert-sorted order: xs[p] = x[token of sorted[p]]; pos is
// int32 scratch [rows] (row id -> sorted position)
cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *sorted, int T, int H, int K,
                               int has_shared, int32_t *pos, uint16_t *xs, int *err, int num_sms,
                               cudaStream_t stream);

// y = (residual +) sum of slot outputs + shared output; residual may be NULL
cudaError_t launch_combine(const uint16_t *Y, const uint16_t *residual, uint16_t *y, int T, int H,
                           int K, int has_shared, int num_sms, cudaStream_t stream);

// offsets = {0, T}, sorted[t] = t: every token in one group, in order
cudaError_t launch_identity_rows(int32_t *offsets, int32_t *sorted, int T, int num_sms,
                                 cudaStream_t stream);

cudaError_t launch_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int T, int H,
                           uint16_t *out, int num_sms, cudaStream_t stream);

cudaError_t launch_pack(const uint16_t *w1, const uint16_t *w3, const uint16_t *w2,
                        const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2, int H, int I,
                        int E, int has_shared, uint16_t *w13_out, uint16_t *w2_out, int num_sms,
                        cudaStream_t stream);

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
