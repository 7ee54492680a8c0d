// ep.cu -- expert-parallel form of the mixture: the routed experts are split
// over R ranks (contiguous expert ranges), each routed assignment travels to
// the owner of its expert and its weighted output travels back.
//
// The method is unchanged ("GLM-5 . MoE transformer block", "All 43 steps",
// Mixture-of-experts equations): no term couples two tokens, so the rows of
// one expert can be computed wherever that expert's weights live.  The pages
// run one expert-parallel group ("ep_size": 1 in the GLM-5 config.json on the
// "Vocabulary projection" page); this file is the form the layer takes when
// the routed experts no longer fit one GPU's share of the node.
//
//   ep_plan_kernel:     from every rank's per-expert counts, where this
//                       rank's rows go (dst_row), and the offsets and row list
//                       of the rows it receives (one group per owned expert)
//   ep_dispatch_kernel: one warp per routed assignment of this rank: the token
//                       row (16-byte vectors), its gate and its back-reference
//                       (source rank, t*K + slot) stored into the owner's
//                       buffers -- plain stores, to peer memory over NVLink
//                       when the owner is another GPU (no staging copy, no TMA
//                       multicast)
//   ep_return_kernel:   one warp per received row: its fp16 weighted output
//                       stored into the source rank's per-slot output buffer
//                       at row t*K + slot, where the single-GPU path writes it
//
// Receive order: by expert, then source rank, then the source's token order,
// which fixes every row's position from the counts alone.  Every index is
// checked against the buffer it addresses; a bad one is skipped and flagged
// (MOE_ERR_BAD_INDEX, or MOE_ERR_WORKSPACE when a receive buffer is too
// small).  No kernel waits on another rank.
#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace {

__device__ __forceinline__ int owner_of(const EpInts &first, int n_ranks, int e) {
  int o = 0;
  while (o + 1 < n_ranks && first.v[o + 1] <= e) ++o;
  return o;
}

}  // namespace

// One CTA of 256 threads (E <= 256) computes the tables; every CTA writes a
// share of the identity row list.
__global__ void __launch_bounds__(256)
    ep_plan_kernel(int n_ranks, int rank, int E, EpInts first, const int32_t *__restrict__ counts_all,
                   int32_t *__restrict__ dst_row, int32_t *__restrict__ recv_offsets,
                   int32_t *__restrict__ recv_sorted, int64_t max_rows, int *err) {
  __shared__ int incl[256];  // inclusive scan over the experts of tot[e] = rows of e, all sources
  const int e = threadIdx.x;
  int tot = 0, before = 0;  // before: rows of e from sources below this rank
  if (e < E) {
    for (int s = 0; s < n_ranks; ++s) {
      const int c = counts_all[s * E + e];
      tot += c;
      if (s < rank) before += c;
    }
  }
  incl[e] = tot;
  __syncthreads();
  for (int d = 1; d < 256; d <<= 1) {  // Hillis-Steele
    const int v = e >= d ? incl[e - d] : 0;
    __syncthreads();
    incl[e] += v;
    __syncthreads();
  }
  // rows of experts [0, g) over all sources, for 0 <= g <= E
  auto start = [&](int g) { return g > 0 ? incl[g - 1] : 0; };
  const int f0 = first.v[rank], f1 = first.v[rank + 1];
  const int total = start(f1) - start(f0);  // rows this rank receives
  if (blockIdx.x == 0) {
    if (e < E) dst_row[e] = start(e) - start(first.v[owner_of(first, n_ranks, e)]) + before;
    if (e < f1 - f0) recv_offsets[e] = start(f0 + e) - start(f0);
    if (e == 0) {
      recv_offsets[f1 - f0] = total;       // end of the last owned expert
      recv_offsets[f1 - f0 + 1] = total;   // an empty shared group
      if (total > max_rows) record_error(err, MOE_ERR_WORKSPACE);
    }
  }
  const int64_t n = total < max_rows ? total : max_rows;
  for (int64_t i = blockIdx.x * 256 + e; i < n; i += static_cast<int64_t>(gridDim.x) * 256)
    recv_sorted[i] = static_cast<int32_t>(i);
}

// One warp per routed position p of this rank's expert-sorted list.
__global__ void __launch_bounds__(256)
    ep_dispatch_kernel(int n_ranks, int rank, int T, int H, int E, int K, EpInts first, EpI64 capacity,
                       const int32_t *__restrict__ dst_row, const uint16_t *__restrict__ x,
                       const float *__restrict__ gate, const int32_t *__restrict__ offsets,
                       const int32_t *__restrict__ sorted, EpPtrs recv_x, EpPtrs recv_gate,
                       EpPtrs recv_src, int *err) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int n_routed = offsets[E];
  if (n_routed < 0 || n_routed > T * K) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(err, MOE_ERR_BAD_INDEX);
    return;
  }
  const int vecs = H / 8;
  for (int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < n_routed; p += warps) {
    int lo = 0, hi = E - 1;  // last e with offsets[e] <= p
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (offsets[mid] <= p)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int e = lo;
    const int a = sorted[p];
    const int o = owner_of(first, n_ranks, e);
    const int64_t dst = static_cast<int64_t>(dst_row[e]) + (p - offsets[e]);
    if (a < 0 || a >= T * K || dst < 0) {
      if (lane == 0) record_error(err, MOE_ERR_BAD_INDEX);
      continue;
    }
    if (dst >= capacity.v[o]) {
      if (lane == 0) record_error(err, MOE_ERR_WORKSPACE);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(a / K) * H);
    uint4 *out = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(recv_x.p[o]) + dst * H);
    for (int v = lane; v < vecs; v += 32) out[v] = src[v];
    if (lane == 0) {
      static_cast<float *>(recv_gate.p[o])[dst] = gate[a];
      int2 *ref = static_cast<int2 *>(recv_src.p[o]);
      ref[dst] = make_int2(rank, a);
    }
  }
  __threadfence_system();  // the peer stores are visible before the caller's barrier
}

// One warp per received row.
__global__ void __launch_bounds__(256)
    ep_return_kernel(int n_ranks, int rows, int H, const int32_t *__restrict__ recv_src,
                     const uint16_t *__restrict__ y_local, EpPtrs dst_y, EpInts dst_rows, int *err) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int vecs = H / 8;
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < rows; i += warps) {
    const int2 ref = reinterpret_cast<const int2 *>(recv_src)[i];
    if (ref.x < 0 || ref.x >= n_ranks || ref.y < 0 || ref.y >= dst_rows.v[ref.x]) {
      if (lane == 0) record_error(err, MOE_ERR_BAD_INDEX);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(y_local + static_cast<size_t>(i) * H);
    uint4 *out = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(dst_y.p[ref.x]) +
                                           static_cast<size_t>(ref.y) * H);
    for (int v = lane; v < vecs; v += 32) out[v] = src[v];
  }
  __threadfence_system();
}

cudaError_t launch_ep_plan(int n_ranks, int rank, int E, const EpInts &expert_first,
                           const int32_t *counts_all, int32_t *dst_row, int32_t *recv_offsets,
                           int32_t *recv_sorted, int64_t max_rows, int *err, int num_sms,
                           cudaStream_t stream) {
  int blocks = static_cast<int>((max_rows + 255) / 256);
  if (blocks > num_sms * 4) blocks = num_sms * 4;
  if (blocks < 1) blocks = 1;
  ep_plan_kernel<<<blocks, 256, 0, stream>>>(n_ranks, rank, E, expert_first, counts_all, dst_row,
                                             recv_offsets, recv_sorted, max_rows, err);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(int n_ranks, int rank, int T, int H, int E, int K,
                               const EpInts &expert_first, const EpI64 &capacity,
                               const int32_t *dst_row, const uint16_t *x, const float *gate,
                               const int32_t *offsets, const int32_t *sorted, const EpPtrs &recv_x,
                               const EpPtrs &recv_gate, const EpPtrs &recv_src, int *err,
                               int num_sms, cudaStream_t stream) {
  int blocks = (T * K + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  if (blocks < 1) blocks = 1;
  ep_dispatch_kernel<<<blocks, 256, 0, stream>>>(n_ranks, rank, T, H, E, K, expert_first, capacity,
                                                 dst_row, x, gate, offsets, sorted, recv_x, recv_gate,
                                                 recv_src, err);
  return cudaGetLastError();
}

cudaError_t launch_ep_return(int n_ranks, int rows, int H, const int32_t *recv_src,
                             const uint16_t *y_local, const EpPtrs &dst_y, const EpInts &dst_rows,
                             int *err, int num_sms, cudaStream_t stream) {
  int blocks = (rows + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  if (blocks < 1) blocks = 1;
  ep_return_kernel<<<blocks, 256, 0, stream>>>(n_ranks, rows, H, recv_src, y_local, dst_y, dst_rows,
                                               err);
  return cudaGetLastError();
}

}  // namespace srm
