// permute.cu -- deterministic expert-sorted permutation of the T*K routing
// assignments (histogram -> exclusive scan -> stable scatter).
//
// The pages route every token to K experts (expert_indices [batch, seq,
// top_k], nnterp GLM-5 page, The API table) and sum the experts' weighted
// outputs; grouping the assignments by expert is how the grouped GEMMs find
// their rows.  Result (identical to a sequential counting sort):
//   counts[g]  rows of group g (g == E: the shared expert, T rows)
//   offsets    exclusive prefix sum of counts, E + 2 entries
//   sorted     row ids of each group in ascending assignment order
//              (routed row id t*K + slot; shared row id T*K + t).
// No step depends on the order in which atomics land: the per-chunk
// histograms only count, and the scatter ranks entries with warp matches and
// per-warp counts in a fixed order.  Three forms: one CTA for small batches;
// one launch with a grid barrier while the 1024-assignment chunks fit one CTA
// per SM; histogram, scan and scatter kernels beyond that.
#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace pm {
constexpr int CHUNK = 1024;  // assignments per chunk
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int MAX_E = 256;
constexpr int SCAN_THREADS = 4 * MAX_E;
}  // namespace pm

int permute_num_chunks(int64_t n_assign) {
  return static_cast<int>((n_assign + pm::CHUNK - 1) / pm::CHUNK);
}

// 1) chunk histograms: scratch[c * E + e] = entries of chunk c equal to e
__global__ void __launch_bounds__(pm::THREADS)
    permute_hist_kernel(const int32_t *__restrict__ idx, int n, int E, int nchunks,
                        int32_t *__restrict__ scratch, int *err) {
  __shared__ int hist[pm::MAX_E];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += pm::THREADS) hist[e] = 0;
  __syncthreads();
  const int end = min(n, (c + 1) * pm::CHUNK);
  for (int i = c * pm::CHUNK + threadIdx.x; i < end; i += pm::THREADS) {
    const int e = idx[i];
    if (e < 0 || e >= E)
      record_error(err, MOE_ERR_BAD_INDEX);
    else
      atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += pm::THREADS) scratch[c * E + e] = hist[e];
}

// 2) one CTA: per-expert running sums over the chunks (turning the scratch
// into each chunk's first destination), counts, and the group offsets.  Four
// threads share an expert, each scanning a quarter of the chunks; for a fixed
// chunk consecutive threads read consecutive experts (coalesced).
__global__ void __launch_bounds__(pm::SCAN_THREADS)
    permute_scan_kernel(int32_t *__restrict__ scratch, int E, int nchunks, int T, int has_shared,
                        int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
  __shared__ int part_sum[4][pm::MAX_E];
  __shared__ int scan[pm::MAX_E];
  const int e = threadIdx.x % pm::MAX_E;
  const int q = threadIdx.x / pm::MAX_E;  // quarter of the chunk range
  const int per = (nchunks + 3) / 4;
  const int c0 = q * per, c1 = min(nchunks, c0 + per);
  int run = 0;
  if (e < E) {
    int c = c0;
    for (; c + 4 <= c1; c += 4) {  // four independent loads in flight
      const int v0 = scratch[(c + 0) * E + e], v1 = scratch[(c + 1) * E + e];
      const int v2 = scratch[(c + 2) * E + e], v3 = scratch[(c + 3) * E + e];
      scratch[(c + 0) * E + e] = run;
      scratch[(c + 1) * E + e] = run + v0;
      scratch[(c + 2) * E + e] = run + v0 + v1;
      scratch[(c + 3) * E + e] = run + v0 + v1 + v2;
      run += v0 + v1 + v2 + v3;
    }
    for (; c < c1; ++c) {
      const int v = scratch[c * E + e];
      scratch[c * E + e] = run;
      run += v;
    }
  }
  part_sum[q][e] = e < E ? run : 0;
  __syncthreads();
  if (q == 0) scan[e] = part_sum[0][e] + part_sum[1][e] + part_sum[2][e] + part_sum[3][e];
  __syncthreads();
  const int tot = scan[e];
  for (int d = 1; d < pm::MAX_E; d <<= 1) {  // inclusive Hillis-Steele scan over experts
    const int v = (q == 0 && e >= d) ? scan[e - d] : 0;
    __syncthreads();
    if (q == 0) scan[e] += v;
    __syncthreads();
  }
  const int excl = scan[e] - tot;
  if (e < E) {
    int before = excl;  // first destination of this quarter
    for (int qq = 0; qq < q; ++qq) before += part_sum[qq][e];
    for (int c = c0; c < c1; ++c) scratch[c * E + e] += before;
    if (q == 0) {
      counts[e] = tot;
      offsets[e] = excl;
    }
  }
  if (threadIdx.x == 0) {
    const int routed = scan[pm::MAX_E - 1];
    counts[E] = has_shared ? T : 0;
    offsets[E] = routed;
    offsets[E + 1] = routed + (has_shared ? T : 0);
  }
}

// 3) stable scatter of each chunk, entries in ascending order.
__global__ void __launch_bounds__(pm::THREADS)
    permute_scatter_kernel(const int32_t *__restrict__ idx, int n, int E, int nchunks,
                           const int32_t *__restrict__ scratch, int T, int has_shared,
                           const int32_t *__restrict__ offsets, int32_t *__restrict__ sorted) {
  __shared__ int cursor[pm::MAX_E];
  __shared__ int wcnt[pm::WARPS][pm::MAX_E];
  const int c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += pm::THREADS) cursor[e] = scratch[c * E + e];
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < pm::CHUNK / pm::THREADS; ++r) {
    for (int k = tid; k < pm::WARPS * pm::MAX_E; k += pm::THREADS) (&wcnt[0][0])[k] = 0;
    __syncthreads();
    const int i = c * pm::CHUNK + r * pm::THREADS + tid;
    int e = i < n ? idx[i] : -1;
    if (e >= E) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt_mask);
    if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(same);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += wcnt[w][e];
      sorted[cursor[e] + before + rank] = i;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += pm::THREADS) {
      int add = 0;
      for (int w = 0; w < pm::WARPS; ++w) add += wcnt[w][ee];
      cursor[ee] += add;
    }
    __syncthreads();
  }
  if (has_shared) {
    const int base = offsets[E];
    const int tk = n;
    for (int t = blockIdx.x * pm::THREADS + tid; t < T; t += gridDim.x * pm::THREADS)
      sorted[base + t] = tk + t;
  }
}

// Small batches (n <= SMALL_N assignments: decode, 4096 tokens at top-4): the same
// histogram -> scan -> stable scatter in ONE CTA, so the permutation costs one
// launch.  Warp w owns the contiguous assignments [w*S*32, (w+1)*S*32) (S steps
// of 32) and keeps them in registers:
//   1) each warp counts its segment per expert (warp matches; one writer per
//      expert per step, so no atomics);
//   2) per expert, an exclusive scan over the warps in order, offset by the
//      expert's first row (exclusive scan of the totals over the experts);
//   3) each warp walks its segment again and writes every entry to its
//      expert's running position: ascending entries keep ascending positions.
namespace pm {
constexpr int SMALL_THREADS = 1024;
constexpr int SMALL_WARPS = SMALL_THREADS / 32;
constexpr int SMALL_N = 4096;  // above this the three-kernel path is faster (16384: 39 us in one CTA)
constexpr int SMALL_STEPS = SMALL_N / SMALL_THREADS;  // 32-entry steps per warp
}  // namespace pm

__global__ void __launch_bounds__(pm::SMALL_THREADS)
    permute_small_kernel(const int32_t *__restrict__ idx, int n, int E, int T, int has_shared,
                         int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                         int32_t *__restrict__ sorted, int *err) {
  __shared__ int whist[pm::SMALL_WARPS][pm::MAX_E];  // counts, then running positions
  __shared__ int wsum[pm::MAX_E / 32];
  __shared__ int routed_total;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int k = tid; k < pm::SMALL_WARPS * pm::MAX_E; k += pm::SMALL_THREADS) (&whist[0][0])[k] = 0;
  const int steps = (n + pm::SMALL_THREADS - 1) / pm::SMALL_THREADS;
  const int seg0 = warp * steps * 32;
  int e_reg[pm::SMALL_STEPS];
#pragma unroll
  for (int j = 0; j < pm::SMALL_STEPS; ++j) {
    const int i = seg0 + j * 32 + lane;
    int e = -1;
    if (j < steps && i < n) {
      e = idx[i];
      if (e < 0 || e >= E) {
        record_error(err, MOE_ERR_BAD_INDEX);
        e = -1;
      }
    }
    e_reg[j] = e;
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < pm::SMALL_STEPS; ++j) {
    if (j >= steps) break;
    const int e = e_reg[j];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && __popc(same & lt_mask) == 0) whist[warp][e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  if (tid < pm::MAX_E) {  // 8 warps: one expert per thread
    const int e = tid;
    int run = 0;
    for (int w = 0; w < pm::SMALL_WARPS; ++w) {
      const int v = whist[w][e];
      whist[w][e] = run;
      run += v;
    }
    int incl = run;  // inclusive scan of the expert totals: within the warp, then across
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    asm volatile("bar.sync 1, %0;" ::"n"(pm::MAX_E));
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const int excl = before + incl - run;
    if (e < E) {
      counts[e] = run;
      offsets[e] = excl;
      for (int w = 0; w < pm::SMALL_WARPS; ++w) whist[w][e] += excl;
    }
    if (e == pm::MAX_E - 1) routed_total = before + incl;
  }
  __syncthreads();
  const int routed = routed_total;
  if (tid == 0) {
    counts[E] = has_shared ? T : 0;
    offsets[E] = routed;
    offsets[E + 1] = routed + (has_shared ? T : 0);
  }
#pragma unroll
  for (int j = 0; j < pm::SMALL_STEPS; ++j) {
    if (j >= steps) break;
    const int e = e_reg[j];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt_mask);
    if (e >= 0) sorted[whist[warp][e] + rank] = seg0 + j * 32 + lane;
    __syncwarp();
    if (e >= 0 && rank == 0) whist[warp][e] += __popc(same);
    __syncwarp();
  }
  if (has_shared)
    for (int t = tid; t < T; t += pm::SMALL_THREADS) sorted[routed + t] = n + t;
}

// Chunked batches whose chunks fit one CTA per SM: the same histogram ->
// scan -> stable scatter in ONE launch (three launches and a one-CTA scan
// otherwise).  Warp w of CTA c owns the contiguous assignments
// [c*CHUNK + w*CHUNK/WARPS, +CHUNK/WARPS) in registers:
//   1) each warp counts its entries per expert (warp matches, one writer per
//      expert per step); per expert, an exclusive scan over the warps, and the
//      chunk's count published to scratch[c * E + e];
//   2) a grid barrier (one arrival per CTA on a counter zeroed before the
//      launch, a bounded wait);
//   3) every CTA reads all chunks' counts: per expert the total and the counts
//      of the chunks before its own; the exclusive scan of the totals over the
//      experts gives the group offsets (the same numbers in every CTA; CTA 0
//      writes counts and offsets);
//   4) each warp writes every entry to its expert's running position: entries
//      ascending (chunk, warp, step, lane) keep ascending positions.
namespace pm {
constexpr int FUSED_STEPS = CHUNK / THREADS;  // 32-entry steps per warp
static_assert(THREADS == MAX_E, "one thread per expert in the offset scan");
}  // namespace pm

__global__ void __launch_bounds__(pm::THREADS)
    permute_fused_kernel(const int32_t *__restrict__ idx, int n, int E, int T, int has_shared,
                         int32_t *__restrict__ scratch, int *grid_counter, int32_t *__restrict__ counts,
                         int32_t *__restrict__ offsets, int32_t *__restrict__ sorted, int *err) {
  __shared__ int whist[pm::WARPS][pm::MAX_E];  // counts, then each warp's running positions
  __shared__ int base[pm::MAX_E];               // first position of this chunk's entries per expert
  __shared__ int wsum[pm::WARPS];
  __shared__ int routed_total;
  const int c = blockIdx.x, nchunks = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int k = tid; k < pm::WARPS * pm::MAX_E; k += pm::THREADS) (&whist[0][0])[k] = 0;
  const int seg0 = c * pm::CHUNK + warp * (pm::CHUNK / pm::WARPS);
  int e_reg[pm::FUSED_STEPS];
#pragma unroll
  for (int j = 0; j < pm::FUSED_STEPS; ++j) {
    const int i = seg0 + j * 32 + lane;
    int e = -1;
    if (i < n) {
      e = idx[i];
      if (e < 0 || e >= E) {
        record_error(err, MOE_ERR_BAD_INDEX);
        e = -1;
      }
    }
    e_reg[j] = e;
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < pm::FUSED_STEPS; ++j) {
    const int e = e_reg[j];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && __popc(same & lt_mask) == 0) whist[warp][e] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  if (tid < E) {
    int run = 0;
    for (int w = 0; w < pm::WARPS; ++w) {
      const int v = whist[w][tid];
      whist[w][tid] = run;
      run += v;
    }
    scratch[c * E + tid] = run;
  }
  __syncthreads();
  if (!grid_barrier(grid_counter, nchunks, err)) return;
  int total = 0, before = 0;
  if (tid < E) {
    for (int cc = 0; cc < nchunks; ++cc) {
      const int v = __ldcg(scratch + cc * E + tid);
      total += v;
      if (cc < c) before += v;
    }
  }
  int incl = total;  // inclusive scan of the totals over the experts: within the warp, then across
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int pre = 0;
  for (int w = 0; w < warp; ++w) pre += wsum[w];
  const int excl = pre + incl - total;
  if (tid < E) {
    base[tid] = excl + before;
    if (c == 0) {
      counts[tid] = total;
      offsets[tid] = excl;
    }
  }
  if (tid == pm::THREADS - 1) routed_total = pre + incl;
  __syncthreads();
  const int routed = routed_total;
  if (c == 0 && tid == 0) {
    counts[E] = has_shared ? T : 0;
    offsets[E] = routed;
    offsets[E + 1] = routed + (has_shared ? T : 0);
  }
#pragma unroll
  for (int j = 0; j < pm::FUSED_STEPS; ++j) {
    const int e = e_reg[j];
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt_mask);
    if (e >= 0) sorted[base[e] + whist[warp][e] + rank] = seg0 + j * 32 + lane;
    __syncwarp();
    if (e >= 0 && rank == 0) whist[warp][e] += __popc(same);
    __syncwarp();
  }
  if (has_shared)
    for (int t = c * pm::THREADS + tid; t < T; t += nchunks * pm::THREADS) sorted[routed + t] = n + t;
}

cudaError_t launch_permute(const int32_t *idx, int T, int E, int K, int has_shared, int32_t *counts,
                           int32_t *offsets, int32_t *sorted, int32_t *scratch, int *err,
                           cudaStream_t stream, int *grid_counter, int num_sms) {
  const int n = T * K;
  if (n <= pm::SMALL_N) {
    permute_small_kernel<<<1, pm::SMALL_THREADS, 0, stream>>>(idx, n, E, T, has_shared, counts,
                                                              offsets, sorted, err);
    return cudaGetLastError();
  }
  const int nchunks = permute_num_chunks(n);
  if (grid_counter && nchunks <= num_sms) {
    cudaError_t e = cudaMemsetAsync(grid_counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    permute_fused_kernel<<<nchunks, pm::THREADS, 0, stream>>>(idx, n, E, T, has_shared, scratch,
                                                              grid_counter, counts, offsets, sorted, err);
    return cudaGetLastError();
  }
  permute_hist_kernel<<<nchunks, pm::THREADS, 0, stream>>>(idx, n, E, nchunks, scratch, err);
  permute_scan_kernel<<<1, pm::SCAN_THREADS, 0, stream>>>(scratch, E, nchunks, T, has_shared, counts,
                                                          offsets);
  permute_scatter_kernel<<<nchunks, pm::THREADS, 0, stream>>>(idx, n, E, nchunks, scratch, T,
                                                              has_shared, offsets, sorted);
  return cudaGetLastError();
}

}  // namespace srm
