// gather.cu -- token rows in expert-sorted order for the up projection.
//
// The up projection of every group reads its rows of x in the expert-sorted
// order moe_permute produced.  Copying them once per step into a contiguous
// buffer lets the tensor-core kernel load plain 128-row TMA tiles (measured:
// per-row tile::gather4 loads starved the tensor pipe).  The copy walks the
// TOKENS in order, reads each row of x once and writes it to the K + 1
// positions its assignments occupy, so x streams from HBM exactly once:
//   1) invert:  pos[sorted[p]] = p              (row id -> sorted position)
//   2) scatter: xs[pos[t*K + k]] = x[t] (k < K),  xs[pos[T*K + t]] = x[t]
#include "common.cuh"
#include "kernels.h"

namespace srm {

__global__ void __launch_bounds__(256)
    invert_rows_kernel(const int32_t *__restrict__ sorted, int rows, int n_rows_y,
                       int32_t *__restrict__ pos, int *err) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < rows; p += gridDim.x * blockDim.x) {
    const int a = sorted[p];
    if (a < 0 || a >= n_rows_y)
      record_error(err, MOE_ERR_BAD_INDEX);
    else
      pos[a] = p;
  }
}

// WPT warps per token (each moves a contiguous part of the row, 8 x 16 bytes
// per lane at a time): one warp per token for large batches, more when there
// are few tokens so that enough bytes are in flight.
__global__ void __launch_bounds__(256)
    scatter_rows_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ pos, int T,
                        int H, int K, int has_shared, int rows, int wpt, uint16_t *__restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // global warp
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int vecs = H / 8;  // 16-byte vectors per row
  const int part = (vecs + wpt - 1) / wpt;
  for (int job = gw; job < T * wpt; job += warps) {
    const int t = job / wpt;
    const int v_begin = (job - t * wpt) * part;
    const int v_end = min(vecs, v_begin + part);
    int dst[17];
    const int n_dst = K + has_shared;
#pragma unroll
    for (int k = 0; k < 17; ++k) {
      int d = -1;
      if (k < K)
        d = pos[t * K + k];
      else if (k == K && has_shared)
        d = pos[T * K + t];
      dst[k] = (d >= 0 && d < rows) ? d : -1;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * H);
    for (int v0 = v_begin; v0 < v_end; v0 += 32 * 8) {
      uint4 buf[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int v = v0 + j * 32 + lane;
        if (v < v_end) buf[j] = __ldcs(src + v);
      }
#pragma unroll
      for (int k = 0; k < 17; ++k) {
        if (k >= n_dst) break;
        if (dst[k] < 0) continue;
        uint4 *out = reinterpret_cast<uint4 *>(xs + static_cast<size_t>(dst[k]) * H);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int v = v0 + j * 32 + lane;
          if (v < v_end) out[v] = buf[j];
        }
      }
    }
  }
}

__global__ void identity_rows_kernel(int32_t *__restrict__ offsets, int32_t *__restrict__ sorted,
                                     int T, int base) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    offsets[0] = 0;
    offsets[1] = T;
  }
  for (int t = i; t < T; t += gridDim.x * blockDim.x) sorted[t] = base + t;
}

cudaError_t launch_identity_rows(int32_t *offsets, int32_t *sorted, int T, int num_sms,
                                 cudaStream_t stream, int base) {
  int blocks = (T + 255) / 256;
  if (blocks > num_sms * 4) blocks = num_sms * 4;
  if (blocks < 1) blocks = 1;
  identity_rows_kernel<<<blocks, 256, 0, stream>>>(offsets, sorted, T, base);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *sorted, int T, int H, int K,
                               int has_shared, int32_t *pos, uint16_t *xs, int *err, int num_sms,
                               cudaStream_t stream) {
  const int rows = T * K + (has_shared ? T : 0);
  const int n_rows_y = rows;
  int blocks = (rows + 255) / 256;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  invert_rows_kernel<<<blocks, 256, 0, stream>>>(sorted, rows, n_rows_y, pos, err);
  int wpt = 1;  // warps per token: aim for at least ~4 warps per SM in flight
  while (wpt < 8 && T * wpt < num_sms * 32) wpt *= 2;
  int tb = (T * wpt + 7) / 8;
  if (tb > num_sms * 16) tb = num_sms * 16;
  scatter_rows_kernel<<<tb, 256, 0, stream>>>(x, pos, T, H, K, has_shared, rows, wpt, xs);
  return cudaGetLastError();
}

}  // namespace srm
