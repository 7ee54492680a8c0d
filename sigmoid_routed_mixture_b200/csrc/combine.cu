// combine.cu -- deterministic un-permute / combine:
//     y[t] = (sum over slots k = 0..K-1, in order, of Y[t*K + k]) + Y[T*K + t]
// in fp32, rounded once to bf16.  Y holds each routing slot's weighted expert
// output (the gate was applied in the down-projection epilogue) and, after the
// T*K routed rows, the shared expert's output; "the shared expert runs after
// the routed ones" (nnterp GLM-5 page, section 03) fixes the order of the
// final addition, and Delta_ffn = y_routed + y_shared ("GLM-5 . MoE
// transformer block", "All 43 steps").  With a residual row the kernel also
// performs the block's x_{n+1} = x'_n + Delta_ffn in the same pass (one
// rounding of the sum).
//
// Pure streaming: each thread owns 8 consecutive columns of one token, loads
// K+1 16-byte vectors of fp16 and stores 16 bytes of bf16.
#include "common.cuh"
#include "kernels.h"

namespace srm {

// 8 fp16 values (16 bytes) added to the fp32 sums
__device__ __forceinline__ void add8v(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[k]));
    acc[2 * k] += f.x;
    acc[2 * k + 1] += f.y;
  }
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint16_t *src) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(src));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[k]));
    acc[2 * k] += f.x;
    acc[2 * k + 1] += f.y;
  }
}

// KK > 0: the kernel for K = KK, every slot row's load issued before the sums
// (more loads in flight per thread); KK = 0: any K.  Same summation order.
template <int KK>
__global__ void __launch_bounds__(256)
    combine_kernel(const uint16_t *__restrict__ Y, const uint16_t *__restrict__ residual,
                   uint16_t *__restrict__ y, int T, int H, int K, int has_shared) {
  const int vecs = H / 8;
  const int64_t total = static_cast<int64_t>(T) * vecs;
  const int64_t tk = static_cast<int64_t>(T) * K;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vecs;
    const int64_t col = (i - t * vecs) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (KK > 0) {
      uint4 v[KK + 1];
#pragma unroll
      for (int k = 0; k < KK; ++k) v[k] = __ldcs(reinterpret_cast<const uint4 *>(Y + (t * KK + k) * H + col));
      if (has_shared) v[KK] = __ldcs(reinterpret_cast<const uint4 *>(Y + (tk + t) * H + col));
#pragma unroll
      for (int k = 0; k < KK; ++k) add8v(acc, v[k]);
      if (has_shared) add8v(acc, v[KK]);
    } else {
      for (int k = 0; k < K; ++k) add8(acc, Y + (t * K + k) * H + col);
      if (has_shared) add8(acc, Y + (tk + t) * H + col);
    }
    if (residual) {  // x_{n+1} = x'_n + Delta_ffn: the block output added to the residual stream
      const uint4 r = *reinterpret_cast<const uint4 *>(residual + t * H + col);
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] = __uint_as_float(w[k] << 16) + acc[2 * k];
        acc[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u) + acc[2 * k + 1];
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4 *>(y + t * H + col) = o;
  }
}

cudaError_t launch_combine(const uint16_t *Y, const uint16_t *residual, uint16_t *y, int T, int H,
                           int K, int has_shared, int num_sms, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(T) * (H / 8);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (K == 8)
    combine_kernel<8><<<static_cast<int>(blocks), 256, 0, stream>>>(Y, residual, y, T, H, K, has_shared);
  else if (K == 4)
    combine_kernel<4><<<static_cast<int>(blocks), 256, 0, stream>>>(Y, residual, y, T, H, K, has_shared);
  else
    combine_kernel<0><<<static_cast<int>(blocks), 256, 0, stream>>>(Y, residual, y, T, H, K, has_shared);
  return cudaGetLastError();
}

}  // namespace srm
