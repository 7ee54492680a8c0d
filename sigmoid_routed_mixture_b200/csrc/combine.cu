// combine.cu -- deterministic un-permute / combine:
//     y[t] = (sum over slots k = 0..K-1, in order, of Y[t*K + k]) + Y[T*K + t]
// in fp32, rounded once to bf16.  Y holds each routing slot's weighted expert
// output (the gate was applied in the down-projection epilogue) and, after the
// T*K routed rows, the shared expert's output; "the shared expert runs after
// the routed ones" (nnterp GLM-5 page, section 03) fixes the order of the
// final addition, and Delta_ffn = y_routed + y_shared ("GLM-5 . MoE
// transformer block", "All 43 steps").
//
// Pure streaming: each thread owns 8 consecutive columns of one token, loads
// K+1 rows of 32 fp32 bytes and stores 16 bytes of bf16.
#include "common.cuh"
#include "kernels.h"

namespace srm {

__device__ __forceinline__ void add8(float (&acc)[8], const float *src) {
  const float4 a = __ldcs(reinterpret_cast<const float4 *>(src));
  const float4 b = __ldcs(reinterpret_cast<const float4 *>(src) + 1);
  acc[0] += a.x;
  acc[1] += a.y;
  acc[2] += a.z;
  acc[3] += a.w;
  acc[4] += b.x;
  acc[5] += b.y;
  acc[6] += b.z;
  acc[7] += b.w;
}

__global__ void __launch_bounds__(256)
    combine_kernel(const float *__restrict__ Y, uint16_t *__restrict__ y, int T, int H, int K,
                   int has_shared) {
  const int vecs = H / 8;
  const int64_t total = static_cast<int64_t>(T) * vecs;
  const int64_t tk = static_cast<int64_t>(T) * K;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / vecs;
    const int64_t col = (i - t * vecs) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) add8(acc, Y + (t * K + k) * H + col);
    if (has_shared) add8(acc, Y + (tk + t) * H + col);
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4 *>(y + t * H + col) = o;
  }
}

cudaError_t launch_combine(const float *Y, uint16_t *y, int T, int H, int K, int has_shared,
                           int num_sms, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(T) * (H / 8);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  combine_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(Y, y, T, H, K, has_shared);
  return cudaGetLastError();
}

}  // namespace srm
