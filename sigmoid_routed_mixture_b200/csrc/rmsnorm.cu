// rmsnorm.cu -- the pre-FFN RMSNorm of the decoder block,
//     x_ffn = RMSNorm(x'_n)  ("GLM-5 . MoE transformer block", "All 43 steps"),
//     x_ffn[t,h] = x[t,h] * gamma[h] / sqrt(mean_h x[t,h]^2 + eps),
// computed in fp32 from the bf16 residual stream and rounded once to bf16 (the
// model dtype); eps is the config's rms_norm_eps (1e-5 on GLM-5 and
// GLM-4.7-Flash).  One warp per token row; the sum of squares is reduced in a
// fixed order (per-lane sequential, then a shuffle tree): deterministic.
#include "common.cuh"
#include "kernels.h"

namespace srm {

__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ gamma, float eps,
                   int T, int H, uint16_t *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int vecs = H / 8;
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    const uint4 *row = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * H);
    float ss = 0.f;
    for (int v = lane; v < vecs; v += 32) {
      const uint4 q = row[v];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = __uint_as_float(w[k] << 16), b = __uint_as_float(w[k] & 0xFFFF0000u);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    uint4 *dst = reinterpret_cast<uint4 *>(out + static_cast<size_t>(t) * H);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(gamma);
    for (int v = lane; v < vecs; v += 32) {
      const uint4 q = row[v], gq = g4[v];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o[k] = pack_bf16x2(__uint_as_float(w[k] << 16) * inv * __uint_as_float(gw[k] << 16),
                           __uint_as_float(w[k] & 0xFFFF0000u) * inv *
                               __uint_as_float(gw[k] & 0xFFFF0000u));
      dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

cudaError_t launch_rmsnorm(const uint16_t *x, const uint16_t *gamma, float eps, int T, int H,
                           uint16_t *out, int num_sms, cudaStream_t stream) {
  int blocks = (T + 7) / 8;
  if (blocks > num_sms * 16) blocks = num_sms * 16;
  rmsnorm_kernel<<<blocks, 256, 0, stream>>>(x, gamma, eps, T, H, out);
  return cudaGetLastError();
}

}  // namespace srm
