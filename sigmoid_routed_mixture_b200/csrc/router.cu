// router.cu -- fused router: logits, sigmoid scores, biased top-K selection
// and renormalised, scaled gates in one kernel.
//
// Definition ("GLM-5 . MoE transformer block", "All 43 steps", Mixture of
// experts):  z = x W_r;  s = sigmoid(z);  E_sel_i = [i in top_K(s + b)];
//            G_i = scale * s_i E_sel_i / sum_j s_j E_sel_j.
// The bias takes part in the choice only; the gates use the un-biased s
// (nnterp GLM-4.7-Flash / GLM-5, section 03, note "The mixture: sigmoid
// scores, a selection bias, renormalized weights").  Ties between equal keys
// go to the lower expert index; the slots come out in descending key order.
//
// One CTA = 64 tokens x all experts (E <= 256).  Stage 1: z for the tile with
// fp32 FMA (bf16 x widened exactly, fp32 W_r, fp32 accumulation; each thread
// owns 8 tokens x NE experts).  Stage 2: z goes to shared memory and each warp
// selects for 8 tokens: every lane holds NE candidate keys and K rounds of a
// warp arg-max (key descending, index ascending) pick the slots; one more
// round gives the (K+1)-th key for the selection margin.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace rt {
constexpr int TT = 64;     // tokens per CTA
constexpr int HC = 32;     // reduction chunk
constexpr int THREADS = 256;
}  // namespace rt

template <int NE>
__global__ void __launch_bounds__(rt::THREADS)
    route_kernel(const uint16_t *__restrict__ x, const float *__restrict__ w_r,
                 const float *__restrict__ bias, int T, int H, int E, int K, float scale,
                 int32_t *__restrict__ idx, float *__restrict__ gate, float *__restrict__ margin) {
  using namespace rt;
  constexpr int EP = NE * 32;  // padded expert count
  extern __shared__ float smem_f[];
  float *xs = smem_f;                  // [TT][HC + 1]
  float *ws = smem_f + TT * (HC + 1);  // [EP][HC + 1]
  float *zs = smem_f;                  // [TT][EP + 1], reused after stage 1

  const int tid = threadIdx.x;
  const int tx = tid & 31;
  const int ty = tid >> 5;
  const int t0 = blockIdx.x * TT;

  float acc[8][NE];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < NE; ++j) acc[i][j] = 0.f;

  for (int h0 = 0; h0 < H; h0 += HC) {
    {  // x tile: 64 tokens x 32 features, 8 bf16 per thread
      const int tt = tid >> 2, part = (tid & 3) * 8;
      const int t = t0 + tt;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T) v = *reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * H + h0 + part);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        xs[tt * (HC + 1) + part + 2 * k] = __uint_as_float(w[k] << 16);
        xs[tt * (HC + 1) + part + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
    // W_r tile: EP experts x 32 features
    for (int i = tid; i < EP * (HC / 4); i += THREADS) {
      const int e = i / (HC / 4), part = (i % (HC / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < E) v = *reinterpret_cast<const float4 *>(w_r + static_cast<size_t>(e) * H + h0 + part);
      ws[e * (HC + 1) + part + 0] = v.x;
      ws[e * (HC + 1) + part + 1] = v.y;
      ws[e * (HC + 1) + part + 2] = v.z;
      ws[e * (HC + 1) + part + 3] = v.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int h = 0; h < HC; ++h) {
      float a[8], b[NE];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = xs[(ty * 8 + i) * (HC + 1) + h];
#pragma unroll
      for (int j = 0; j < NE; ++j) b[j] = ws[(tx + 32 * j) * (HC + 1) + h];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < NE; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < NE; ++j) zs[(ty * 8 + i) * (EP + 1) + tx + 32 * j] = acc[i][j];
  __syncthreads();

  // ---- selection: warp `ty` handles tokens ty*8 .. ty*8+7 of the tile
  float bj[NE];
#pragma unroll
  for (int j = 0; j < NE; ++j) {
    const int e = tx + 32 * j;
    bj[j] = e < E ? bias[e] : 0.f;
  }
  for (int i = 0; i < 8; ++i) {
    const int tt = ty * 8 + i;
    const int t = t0 + tt;
    if (t >= T) break;  // uniform across the warp
    float key[NE], sv[NE];
#pragma unroll
    for (int j = 0; j < NE; ++j) {
      const int e = tx + 32 * j;
      const float sj = sigmoidf_(zs[tt * (EP + 1) + e]);
      sv[j] = sj;
      key[j] = e < E ? sj + bj[j] : -INFINITY;
    }
    int my_e = 0;
    float my_s = 0.f, kth_key = 0.f, next_key = -INFINITY;
    const int rounds = K < E ? K + 1 : K;
    for (int k = 0; k < rounds; ++k) {
      float bk = -INFINITY, bs = 0.f;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < NE; ++j) {
        if (key[j] > bk) {  // j ascending = expert index ascending: strict > keeps the lower
          bk = key[j];
          be = tx + 32 * j;
          bs = sv[j];
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        if (ok > bk || (ok == bk && oe < be)) {
          bk = ok;
          be = oe;
          bs = os;
        }
      }
      if (k == K) {
        next_key = bk;
        break;
      }
      if (tx == k) {
        my_e = be;
        my_s = bs;
      }
      if (k == K - 1) kth_key = bk;
#pragma unroll
      for (int j = 0; j < NE; ++j)
        if (be == tx + 32 * j) key[j] = -INFINITY;
    }
    float denom = 0.f;
    for (int k = 0; k < K; ++k) denom += __shfl_sync(0xffffffffu, my_s, k);
    if (tx < K) {
      idx[static_cast<size_t>(t) * K + tx] = my_e;
      gate[static_cast<size_t>(t) * K + tx] = scale * my_s / denom;
    }
    if (margin && tx == 0) margin[t] = K < E ? kth_key - next_key : INFINITY;
  }
}

template <int NE>
static cudaError_t launch_ne(const uint16_t *x, const float *w_r, const float *bias, int T, int H,
                             int E, int K, float scale, int32_t *idx, float *gate, float *margin,
                             cudaStream_t stream) {
  using namespace rt;
  constexpr int EP = NE * 32;
  const size_t stage1 = sizeof(float) * (TT * (HC + 1) + EP * (HC + 1));
  const size_t stage2 = sizeof(float) * TT * (EP + 1);
  const size_t smem = stage1 > stage2 ? stage1 : stage2;
  cudaError_t e = cudaFuncSetAttribute(route_kernel<NE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = (T + TT - 1) / TT;
  route_kernel<NE><<<grid, THREADS, smem, stream>>>(x, w_r, bias, T, H, E, K, scale, idx, gate,
                                                   margin);
  return cudaGetLastError();
}

cudaError_t launch_route(const uint16_t *x, const float *w_r, const float *bias, int T, int H, int E,
                         int K, float scale, int32_t *idx, float *gate, float *margin,
                         cudaStream_t stream) {
  if (E <= 32) return launch_ne<1>(x, w_r, bias, T, H, E, K, scale, idx, gate, margin, stream);
  if (E <= 64) return launch_ne<2>(x, w_r, bias, T, H, E, K, scale, idx, gate, margin, stream);
  if (E <= 128) return launch_ne<4>(x, w_r, bias, T, H, E, K, scale, idx, gate, margin, stream);
  return launch_ne<8>(x, w_r, bias, T, H, E, K, scale, idx, gate, margin, stream);
}

}  // namespace srm
