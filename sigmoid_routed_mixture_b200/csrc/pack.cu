// pack.cu -- one-time re-layout of the expert weights for the grouped GEMMs.
//   w13_out [(E+1)*2I][H]: group g, unit j (32 rows) = W1_g rows 16j..16j+15
//       then W3_g rows 16j..16j+15, so the 32 tensor-memory lanes one warp
//       reads in the up projection's epilogue hold gate and up of the same 16
//       features; the gate-then-up order is the fused gate_up_proj order of
//       the nnterp GLM-4 page (section 03, "The MLP is GLM's fused one").
//   w2_out [(E+1)*H][I]: W2_g for g < E, the shared expert's W2 as group E,
//       converted from bf16 to fp16 (the down projection multiplies fp16 h by
//       fp16 W2; the conversion is exact for |w| in [2^-17, 65504]; values it
//       changes are counted into an optional device counter).
// A missing shared expert (has_shared == 0) leaves group E zero.
#include "common.cuh"
#include "kernels.h"

namespace srm {

__global__ void __launch_bounds__(256)
    pack_w13_kernel(const uint16_t *__restrict__ w1, const uint16_t *__restrict__ w3,
                    const uint16_t *__restrict__ ws1, const uint16_t *__restrict__ ws3, int H, int I,
                    int E, int has_shared, uint16_t *__restrict__ out) {
  const int vecs = H / 8;
  const int64_t rows = static_cast<int64_t>(E + 1) * 2 * I;
  const int64_t total = rows * vecs;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vecs;
    const int64_t col = (i - r * vecs) * 8;
    const int64_t g = r / (2 * I);
    const int64_t within = r - g * 2 * I;
    const int64_t j = within / 32, k = within % 32;
    const int64_t src_row = j * 16 + (k & 15);
    const bool up = k >= 16;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (g < E) {
      const uint16_t *src = (up ? w3 : w1) + (g * I + src_row) * H + col;
      v = *reinterpret_cast<const uint4 *>(src);
    } else if (has_shared) {
      const uint16_t *src = (up ? ws3 : ws1) + src_row * H + col;
      v = *reinterpret_cast<const uint4 *>(src);
    }
    *reinterpret_cast<uint4 *>(out + r * H + col) = v;
  }
}

// fp16 bit pattern -> float (exact)
__device__ __forceinline__ float f16_bits_to_float(uint32_t bits) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

__global__ void __launch_bounds__(256)
    pack_w2_kernel(const uint16_t *__restrict__ w2, const uint16_t *__restrict__ ws2, int H, int I,
                   int E, int has_shared, uint16_t *__restrict__ out, int32_t *inexact) {
  int n_inexact = 0;  // this thread's W2 values whose fp16 copy is not exact
  const int vecs = I / 8;
  const int64_t rows = static_cast<int64_t>(E + 1) * H;
  const int64_t total = rows * vecs;
  const int64_t routed_rows = static_cast<int64_t>(E) * H;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vecs;
    const int64_t col = (i - r * vecs) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < routed_rows)
      v = *reinterpret_cast<const uint4 *>(w2 + r * I + col);
    else if (has_shared)
      v = *reinterpret_cast<const uint4 *>(ws2 + (r - routed_rows) * I + col);
    // bf16 -> fp16: exact for |w| in [2^-17, 65504]; smaller magnitudes keep
    // fp16's subnormal spacing 2^-24, larger ones saturate
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    bool sat = false;  // bf16 weights beyond the fp16 range saturate
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
      w[k] = pack_f16x2_sat(lo, hi, sat);
      n_inexact += (f16_bits_to_float(w[k] & 0xFFFFu) != lo) + (f16_bits_to_float(w[k] >> 16) != hi);
    }
    *reinterpret_cast<uint4 *>(out + r * I + col) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (inexact) {
    n_inexact = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(n_inexact));
    if ((threadIdx.x & 31) == 0 && n_inexact) atomicAdd(inexact, n_inexact);
  }
}

cudaError_t launch_pack(const uint16_t *w1, const uint16_t *w3, const uint16_t *w2,
                        const uint16_t *ws1, const uint16_t *ws3, const uint16_t *ws2, int H, int I,
                        int E, int has_shared, uint16_t *w13_out, uint16_t *w2_out,
                        int32_t *w2_inexact, int num_sms, cudaStream_t stream) {
  const int grid = num_sms * 8;
  pack_w13_kernel<<<grid, 256, 0, stream>>>(w1, w3, ws1, ws3, H, I, E, has_shared, w13_out);
  pack_w2_kernel<<<grid, 256, 0, stream>>>(w2, ws2, H, I, E, has_shared, w2_out, w2_inexact);
  return cudaGetLastError();
}

}  // namespace srm
