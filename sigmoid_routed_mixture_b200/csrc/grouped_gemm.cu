// grouped_gemm.cu -- the two expert contractions of the mixture on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// fed by TMA, as one persistent, warp-specialised kernel template.
//
// Definition ("GLM-5 . MoE transformer block", "All 43 steps", Mixture of
// experts): per expert i and token row x,
//     g = x W1_i,  u = x W3_i,  a = g sigmoid(g),  h = a (.) u,  E_i = h W2_i,
// and the shared expert the same way at weight 1; the routed outputs are
// weighted by G_i ("expert_outputs: each routing slot's weighted expert
// output", nnterp GLM-5 page, The API table).
//
//   kUp   : for every group g (routed experts 0..E-1, shared expert E) and its
//           rows, [g | u] = xs_rows . W13_g^T where xs holds the token rows in
//           expert-sorted order (gather.cu); epilogue h = silu(g) * u -> fp16 h[row][I] (three more mantissa
//           bits than bf16 at the same tensor-core rate; |h| saturates at
//           65504).
//   kDown : Y[a] = G[a] * (h_rows . W2_g^T) in fp16 x fp16 (W2 packed as
//           fp16, an exact conversion of bf16 weights in fp16's normal
//           range), rows of h contiguous, epilogue
//           multiplies by the routing gate (1 for the shared expert) and
//           scatters fp32 rows to their (token, slot) position a (fp32 so that
//           the only roundings after the tensor cores are h and the final y).
//
// Tiling: one work tile = 128 rows x 256 output columns, K loop in steps of
// 64 (one 128-byte swizzle atom), 4-stage TMA ring, two 128x256 fp32
// accumulators in tensor memory (512 columns) so the epilogue of one tile
// overlaps the main loop of the next.  Warp roles (6 warps):
//   warp 0: TMA producer (one lane issues the A and B tile loads)
//   warp 1: tensor-memory allocation + single-thread MMA issue
//   warps 2-5: epilogue (tensor memory -> registers -> global)
// Work tiles are (group, 128-row block, 256-column block), column block
// fastest, dealt round-robin over a grid of one CTA per SM; the per-group
// row-block counts come from the group offsets on the device, so the host
// never synchronises.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace gg {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators
constexpr int MAX_GROUPS = 257;

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int mma_consumed;
  int total_mtiles;
  int tile_start[MAX_GROUPS + 1];
  int grp_off[MAX_GROUPS + 1];
};
constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + sizeof(Smem);
}  // namespace gg

struct TileCoord {
  int g;          // group
  int row_base;   // first row of the tile in the expert-sorted order
  int rows;       // valid rows in the tile (1..128)
  int n0;         // first output column
};

__device__ __forceinline__ TileCoord decode_tile(const gg::Smem &s, int groups, int n_tiles,
                                                 int tile) {
  const int mt = tile / n_tiles;
  const int nt = tile - mt * n_tiles;
  int lo = 0, hi = groups - 1;  // last g with tile_start[g] <= mt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= mt)
      lo = mid;
    else
      hi = mid - 1;
  }
  TileCoord c;
  c.g = lo;
  c.row_base = s.grp_off[lo] + (mt - s.tile_start[lo]) * gg::BM;
  c.rows = min(gg::BM, s.grp_off[lo + 1] - c.row_base);
  c.n0 = nt * gg::BN;
  return c;
}

template <int kMode>
__global__ void __launch_bounds__(gg::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_b, GemmArgs p) {
  using namespace gg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sA = base;
  uint8_t *sB = base + STAGES * A_BYTES;
  Smem &s = *reinterpret_cast<Smem *>(base + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int groups = p.groups;
  const int n_tiles = p.n_total / BN;
  const int kblocks = p.k_total / BK;
  // up: bf16 x times bf16 W13; down: fp16 h times fp16 W2
  constexpr uint32_t IDESC = umma_idesc_f32acc(BM, BN, kMode == kUp ? 1u : 0u);

  // ---- prologue: barriers, tensor memory, per-group tile starts
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    s.mma_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0) {
    // group offsets and an exclusive scan of ceil(count / BM) over the groups
    const int per = (groups + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int g = g0; g < min(g0 + per, groups); ++g) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      s.grp_off[g] = o0;
      local += (o1 - o0 + BM - 1) / BM;
    }
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < min(g0 + per, groups); ++g) {
      s.tile_start[g] = run;
      run += (p.offsets[g + 1] - p.offsets[g] + BM - 1) / BM;
    }
    if (lane == 31) {
      s.total_mtiles = incl;
      s.tile_start[groups] = incl;
      s.grp_off[groups] = p.offsets[groups];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = s.total_mtiles * n_tiles;
  volatile int *abort_flag = &s.abort_flag;
  int issued = 0;  // k-blocks armed by the producer (lane 0's count)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t stage = 0, phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(s, groups, n_tiles, tile);
      const int b_row = c.g * p.n_total + c.n0;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&s.full[stage], STAGE_BYTES);
        __syncwarp();
        if (lane == 0) {
          tma_load_2d(sA + stage * A_BYTES, &tmap_a, &s.full[stage], kb * BK, c.row_base);
          tma_load_2d(sB + stage * B_BYTES, &tmap_b, &s.full[stage], kb * BK, b_row);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
    int consumed = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&s.full[stage], phase, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        ++consumed;
        if (lane == 0) {
          const uint32_t a_addr = smem_addr(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_addr(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            umma_bf16(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32),
                      IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&s.empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&s.tfull[acc]);
      __syncwarp();
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) s.mma_consumed = consumed;
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(s, groups, n_tiles, tile);
      if (!mbar_wait(&s.tfull[acc], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      bool valid = row < c.rows;
      int a = valid ? p.sorted[c.row_base + row] : 0;
      if (valid && (a < 0 || a >= p.n_rows_y)) {
        record_error(p.err, MOE_ERR_BAD_INDEX);
        valid = false;
      }
      const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      if (kMode == kUp) {
        // columns 0..127 of the tile are gate rows, 128..255 the matching up rows
        uint16_t *hrow = reinterpret_cast<uint16_t *>(p.out) +
                         static_cast<size_t>(c.row_base + row) * p.out_ld + c.n0 / 2;
#pragma unroll 1
        for (int ch = 0; ch < BN / 2 / 32; ++ch) {
          uint32_t gr[32], ur[32];
          tmem_ld32(taddr + ch * 32, gr);
          tmem_ld32(taddr + BN / 2 + ch * 32, ur);
          tmem_ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(gr[2 * j]), g1 = __uint_as_float(gr[2 * j + 1]);
              const float u0 = __uint_as_float(ur[2 * j]), u1 = __uint_as_float(ur[2 * j + 1]);
              packed[j] = pack_f16x2_sat(g0 * sigmoidf_(g0) * u0, g1 * sigmoidf_(g1) * u1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(hrow + ch * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                  packed[4 * v + 3]);
          }
        }
      } else {
        const float gv = (a < p.tk) ? p.gate[valid ? a : 0] : 1.0f;
        float *yrow = reinterpret_cast<float *>(p.out) + static_cast<size_t>(a) * p.out_ld + c.n0;
#pragma unroll 1
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(taddr + ch * 32, r);
          tmem_ld_wait();
          if (valid) {
            float4 *dst = reinterpret_cast<float4 *>(yrow + ch * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(gv * __uint_as_float(r[4 * v]), gv * __uint_as_float(r[4 * v + 1]),
                                   gv * __uint_as_float(r[4 * v + 2]), gv * __uint_as_float(r[4 * v + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tempty[acc]);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- teardown.  On the error path wait (bounded) for copies and MMAs still
  // in flight before the shared and tensor memory are given back.
  __syncthreads();
  if (s.abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int i = s.mma_consumed; i < issued; ++i) {
        const uint32_t a = smem_addr(&s.full[i % STAGES]);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(a, static_cast<uint32_t>((i / STAGES) & 1)) &&
               global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    if (warp == 1 && lane == 0) {
      umma_commit(&s.drain);
      const uint32_t a = smem_addr(&s.drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(a, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

size_t grouped_gemm_smem_bytes() { return gg::SMEM_BYTES; }

template <int kMode>
static cudaError_t launch_mode(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p,
                               int grid, cudaStream_t stream) {
  auto kern = grouped_gemm_kernel<kMode>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, gg::THREADS, gg::SMEM_BYTES, stream>>>(ta, tb, p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int mode, const CUtensorMap &ta, const CUtensorMap &tb,
                                const GemmArgs &p, int grid, cudaStream_t stream) {
  if (mode == kUp) return launch_mode<kUp>(ta, tb, p, grid, stream);
  return launch_mode<kDown>(ta, tb, p, grid, stream);
}

}  // namespace srm
