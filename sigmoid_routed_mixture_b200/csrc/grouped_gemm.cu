// grouped_gemm.cu -- the two expert contractions of the mixture on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// fed by TMA, as one persistent, warp-specialised kernel template that runs
// on CTA pairs.
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
//           expert-sorted order (gather.cu); epilogue h = silu(g) * u -> fp16
//           h[row][I] (three more mantissa bits than bf16 at the same
//           tensor-core rate; |h| saturates at 65504, flagged MOE_ERR_RANGE).
//   kDown : Y[a] = G[a] * (h_rows . W2_g^T) in fp16 x fp16 (W2 packed as
//           fp16, an exact conversion of bf16 weights in fp16's normal
//           range), rows of h contiguous, epilogue multiplies by the routing
//           gate (1 for the shared expert) and scatters fp16 rows to their
//           (token, slot) position a (fp16: 8x finer rounding than bf16 in
//           the same two bytes; saturation at 65504 is flagged MOE_ERR_RANGE).
//
// Tiling: a cluster of two CTAs (a CTA pair) owns one work tile of 256 rows x
// 256 output columns: each CTA loads its 128 rows of A and 128 of the 256
// rows of B (so every B byte crosses L2 once per pair, not once per CTA), and
// the leader CTA issues tcgen05.mma.cta_group::2 with M = 256 that reads both
// CTAs' shared memory and leaves each CTA's 128 x 256 fp32 accumulator in its
// own tensor memory.  K loop in steps of 64 (one 128-byte swizzle atom), a
// 6-stage TMA ring per CTA, two accumulators per CTA (512 TMEM columns) so the
// epilogue of one tile overlaps the main loop of the next.
// Warp roles (6 warps per CTA):
//   warp 0: TMA producer (one lane issues the CTA's A and B tile loads)
//   warp 1: tensor-memory allocation; in the leader also single-thread MMA issue
//   warps 2-5: epilogue (tensor memory -> registers -> global)
// Work tiles are (group, 256-column block, row block), row block fastest; a
// unit (CTA pair or single CTA) takes its next tile from a global atomic
// counter when it is ready for one, so tiles that share a weight tile start
// together; the per-group row-block counts come from the group offsets on the
// device, so the host never synchronises.
//
// Barrier protocol of a pair (no TMA multicast anywhere):
//   full[s]   (leader's)  producer of the leader arms it with both CTAs' bytes;
//                         both CTAs' loads complete on it
//   empty[s]  (each CTA)  the leader's commit multicasts to both when the
//                         MMAs reading stage s are done
//   tfull[a]  (each CTA)  the leader's commit multicasts to both when
//                         accumulator a is complete
//   tempty[a] (leader's)  the 4 epilogue warps of each CTA arrive (8 in all)
//                         when they have drained accumulator a
//   tile_full[i] (each)   the leader's producer publishes tile id i (ring of 4)
//                         into both CTAs' shared memory and arrives on both
//   tile_empty[i] (leader's) the epilogue warps of both CTAs release ring slot i
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace gg {
constexpr int BM = 128;        // rows per CTA
constexpr int BN = 256;        // output columns per tile
constexpr int BK = 64;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators
constexpr int MAX_GROUPS = 257;
constexpr int MAX_STAGES = 6;
constexpr int TILE_RING = 4;  // tile ids in flight between the scheduler and the roles

// kPair: a CTA pair shares each 256-row tile (M = 256, each CTA loads half of
// B); solo: one CTA per 128-row tile (M = 128, the CTA loads all of B).
template <bool kPair>
struct Cfg {
  static constexpr int TILE_M = kPair ? 2 * BM : BM;
  static constexpr int B_ROWS = kPair ? BN / 2 : BN;     // B rows loaded per CTA
  static constexpr int STAGES = kPair ? 6 : 4;
  static constexpr int A_BYTES = BM * BK * 2;            // 16 KB
  static constexpr int B_BYTES = B_ROWS * BK * 2;        // 16 or 32 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TX_BYTES = (kPair ? 2 : 1) * STAGE_BYTES;
  static constexpr uint32_t EPI_ARRIVALS = kPair ? 8 : 4;
};

struct Smem {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tile_full[TILE_RING];
  uint64_t tile_empty[TILE_RING];
  int tile_ring[TILE_RING];
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
template <bool kPair>
constexpr size_t smem_bytes() {
  return 1024 /*alignment slack*/ + Cfg<kPair>::STAGES * Cfg<kPair>::STAGE_BYTES + sizeof(Smem);
}
}  // namespace gg

struct TileCoord {
  int g;          // group
  int row_base;   // first row of this CTA's half of the tile (expert-sorted order)
  int rows;       // valid rows of this CTA's half (0..128)
  int n0;         // first output column
};

// Tiles of group g occupy [tile_start[g] * n_tiles, tile_start[g+1] * n_tiles)
// and inside a group the row block runs fastest: the units working at the same
// moment share each 256-column weight tile (one DRAM read serves all the
// group's row blocks) instead of spreading over many weight tiles that evict
// one another from L2.  A group with more than m_chunk row blocks (the shared
// expert at large batches) is walked in chunks of m_chunk row blocks, each
// chunk through all column blocks, so that the chunk's rows stay in L2 while
// every column block reads them (a whole 16384-token group would not fit and
// would be re-read from DRAM once per column block).
template <bool kPair>
__device__ __forceinline__ TileCoord decode_tile(const gg::Smem &s, int groups, int n_tiles,
                                                 int m_chunk, int tile, int rank) {
  const int mt_flat = tile / n_tiles;
  int lo = 0, hi = groups - 1;  // last g with tile_start[g] <= mt_flat
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= mt_flat)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int mblocks = s.tile_start[lo + 1] - s.tile_start[lo];
  const int local = tile - s.tile_start[lo] * n_tiles;
  const int chunk = local / (m_chunk * n_tiles);
  const int m0 = chunk * m_chunk;
  const int cm = min(m_chunk, mblocks - m0);  // row blocks in this chunk
  const int r = local - m0 * n_tiles;
  const int nt = r / cm;
  const int mt = m0 + (r - nt * cm);
  TileCoord c;
  c.g = lo;
  c.row_base = s.grp_off[lo] + mt * gg::Cfg<kPair>::TILE_M + rank * gg::BM;
  c.rows = max(0, min(gg::BM, s.grp_off[lo + 1] - c.row_base));
  c.n0 = nt * gg::BN;
  return c;
}

template <int kMode, bool kPair>
__device__ __forceinline__ void grouped_gemm_body(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                                                  const GemmArgs &p) {
  using namespace gg;
  using C = Cfg<kPair>;
  constexpr int STAGES = C::STAGES;
  constexpr int A_BYTES = C::A_BYTES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int TILE_M = C::TILE_M;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sA = base;
  uint8_t *sB = base + STAGES * A_BYTES;
  Smem &s = *reinterpret_cast<Smem *>(base + STAGES * C::STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int groups = p.groups;
  const int n_tiles = p.n_total / BN;
  const int kblocks = p.k_total / BK;
  // row blocks per chunk: about 48 MB of A rows (16-bit operands)
  const int m_chunk = max(1, (48 << 20) / (TILE_M * p.k_total * 2));
  // up: bf16 x times bf16 W13; down: fp16 h times fp16 W2
  constexpr uint32_t IDESC = umma_idesc_f32acc(TILE_M, BN, kMode == kUp ? 1u : 0u);

  // ---- prologue: barriers, tensor memory, per-group tile starts
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], C::EPI_ARRIVALS);
    }
    for (int i = 0; i < TILE_RING; ++i) {
      mbar_init(&s.tile_full[i], 1);
      mbar_init(&s.tile_empty[i], C::EPI_ARRIVALS);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    s.mma_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&s.tmem_base, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s.tmem_base, TMEM_COLS);
      tmem_relinquish();
    }
  }
  if (warp == 0) {
    // group offsets and an exclusive scan of ceil(count / TILE_M) over the groups
    const int per = (groups + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int g = g0; g < min(g0 + per, groups); ++g) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      s.grp_off[g] = o0;
      local += (o1 - o0 + TILE_M - 1) / TILE_M;
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
      run += (p.offsets[g + 1] - p.offsets[g] + TILE_M - 1) / TILE_M;
    }
    if (lane == 31) {
      s.total_mtiles = incl;
      s.tile_start[groups] = incl;
      s.grp_off[groups] = p.offsets[groups];
    }
  }
  tc_fence_before();
  if (kPair)
    cluster_sync();  // the peer's barriers are initialised before any remote use
  else
    __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s.tmem_base;
  const int total_tiles = s.total_mtiles * n_tiles;
  volatile int *abort_flag = &s.abort_flag;
  int issued = 0;  // k-blocks this CTA's producer has loaded

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The leader's producer is also the tile scheduler: it takes the next
    // tile from the global counter, so tiles sharing a weight tile (one
    // group's row blocks) start at nearly the same moment on whichever units
    // are free, and publishes the id to its own CTA and to the peer through
    // the tile ring.
    uint32_t stage = 0, phase = 0, ts = 0, tph = 0;
    while (true) {
      if (leader) {
        if (!mbar_wait(&s.tile_empty[ts], tph ^ 1u, abort_flag, p.err)) break;
        if (lane == 0) {
          int t = atomicAdd(p.tile_counter, 1);
          if (t >= total_tiles) t = -1;
          s.tile_ring[ts] = t;
          mbar_arrive(&s.tile_full[ts]);
          if (kPair) {
            st_shared_remote(cluster_map(&s.tile_ring[ts], 1), t);
            mbar_arrive_remote(cluster_map(&s.tile_full[ts], 1));
          }
        }
        __syncwarp();
      }
      if (!mbar_wait(&s.tile_full[ts], tph, abort_flag, p.err, kPair)) break;
      const int tile = *reinterpret_cast<volatile int *>(&s.tile_ring[ts]);
      if (++ts == TILE_RING) {
        ts = 0;
        tph ^= 1u;
      }
      if (tile < 0 || p.stall) break;
      const TileCoord c = decode_tile<kPair>(s, groups, n_tiles, m_chunk, tile, rank);
      const int b_row = c.g * p.n_total + c.n0 + rank * C::B_ROWS;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&s.full[stage], C::TX_BYTES);
          if (kPair) {
            const uint32_t full_leader = cluster_map(&s.full[stage], 0);
            tma_load_2d_pair(sA + stage * A_BYTES, &tmap_a, full_leader, kb * BK, c.row_base);
            tma_load_2d_pair(sB + stage * B_BYTES, &tmap_b, full_leader, kb * BK, b_row);
          } else {
            tma_load_2d(sA + stage * A_BYTES, &tmap_a, &s.full[stage], kb * BK, c.row_base);
            tma_load_2d(sB + stage * B_BYTES, &tmap_b, &s.full[stage], kb * BK, b_row);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, ts = 0, tph = 0;
      int consumed = 0;
      while (true) {
        if (!mbar_wait(&s.tile_full[ts], tph, abort_flag, p.err)) break;
        const int tile = *reinterpret_cast<volatile int *>(&s.tile_ring[ts]);
        if (++ts == TILE_RING) {
          ts = 0;
          tph ^= 1u;
        }
        if (tile < 0) break;
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
              if (kPair)
                umma_pair(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32),
                          IDESC, (kb | k) != 0 ? 1u : 0u);
              else
                umma_bf16(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32),
                          IDESC, (kb | k) != 0 ? 1u : 0u);
            }
            if (kPair)
              umma_commit_pair(&s.empty[stage], 0x3);
            else
              umma_commit(&s.empty[stage]);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) {
          if (kPair)
            umma_commit_pair(&s.tfull[acc], 0x3);
          else
            umma_commit(&s.tfull[acc]);
        }
        __syncwarp();
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (lane == 0) s.mma_consumed = consumed;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    uint32_t acc = 0, acc_phase = 0, ts = 0, tph = 0;
    while (true) {
      if (!mbar_wait(&s.tile_full[ts], tph, abort_flag, p.err, kPair)) break;
      const int tile = *reinterpret_cast<volatile int *>(&s.tile_ring[ts]);
      const uint32_t slot = ts;
      if (++ts == TILE_RING) {
        ts = 0;
        tph ^= 1u;
      }
      if (tile < 0) break;
      const TileCoord c = decode_tile<kPair>(s, groups, n_tiles, m_chunk, tile, rank);
      if (!mbar_wait(&s.tfull[acc], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      bool valid = row < c.rows;
      int a = valid ? p.sorted[c.row_base + row] : 0;
      if (valid && (a < 0 || a >= p.n_rows_y)) {
        record_error(p.err, MOE_ERR_BAD_INDEX);
        valid = false;
      }
      const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(q * 32) << 16);
      bool sat = false;
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
              packed[j] = pack_f16x2_sat(g0 * sigmoidf_(g0) * u0, g1 * sigmoidf_(g1) * u1, sat);
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
        uint16_t *yrow = reinterpret_cast<uint16_t *>(p.out) + static_cast<size_t>(a) * p.out_ld + c.n0;
#pragma unroll 1
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(taddr + ch * 32, r);
          tmem_ld_wait();
          if (valid) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              packed[j] = pack_f16x2_sat(gv * __uint_as_float(r[2 * j]), gv * __uint_as_float(r[2 * j + 1]), sat);
            uint4 *dst = reinterpret_cast<uint4 *>(yrow + ch * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2],
                                  packed[4 * v + 3]);
          }
        }
      }
      if (sat) record_error(p.err, MOE_ERR_RANGE);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // the accumulator is drained and, past tfull, every reader of this tile
        // id (both producers, the MMA warp) has read it: free both
        if (leader) {
          mbar_arrive(&s.tempty[acc]);
          mbar_arrive(&s.tile_empty[slot]);
        } else {
          mbar_arrive_remote(cluster_map(&s.tempty[acc], 0));
          mbar_arrive_remote(cluster_map(&s.tile_empty[slot], 0));
        }
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- teardown.  On the error path wait (bounded) for copies and MMAs still
  // in flight before shared and tensor memory are given back; then both CTAs
  // of the pair meet so neither leaves while the other may still touch its
  // shared memory.
  __syncthreads();
  if (s.abort_flag) {
    if (warp == 0 && lane == 0) {
      // the leader's full barriers count both CTAs' bytes; the peer waits a
      // bounded time for its own copies to land
      const uint64_t t0 = global_timer_ns();
      if (leader) {
        for (int i = s.mma_consumed; i < issued; ++i) {
          const uint32_t a = smem_addr(&s.full[i % STAGES]);
          while (!mbar_try_wait(a, static_cast<uint32_t>((i / STAGES) & 1)) &&
                 global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      } else {
        while (global_timer_ns() - t0 < 1000000ull) {
        }
      }
    }
    if (warp == 1 && lane == 0 && leader) {
      if (kPair)
        umma_commit_pair(&s.drain, 0x1);
      else
        umma_commit(&s.drain);
      const uint32_t a = smem_addr(&s.drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(a, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (kPair)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int kMode>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gg::THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                             const __grid_constant__ CUtensorMap tmap_b, GemmArgs p) {
  grouped_gemm_body<kMode, true>(tmap_a, tmap_b, p);
}

template <int kMode>
__global__ void __launch_bounds__(gg::THREADS, 1)
    grouped_gemm_solo_kernel(const __grid_constant__ CUtensorMap tmap_a,
                             const __grid_constant__ CUtensorMap tmap_b, GemmArgs p) {
  grouped_gemm_body<kMode, false>(tmap_a, tmap_b, p);
}

bool gemm_use_pairs(int64_t T, int K, int E) { return T * K >= 512LL * E; }

int gemm_b_box_rows(bool pair) { return pair ? gg::Cfg<true>::B_ROWS : gg::Cfg<false>::B_ROWS; }

template <int kMode>
static cudaError_t launch_mode(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &p,
                               bool pair, int num_sms, cudaStream_t stream) {
  static int cached_units[2][2][64] = {{{0}}};
  int dev = 0;
  cudaGetDevice(&dev);
  int &units = cached_units[kMode][pair ? 1 : 0][dev & 63];
  if (pair) {
    auto kern = grouped_gemm_pair_kernel<kMode>;
    constexpr size_t smem = gg::smem_bytes<true>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (units == 0) {  // persistent: as many CTA pairs as can be resident at once
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(num_sms & ~1);
      cfg.blockDim = dim3(gg::THREADS);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters <= 0)
        clusters = num_sms / 2;
      units = clusters;
    }
    kern<<<2 * units, gg::THREADS, smem, stream>>>(ta, tb, p);
  } else {
    auto kern = grouped_gemm_solo_kernel<kMode>;
    constexpr size_t smem = gg::smem_bytes<false>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, gg::THREADS, smem, stream>>>(ta, tb, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int mode, bool pair, const CUtensorMap &ta, const CUtensorMap &tb,
                                const GemmArgs &p, int num_sms, cudaStream_t stream) {
  if (mode == kUp) return launch_mode<kUp>(ta, tb, p, pair, num_sms, stream);
  return launch_mode<kDown>(ta, tb, p, pair, num_sms, stream);
}

}  // namespace srm
