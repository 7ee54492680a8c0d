// grouped_gemm.cu -- the two expert contractions of the mixture on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory),
// fed by TMA, as one persistent, warp-specialised kernel template that runs
// on CTA pairs (or single CTAs for small batches).
//
// Definition ("GLM-5 . MoE transformer block", "All 43 steps", Mixture of
// experts): per expert i and token row x,
//     g = x W1_i,  u = x W3_i,  a = g sigmoid(g),  h = a (.) u,  E_i = h W2_i,
// and the shared expert the same way at weight 1; the routed outputs are
// weighted by G_i ("expert_outputs: each routing slot's weighted expert
// output", nnterp GLM-5 page, The API table).
//
// Operand roles: the WEIGHTS are the MMA's M side and the TOKENS its N side,
// D^T[weight row][token] = W_g[weight rows] . X[tokens]^T.  M is fixed (256
// weight rows per CTA pair, 128 per single CTA), and N, the tile's token
// count, can be any multiple of 16 up to 256: a group whose row count is not a
// multiple of 256 pads its last tile to 16 rows, not to 256 (with tokens on
// the M side, 16.8% of the rows of the 16384-token GLM-5 block were padding).
// (Measured on B200: a k-block of a pair tile takes about as long at 16 tokens
// as at 256, so such a tail still costs about a full tile's time.)
//
//   kUp   : for every group g (routed experts 0..E-1, shared expert E), the
//           packed W13_g rows against its token rows (xs: token rows in
//           expert-sorted order, gather.cu).  W13 is packed in units of 32
//           rows, 16 gate rows then the 16 matching up rows, so a warp's 32
//           TMEM lanes hold gate and up of 16 features; each 32-token chunk
//           is transposed through shared memory so that a lane holds one
//           token's 16 gate and 16 up values: h = silu(g) * u -> fp16
//           h[row][I] (three more mantissa bits than bf16 at the same
//           tensor-core rate; |h| saturates at 65504, flagged MOE_ERR_RANGE).
//   kDown : W2_g rows (output features, fp16; an exact conversion of bf16
//           weights in fp16's normal range) against the token rows of h
//           (fp16); epilogue multiplies by the routing gate (1 for the shared
//           expert) and stores fp16 to the row's (token, slot) position
//           (saturation at 65504 flagged MOE_ERR_RANGE).
//
// Tiling: a work tile is (group, weight block of 256 rows, token block of up
// to 256 rows).  On a CTA pair each CTA loads 128 of the weight rows and half
// of the tile's token rows (N/2: one 128-row TMA box for a full tile, boxes of
// 32 rows for a group's last, partial one), the leader issues
// tcgen05.mma.cta_group::2 with M = 256 and N = the tile's token count
// rounded up to 16, and each CTA receives its 128 weight rows x N tokens in
// its own tensor memory.  K loop in steps of 64 (one 128-byte swizzle atom), a
// 6-stage TMA ring per CTA (8 for single CTAs), two accumulators of 256
// columns so the epilogue of one tile overlaps the main loop of the next.
// Warp roles (6 warps per CTA):
//   warp 0: TMA producer (one lane issues the CTA's weight and token loads)
//   warp 1: tensor-memory allocation; in the leader also single-thread MMA issue
//   warps 2-5: epilogue (tensor memory -> registers -> global)
// Work tiles are ordered (group, weight block, token block), token block
// fastest; a unit (CTA pair or single CTA) takes its tiles from a global
// atomic counter (the leader keeps two ids published ahead), so the tiles that share a weight
// block start together and read it from DRAM once; the per-group token-block
// counts come from the group offsets on the device, so the host never
// synchronises.
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
constexpr int BM = 128;        // weight rows per CTA (tensor-memory lanes)
constexpr int BK = 64;
constexpr int TOK_BOX = 32;    // token rows per TMA box of a tail tile
constexpr int TOK_BOX_BIG = 128;  // token rows per TMA box when a CTA's rows are a multiple of it
#ifndef SRM_GEMM_EPI_WARPS
#define SRM_GEMM_EPI_WARPS 4
#endif
constexpr int EPI_WARPS = SRM_GEMM_EPI_WARPS;  // 4, or 8 (two per tensor-memory lane quarter)
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int MAX_GROUPS = 257;
constexpr int MAX_STAGES = 8;
constexpr int TILE_RING = 4;  // tile ids in flight between the scheduler and the roles

// kPair: a CTA pair shares each tile (M = 256 weight rows, each CTA loads 128
// of them and half of up to 256 tokens).  Solo (small batches, where the
// experts hold a few rows each and the weights stream from HBM): one CTA per
// tile, M = 128, up to 64 tokens, so that a stage is 16 KB of weights + 8 KB
// of tokens and 8 of them keep 128 KB of weights in flight per SM.
template <bool kPair>
struct Cfg {
  static constexpr int BT = kPair ? 256 : 64;           // tokens per tile (largest MMA N)
  static constexpr int W_BLOCK = kPair ? 2 * BM : BM;   // weight rows per tile (MMA M)
  static constexpr int TOK_ROWS = kPair ? BT / 2 : BT;  // token rows one CTA holds at most
  static constexpr int STAGES = kPair ? (EPI_WARPS == 8 ? 5 : 6) : (EPI_WARPS == 8 ? 7 : 8);
  static constexpr int A_BYTES = BM * BK * 2;           // 16 KB of weights
  static constexpr int B_BYTES = TOK_ROWS * BK * 2;     // 16 or 8 KB of token rows at most
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BT;  // two accumulators (512 or 128 columns)
  static constexpr uint32_t EPI_ARRIVALS = (kPair ? 2 : 1) * EPI_WARPS;
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
  float epi[EPI_WARPS][32][33];  // one 32 x 32 transpose buffer per epilogue warp (padded rows)
};
template <bool kPair>
constexpr size_t smem_bytes() {
  return 1024 /*alignment slack*/ + Cfg<kPair>::STAGES * Cfg<kPair>::STAGE_BYTES + sizeof(Smem);
}
static_assert(smem_bytes<true>() <= 232448 && smem_bytes<false>() <= 232448,
              "grouped GEMM shared memory above 227 KB");
}  // namespace gg

struct TileCoord {
  int g;          // group
  int row_base;   // first token row of the tile (expert-sorted order)
  int rows;       // valid token rows (1 .. BT)
  int n;          // MMA N: rows rounded up to 16
  int w0;         // first weight row of the tile within the group
};

// Tiles of group g occupy [tile_start[g] * n_tiles, tile_start[g+1] * n_tiles)
// and inside a group the token block runs fastest: the units working at the
// same moment share each 256-row weight block (one DRAM read serves all the
// group's token blocks) instead of spreading over many weight blocks that
// evict one another from L2.  A group with more than m_chunk token blocks (the
// shared expert at large batches) is walked in chunks of m_chunk token blocks,
// each chunk through all weight blocks, so that the chunk's token rows stay in
// L2 while every weight block reads them (a whole 16384-token group would not
// fit and would be re-read from DRAM once per weight block).
template <bool kPair>
__device__ __forceinline__ TileCoord decode_tile(const gg::Smem &s, int groups, int n_tiles,
                                                 int m_chunk, int tile) {
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
  const int cm = min(m_chunk, mblocks - m0);  // token blocks in this chunk
  const int r = local - m0 * n_tiles;
  const int nt = r / cm;
  const int mt = m0 + (r - nt * cm);
  constexpr int BT = gg::Cfg<kPair>::BT;
  TileCoord c;
  c.g = lo;
  c.row_base = s.grp_off[lo] + mt * BT;
  c.rows = max(0, min(BT, s.grp_off[lo + 1] - c.row_base));
  c.n = max(16, (c.rows + 15) & ~15);
  c.w0 = nt * gg::Cfg<kPair>::W_BLOCK;
  return c;
}

// fp32 -> fp16 bits (round to nearest even), saturating at +-65504 (sets sat)
__device__ __forceinline__ uint16_t f16_sat(float v, bool &sat) {
  sat |= !(fabsf(v) <= 65504.f);
  return __half_as_ushort(__float2half_rn(fminf(fmaxf(v, -65504.f), 65504.f)));
}

template <int kMode, bool kPair>
__device__ __forceinline__ void grouped_gemm_body(const CUtensorMap &tmap_tok, const CUtensorMap &tmap_tok_big,
                                                  const CUtensorMap &tmap_w, const GemmArgs &p) {
  using namespace gg;
  using C = Cfg<kPair>;
  constexpr int BT = C::BT;
  constexpr uint32_t TMEM_COLS = C::TMEM_COLS;
  constexpr int STAGES = C::STAGES;
  constexpr int A_BYTES = C::A_BYTES;
  constexpr int B_BYTES = C::B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t *sA = base;                   // weights
  uint8_t *sB = base + STAGES * A_BYTES;  // token rows
  Smem &s = *reinterpret_cast<Smem *>(base + STAGES * C::STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int groups = p.groups;
  const int n_tiles = p.n_total / C::W_BLOCK;
  const int kblocks = p.k_total / BK;
  // token blocks per chunk: about 48 MB of token rows (16-bit operands)
  const int m_chunk = max(1, (48 << 20) / (BT * p.k_total * 2));
  // up: bf16 W13 times bf16 x; down: fp16 W2 times fp16 h
  constexpr uint32_t AB_BF16 = kMode == kUp ? 1u : 0u;

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
    tma_prefetch_desc(&tmap_tok);
    tma_prefetch_desc(&tmap_tok_big);
    tma_prefetch_desc(&tmap_w);
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
    // group offsets and an exclusive scan of ceil(count / BT) over the
    // groups.  Offsets come from the caller: a group whose range is not
    // 0 <= o0 <= o1 <= n_rows_y (or a first offset other than 0, which is how
    // the allocation-free permutation flags a bad id) gets no tiles and is
    // flagged MOE_ERR_BAD_INDEX, so no row outside the buffers is touched.
    // A group's end is the next group's raw start, so a valid group keeps its
    // own bounds even when its neighbour is rejected.
    auto token_blocks = [&](int g) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      if (o0 < 0 || o1 < o0 || o1 > p.n_rows_y || (g == 0 && o0 != 0)) {
        record_error(p.err, MOE_ERR_BAD_INDEX);
        return 0;
      }
      return (o1 - o0 + BT - 1) / BT;
    };
    const int per = (groups + 31) / 32;
    const int g0 = lane * per;
    int local = 0;
    for (int g = g0; g < min(g0 + per, groups); ++g) {
      s.grp_off[g] = p.offsets[g];
      local += token_blocks(g);
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
      run += token_blocks(g);
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
    // tile from the global counter, so tiles sharing a weight block (one
    // group's token blocks) start at nearly the same moment on whichever units
    // are free, and publishes the id to its own CTA and to the peer through
    // the tile ring.
    uint32_t stage = 0, phase = 0, ts = 0, tph = 0;
    // The leader keeps LOOKAHEAD tile ids published ahead of the tile it loads,
    // so the counter's round trip and the signal to the peer are off the
    // critical path: when one tile's last loads are issued the next id is
    // already known (measured: a per-tile bubble of ~2.8 k cycles otherwise).
    constexpr int LOOKAHEAD = 2;
    uint32_t ps = 0, pph = 0;  // next ring slot to publish and its phase
    int published = 0, consumed = 0;
    bool last_published = false;
    bool pub_ok = true;
    while (true) {
      while (leader && !last_published && published - consumed < LOOKAHEAD) {
        if (!mbar_wait(&s.tile_empty[ps], pph ^ 1u, abort_flag, p.err)) {
          pub_ok = false;
          break;
        }
        int t = 0;
        if (lane == 0) {
          t = atomicAdd(p.tile_counter, 1);
          if (t >= total_tiles) t = -1;
          s.tile_ring[ps] = t;
          mbar_arrive(&s.tile_full[ps]);
          if (kPair) {
            st_shared_remote(cluster_map(&s.tile_ring[ps], 1), t);
            mbar_arrive_remote(cluster_map(&s.tile_full[ps], 1));
          }
        }
        t = __shfl_sync(0xffffffffu, t, 0);
        last_published = t < 0;
        ++published;
        if (++ps == TILE_RING) {
          ps = 0;
          pph ^= 1u;
        }
      }
      if (!pub_ok) break;
      if (!mbar_wait(&s.tile_full[ts], tph, abort_flag, p.err, kPair)) break;
      ++consumed;
      const int tile = *reinterpret_cast<volatile int *>(&s.tile_ring[ts]);
      if (++ts == TILE_RING) {
        ts = 0;
        tph ^= 1u;
      }
      if (tile < 0 || p.stall) break;
      const TileCoord c = decode_tile<kPair>(s, groups, n_tiles, m_chunk, tile);
      const int w_row = c.g * p.n_total + c.w0 + rank * BM;   // this CTA's weight rows
      const int tok_rows = kPair ? c.n / 2 : c.n;             // this CTA's token rows
      const int tok_row0 = c.row_base + rank * tok_rows;
      // full tiles: one or two 128-row boxes (each TMA instruction costs issue
      // time on the single producer lane); tails: 32-row boxes
      const bool big = tok_rows % TOK_BOX_BIG == 0;
      const int box_rows = big ? TOK_BOX_BIG : TOK_BOX;
      const CUtensorMap *tmap_b = big ? &tmap_tok_big : &tmap_tok;
      const int nb = (tok_rows + box_rows - 1) / box_rows;
      const uint32_t tx = (kPair ? 2u : 1u) * static_cast<uint32_t>(A_BYTES + nb * box_rows * BK * 2);
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&s.full[stage], tx);
          uint8_t *b_dst = sB + stage * B_BYTES;
          if (kPair) {
            const uint32_t full_leader = cluster_map(&s.full[stage], 0);
            tma_load_2d_pair(sA + stage * A_BYTES, &tmap_w, full_leader, kb * BK, w_row);
            for (int j = 0; j < nb; ++j)
              tma_load_2d_pair(b_dst + j * box_rows * BK * 2, tmap_b, full_leader, kb * BK,
                               tok_row0 + j * box_rows);
          } else {
            tma_load_2d(sA + stage * A_BYTES, &tmap_w, &s.full[stage], kb * BK, w_row);
            for (int j = 0; j < nb; ++j)
              tma_load_2d(b_dst + j * box_rows * BK * 2, tmap_b, &s.full[stage], kb * BK,
                          tok_row0 + j * box_rows);
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
        const TileCoord c = decode_tile<kPair>(s, groups, n_tiles, m_chunk, tile);
        const uint32_t idesc = umma_idesc_f32acc(C::W_BLOCK, c.n, AB_BF16);
        if (!mbar_wait(&s.tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BT;
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
                          idesc, (kb | k) != 0 ? 1u : 0u);
              else
                umma_bf16(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32),
                          idesc, (kb | k) != 0 ? 1u : 0u);
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
    // Warp q = warp % 4 may read tensor-memory lanes 32q .. 32q+31: this
    // CTA's weight rows w0 + rank*128 + 32q + lane, one lane per weight row,
    // the tile's tokens along the columns.
    const int q = warp & 3;
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
      const TileCoord c = decode_tile<kPair>(s, groups, n_tiles, m_chunk, tile);
      const int wr = c.w0 + static_cast<int>(rank) * BM + q * 32;  // this warp's first weight row
      constexpr int CHUNKS = BT / 32;
      // kDown: each token's destination row and gate, lane holding tokens
      // lane + 32m.  They do not depend on the accumulator, so they are read
      // while the tile's MMAs still run.
      int my_a[CHUNKS];
      float my_g[CHUNKS];
      if (kMode == kDown) {
#pragma unroll
        for (int m = 0; m < CHUNKS; ++m)
          my_a[m] = 32 * m + lane < c.rows ? p.sorted[c.row_base + 32 * m + lane] : -1;
#pragma unroll
        for (int m = 0; m < CHUNKS; ++m) {
          my_g[m] = 0.f;
          if (32 * m + lane < c.rows) {
            if (my_a[m] < 0 || my_a[m] >= p.n_rows_y) {
              record_error(p.err, MOE_ERR_BAD_INDEX);
              my_a[m] = -1;
            } else {
              my_g[m] = my_a[m] < p.tk ? p.gate[my_a[m]] : 1.0f;
            }
          }
        }
      }
      if (!mbar_wait(&s.tfull[acc], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * BT + (static_cast<uint32_t>(q * 32) << 16);
      bool sat = false;
      // 32-token chunks (each read from tensor memory and waited for before use)
#pragma unroll
      for (int m = 0; m < CHUNKS; ++m) {
        if (32 * m >= c.n) break;  // uniform across the warp
        if (EPI_WARPS == 8 && (m & 1) != ((warp - 2) >> 2)) continue;  // the other warp of this quarter
        uint32_t cv[32];
        tmem_ld32(taddr + 32 * m, cv);
        tmem_ld_wait();
        // transpose the 32 weight rows x 32 tokens chunk through this warp's
        // buffer (row stride 33: both passes conflict-free), so that lane l
        // owns token 32m + l and reads its 32 values from its own row
        float(&buf)[32][33] = s.epi[warp - 2];
#pragma unroll
        for (int k = 0; k < 32; ++k) buf[k][lane] = __uint_as_float(cv[k]);
        __syncwarp();
        if (kMode == kUp) {
          // rows 0-15 of the chunk are the gate rows of features j0 .. j0+15,
          // rows 16-31 the matching up rows (the 32-row packing unit): lane l
          // computes h = silu(g) * u of its token for the 16 features and
          // writes them as two 16-byte stores (32 contiguous bytes of its h row)
          if (32 * m + lane < c.rows) {
            uint32_t packed[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float g0 = buf[lane][2 * j], g1 = buf[lane][2 * j + 1];
              const float u0 = buf[lane][16 + 2 * j], u1 = buf[lane][16 + 2 * j + 1];
              packed[j] = pack_f16x2_sat(silu_approx(g0) * u0, silu_approx(g1) * u1, sat);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) +
                                                   static_cast<size_t>(c.row_base + 32 * m + lane) * p.out_ld +
                                                   wr / 2);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
        } else {
          // lane l: its token's destination and gate, its 32 output features
          // (64 contiguous bytes of the slot row) in four 16-byte stores
          if (my_a[m] >= 0) {
            const float gv = my_g[m];
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              packed[j] = pack_f16x2_sat(gv * buf[lane][2 * j], gv * buf[lane][2 * j + 1], sat);
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) +
                                                   static_cast<size_t>(my_a[m]) * p.out_ld + wr);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(packed[4 * v4], packed[4 * v4 + 1], packed[4 * v4 + 2], packed[4 * v4 + 3]);
          }
        }
        __syncwarp();  // the buffer is read before the next chunk overwrites it
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
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_tok,
                             const __grid_constant__ CUtensorMap tmap_tok_big,
                             const __grid_constant__ CUtensorMap tmap_w, GemmArgs p) {
  grouped_gemm_body<kMode, true>(tmap_tok, tmap_tok_big, tmap_w, p);
}

template <int kMode>
__global__ void __launch_bounds__(gg::THREADS, 1)
    grouped_gemm_solo_kernel(const __grid_constant__ CUtensorMap tmap_tok,
                             const __grid_constant__ CUtensorMap tmap_tok_big,
                             const __grid_constant__ CUtensorMap tmap_w, GemmArgs p) {
  grouped_gemm_body<kMode, false>(tmap_tok, tmap_tok_big, tmap_w, p);
}

// CTA pairs unless the experts average fewer than 8 rows each (decode), where
// single CTAs keep more weight bytes in flight per SM
bool gemm_use_pairs(int64_t T, int K, int E) { return T * K >= 8LL * (E > 0 ? E : 1); }

int gemm_tok_box_rows() { return gg::TOK_BOX; }
int gemm_tok_big_box_rows() { return gg::TOK_BOX_BIG; }
int gemm_w_box_rows() { return gg::BM; }

template <int kMode>
static cudaError_t launch_mode(const TokMaps &tok, const CUtensorMap &tw, const GemmArgs &p, bool pair,
                               int num_sms, cudaStream_t stream) {
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
    kern<<<2 * units, gg::THREADS, smem, stream>>>(tok.small, tok.big, tw, p);
  } else {
    auto kern = grouped_gemm_solo_kernel<kMode>;
    constexpr size_t smem = gg::smem_bytes<false>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<num_sms, gg::THREADS, smem, stream>>>(tok.small, tok.big, tw, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int mode, bool pair, const TokMaps &tok, const CUtensorMap &tw,
                                const GemmArgs &p, int num_sms, cudaStream_t stream) {
  if (mode == kUp) return launch_mode<kUp>(tok, tw, p, pair, num_sms, stream);
  return launch_mode<kDown>(tok, tw, p, pair, num_sms, stream);
}

}  // namespace srm
