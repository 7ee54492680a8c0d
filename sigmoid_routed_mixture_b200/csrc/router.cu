// router.cu -- the router in one kernel: logits on the tensor cores, then
// sigmoid scores, biased top-K selection and renormalised, scaled gates.
//
// Definition ("GLM-5 . MoE transformer block", "All 43 steps", Mixture of
// experts):  z = x W_r;  s = sigmoid(z);  E_sel_i = [i in top_K(s + b)];
//            G_i = scale * s_i E_sel_i / sum_j s_j E_sel_j.
// The bias takes part in the choice only; the gates use the un-biased s
// (nnterp GLM-4.7-Flash / GLM-5, section 03, note "The mixture: sigmoid
// scores, a selection bias, renormalized weights").  Ties between equal keys
// go to the lower expert index; the slots come out in descending key order.
//
// W_r is fp32 and x is bf16.  W_r is split exactly-to-fp32-precision into
// three bf16 parts (hi = bf16(W), mid = bf16(W - hi), lo = bf16(W - hi - mid);
// what is left is below 2^-24 |W|), so z = x.hi + x.mid + x.lo with every
// product exact and fp32 accumulation: fp32-accurate logits at bf16 tensor-
// core speed.
//   1) router_split_kernel: W_r -> [3][E_pad][H] bf16 (E_pad = E rounded up
//      to 64, padding rows zero).  A property of the weights: moe_pack_router
//      runs it once; moe_route (fp32 W_r given per call) runs it every call.
//   2) router_kernel: 128 tokens x E_pad experts per CTA, tcgen05.mma
//      kind::f16 (bf16) into tensor memory, TMA-fed ring, short accumulation
//      chains promoted to fp32 registers (see below), then the selection in
//      the same kernel:
//        - one CTA per 128 tokens (no split of H): the epilogue warps stage
//          their fp32 z rows in shared memory (the drained operand ring); one
//          thread per (token, half of the experts) builds a sorted top-(K+1)
//          list of (key, expert) in registers, the halves merge, and the
//          first half's thread writes experts, gates and margin.  z never
//          reaches global memory unless asked for.
//        - few 128-token tiles (decode): the H range is split over S CTAs;
//          each writes fp32 partial logits (whole rows, through shared
//          memory), all CTAs of the grid (at most one per SM, so all resident
//          together) meet at a bounded grid barrier, then every CTA takes
//          some tokens, sums the S partials in a fixed order (deterministic)
//          and selects: a CTA-wide ranking for a single token, otherwise K + 1
//          rounds of a warp arg-max (key descending, index ascending) per token
//          (two tokens' rounds interleaved per warp up to 64 experts).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace srm {

namespace rt {
constexpr int BM = 128;
constexpr int BK = 64;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;  // warp 0 TMA, warp 1 MMA + TMEM, 8 epilogue warps
#ifndef SRM_ROUTER_CHUNK
#define SRM_ROUTER_CHUNK 2
#endif
constexpr int CHUNK = SRM_ROUTER_CHUNK;       // k-blocks per tensor-core accumulation chain
constexpr int A_BYTES = BM * BK * 2;
constexpr int MAX_SMEM = 232448;  // 227 KB dynamic shared memory per CTA
}  // namespace rt

int router_e_pad(int E) { return (E + 63) / 64 * 64; }

int router_stage_bytes(int e_pad) { return rt::A_BYTES + 3 * e_pad * rt::BK * 2; }

struct RouterSmem;
int router_stages(int e_pad, bool pair);

constexpr int kMaxSplits = 96;       // up to 96 CTAs stream W_r at decode (one k-block each at H 6144)
constexpr int kRowBatch = 8;         // token rows a CTA reduces and selects at a time after a split
constexpr int kRankRows = 1;         // a batch of this many rows takes the CTA-wide rank selection
constexpr int kPairMinTiles = 9;     // from this many 128-token tiles on, CTA pairs

// Upper bound of the split count for any SM count (sizes the partials).
int router_splits(int T, int H) {
  const int m_tiles = (T + rt::BM - 1) / rt::BM;
  const int kblocks = H / rt::BK;
  int s = 148 / (m_tiles > 0 ? m_tiles : 1);
  const int max_s = kblocks > 0 ? kblocks : 1;
  if (s > max_s) s = max_s;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  return s;
}

// ---------------------------------------------------------------- 1) split

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Eight consecutive weights per thread: two 16-byte loads, three 16-byte stores.
__global__ void __launch_bounds__(256)
    router_split_kernel(const float *__restrict__ w_r, int E, int e_pad, int H,
                        uint16_t *__restrict__ wsplit) {
  const int64_t n = static_cast<int64_t>(e_pad) * H;
  const int64_t n8 = n / 8;  // H is a multiple of 256
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = (i * 8) / H;
    float w[8];
    if (e < E) {
      const float4 a = reinterpret_cast<const float4 *>(w_r)[2 * i];
      const float4 b = reinterpret_cast<const float4 *>(w_r)[2 * i + 1];
      w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0.f;
    }
    uint16_t hi[8], mid[8], lo[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      hi[k] = bf16_rn_bits(w[k]);
      const float r1 = w[k] - bf16_bits_to_float(hi[k]);
      mid[k] = bf16_rn_bits(r1);
      const float r2 = r1 - bf16_bits_to_float(mid[k]);
      lo[k] = bf16_rn_bits(r2);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(wsplit);
    dst[i] = make_uint4(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16),
                        hi[4] | (uint32_t(hi[5]) << 16), hi[6] | (uint32_t(hi[7]) << 16));
    dst[n8 + i] = make_uint4(mid[0] | (uint32_t(mid[1]) << 16), mid[2] | (uint32_t(mid[3]) << 16),
                             mid[4] | (uint32_t(mid[5]) << 16), mid[6] | (uint32_t(mid[7]) << 16));
    dst[2 * n8 + i] = make_uint4(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16),
                                 lo[4] | (uint32_t(lo[5]) << 16), lo[6] | (uint32_t(lo[7]) << 16));
  }
}

// ---------------------------------------------------------------- 2) logits + selection

// The tensor core's fp32 accumulator loses precision over long chains of
// MMAs (measured on B200: max |dz| 1.5e-4 after 1152 chained MMAs against
// 4e-6 for an fp32 blocked sum).  So each chunk of CHUNK k-blocks goes to one
// of two ping-pong accumulators, starting from zero, and the epilogue warps
// add every finished chunk into fp32 registers: no accumulation chain is
// longer than CHUNK * 12 MMAs.
struct RouterSmem {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int mma_consumed;
};

struct RouteOut {
  const float *bias;
  int32_t *idx;
  float *gate;
  float *margin;  // may be null
  float *logits;  // may be null: [T][E]
  float scale;
  int T, E, K;
};

// Selection for R tokens by one warp, R independent chains interleaved so the
// shuffles of one token hide the latency of the other's (row r of z at
// zs + r * zstride in shared memory; rows with valid[r] false are computed on
// and not written): s = sigmoid(z), key = s + b, K rounds of a warp arg-max
// (key descending, equal keys to the lower index), one more round for the
// margin; gates = scale * s / sum of the selected s in rank order.  bias_r[j]
// holds bias[lane + 32 j] (this lane's experts).
template <int NE, int R>
__device__ __forceinline__ void select_tokens(const float *zs, int zstride, const int (&t)[R],
                                              const bool (&valid)[R], const float (&bias_r)[NE],
                                              const RouteOut &o, int lane) {
  float key[R][NE], sv[R][NE];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int j = 0; j < NE; ++j) {
      const int e = lane + 32 * j;
      float z = 0.f;
      if (e < o.E) {
        z = zs[r * zstride + e];
        if (o.logits && valid[r]) o.logits[static_cast<size_t>(t[r]) * o.E + e] = z;
      }
      const float sj = sigmoidf_(z);
      sv[r][j] = sj;
      key[r][j] = e < o.E ? sj + bias_r[j] : -INFINITY;
    }
  }
  int my_e[R];
  float my_s[R], kth_key[R], next_key[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    my_e[r] = 0;
    my_s[r] = 0.f;
    kth_key[r] = 0.f;
    next_key[r] = -INFINITY;
  }
  const int K = o.K;
  const int rounds = K < o.E ? K + 1 : K;
  for (int k = 0; k < rounds; ++k) {
    float bk[R], bs[R];
    int be[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      bk[r] = -INFINITY;
      bs[r] = 0.f;
      be[r] = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < NE; ++j) {
        if (key[r][j] > bk[r]) {  // j ascending = expert index ascending: strict > keeps the lower
          bk[r] = key[r][j];
          be[r] = lane + 32 * j;
          bs[r] = sv[r][j];
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk[r], off);
        const int oe = __shfl_xor_sync(0xffffffffu, be[r], off);
        const float os = __shfl_xor_sync(0xffffffffu, bs[r], off);
        if (ok > bk[r] || (ok == bk[r] && oe < be[r])) {
          bk[r] = ok;
          be[r] = oe;
          bs[r] = os;
        }
      }
    }
    if (k == K) {  // the margin round (only when K < E): nothing is taken
#pragma unroll
      for (int r = 0; r < R; ++r) next_key[r] = bk[r];
      break;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (lane == k) {
        my_e[r] = be[r];
        my_s[r] = bs[r];
      }
      if (k == K - 1) kth_key[r] = bk[r];
#pragma unroll
      for (int j = 0; j < NE; ++j)
        if (be[r] == lane + 32 * j) key[r][j] = -INFINITY;
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float denom = 0.f;
    for (int k = 0; k < K; ++k) denom += __shfl_sync(0xffffffffu, my_s[r], k);
    if (!valid[r]) continue;
    if (lane < K) {
      o.idx[static_cast<size_t>(t[r]) * K + lane] = my_e[r];
      o.gate[static_cast<size_t>(t[r]) * K + lane] = o.scale * my_s[r] / denom;
    }
    if (o.margin && lane == 0) o.margin[t[r]] = K < o.E ? kth_key[r] - next_key[r] : INFINITY;
  }
}

// Sorted insert into a top-LK list (keys descending).  Experts arrive in
// ascending index order and an entry is passed only by a strictly greater key,
// so equal keys keep ascending expert order.  A NaN key is never inserted.
template <int LK>
__device__ __forceinline__ void top_insert(float (&lk)[LK], int (&le)[LK], float key, int e) {
  bool c[LK];
#pragma unroll
  for (int j = 0; j < LK; ++j) c[j] = key > lk[j];
#pragma unroll
  for (int j = LK - 1; j > 0; --j) {
    lk[j] = c[j] ? (c[j - 1] ? lk[j - 1] : key) : lk[j];
    le[j] = c[j] ? (c[j - 1] ? le[j - 1] : e) : le[j];
  }
  if (c[0]) {
    lk[0] = key;
    le[0] = e;
  }
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Selection for a staged tile of z rows, one thread per (row, half of the
// experts): the thread scans experts [hf*HALF, min(E, (hf+1)*HALF)) of its row
// in index order (s = sigmoid(z), key = s + b) into a sorted top-LK list
// (LK > K).  The second half's lists pass through shared memory and the first
// half's thread inserts them after its own (all their experts are higher, so
// the order stays key descending, then expert ascending); it then holds the
// token's K experts and the (K+1)-th key, and writes experts, gates
// (scale * s / sum of the selected s, summed in rank order) and the margin.
// All 32 * EPI_WARPS epilogue threads call this (it contains a named barrier);
// `work` false skips the computation only.
template <int LK, int HALF>
__device__ __forceinline__ void select_staged(const float *zr, const float *bias_s, float *list_k,
                                              int *list_e, int row, int hf, int t, bool work,
                                              const RouteOut &o) {
  float lk[LK];
  int le[LK];
#pragma unroll
  for (int j = 0; j < LK; ++j) {
    lk[j] = -INFINITY;
    le[j] = 0x7fffffff;
  }
  const int e0 = hf * HALF;
  const int e1 = min(o.E, e0 + HALF);
  if (work) {
#pragma unroll 1
    for (int e = e0; e < e1; e += 4) {
      const float4 z4 = *reinterpret_cast<const float4 *>(zr + e);
      const float4 b4 = *reinterpret_cast<const float4 *>(bias_s + e);
      const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
      const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (e + i < e1) top_insert<LK>(lk, le, sigmoidf_(zz[i]) + bb[i], e + i);
    }
  }
  if (hf == 1) {
#pragma unroll
    for (int j = 0; j < LK; ++j) {
      list_k[j * rt::BM + row] = lk[j];
      list_e[j * rt::BM + row] = le[j];
    }
  }
  named_barrier(1, 32 * rt::EPI_WARPS);
  if (hf != 0 || !work) return;
#pragma unroll
  for (int j = 0; j < LK; ++j) top_insert<LK>(lk, le, list_k[j * rt::BM + row], list_e[j * rt::BM + row]);
  const int K = o.K;
  float sk[LK];
  float denom = 0.f, kth = 0.f, nxt = -INFINITY;
#pragma unroll
  for (int k = 0; k < LK; ++k) {
    sk[k] = 0.f;
    if (k < K) {
      sk[k] = le[k] < o.E ? sigmoidf_(zr[le[k]]) : 0.f;
      denom += sk[k];
    }
    if (k == K - 1) kth = lk[k];
    if (k == K) nxt = lk[k];
  }
#pragma unroll
  for (int k = 0; k < LK; ++k) {
    if (k < K) {
      o.idx[static_cast<size_t>(t) * K + k] = le[k];
      o.gate[static_cast<size_t>(t) * K + k] = o.scale * sk[k] / denom;
    }
  }
  if (o.margin) o.margin[t] = K < o.E ? kth - nxt : INFINITY;
}

// Selection for up to kRankRows tokens by the whole CTA (a decode-sized batch
// after a split, where one warp per token would leave the latency of its
// rounds exposed).  Thread e < E_PAD owns expert e of every row: key =
// sigmoid(z) + b.  "a beats b" is the selection order: a larger key, or an
// equal key and a lower expert.  (1) Each thread counts the experts of its own
// warp that beat it; the (at most K + 1) it leaves beaten by at most K of them
// are the warp's candidates, kept in LKS slots (LKC rounded up to a multiple
// of four, for 16-byte loads; the rest padding that beats nothing).  (2) A
// candidate's count of the beating candidates of all warps is
// its rank in the whole row whenever that rank is at most K: an expert that
// beats it either is a candidate or is beaten by K + 1 candidates of its warp
// that also beat it, which puts the rank above K anyway.  Ranks 0..K-1 are the
// K slots in order, rank K gives the margin.  NaN and -inf keys are never
// selected, as in the other selection paths.  All threads of the CTA call this
// (it has __syncthreads); rows r < nb sit at zs + r * zstride.
template <int E_PAD, int LKC>
__device__ __forceinline__ void select_rank_rows(const float *zs, int zstride, int nb, float my_bias,
                                                 float *scratch, int t0, int t_step, const RouteOut &o) {
  constexpr int NWARP = E_PAD / 32;
  constexpr int R = kRankRows;
  constexpr int LKS = (LKC + 3) / 4 * 4;                           // slots per warp (16-byte rows)
  float *key_s = scratch;                                          // [R][E_PAD]
  float *cand_k = key_s + R * E_PAD;                               // [R][NWARP][LKS]
  int *cand_e = reinterpret_cast<int *>(cand_k + R * NWARP * LKS);  // [R][NWARP][LKS]
  float *sel_k = reinterpret_cast<float *>(cand_e + R * NWARP * LKS);  // [R][17]
  float *sel_s = sel_k + R * 17;                                   // [R][17]
  int *sel_e = reinterpret_cast<int *>(sel_s + R * 17);            // [R][17]
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int K = o.K;
  const bool mine = tid < o.E;
  float key[R], sv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    key[r] = -INFINITY;
    sv[r] = 0.f;
    if (r < nb && tid < E_PAD) {
      if (mine) {
        const float z = zs[r * zstride + tid];
        if (o.logits) o.logits[static_cast<size_t>(t0 + r * t_step) * o.E + tid] = z;
        sv[r] = sigmoidf_(z);
        key[r] = sv[r] + my_bias;
      }
      key_s[r * E_PAD + tid] = key[r];
    }
  }
  if (tid < R * 17) {
    sel_k[tid] = 0.f;
    sel_s[tid] = 0.f;
    sel_e[tid] = 0x7fffffff;
  }
  __syncthreads();
  bool cand[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    cand[r] = false;
    if (r < nb && w < NWARP) {
      const float4 *wk = reinterpret_cast<const float4 *>(key_s + r * E_PAD + 32 * w);
      int beaten = 0;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 k4 = wk[j4];
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) beaten += (4 * j4 + i < lane) ? (kk[i] >= key[r]) : (kk[i] > key[r]);
      }
      cand[r] = mine && key[r] > -INFINITY && beaten <= K;  // NaN compares false
      const unsigned m = __ballot_sync(0xffffffffu, cand[r]);
      const int n = __popc(m);
      if (cand[r]) {  // candidates fill slots 0..n-1
        const int slot = __popc(m & ((1u << lane) - 1u));
        cand_k[(r * NWARP + w) * LKS + slot] = key[r];
        cand_e[(r * NWARP + w) * LKS + slot] = tid;
      }
      if (lane >= n && lane < LKS) {  // lane l pads slot l
        cand_k[(r * NWARP + w) * LKS + lane] = -INFINITY;
        cand_e[(r * NWARP + w) * LKS + lane] = 0x7fffffff;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (cand[r]) {
      int rank = 0;
      const float4 *ck = reinterpret_cast<const float4 *>(cand_k + r * NWARP * LKS);
      const int4 *ce = reinterpret_cast<const int4 *>(cand_e + r * NWARP * LKS);
#pragma unroll
      for (int i = 0; i < NWARP * LKS / 4; ++i) {
        const float4 kc = ck[i];
        const int4 ec = ce[i];
        rank += (kc.x > key[r]) || (kc.x == key[r] && ec.x < tid);
        rank += (kc.y > key[r]) || (kc.y == key[r] && ec.y < tid);
        rank += (kc.z > key[r]) || (kc.z == key[r] && ec.z < tid);
        rank += (kc.w > key[r]) || (kc.w == key[r] && ec.w < tid);
      }
      if (rank <= K) {
        sel_k[r * 17 + rank] = key[r];
        if (rank < K) {
          sel_s[r * 17 + rank] = sv[r];
          sel_e[r * 17 + rank] = tid;
        }
      }
    }
  }
  __syncthreads();
  if (tid < nb * K) {
    const int r = tid / K, k = tid - r * K;
    const int t = t0 + r * t_step;
    float denom = 0.f;
    for (int i = 0; i < K; ++i) denom += sel_s[r * 17 + i];
    o.idx[static_cast<size_t>(t) * K + k] = sel_e[r * 17 + k];
    o.gate[static_cast<size_t>(t) * K + k] = o.scale * sel_s[r * 17 + k] / denom;
    if (k == 0 && o.margin) o.margin[t] = K < o.E ? sel_k[r * 17 + K - 1] - sel_k[r * 17 + K] : INFINITY;
  }
}

// NH = e_pad / 64: each epilogue thread keeps half a row (e_pad / 2 columns).
// kSplit: the H range is split over gridDim.y CTAs (partials + grid barrier).
// kPair (enough token tiles; with or without a split): clusters of two CTAs run tcgen05.mma.cta_group::2
// with M = 256 tokens; each CTA loads its 128 token rows and half of every
// part's expert rows, so each byte of the split W_r crosses L2 once per 256
// tokens instead of once per 128, and a stage is small enough for 3 of them.
template <int NH, bool kSplit, bool kPair>
__global__ void __launch_bounds__(rt::THREADS, 1)
    router_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  int kb_per_split, int kblocks, int stages, uint32_t tmem_cols,
                  float *__restrict__ zp, int *grid_counter, RouteOut o, int *err) {
  using namespace rt;
  constexpr int e_pad = NH * 64;
  constexpr int HALF = e_pad / 2;
  constexpr int NE = e_pad / 32;         // experts per lane in the selection
  constexpr int ZS = e_pad + 4;          // shared-memory row stride of staged z (floats)
  constexpr int W_ROWS = kPair ? e_pad / 2 : e_pad;  // expert rows of each part this CTA loads
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  constexpr int stage_bytes = A_BYTES + 3 * W_ROWS * BK * 2;
  RouterSmem &s = *reinterpret_cast<RouterSmem *>(base + stages * stage_bytes);
  float *zs = reinterpret_cast<float *>(base);  // staged z rows, over the drained ring

  const int T = o.T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int m0 = blockIdx.x * BM;  // a pair's two CTAs are x = 2p, 2p + 1: tokens 256p, 256p + 128
  const int split = blockIdx.y;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(kblocks, kb0 + kb_per_split);
  const int nchunks = (kb1 - kb0 + CHUNK - 1) / CHUNK;
  constexpr uint32_t part_bytes = static_cast<uint32_t>(W_ROWS) * BK * 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], (kPair ? 2 : 1) * EPI_WARPS);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    s.mma_consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&s.tmem_base, tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s.tmem_base, tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kPair)
    cluster_sync();  // the peer's barriers are initialised before any remote use
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int *abort_flag = &s.abort_flag;
  int issued = 0;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    uint32_t stage = 0, phase = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&s.empty[stage], phase ^ 1u, abort_flag, err)) break;
      if (lane == 0) {
        uint8_t *st = base + stage * stage_bytes;
        if (kPair) {
          // both CTAs' copies complete on the leader's barrier
          if (leader) mbar_arrive_expect_tx(&s.full[stage], 2 * stage_bytes);
          const uint32_t full_leader = cluster_map(&s.full[stage], 0);
          tma_load_2d_pair(st, &tmap_x, full_leader, kb * BK, m0);
          for (int part = 0; part < 3; ++part)
            tma_load_2d_pair(st + A_BYTES + part * part_bytes, &tmap_w, full_leader, kb * BK,
                             part * e_pad + static_cast<int>(rank) * W_ROWS);
        } else {
          mbar_arrive_expect_tx(&s.full[stage], stage_bytes);
          tma_load_2d(st, &tmap_x, &s.full[stage], kb * BK, m0);
          for (int part = 0; part < 3; ++part)
            tma_load_2d(st + A_BYTES + part * part_bytes, &tmap_w, &s.full[stage], kb * BK,
                        part * e_pad);
        }
      }
      __syncwarp();
      ++issued;
      if (++stage == static_cast<uint32_t>(stages)) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (the leader of a pair)
    if (kPair && !leader) {
      // nothing to issue: the leader's MMAs read this CTA's shared memory
    } else {
    const uint32_t idesc = umma_idesc_f32acc(kPair ? 2 * BM : BM, e_pad, 1u);
    uint32_t stage = 0, phase = 0;
    int consumed = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const uint32_t slot = c & 1;
      if (!mbar_wait(&s.tempty[slot], ((c >> 1) & 1) ^ 1u, abort_flag, err)) break;
      tc_fence_after();
      const uint32_t d = tmem + slot * e_pad;
      const int ka = kb0 + c * CHUNK, kz = min(kb1, ka + CHUNK);
      for (int kb = ka; kb < kz; ++kb) {
        if (!mbar_wait(&s.full[stage], phase, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        ++consumed;
        if (lane == 0) {
          const uint32_t a_addr = smem_addr(base + stage * stage_bytes);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint32_t b_addr = a_addr + A_BYTES + part * part_bytes;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint32_t accum = (kb > ka || part > 0 || k > 0) ? 1u : 0u;
              if (kPair)
                umma_pair(d, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32), idesc,
                          accum);
              else
                umma_bf16(d, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32), idesc,
                          accum);
            }
          }
          if (kPair)
            umma_commit_pair(&s.empty[stage], 0x3);
          else
            umma_commit(&s.empty[stage]);
        }
        __syncwarp();
        if (++stage == static_cast<uint32_t>(stages)) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && lane == 0) {
        if (kPair)
          umma_commit_pair(&s.tfull[slot], 0x3);
        else
          umma_commit(&s.tfull[slot]);
      }
      __syncwarp();
    }
    if (lane == 0) s.mma_consumed = consumed;
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // warps 2..9: lane quarter q = warp % 4 (the TMEM lanes this warp may
    // read), column half hf; each thread owns row q*32 + lane, HALF columns
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int t = m0 + row;
    float acc[HALF];
#pragma unroll
    for (int j = 0; j < HALF; ++j) acc[j] = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const uint32_t slot = c & 1;
      if (!mbar_wait(&s.tfull[slot], (c >> 1) & 1, abort_flag, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem + slot * e_pad + hf * HALF + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < HALF / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(taddr + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[cc * 32 + j] += __uint_as_float(r[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (!kPair || leader)
          mbar_arrive(&s.tempty[slot]);
        else
          mbar_arrive_remote(cluster_map(&s.tempty[slot], 0));
      }
    }
    const int epi_tid = threadIdx.x - 64;
    const int rows = min(BM, T - m0);
    if (kSplit) {
      // The partials go out through the drained ring (below): row per thread
      // into shared memory, then whole rows per warp, so the stores coalesce.
      if (ok) {
        float4 *d4 = reinterpret_cast<float4 *>(zs + row * ZS + hf * HALF);
#pragma unroll
        for (int v = 0; v < HALF / 4; ++v)
          d4[v] = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
      }
      named_barrier(1, 32 * EPI_WARPS);
      if (!*abort_flag) {
        constexpr int V = e_pad / 4;
        float4 *dst = reinterpret_cast<float4 *>(zp + (static_cast<size_t>(split) * T + m0) * e_pad);
        for (int i = epi_tid; i < rows * V; i += 32 * EPI_WARPS) {
          const int r = i / V, c = i - r * V;
          dst[i] = *reinterpret_cast<const float4 *>(zs + r * ZS + 4 * c);
        }
      }
    } else {
      // Every MMA has completed (its tfull arrived) and so has every copy it
      // read: the operand ring is free.  Stage the 128 x e_pad tile of z there
      // (row stride ZS floats: the 8 rows of one 16-byte store phase fall in
      // distinct banks), then each epilogue warp selects for 16 tokens.
      if (ok) {
        float4 *d4 = reinterpret_cast<float4 *>(zs + row * ZS + hf * HALF);
#pragma unroll
        for (int v = 0; v < HALF / 4; ++v)
          d4[v] = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
      }
      // The bias and the second half's lists sit after the staged rows.
      float *bias_s = zs + BM * ZS;
      float *list_k = bias_s + e_pad;
      int *list_e = reinterpret_cast<int *>(list_k + 17 * BM);
      for (int e = epi_tid; e < e_pad; e += 32 * EPI_WARPS) bias_s[e] = e < o.E ? o.bias[e] : 0.f;
      named_barrier(1, 32 * EPI_WARPS);
      const bool work = !*abort_flag;  // guards work only: every thread takes the barriers
      if (work && o.logits) {
        for (int i = epi_tid; i < rows * o.E; i += 32 * EPI_WARPS) {
          const int r = i / o.E, c = i - r * o.E;
          o.logits[static_cast<size_t>(m0 + r) * o.E + c] = zs[r * ZS + c];
        }
      }
      if (o.K < 9)
        select_staged<9, HALF>(zs + row * ZS, bias_s, list_k, list_e, row, hf, t, work && t < T, o);
      else
        select_staged<17, HALF>(zs + row * ZS, bias_s, list_k, list_e, row, hf, t, work && t < T, o);
    }
  }

  __syncthreads();
  if (s.abort_flag) {  // error path: let copies and MMAs in flight land first
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = global_timer_ns();
      if (leader) {
        // (a pair's leader barriers count both CTAs' copies)
        for (int i = s.mma_consumed; i < issued; ++i) {
          const uint32_t a = smem_addr(&s.full[i % stages]);
          while (!mbar_try_wait(a, static_cast<uint32_t>((i / stages) & 1)) &&
                 global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      } else {  // the peer gives its own copies a bounded time to land
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
  if (kPair) cluster_sync();  // neither CTA leaves while the other may touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    if (kPair)
      tmem_dealloc_pair(tmem, tmem_cols);
    else
      tmem_dealloc(tmem, tmem_cols);
  }

  if (kSplit) {
    // Every CTA's partials are written; after the grid barrier CTA c takes the
    // tokens t = c, c + C, c + 2C, ... (C CTAs in the grid), a batch of rows at a time.
    // All its threads sum the S partials of those rows: groups of eight splits
    // in a fixed tree ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7)) (a
    // shorter last group in split order), then the group sums in group order
    // (deterministic whichever CTA does it; every load of a group is
    // independent, so a few round trips to L2 cover all S splits); the rows
    // land in shared memory and each warp selects for one row at a time.
    const int splits = gridDim.y;
    // this thread's expert's bias for the CTA-wide selection, fetched while the grid meets
    const float my_bias = static_cast<int>(threadIdx.x) < o.E ? o.bias[threadIdx.x] : 0.f;
    if (!grid_barrier(grid_counter, gridDim.x * gridDim.y, err)) return;
    float bias_r[NE];
#pragma unroll
    for (int j = 0; j < NE; ++j) {
      const int e = lane + 32 * j;
      bias_r[j] = e < o.E ? o.bias[e] : 0.f;
    }
    constexpr int V = e_pad / 4;  // float4 columns of a row
    const int n_ctas = gridDim.x * gridDim.y;
    const int cta = blockIdx.y * gridDim.x + blockIdx.x;
    const int n_rows = cta < T ? (T - 1 - cta) / n_ctas + 1 : 0;
    const int groups = (splits + 7) / 8;
    const size_t plane4 = static_cast<size_t>(T) * V;  // float4s per split
    const float4 *zp4 = reinterpret_cast<const float4 *>(zp);
    float4 *part = reinterpret_cast<float4 *>(zs + kRowBatch * ZS);  // [groups][kRowBatch][V]
    const int n_warps = blockDim.x >> 5;
    // rows per batch: all of the CTA's rows (up to 128) when the splits form one
    // group, so one pass of loads and one round of warps cover them; kRowBatch
    // when the group sums need the `part` buffer
    const int rb = groups == 1 ? BM : kRowBatch;
    for (int r0 = 0; r0 < n_rows; r0 += rb) {
      const int nb = min(rb, n_rows - r0);
      // Up to three items per thread, all their loads issued before any sum, so
      // one round trip to L2 covers the thread's share of the splits.
      const int n_items = groups * nb * V;
      constexpr int U = 3;
      for (int i0 = threadIdx.x; i0 < n_items; i0 += U * blockDim.x) {
        float4 a[U][8];
        int n[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * blockDim.x;
          n[u] = 0;
          if (i < n_items) {
            const int g = i / (nb * V);
            const int r = (i - g * nb * V) / V;
            const int c = i - g * nb * V - r * V;
            const int t = cta + (r0 + r) * n_ctas;
            const float4 *q = zp4 + static_cast<size_t>(t) * V + c + static_cast<size_t>(8 * g) * plane4;
            n[u] = min(8, splits - 8 * g);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              if (k < n[u]) a[u][k] = __ldcg(q + k * plane4);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * blockDim.x;
          if (i >= n_items) continue;
          const int g = i / (nb * V);
          const int r = (i - g * nb * V) / V;
          const int c = i - g * nb * V - r * V;
          float4 sum;
          if (n[u] == 8) {
            sum.x = ((a[u][0].x + a[u][1].x) + (a[u][2].x + a[u][3].x)) + ((a[u][4].x + a[u][5].x) + (a[u][6].x + a[u][7].x));
            sum.y = ((a[u][0].y + a[u][1].y) + (a[u][2].y + a[u][3].y)) + ((a[u][4].y + a[u][5].y) + (a[u][6].y + a[u][7].y));
            sum.z = ((a[u][0].z + a[u][1].z) + (a[u][2].z + a[u][3].z)) + ((a[u][4].z + a[u][5].z) + (a[u][6].z + a[u][7].z));
            sum.w = ((a[u][0].w + a[u][1].w) + (a[u][2].w + a[u][3].w)) + ((a[u][4].w + a[u][5].w) + (a[u][6].w + a[u][7].w));
          } else {
            sum = a[u][0];
#pragma unroll
            for (int k = 1; k < 8; ++k) {
              if (k < n[u]) {
                sum.x += a[u][k].x;
                sum.y += a[u][k].y;
                sum.z += a[u][k].z;
                sum.w += a[u][k].w;
              }
            }
          }
          if (groups == 1)
            *reinterpret_cast<float4 *>(zs + r * ZS + 4 * c) = sum;
          else
            part[(g * kRowBatch + r) * V + c] = sum;
        }
      }
      __syncthreads();
      if (groups > 1) {
        for (int i = threadIdx.x; i < nb * V; i += blockDim.x) {
          const int r = i / V, c = i - r * V;
          float4 sum = part[r * V + c];
          for (int g = 1; g < groups; ++g) {
            const float4 v = part[(g * kRowBatch + r) * V + c];
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
          }
          *reinterpret_cast<float4 *>(zs + r * ZS + 4 * c) = sum;
        }
        __syncthreads();
      }
      if (nb <= kRankRows) {  // few rows: the whole CTA ranks their experts together
        if (o.K < 9)
          select_rank_rows<e_pad, 9>(zs, ZS, nb, my_bias, reinterpret_cast<float *>(part), cta + r0 * n_ctas,
                                     n_ctas, o);
        else
          select_rank_rows<e_pad, 17>(zs, ZS, nb, my_bias, reinterpret_cast<float *>(part), cta + r0 * n_ctas,
                                      n_ctas, o);
      } else {
        // up to 64 experts, two rows per warp at a time (a lone last row is paired with
        // itself, the copy not written): 64 experts top-4 at 4096 tokens over 128 CTAs, 21.0
        // against 22.9 us; with 256 experts the two rows' keys spill and one row is faster
        // (8192 GLM-5 tokens: 122 against 134 us)
        constexpr int RW = NE <= 2 ? 2 : 1;
        for (int r = RW * warp; r < nb; r += RW * n_warps) {
          const int rr = min(r + RW - 1, nb - 1);
          if constexpr (RW == 2) {
            const int t2[2] = {cta + (r0 + r) * n_ctas, cta + (r0 + rr) * n_ctas};
            const bool v2[2] = {true, r + 1 < nb};
            select_tokens<NE, 2>(zs + r * ZS, static_cast<int>(rr - r) * ZS, t2, v2, bias_r, o, lane);
          } else {
            const int t1[1] = {cta + (r0 + r) * n_ctas};
            const bool v1[1] = {true};
            select_tokens<NE, 1>(zs + r * ZS, 0, t1, v1, bias_r, o, lane);
          }
        }
      }
      __syncthreads();
    }
  }
}

int router_stages(int e_pad, bool pair = false) {
  const int stage = rt::A_BYTES + 3 * (pair ? e_pad / 2 : e_pad) * rt::BK * 2;
  int s = static_cast<int>((rt::MAX_SMEM - 1024 - sizeof(RouterSmem)) / stage);
  return s > 4 ? 4 : s;
}

// ---------------------------------------------------------------- launch

size_t router_smem_bytes(int e_pad, bool pair) {
  const int stage = rt::A_BYTES + 3 * (pair ? e_pad / 2 : e_pad) * rt::BK * 2;
  return 1024 + static_cast<size_t>(router_stages(e_pad, pair)) * stage + sizeof(RouterSmem);
}


template <int NH, bool kSplit, bool kPair>
static cudaError_t launch_router_kernel(dim3 grid, const CUtensorMap &tmap_x, const CUtensorMap &tmap_w,
                                        int kb_per, int kblocks, float *zp, int *grid_counter,
                                        const RouteOut &o, int *err, cudaStream_t stream) {
  constexpr int e_pad = NH * 64;
  const size_t smem = router_smem_bytes(e_pad, kPair);
  const int stages = router_stages(e_pad, kPair);
  // the selection stages z rows, the bias and 17-entry lists over the drained ring
  const size_t staged = (static_cast<size_t>(rt::BM) * (e_pad + 4) + e_pad + 2 * 17 * rt::BM) * 4;
  // after a split: kRowBatch staged rows and up to ceil(kMaxSplits / 8) group sums of them
  const size_t reduced = static_cast<size_t>(kRowBatch) * ((e_pad + 4) + (kMaxSplits + 7) / 8 * e_pad) * 4;
  if (kSplit && reduced > static_cast<size_t>(stages) * (rt::A_BYTES + 3 * (kPair ? e_pad / 2 : e_pad) * rt::BK * 2))
    return cudaErrorInvalidValue;
  if (staged > static_cast<size_t>(stages) * (rt::A_BYTES + 3 * (kPair ? e_pad / 2 : e_pad) * rt::BK * 2))
    return cudaErrorInvalidValue;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * e_pad)) cols <<= 1;  // two ping-pong accumulators
  auto kern = router_kernel<NH, kSplit, kPair>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (!kPair) {
    kern<<<grid, rt::THREADS, smem, stream>>>(tmap_x, tmap_w, kb_per, kblocks, stages, cols, zp,
                                              grid_counter, o, err);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(rt::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmap_x, tmap_w, kb_per, kblocks, stages, cols, zp, grid_counter,
                            o, err);
}

cudaError_t launch_router_split(const float *w_r, int E, int H, uint16_t *wsplit, int num_sms,
                                cudaStream_t stream) {
  router_split_kernel<<<num_sms * 4, 256, 0, stream>>>(w_r, E, router_e_pad(E), H, wsplit);
  return cudaGetLastError();
}

// CTA pairs (256 tokens per pair, each CTA loading half of every W_r part)
// once there are enough token tiles: every token tile reads the whole split
// W_r from L2, so pairs halve that traffic.  A few tiles (decode) stay single
// CTAs, which spread W_r over many splits.
bool router_use_pairs(int T, int H, int num_sms) {
  (void)H;
  (void)num_sms;
  return (T + rt::BM - 1) / rt::BM >= kPairMinTiles;
}

int router_grid_splits(int T, int H, int num_sms) {
  const int m_tiles = (T + rt::BM - 1) / rt::BM;
  const bool pair = router_use_pairs(T, H, num_sms);
  const int ctas = pair ? (m_tiles + 1) / 2 * 2 : m_tiles;  // CTAs per split
  int s = router_splits(T, H);
  const int fit = num_sms / (ctas > 0 ? ctas : 1);  // the whole grid resident at once
  if (s > fit) s = fit;
  if (s < 1) s = 1;
  const int kblocks = H / rt::BK;
  const int kb_per = (kblocks + s - 1) / s;
  return (kblocks + kb_per - 1) / kb_per;  // splits that get at least one k-block
}

int router_w_box_rows(int E, bool pair) { return pair ? router_e_pad(E) / 2 : router_e_pad(E); }


cudaError_t launch_route(const CUtensorMap &tmap_x, const CUtensorMap &tmap_w, const float *bias, int T,
                         int H, int E, int K, float scale, float *zp, int *grid_counter,
                         int32_t *idx, float *gate, float *margin, float *logits, int *err,
                         int num_sms, cudaStream_t stream) {
  const int kblocks = H / rt::BK;
  const int splits = router_grid_splits(T, H, num_sms);
  const int kb_per = (kblocks + splits - 1) / splits;
  const bool pair = router_use_pairs(T, H, num_sms);  // the tensor map's box follows the same rule
  const int m_tiles = (T + rt::BM - 1) / rt::BM;
  dim3 grid(pair ? (m_tiles + 1) / 2 * 2 : m_tiles, splits);
  RouteOut o;
  o.bias = bias;
  o.idx = idx;
  o.gate = gate;
  o.margin = margin;
  o.logits = logits;
  o.scale = scale;
  o.T = T;
  o.E = E;
  o.K = K;
  const int nh = router_e_pad(E) / 64;
#define SRM_ROUTER_CASES(SPLIT, PAIR)                                                                       \
  switch (nh) {                                                                                            \
    case 1: return launch_router_kernel<1, SPLIT, PAIR>(grid, tmap_x, tmap_w, kb_per, kblocks, zp,         \
                                                        grid_counter, o, err, stream);                     \
    case 2: return launch_router_kernel<2, SPLIT, PAIR>(grid, tmap_x, tmap_w, kb_per, kblocks, zp,         \
                                                        grid_counter, o, err, stream);                     \
    case 3: return launch_router_kernel<3, SPLIT, PAIR>(grid, tmap_x, tmap_w, kb_per, kblocks, zp,         \
                                                        grid_counter, o, err, stream);                     \
    default: return launch_router_kernel<4, SPLIT, PAIR>(grid, tmap_x, tmap_w, kb_per, kblocks, zp,        \
                                                         grid_counter, o, err, stream);                    \
  }
  if (splits > 1) {
    if (pair) {
      SRM_ROUTER_CASES(true, true)
    }
    SRM_ROUTER_CASES(true, false)
  }
  if (pair) {
    SRM_ROUTER_CASES(false, true)
  }
  SRM_ROUTER_CASES(false, false)
#undef SRM_ROUTER_CASES
}

}  // namespace srm
