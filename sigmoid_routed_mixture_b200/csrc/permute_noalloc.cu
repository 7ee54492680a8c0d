// permute_noalloc.cu -- moe_permute for callers that cannot allocate device
// memory.
//
// moe_permute needs a little scratch (per-chunk expert counts and an error
// word), which it takes from the caller's workspace.  Some callers have no
// workspace to give: a host that has handed all device memory to its own
// pool, a runtime that forbids cudaMalloc on the serving path because it
// synchronises the whole device, or a plugin that only ever sees the tensors
// it is given.  moe_permute_noalloc does the same work with its scratch in
// the file-scope array below instead, so the caller passes only inputs and
// outputs.
//
// Limits and sharing (also stated in include/srm_moe.h):
//   - the array holds counts for at most kMaxChunks chunks of 1024
//     assignments: T * K <= 262144 (for example 32768 tokens at top-8);
//     larger calls are rejected with MOE_ERR_UNSUPPORTED;
//   - every GPU that loads the library keeps this array (257 KB) until the
//     process exits;
//   - all calls share it, and it keeps the last call's contents: each call
//     clears the error word first; calls that overlap on the GPU (different
//     streams, no ordering between them) race on it and must be avoided.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/srm_moe.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int kMaxE = 256;
constexpr int kMaxChunks = 256;                   // chunks of 1024 assignments
constexpr int64_t kMaxAssignments = 262144;       // kMaxChunks * 1024
constexpr int kErrWords = 64;                     // word 0 = error flag; keeps counts 256-B aligned
constexpr int kDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kErrWords + kMaxE * kMaxChunks];

// Address of g_permute_scratch on each device, looked up once per device with
// that device current (in host code the symbol is only a host-side handle).
// The address is kept for the life of the process: a cudaDeviceReset after the
// first call may move the array, so resetting a device that this entry point
// has used is not supported.
std::mutex g_mutex;
int32_t *g_scratch_ptr[kDevices] = {nullptr};

moe_status_t scratch_for_current_device(int32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MOE_ERR_CUDA;
  if (dev >= kDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t *>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

// A skipped (out-of-range) expert id is reported in-band: offsets[0], always
// 0 otherwise, becomes -1.
__global__ void flag_bad_index_kernel(const int32_t *err, int32_t *offsets) {
  if (threadIdx.x == 0 && blockIdx.x == 0 && *err != 0) offsets[0] = -1;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const moe_cfg_t *cfg, const int32_t *topk_idx,
                                            int32_t *counts, int32_t *offsets, int32_t *sorted,
                                            void *stream) {
  if (!cfg) return MOE_ERR_ARG;
  if (cfg->T < 0 || cfg->E <= 0 || cfg->K <= 0 || cfg->K > cfg->E ||
      (cfg->has_shared != 0 && cfg->has_shared != 1))
    return MOE_ERR_ARG;
  if (cfg->E > kMaxE || cfg->K > 16) return MOE_ERR_UNSUPPORTED;
  if (cfg->T * static_cast<int64_t>(cfg->K) > kMaxAssignments) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_ARG;
  if (cfg->T > 0 && (!topk_idx || !sorted)) return MOE_ERR_ARG;
  if (!aligned4(counts) || !aligned4(offsets) || (topk_idx && !aligned4(topk_idx)) ||
      (sorted && !aligned4(sorted)))
    return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * (cfg->E + 1), s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (cfg->E + 2), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  int32_t *scratch = nullptr;
  const moe_status_t st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  int *err = reinterpret_cast<int *>(scratch);
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (srm::launch_permute(topk_idx, static_cast<int>(cfg->T), cfg->E, cfg->K, cfg->has_shared,
                          counts, offsets, sorted, scratch + kErrWords, err, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  flag_bad_index_kernel<<<1, 32, 0, s>>>(err, offsets);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
