// moe_dispatch: per-expert histogram, exclusive scan and stable scatter.
//
// Restates, for all experts at once and without a host round trip, what the
// moe-forward code excerpt of "DeepSeek-V3.2-Exp · Mixture of experts" does
// with torch.bincount(indices) and, per expert, torch.where(indices == i):
// every expert's (token, slot) pairs, tokens ascending.
//
// The pairs are cut into chunks of CHUNK_TOKENS tokens:
//  1. dispatch_hist:    per-chunk expert histograms (shared-memory atomics).
//  2. dispatch_scan:    per expert, an exclusive scan over chunks; then an
//                       exclusive scan over experts gives offsets; each
//                       chunk's base row for each expert is their sum.
//  3. dispatch_scatter: one warp per chunk walks its pairs in order, 32 at a
//                       time; lanes holding the same expert rank themselves
//                       with __match_any_sync, so the order inside an expert
//                       is the pair order (token ascending) -- deterministic.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "dispatch_dev.cuh"
#include "moe_dispatch.h"

namespace moe {
namespace {

using grouping::CHUNK_TOKENS;

__global__ void __launch_bounds__(256) dispatch_hist(const int32_t *__restrict__ idx, int T, int k,
                                                     int E, int32_t *__restrict__ chunk_hist,
                                                     int32_t *status) {
  extern __shared__ int32_t h[];
  grouping::hist_chunk(idx, T, k, E, blockIdx.x, chunk_hist, status, h);
}

// One block of >= E threads (E <= 1024).
__global__ void __launch_bounds__(1024) dispatch_scan(int32_t *__restrict__ chunk_hist,
                                                      int nchunks, int E,
                                                      int32_t *__restrict__ counts,
                                                      int32_t *__restrict__ offsets) {
  __shared__ int32_t warp_tot[32];
  grouping::scan_chunks(chunk_hist, nchunks, E, counts, offsets, warp_tot);
}

// One warp per chunk.
__global__ void __launch_bounds__(32) dispatch_scatter(const int32_t *__restrict__ idx, int T,
                                                       int k, int E,
                                                       const int32_t *__restrict__ chunk_base,
                                                       const int32_t *__restrict__ offsets,
                                                       int32_t *__restrict__ sorted_token,
                                                       int32_t *__restrict__ slot_of) {
  extern __shared__ int32_t base[];
  grouping::scatter_chunk(idx, T, k, E, blockIdx.x, chunk_base, offsets, sorted_token, slot_of,
                          base);
}

// ------------------------------------------------- no-allocation variant
//
// Scratch for moe_dispatch_build_noalloc: the per-chunk histograms live in
// this file-scope device array instead of a caller-provided workspace.  Every
// GPU that loads the library holds it until the process exits.
constexpr int64_t NOALLOC_SCRATCH_INTS = (int64_t)1 << 18;  // 1 MiB
__device__ __align__(256) int32_t g_noalloc_scratch[NOALLOC_SCRATCH_INTS];

constexpr int MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
// per device: the scratch array's device address and the id of the context
// it was looked up in (a context that is destroyed and created again, as
// after cudaDeviceReset, loads the module anew, possibly elsewhere)
int32_t *g_noalloc_ptr[MAX_DEVICES] = {};
unsigned long long g_noalloc_ctx[MAX_DEVICES] = {};

// Unique id of the current context (0 when the driver cannot tell).
unsigned long long current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    looked = true;
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the
// array's name only stands for a host-side symbol, so the address is looked up
// (with the device current) on the first call in each context and cached.
moe_status noalloc_scratch(int32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  // no current context yet (id 0): the look-up below makes the runtime's
  // primary context current, and the id is read again after it
  const unsigned long long ctx = current_ctx_id();
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<int32_t *>(ptr);
    g_noalloc_ctx[dev] = current_ctx_id();
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_EXPORT size_t moe_dispatch_workspace_size(const moe_cfg *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  const int64_t nchunks = (T + CHUNK_TOKENS - 1) / CHUNK_TOKENS;
  return align_up((size_t)(nchunks > 0 ? nchunks : 1) * cfg->n_routed * sizeof(int32_t), 256);
}

MOE_EXPORT moe_status moe_dispatch_build(const moe_cfg *cfg, int64_t T, const int32_t *indices,
                                         int32_t *counts, int32_t *offsets,
                                         int32_t *sorted_token, int32_t *slot_of, void *ws,
                                         size_t ws_bytes, int32_t *dev_status,
                                         moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || T * (int64_t)cfg->topk >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
  if (!counts || !offsets || !ws) return MOE_ERR_INVALID;
  if (T > 0 && (!indices || !sorted_token || !slot_of)) return MOE_ERR_INVALID;
  if (cfg->n_routed > 1024) return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < moe_dispatch_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const int E = cfg->n_routed, k = cfg->topk;
  const int nchunks = (int)((T + CHUNK_TOKENS - 1) / CHUNK_TOKENS);
  int32_t *chunk_hist = static_cast<int32_t *>(ws);
  const size_t hsmem = (size_t)E * sizeof(int32_t);
  if (nchunks > 0) {
    dispatch_hist<<<nchunks, 256, hsmem, s>>>(indices, (int)T, k, E, chunk_hist, dev_status);
    if ((st = launch_status()) != MOE_OK) return st;
  }
  const int scan_threads = (E + 31) / 32 * 32;
  dispatch_scan<<<1, scan_threads, 0, s>>>(chunk_hist, nchunks, E, counts, offsets);
  if ((st = launch_status()) != MOE_OK) return st;
  if (nchunks > 0) {
    dispatch_scatter<<<nchunks, 32, hsmem, s>>>(indices, (int)T, k, E, chunk_hist, offsets,
                                                sorted_token, slot_of);
    if ((st = launch_status()) != MOE_OK) return st;
  }
  return MOE_OK;
}

MOE_EXPORT moe_status moe_dispatch_build_noalloc(const moe_cfg *cfg, int64_t T,
                                                 const int32_t *indices, int32_t *counts,
                                                 int32_t *offsets, int32_t *sorted_token,
                                                 int32_t *slot_of, int32_t *dev_status,
                                                 moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID;
  const size_t need = moe_dispatch_workspace_size(cfg, T);
  if (need > (size_t)NOALLOC_SCRATCH_INTS * sizeof(int32_t)) return MOE_ERR_WORKSPACE;
  int32_t *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != MOE_OK) return st;
  // the histogram pass writes every scratch entry the later passes read, so
  // nothing has to be cleared between calls
  return moe_dispatch_build(cfg, T, indices, counts, offsets, sorted_token, slot_of, scratch,
                            (size_t)NOALLOC_SCRATCH_INTS * sizeof(int32_t), dev_status, stream);
}
