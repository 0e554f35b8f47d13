// The token grouping as device functions, shared by the moe_dispatch kernels
// and the fused decode kernel of moe_experts: per-chunk expert histograms,
// exclusive scans, and the stable scatter into expert-contiguous order (the
// bincount / torch.where steps of the moe-forward excerpt of
// "DeepSeek-V3.2-Exp · Mixture of experts", for all experts at once).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {
namespace {
namespace grouping {

constexpr int CHUNK_TOKENS = 64;

// Histogram of chunk `chunk` (a whole block; h is shared memory of E ints);
// writes chunk_hist[chunk][e].
__device__ __forceinline__ void hist_chunk(const int32_t *__restrict__ idx, int T, int k, int E,
                                           int chunk, int32_t *__restrict__ chunk_hist,
                                           int32_t *status, int32_t *h) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int t0 = chunk * CHUNK_TOKENS;
  const int n = min(CHUNK_TOKENS, T - t0) * k;
  const int32_t *src = idx + (size_t)t0 * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = src[i];
    if (e < 0 || e >= E)
      set_status(status, MOE_ERR_RANGE);
    else
      atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)chunk * E + e] = h[e];
}

// Per expert, an exclusive scan over the chunks (each chunk's first row
// within the expert's rows, left in chunk_hist), then over the experts:
// counts and offsets.  One block of >= E threads (E <= 1024); warp_tot is
// shared memory of 32 ints.
__device__ __forceinline__ void scan_chunks(int32_t *__restrict__ chunk_hist, int nchunks, int E,
                                            int32_t *__restrict__ counts,
                                            int32_t *__restrict__ offsets, int32_t *warp_tot) {
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    // eight chunks' loads in flight before their stores
    int c = 0;
    for (; c + 8 <= nchunks; c += 8) {
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = chunk_hist[(size_t)(c + q) * E + e];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        chunk_hist[(size_t)(c + q) * E + e] = run;
        run += v[q];
      }
    }
    for (; c < nchunks; ++c) {
      const int v = chunk_hist[(size_t)c * E + e];
      chunk_hist[(size_t)c * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  // exclusive scan of run over e: warp inclusive scans, then warp totals
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  int v = (e < E) ? run : 0;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_tot[w] = inc;
  __syncthreads();
  if (w == 0) {
    const int nw = (blockDim.x + 31) / 32;
    int t = lane < nw ? warp_tot[lane] : 0;
    int tinc = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, tinc, off);
      if (lane >= off) tinc += o;
    }
    warp_tot[lane] = tinc - t;  // exclusive prefix of the warp totals
  }
  __syncthreads();
  const int excl = inc - v + warp_tot[w];
  if (e < E) {
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + v;
  }
}

// The stable scatter of chunk `chunk` by one warp: chunk_base holds each
// chunk's first row within each expert, offsets each expert's first row;
// base is that warp's shared memory of E ints.
__device__ __forceinline__ void scatter_chunk(const int32_t *__restrict__ idx, int T, int k, int E,
                                              int chunk, const int32_t *__restrict__ chunk_base,
                                              const int32_t *__restrict__ offsets,
                                              int32_t *__restrict__ sorted_token,
                                              int32_t *__restrict__ slot_of, int32_t *base) {
  const int lane = threadIdx.x % 32;
  for (int e = lane; e < E; e += 32) base[e] = chunk_base[(size_t)chunk * E + e] + offsets[e];
  __syncwarp();
  const int t0 = chunk * CHUNK_TOKENS;
  const int n = min(CHUNK_TOKENS, T - t0) * k;
  const size_t flat0 = (size_t)t0 * k;
  const unsigned lt = (1u << lane) - 1u;
  // the indices of eight rounds of 32 slots are loaded before the rounds run
  for (int i00 = 0; i00 < n; i00 += 256) {
    int ev[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i00 + 32 * j + lane;
      ev[j] = i < n ? idx[flat0 + i] : -1;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i0 = i00 + 32 * j;
      if (i0 >= n) break;
      const int i = i0 + lane;
      const int e = ev[j];
      const bool ok = i < n && e >= 0 && e < E;
      const int key = ok ? e : -1 - lane;  // invalid lanes get a key of their own
      const unsigned same = __match_any_sync(0xffffffffu, key);
      if (ok) {
        const int rank = __popc(same & lt);
        const int pos = base[e] + rank;
        sorted_token[pos] = t0 + i / k;
        slot_of[flat0 + i] = pos;
      }
      __syncwarp();
      // the highest lane of each group advances that expert's next free row
      if (ok && (same >> lane) == 1u) base[e] += __popc(same);
      __syncwarp();
    }
  }
}

}  // namespace grouping
}  // namespace
}  // namespace moe
