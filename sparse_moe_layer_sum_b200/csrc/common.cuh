// Helpers shared by the four MoE block libraries (header-only, compiled into
// each library separately).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_common.h"

#define MOE_EXPORT extern "C" __attribute__((visibility("default")))

namespace moe {

static inline cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Checks a config for consistency; returns MOE_OK or MOE_ERR_INVALID.
static inline moe_status check_cfg(const moe_cfg *c) {
  if (!c) return MOE_ERR_INVALID;
  if (c->dim <= 0 || c->n_routed <= 0 || c->n_groups <= 0 || c->topk_groups <= 0 ||
      c->topk <= 0 || c->inter <= 0 || c->n_shared < 0)
    return MOE_ERR_INVALID;
  if (c->n_routed % c->n_groups != 0) return MOE_ERR_INVALID;
  if (c->topk_groups > c->n_groups) return MOE_ERR_INVALID;
  if (c->topk > c->topk_groups * (c->n_routed / c->n_groups)) return MOE_ERR_INVALID;
  if (c->score_func != MOE_SCORE_SIGMOID && c->score_func != MOE_SCORE_SOFTMAX)
    return MOE_ERR_INVALID;
  if (c->has_bias != 0 && c->has_bias != 1) return MOE_ERR_INVALID;
  if (c->has_bias && c->n_groups > 1 && c->n_routed / c->n_groups < 2) return MOE_ERR_INVALID;
  return MOE_OK;
}

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static inline moe_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Records the first device-side error in the caller's status word.
__device__ __forceinline__ void set_status(int32_t *st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

}  // namespace moe
