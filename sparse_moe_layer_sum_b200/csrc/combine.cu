// moe_combine: y[t] = sum_j weights[t,j] * out_perm[slot_of[t,j]] + out_shared[t].
//
// The moe-forward code excerpt of "DeepSeek-V3.2-Exp · Mixture of experts"
// accumulates into an fp32 zero tensor: each routed expert's output times the
// token's gate, then the shared expert's output.  One CTA per token reads its
// k expert rows (found through slot_of) and its shared row with 16-byte
// loads and writes y once, summing in a fixed order (j ascending, shared
// last) so the result is deterministic.
#include "common.cuh"
#include "moe_combine.h"

namespace moe {
namespace {

constexpr int CB_THREADS = 256;

__global__ void __launch_bounds__(CB_THREADS) combine_kernel(
    const float *__restrict__ weights, const int32_t *__restrict__ slot_of,
    const float *__restrict__ out_perm, const float *__restrict__ out_shared,
    float *__restrict__ y, int k, int D, int64_t nrows, int32_t *status) {
  __shared__ int64_t row[32];
  __shared__ float gate[32];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    const int32_t s = slot_of[t * k + threadIdx.x];
    if (s < 0 || s >= nrows) {
      set_status(status, MOE_ERR_RANGE);
      row[threadIdx.x] = -1;
    } else {
      row[threadIdx.x] = s;
    }
    gate[threadIdx.x] = weights[t * k + threadIdx.x];
  }
  __syncthreads();
  const int D4 = D / 4;
  const float4 *op = reinterpret_cast<const float4 *>(out_perm);
  const float4 *sp = reinterpret_cast<const float4 *>(out_shared);
  float4 *yp = reinterpret_cast<float4 *>(y);
  for (int c = threadIdx.x; c < D4; c += CB_THREADS) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int64_t r = row[j];
      if (r < 0) continue;
      const float4 o = __ldcs(op + r * D4 + c);  // read once: stream past L2
      const float g = gate[j];
      acc.x = __fmaf_rn(g, o.x, acc.x);
      acc.y = __fmaf_rn(g, o.y, acc.y);
      acc.z = __fmaf_rn(g, o.z, acc.z);
      acc.w = __fmaf_rn(g, o.w, acc.w);
    }
    if (sp) {
      const float4 o = __ldcs(sp + t * D4 + c);
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }
    yp[t * D4 + c] = acc;
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_EXPORT moe_status moe_combine(const moe_cfg *cfg, int64_t T, const float *weights,
                                  const int32_t *slot_of, const float *out_perm,
                                  const float *out_shared, float *y, int32_t *dev_status,
                                  moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || T * (int64_t)cfg->topk >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!weights || !slot_of || !out_perm || !y) return MOE_ERR_INVALID;
  if (cfg->n_shared > 0 && !out_shared) return MOE_ERR_INVALID;
  if (cfg->dim % 4 != 0 || cfg->topk > 32) return MOE_ERR_UNSUPPORTED;
  combine_kernel<<<(unsigned)T, CB_THREADS, 0, as_stream(stream)>>>(
      weights, slot_of, out_perm, cfg->n_shared > 0 ? out_shared : nullptr, y, cfg->topk,
      cfg->dim, T * cfg->topk, dev_status);
  return launch_status();
}
