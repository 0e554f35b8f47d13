/*
 * moe_combine.h -- the weighted sum into the fp32 block output.
 *
 * The moe-forward code excerpt of "DeepSeek-V3.2-Exp · Mixture of experts"
 * starts from an fp32 zero tensor y, adds every routed expert's output times
 * the token's gate weight, then adds the shared expert's output.  Here:
 *   y[t,:] = sum_{j=0..topk-1} weights[t,j] * out_perm[slot_of[t*topk+j], :]
 *            + out_shared[t,:]
 * in fp32, in that fixed order (j ascending, shared last), so the result is
 * deterministic and reproducible run to run.
 */
#ifndef MOE_COMBINE_H
#define MOE_COMBINE_H
#include "moe_common.h"
#ifdef __cplusplus
extern "C" {
#endif

/*
 * weights    [T, topk] fp32 from moe_router_forward
 * slot_of    [T, topk] int32 from moe_dispatch_build
 * out_perm   [T * topk, dim] fp32 from moe_experts_forward
 * out_shared [T, dim] fp32, or NULL when n_shared == 0
 * y          [T, dim] fp32 out (overwritten)
 * Limits: dim % 4 == 0.  A slot outside [0, T*topk) writes MOE_ERR_RANGE to
 * dev_status and that term is skipped.
 */
moe_status moe_combine(const moe_cfg *cfg, int64_t T, const float *weights,
                       const int32_t *slot_of, const float *out_perm, const float *out_shared,
                       float *y, int32_t *dev_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
