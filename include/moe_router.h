/*
 * moe_router.h -- the gate of the MoE block.
 *
 * Computes, for every token t (page "DeepSeek-V3.2-Exp · Router", the four
 * equations under "All 4 steps" and the gate-forward code excerpt):
 *   z[t,e] = sum_d x[t,d] * W_r[e,d]                 fp32 accumulation
 *   s[t,e] = sigmoid(z[t,e])        (score_func = MOE_SCORE_SIGMOID)
 *          | softmax_e(z[t,:])      (score_func = MOE_SCORE_SOFTMAX)
 *   c[t,e] = s[t,e] + bias[e]       (has_bias; the bias only selects)
 *   group q score = sum of its two largest c (has_bias) | its largest c
 *   keep the topk_groups best groups; mask the others' experts with -inf
 *   indices[t,:] = the topk largest masked c, descending, ties to the lower
 *                  expert index
 *   weights[t,j] = s[t, indices[t,j]], divided by their sum (sigmoid only),
 *                  times route_scale
 * All score and decision arithmetic is fp32, as in the excerpt (x and the
 * weight are cast to float); sigmoid and softmax use the IEEE expf and
 * divisions of the CUDA runtime (no fast-math approximations).
 */
#ifndef MOE_ROUTER_H
#define MOE_ROUTER_H
#include "moe_common.h"
#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of device workspace moe_router_forward needs for T tokens. */
size_t moe_router_workspace_size(const moe_cfg *cfg, int64_t T);

/*
 * x        [T, dim]      x_dt = MOE_BF16 or MOE_F32 (converted exactly to fp32)
 * w_r      [n_routed, dim] fp32
 * bias     [n_routed] fp32, required when cfg->has_bias, ignored otherwise
 * weights  [T, topk] fp32 out
 * indices  [T, topk] int32 out, in [0, n_routed)
 * sel_gap  [T] fp32 out, optional (NULL): the smallest score gap behind any
 *          of the token's decisions (kept/dropped group boundary, chosen/
 *          unchosen expert boundary, and consecutive chosen experts); a gap
 *          near zero marks a near-tie whose outcome depends on rounding
 * ws       device workspace of moe_router_workspace_size(cfg, T) bytes
 * Limits: n_routed <= 1024, n_groups <= 32 dividing n_routed, topk <= 32,
 * topk <= topk_groups * n_routed / n_groups, dim % 4 == 0.
 * Returns MOE_OK, or MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED /
 * MOE_ERR_WORKSPACE before any launch, or MOE_ERR_CUDA if a launch failed.
 * T == 0 launches nothing and returns MOE_OK.
 */
moe_status moe_router_forward(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                              const float *w_r, const float *bias, float *weights,
                              int32_t *indices, float *sel_gap, void *ws, size_t ws_bytes,
                              int32_t *dev_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
