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

/*
 * Preparation of the router weight, done once when the weights are loaded.
 *
 * On the tensor-core scoring path (bf16 x, T >= 32, n_routed a multiple of
 * 128, dim a multiple of 64) z = x W_r^T is computed as x hi^T + x mid^T +
 * x lo^T with three bf16 matrices whose sum is W_r exactly (each holds the
 * next 8 significant bits of every element; the remainders are exact in
 * fp32), so every product is exact and z carries only fp32 accumulation
 * error, as the excerpt's fp32 linear would.  moe_router_forward writes
 * that split into its workspace on every call; moe_router_prepare writes it
 * once into a caller-owned buffer, and moe_router_forward_prepared reads it
 * from there.
 *
 * moe_router_prepare_size: bytes of the split (3 * n_routed * dim * 2), or 0
 * when the tensor-core path cannot apply to cfg (or cfg is invalid).
 * moe_router_prepare: w_r [n_routed, dim] fp32 -> prep (device, caller-owned,
 * prep_bytes >= moe_router_prepare_size(cfg)); enqueued on `stream`.
 * Returns MOE_ERR_UNSUPPORTED when the size is 0, MOE_ERR_WORKSPACE when
 * prep_bytes is too small, MOE_ERR_INVALID for NULL pointers.  prep must be
 * prepared again whenever w_r changes.
 */
size_t moe_router_prepare_size(const moe_cfg *cfg);
moe_status moe_router_prepare(const moe_cfg *cfg, const float *w_r, void *prep,
                              size_t prep_bytes, moe_stream_t stream);

/*
 * moe_router_forward with the prepared split of w_r: identical results, one
 * launch fewer.  `prep` (required, from moe_router_prepare on this w_r) is
 * read when the tensor-core path applies; otherwise the call scores from
 * w_r exactly as moe_router_forward does.  All other arguments, limits and
 * errors are those of moe_router_forward (the same workspace size).
 */
moe_status moe_router_forward_prepared(const moe_cfg *cfg, int64_t T, const void *x,
                                       moe_dtype x_dt, const float *w_r, const void *prep,
                                       const float *bias, float *weights, int32_t *indices,
                                       float *sel_gap, void *ws, size_t ws_bytes,
                                       int32_t *dev_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
