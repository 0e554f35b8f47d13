/*
 * moe_dispatch.h -- grouping of tokens by expert.
 *
 * The moe-forward code excerpt of "DeepSeek-V3.2-Exp · Mixture of experts"
 * counts the tokens of every expert with a bincount of the router indices and
 * gathers each expert's rows with torch.where(indices == i), which lists the
 * (token, slot) pairs in row-major order.  This library produces the same
 * grouping for all experts at once, on the device, without a host round trip:
 *   counts[e]        number of pairs (t, j) with indices[t,j] == e
 *   offsets[e]       exclusive prefix sum of counts; offsets[n_routed] = T*topk
 *   sorted_token[p]  token of row p of the expert-contiguous order; rows
 *                    offsets[e] .. offsets[e+1]-1 belong to expert e and list
 *                    its tokens in ascending order (the torch.where order)
 *   slot_of[t*topk+j] row p at which pair (t, j) was placed
 * The result is fully determined (stable), so it is bit-exact by design.
 */
#ifndef MOE_DISPATCH_H
#define MOE_DISPATCH_H
#include "moe_common.h"
#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of device workspace moe_dispatch_build needs for T tokens. */
size_t moe_dispatch_workspace_size(const moe_cfg *cfg, int64_t T);

/*
 * indices      [T, topk] int32 in; a token's topk experts must be distinct
 * counts       [n_routed] int32 out
 * offsets      [n_routed + 1] int32 out
 * sorted_token [T * topk] int32 out
 * slot_of      [T * topk] int32 out
 * An index outside [0, n_routed) is not placed; MOE_ERR_RANGE is written to
 * dev_status and the outputs for that call are unspecified.
 * Limits: n_routed <= 1024, T * topk < 2^31.
 */
moe_status moe_dispatch_build(const moe_cfg *cfg, int64_t T, const int32_t *indices,
                              int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                              int32_t *slot_of, void *ws, size_t ws_bytes,
                              int32_t *dev_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
