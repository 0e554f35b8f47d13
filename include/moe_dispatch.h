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

/*
 * moe_dispatch_build without a workspace argument, for callers that hold
 * only their input and output buffers and have no way to obtain device
 * memory for scratch space -- for instance a host framework that hands a
 * kernel its tensors but no allocator, or a process whose device memory is
 * entirely owned by another allocator.  (The pages have no counterpart; this
 * is a convenience of this library.)
 *
 * The scratch space is a fixed array of 1 MiB inside this library, which
 * every GPU that loads the library holds until the process exits.  It covers
 * ceil(T / 64) * n_routed <= 262144 (for example T up to 65536 tokens with
 * 256 experts); larger calls return MOE_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up the array's device address with that
 * device current (and caches it, together with the id of the context it
 * belongs to; a later call in a new context of that device, for instance
 * after cudaDeviceReset, looks it up again), so make the first call in each
 * context before any stream capture.  This entry point allocates and frees no memory.  All calls share
 * the one array: calls that may overlap on the GPU (other streams, other
 * threads) race on it and must be serialised by the caller.  Outputs,
 * limits and errors are those of moe_dispatch_build.
 */
moe_status moe_dispatch_build_noalloc(const moe_cfg *cfg, int64_t T, const int32_t *indices,
                                      int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                                      int32_t *slot_of, int32_t *dev_status,
                                      moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
