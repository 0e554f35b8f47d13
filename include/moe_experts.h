/*
 * moe_experts.h -- the routed experts and the shared expert.
 *
 * Every expert is a bias-free SwiGLU MLP, w2(silu(w1 x) * w3 x) with
 * silu(a) = a * sigmoid(a): the pages print only the constructor
 * Expert(dim, moe_inter_dim) (moe-init excerpt of "DeepSeek-V3.2-Exp ·
 * Mixture of experts"), and three bias-free [inter, dim] / [dim, inter]
 * matrices match the per-expert count 3 * 7168 * 2048 = 44,040,192 of that
 * page's "Exact per-instance accounting" table.  The shared expert (MLP of
 * n_shared * moe_inter_dim features) is applied to every token.
 *
 * Computes, for the rows that moe_dispatch_build grouped by expert:
 *   h[p,:]   = round_act(silu(x[t] w1_e^T) * (x[t] w3_e^T))  t = sorted_token[p]
 *   out_perm[p,:]   = h[p,:] w2_e^T           p in [offsets[e], offsets[e+1])
 *   out_shared[t,:] = same expert on x[t] with the shared weights, every t
 * Accumulation is fp32; h is rounded once to the activation dtype (it is the
 * second matmul's operand); outputs are fp32 and not yet multiplied by the
 * gates (moe_combine applies them, as the excerpt multiplies the expert's
 * output by the weight before adding it into y).  Experts with no rows
 * launch no work (the excerpt skips them).
 */
#ifndef MOE_EXPERTS_H
#define MOE_EXPERTS_H
#include "moe_common.h"
#ifdef __cplusplus
extern "C" {
#endif

/*
 * Weights of all n_routed + n_shared experts, stacked: routed experts
 * 0 .. n_routed-1, then the shared expert(s).
 *   w1, w3  [n_routed + n_shared, inter, dim]
 *   w2      [n_routed + n_shared, dim, inter]
 *   w_dt    MOE_BF16, MOE_F32 or MOE_E4M3
 *   s1, s3  [n_routed + n_shared, inter/128, dim/128] fp32 (MOE_E4M3 only)
 *   s2      [n_routed + n_shared, dim/128, inter/128] fp32 (MOE_E4M3 only)
 * For MOE_E4M3 the weight is value(q) * scale of its 128 x 128 block.
 *   act_e4m3  0: the matmuls take bf16 activations (e4m3 weights are
 *             expanded to fp16 on the fly, fp16 x fp16 MMAs).
 *             1 (MOE_E4M3 weights only): FP8 x FP8 -- each expert row of x
 *             and each row of the hidden h (after its bf16 rounding) is
 *             quantised to e4m3 with one fp32 scale per row, row amax / 448
 *             (the weights' rule; an all-zero row has scale 0), and the
 *             matmuls run as e4m3 x e4m3 tensor-core MMAs; each 128-wide
 *             k-block's partial sum is scaled by its weight block's scale in
 *             fp32, and the row's scale is applied to the total.  The pages
 *             name FP8 experts but no activation format; this path trades
 *             about 5% rms of extra error for twice the tensor throughput.
 *             Needs dim % 256 == 0 and inter % 128 == 0.
 */
typedef struct {
  const void *w1, *w3, *w2;
  moe_dtype w_dt;
  const float *s1, *s3, *s2;
  int32_t act_e4m3;
} moe_expert_weights;

/* Bytes of device workspace moe_experts_forward needs (for MOE_E4M3 weights,
 * enough for either activation path). */
size_t moe_experts_workspace_size(const moe_cfg *cfg, int64_t T, moe_dtype x_dt,
                                  moe_dtype w_dt);

/*
 * x            [T, dim], x_dt = MOE_BF16 or MOE_F32
 * offsets      [n_routed + 1] int32 from moe_dispatch_build
 * sorted_token [T * topk] int32 from moe_dispatch_build
 * out_perm     [T * topk, dim] fp32 out, row p = expert output of row p
 * out_shared   [T, dim] fp32 out (may be NULL when n_shared == 0)
 * Paths: bf16 activations with bf16 or e4m3 weights run on the tcgen05
 * tensor cores (dim % 128 == 0, inter % 128 == 0); any other combination
 * (fp32 activations or weights) runs on the CUDA cores in fp32.
 * Limits: n_shared <= 1, T * topk < 2^31.
 * Device errors: MOE_ERR_TIMEOUT if a pipeline wait expired (the kernel then
 * stops early; outputs are unspecified).
 */
moe_status moe_experts_forward(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                               const moe_expert_weights *w, const int32_t *offsets,
                               const int32_t *sorted_token, float *out_perm, float *out_shared,
                               void *ws, size_t ws_bytes, int32_t *dev_status,
                               moe_stream_t stream);

/*
 * The experts and the weighted combine in one pass: the second matmul's
 * epilogue adds gate(t, e) * expert_e(x[t]) for every routed row, and the
 * shared expert's output with gate 1, straight into the fp32 block output
 *   y[t,:] = sum_j weights[t,j] * expert_{indices[t,j]}(x[t,:]) + shared(x[t,:])
 * with fp32 reductions (the "y[idx] += expert(x[idx]) * weight" accumulation
 * of the moe-forward excerpt, run for all experts at once).  y is zeroed by
 * the call first.  No per-slot expert outputs are written, which saves their
 * round trip through memory; in exchange the order of the fp32 additions
 * into y is not fixed, so results may differ in the last bits from run to
 * run (use moe_experts_forward + moe_combine for bit-reproducible sums).
 * indices, weights [T, topk] from moe_router_forward; y [T, dim] fp32 out,
 * 16-byte aligned (the epilogue adds 16-byte vectors into it; otherwise
 * MOE_ERR_INVALID).
 */
moe_status moe_experts_forward_combine(const moe_cfg *cfg, int64_t T, const void *x,
                                       moe_dtype x_dt, const moe_expert_weights *w,
                                       const int32_t *offsets, const int32_t *sorted_token,
                                       const int32_t *indices, const float *weights, float *y,
                                       void *ws, size_t ws_bytes, int32_t *dev_status,
                                       moe_stream_t stream);

/*
 * Expert parallelism: the experts split over `world` ranks (GPUs), as the
 * moe-init excerpt of "DeepSeek-V3.2-Exp · Mixture of experts" splits them
 * (n_local_experts = n_routed / world_size, experts_start_idx = rank *
 * n_local_experts) and the moe-forward excerpt sums the ranks' partial
 * outputs (dist.all_reduce(y)).  Rank r runs the routed experts
 * [r * E / world, (r + 1) * E / world) on the tokens routed to them, and the
 * shared expert on its slice of the tokens [floor(r * T / world),
 * floor((r + 1) * T / world)) -- every shared-expert row is computed by
 * exactly one rank, so the sum over ranks is the block output.  The router
 * and the dispatch run on every rank on the full batch (x is replicated).
 */
typedef struct {
  int32_t rank, world;
} moe_ep_shard;

/*
 * The shard of `shard->rank`: out[0..3] = first and end routed expert, first
 * and end token of the shared expert's slice.  Host only (no device call).
 * Returns MOE_ERR_INVALID for a bad config, T < 0 or rank outside
 * [0, world), MOE_ERR_UNSUPPORTED when world does not divide n_routed.
 */
moe_status moe_ep_plan(const moe_cfg *cfg, int64_t T, const moe_ep_shard *shard, int32_t *out);

/*
 * moe_experts_forward_combine for one expert-parallel rank: y (zeroed
 * first) receives the rank's partial sum, gate * expert output for the
 * routed rows of its experts plus the shared expert's output on its token
 * slice; the caller adds the ranks' y (an all-reduce).  w holds only the
 * rank's weights: its n_routed / world routed experts in order, then the
 * shared expert ([n_routed / world + n_shared, ...] stacked as above).
 * offsets, sorted_token, indices and weights are those of the whole batch.
 * Limits and errors as moe_experts_forward_combine and moe_ep_plan.
 */
moe_status moe_experts_forward_combine_ep(const moe_cfg *cfg, int64_t T, const void *x,
                                          moe_dtype x_dt, const moe_expert_weights *w,
                                          const moe_ep_shard *shard, const int32_t *offsets,
                                          const int32_t *sorted_token, const int32_t *indices,
                                          const float *weights, float *y, void *ws,
                                          size_t ws_bytes, int32_t *dev_status,
                                          moe_stream_t stream);

/*
 * The whole block for a decode-sized batch in one launch: routing (as
 * moe_router_forward, with fp32 FMA scores), the token grouping (as
 * moe_dispatch_build), the experts and the weighted scatter into y (as
 * moe_experts_forward_combine) run as phases of one persistent kernel with
 * one block per SM, separated by grid-wide barriers; a CUDA cooperative
 * launch keeps every block resident.  Each barrier wait is bounded (1 s):
 * a block that gives up records MOE_ERR_TIMEOUT in dev_status and returns.
 * No counterpart on the pages beyond the block itself; it removes the
 * launch gaps between the block's kernels at decode.
 *   x         [T, dim] bf16; w_r [n_routed, dim] fp32; bias [n_routed] fp32
 *   w         bf16 expert weights (act_e4m3 = 0)
 *   weights, indices [T, topk], sel_gap [T] (may be NULL): as moe_router_forward
 *   counts [n_routed], offsets [n_routed + 1], sorted_token, slot_of
 *             [T * topk]: as moe_dispatch_build
 *   y         [T, dim] fp32 out (zeroed by the call first), 16-byte aligned
 *   ws        moe_block_decode_workspace_size(cfg, T) bytes
 * Limits: the decode regime, T * topk <= 16 * n_routed; n_routed <= 256,
 * n_groups <= 32, topk <= 32, n_shared == 1, dim and inter multiples of 128;
 * otherwise MOE_ERR_UNSUPPORTED.  T == 0 launches nothing.
 */
size_t moe_block_decode_workspace_size(const moe_cfg *cfg, int64_t T);
moe_status moe_block_forward_decode(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                                    const float *w_r, const float *bias,
                                    const moe_expert_weights *w, float *weights,
                                    int32_t *indices, float *sel_gap, int32_t *counts,
                                    int32_t *offsets, int32_t *sorted_token, int32_t *slot_of,
                                    float *y, void *ws, size_t ws_bytes, int32_t *dev_status,
                                    moe_stream_t stream);

/*
 * The two halves of moe_experts_forward, for callers that schedule them
 * separately (moe_experts_forward(...) == moe_experts_up(...) followed by
 * moe_experts_down(...) on the same stream and workspace).
 *   moe_experts_up    gathers the expert-contiguous rows and computes
 *                     h = round_act(silu(x w1^T) * (x w3^T)) for every row
 *                     into the workspace
 *   moe_experts_down  reads h from the workspace that moe_experts_up filled
 *                     (same cfg, T, dtypes and offsets) and writes out_perm and
 *                     out_shared
 */
moe_status moe_experts_up(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                          const moe_expert_weights *w, const int32_t *offsets,
                          const int32_t *sorted_token, void *ws, size_t ws_bytes,
                          int32_t *dev_status, moe_stream_t stream);
moe_status moe_experts_down(const moe_cfg *cfg, int64_t T, moe_dtype x_dt,
                            const moe_expert_weights *w, const int32_t *offsets,
                            float *out_perm, float *out_shared, void *ws, size_t ws_bytes,
                            int32_t *dev_status, moe_stream_t stream);

/*
 * The activation quantiser of the FP8 x FP8 path (act_e4m3 = 1), on its own:
 * each row of src [rows, K] bf16 gets one scale, amax / 448 (fp32, IEEE
 * division), and codes e4m3(v * fp32(1 / scale)) (IEEE reciprocal, round to
 * nearest even, saturated to +-448); an all-zero row has scale 0 and codes 0.
 *   q       [rows, K] uint8 out (e4m3 codes, row-major)
 *   scales  [rows] fp32 out
 * No counterpart on the pages, which name FP8 experts but no activation
 * format (the weights' amax / 448 block rule applied to a row).
 * Limits: K % 4 == 0, rows < 2^31, src and q 8- and 4-byte aligned.
 * Returns MOE_ERR_INVALID for bad sizes or NULL pointers (rows == 0
 * launches nothing).
 */
moe_status moe_quantize_e4m3_rows(const void *src, int64_t rows, int32_t K, uint8_t *q,
                                  float *scales, moe_stream_t stream);

/*
 * Profiling: register up to five caller-owned cudaEvent_t handles that later
 * calls record on their stream: [0] before the row gather, [1] before the
 * first GEMM, [2] after it, [3] before the second GEMM, [4] after it.  n = 0
 * stops the recording.  Process-wide and not thread-safe; meant for
 * benchmarks.  Returns MOE_ERR_INVALID for n outside [0, 5].
 */
moe_status moe_experts_set_profile_events(void *const *events, int32_t n);

/*
 * Self-test of the bounded pipeline wait used by the tensor-core kernels:
 * one CTA waits on a barrier that nothing signals, with a limit of
 * `limit_ns` nanoseconds, then writes MOE_ERR_TIMEOUT to dev_status and
 * returns.  The context stays usable.  limit_ns must be in (0, 2e9].
 */
moe_status moe_experts_selftest_wait(int64_t limit_ns, int32_t *dev_status,
                                     moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
