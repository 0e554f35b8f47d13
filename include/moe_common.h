/*
 * moe_common.h -- types shared by the four MoE block libraries
 * (moe_router, moe_dispatch, moe_experts, moe_combine).
 *
 * The block is the forward pass of one DeepSeek-V3/R1 Mixture-of-Experts FFN
 * layer as the pages "DeepSeek-V3.2-Exp · Router" and "DeepSeek-V3.2-Exp ·
 * Mixture of experts" describe it: a router that picks k of E experts per
 * token from the best groups, a grouping of tokens by expert, the routed
 * experts plus the shared expert, and a weighted sum into an fp32 output.
 *
 * Conventions common to every entry point:
 *  - All pointers to tensors are DEVICE pointers, allocated and owned by the
 *    caller.  The libraries never allocate, free or synchronise; every call
 *    enqueues its kernels on the stream passed in and returns.
 *  - Tensors are dense row-major.  Matrices follow the nn.Linear layout
 *    [out, in] (y = x W^T), as the router weight [n_routed_experts, dim] of
 *    the gate-init excerpt.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns a negative moe_status and launches nothing.
 *  - Errors found on the device (an expert index out of range, a pipeline
 *    wait that ran out of time) are written to the optional device status
 *    word `dev_status` (int32, zero-initialised by the caller; the first error
 *    wins).  Read it with an ordinary device-to-host copy after the stream has
 *    finished.  NULL disables the report.
 *  - Each library that needs scratch memory exports a *_workspace_size()
 *    query; the caller passes a device buffer at least that large (256-byte
 *    aligned) and its size.
 */
#ifndef MOE_COMMON_H
#define MOE_COMMON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's stream handle); 0 is the legacy default stream. */
typedef struct CUstream_st *moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = -1,     /* null pointer, negative size, inconsistent config */
  MOE_ERR_UNSUPPORTED = -2, /* valid but not implemented (dtype or shape)       */
  MOE_ERR_WORKSPACE = -3,   /* workspace smaller than *_workspace_size()        */
  MOE_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed             */
  MOE_ERR_TIMEOUT = -5,     /* device: a bounded pipeline wait expired          */
  MOE_ERR_RANGE = -6        /* device: an expert index outside [0, n_routed)    */
} moe_status;

typedef enum {
  MOE_F32 = 0,  /* IEEE binary32                                  */
  MOE_BF16 = 1, /* bfloat16                                       */
  MOE_E4M3 = 2  /* float8 e4m3 ("fn": no infinities), weights only */
} moe_dtype;

typedef enum {
  MOE_SCORE_SIGMOID = 0, /* s = sigmoid(z); gates renormalised to sum 1 */
  MOE_SCORE_SOFTMAX = 1  /* s = softmax(z); gates not renormalised      */
} moe_score_func;

/*
 * Block hyper-parameters, named after the gate-init and moe-init excerpts:
 *   dim          model width D (7168 for V3)
 *   n_routed     routed experts E (256)
 *   n_groups     expert groups G (8); experts q*E/G .. (q+1)*E/G-1 form group q
 *   topk_groups  groups kept per token (4)
 *   topk         experts per token k (8)
 *   inter        expert intermediate width I (2048)
 *   n_shared     shared experts S (1), applied to every token with weight 1
 *   route_scale  gate scale (2.5)
 *   score_func   moe_score_func
 *   has_bias     1: a per-expert bias is added to the scores for selection
 *                only, and a group scores the sum of its two largest biased
 *                scores; 0: no bias, a group scores its largest score.
 */
typedef struct {
  int32_t dim, n_routed, n_groups, topk_groups, topk, inter, n_shared;
  float route_scale;
  int32_t score_func;
  int32_t has_bias;
} moe_cfg;

static inline const char *moe_status_name(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID: return "MOE_ERR_INVALID";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_RANGE: return "MOE_ERR_RANGE";
    default: return "MOE_ERR_UNKNOWN";
  }
}

#ifdef __cplusplus
}
#endif
#endif /* MOE_COMMON_H */
