// moe_router: scores, group-limited top-k selection and gate weights.
//
// Page "DeepSeek-V3.2-Exp · Router": z = x W_r, s = sigmoid(z) (or softmax),
// the top-8 experts of s + b inside the best 4 of 8 groups (a group scores
// the sum of its two largest biased scores), and gates G_i = 2.5 s_i /
// sum_j s_j over the chosen experts -- the four equations under "All 4 steps"
// and the gate-forward code excerpt under "Code".
//
// Two kernels:
//  1. router_scores: z = x W_r^T in fp32 on the CUDA cores (tiled, with a
//     deterministic split over dim when there are too few token tiles to
//     fill the GPU).  fp32 inputs and fp32 FMA: the excerpt scores in fp32.
//  2. router_select: one warp per token; sums the split partials in a fixed
//     order, applies sigmoid/softmax and the bias, picks groups and experts
//     with warp-shuffle arg-max rounds and writes gates, indices and the
//     smallest decision gap.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "moe_router.h"

namespace moe {
namespace {

constexpr int SC_BM = 64, SC_BN = 64, SC_BK = 16, SC_THREADS = 256;
constexpr int SEL_WARPS = 8;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// z_part[split][t][e] = sum over this split's columns d of x[t,d] * w[e,d].
template <typename XT>
__global__ void __launch_bounds__(SC_THREADS) router_scores(const XT *__restrict__ x,
                                                            const float *__restrict__ w,
                                                            float *__restrict__ z_part, int T,
                                                            int E, int D, int cols_per_split) {
  __shared__ float xs[SC_BK][SC_BM + 4];
  __shared__ float ws[SC_BK][SC_BN + 4];
  const int m0 = blockIdx.x * SC_BM, n0 = blockIdx.y * SC_BN;
  const int kbeg = blockIdx.z * cols_per_split;
  const int kend = min(D, kbeg + cols_per_split);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kend; k0 += SC_BK) {
    for (int i = threadIdx.x; i < SC_BM * SC_BK; i += SC_THREADS) {
      const int r = i / SC_BK, c = i % SC_BK;
      const int gr = m0 + r, gc = k0 + c;
      xs[c][r] = (gr < T && gc < kend) ? to_f32(x[(size_t)gr * D + gc]) : 0.f;
      const int er = n0 + r;
      ws[c][r] = (er < E && gc < kend) ? w[(size_t)er * D + gc] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SC_BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float *out = z_part + (size_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = m0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = n0 + tx * 4 + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// Warp arg-max over (value, index): larger value wins, equal values go to
// the lower index.  Returns the winner in every lane.
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

struct SelectArgs {
  const float *z_part;
  int nsplit;
  const float *bias;
  float *weights;
  int32_t *indices;
  float *sel_gap;
  int T, E, G, Gk, k;
  float route_scale;
  int softmax;
};

// One warp per token.  Shared memory per warp: s[E] and c[E].
__global__ void __launch_bounds__(SEL_WARPS * 32) router_select(SelectArgs a) {
  extern __shared__ float sel_smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * SEL_WARPS + warp;
  if (t >= a.T) return;
  const int E = a.E;
  float *s = sel_smem + (size_t)warp * 2 * E;
  float *c = s + E;
  const float NEG_INF = -INFINITY;

  // z (split partials summed in split order), then s and c = s + b
  float zmax = NEG_INF;
  for (int e = lane; e < E; e += 32) {
    float z = 0.f;
    for (int p = 0; p < a.nsplit; ++p) z += a.z_part[((size_t)p * a.T + t) * E + e];
    s[e] = z;
    zmax = fmaxf(zmax, z);
  }
  if (a.softmax) {
    zmax = warp_max(zmax);
    float part = 0.f;
    for (int e = lane; e < E; e += 32) {
      const float ez = expf(s[e] - zmax);
      s[e] = ez;
      part += ez;
    }
    const float tot = warp_sum(part);
    for (int e = lane; e < E; e += 32) s[e] = s[e] / tot;
  } else {
    for (int e = lane; e < E; e += 32) s[e] = 1.0f / (1.0f + expf(-s[e]));
  }
  for (int e = lane; e < E; e += 32) c[e] = a.bias ? s[e] + a.bias[e] : s[e];
  __syncwarp();

  // group selection: lane q scores group q
  const int P = E / a.G;
  float gap = INFINITY;
  uint32_t kept = 0xffffffffu;
  if (a.G > 1) {
    float gs = NEG_INF;
    if (lane < a.G) {
      float m1 = NEG_INF, m2 = NEG_INF;
      for (int i = 0; i < P; ++i) {
        const float v = c[lane * P + i];
        if (v > m1) {
          m2 = m1;
          m1 = v;
        } else if (v > m2) {
          m2 = v;
        }
      }
      gs = a.bias ? m1 + m2 : m1;
    }
    kept = 0;
    float prev = 0.f;
    const int rounds = a.Gk < a.G ? a.Gk + 1 : a.Gk;
    for (int r = 0; r < rounds; ++r) {
      float v = (lane < a.G && !((kept >> lane) & 1u)) ? gs : NEG_INF;
      int i = (lane < a.G && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
      warp_argmax(v, i);
      if (r < a.Gk) {
        kept |= 1u << i;
        prev = v;
      } else {
        gap = fminf(gap, prev - v);  // last kept group minus best dropped group
      }
    }
  }

  // expert selection: lane owns experts lane, lane+32, ...; k arg-max rounds
  // over the biased scores of the kept groups, plus one round for the first
  // expert left out
  uint32_t taken = 0;  // bit m: expert lane + 32 m already chosen
  float prev_v = 0.f;
  int chosen_i = 0;
  const int rounds = a.k < E ? a.k + 1 : a.k;
  for (int r = 0; r < rounds; ++r) {
    float v = NEG_INF;
    int i = 0x7fffffff;
    for (int m = 0, e = lane; e < E; ++m, e += 32) {
      if ((taken >> m) & 1u) continue;
      const float ce = ((kept >> (e / P)) & 1u) ? c[e] : NEG_INF;
      if (ce > v || (ce == v && e < i)) {
        v = ce;
        i = e;
      }
    }
    warp_argmax(v, i);
    if (r < a.k) {
      if (i % 32 == lane) taken |= 1u << (i / 32);
      if (r > 0) gap = fminf(gap, prev_v - v);  // consecutive chosen experts
      prev_v = v;
      if (lane == r) chosen_i = i;
    } else {
      gap = fminf(gap, prev_v - v);  // k-th chosen minus first left out
    }
  }

  // gates: unbiased scores of the chosen experts, summed in choice order
  float w = (lane < a.k) ? s[chosen_i] : 0.f;
  float tot = 0.f;
  for (int j = 0; j < a.k; ++j) tot += __shfl_sync(0xffffffffu, w, j);
  if (lane < a.k) {
    if (!a.softmax) w = w / tot;
    w = w * a.route_scale;
    a.weights[(size_t)t * a.k + lane] = w;
    a.indices[(size_t)t * a.k + lane] = chosen_i;
  }
  if (a.sel_gap && lane == 0) a.sel_gap[t] = gap;
}

struct Plan {
  int nsplit, cols_per_split;
};

Plan plan_scores(const moe_cfg *c, int64_t T) {
  const int mt = (int)((T + SC_BM - 1) / SC_BM);
  const int nt = (c->n_routed + SC_BN - 1) / SC_BN;
  const int tiles = mt * nt;
  const int target = 296;  // about two CTAs per SM on a 148-SM part
  int max_split = c->dim / 256;
  if (max_split < 1) max_split = 1;
  int nsplit = (target + tiles - 1) / tiles;
  if (nsplit > max_split) nsplit = max_split;
  if (nsplit < 1) nsplit = 1;
  int cps = (c->dim + nsplit - 1) / nsplit;
  cps = (cps + SC_BK - 1) / SC_BK * SC_BK;
  nsplit = (c->dim + cps - 1) / cps;
  return {nsplit, cps};
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_EXPORT size_t moe_router_workspace_size(const moe_cfg *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  const Plan p = plan_scores(cfg, T);
  return align_up((size_t)p.nsplit * (size_t)T * cfg->n_routed * sizeof(float), 256);
}

MOE_EXPORT moe_status moe_router_forward(const moe_cfg *cfg, int64_t T, const void *x,
                                         moe_dtype x_dt, const float *w_r, const float *bias,
                                         float *weights, int32_t *indices, float *sel_gap,
                                         void *ws, size_t ws_bytes, int32_t *dev_status,
                                         moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || T > (int64_t)1 << 30) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!x || !w_r || !weights || !indices || !ws) return MOE_ERR_INVALID;
  if (cfg->has_bias && !bias) return MOE_ERR_INVALID;
  if (x_dt != MOE_F32 && x_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->n_routed > 1024 || cfg->n_groups > 32 || cfg->topk > 32 || cfg->dim % 4 != 0)
    return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < moe_router_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;

  cudaStream_t s = as_stream(stream);
  const Plan p = plan_scores(cfg, T);
  float *z_part = static_cast<float *>(ws);
  dim3 grid((unsigned)((T + SC_BM - 1) / SC_BM), (unsigned)((cfg->n_routed + SC_BN - 1) / SC_BN),
            (unsigned)p.nsplit);
  if (x_dt == MOE_BF16)
    router_scores<__nv_bfloat16><<<grid, SC_THREADS, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(x), w_r, z_part, (int)T, cfg->n_routed, cfg->dim,
        p.cols_per_split);
  else
    router_scores<float><<<grid, SC_THREADS, 0, s>>>(static_cast<const float *>(x), w_r, z_part,
                                                     (int)T, cfg->n_routed, cfg->dim,
                                                     p.cols_per_split);
  if ((st = launch_status()) != MOE_OK) return st;

  SelectArgs a;
  a.z_part = z_part;
  a.nsplit = p.nsplit;
  a.bias = cfg->has_bias ? bias : nullptr;
  a.weights = weights;
  a.indices = indices;
  a.sel_gap = sel_gap;
  a.T = (int)T;
  a.E = cfg->n_routed;
  a.G = cfg->n_groups;
  a.Gk = cfg->topk_groups;
  a.k = cfg->topk;
  a.route_scale = cfg->route_scale;
  a.softmax = cfg->score_func == MOE_SCORE_SOFTMAX;
  const size_t smem = (size_t)SEL_WARPS * 2 * cfg->n_routed * sizeof(float);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(router_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  router_select<<<(unsigned)((T + SEL_WARPS - 1) / SEL_WARPS), SEL_WARPS * 32, smem, s>>>(a);
  (void)dev_status;
  return launch_status();
}
