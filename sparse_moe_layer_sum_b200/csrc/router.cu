// moe_router: scores, group-limited top-k selection and gate weights.
//
// Page "DeepSeek-V3.2-Exp · Router": z = x W_r, s = sigmoid(z) (or softmax),
// the top-8 experts of s + b inside the best 4 of 8 groups (a group scores
// the sum of its two largest biased scores), and gates G_i = 2.5 s_i /
// sum_j s_j over the chosen experts -- the four equations under "All 4 steps"
// and the gate-forward code excerpt under "Code".
//
// The scores z = x W_r^T are fp32-accurate either way:
//  1a. bf16 x (T >= 32, experts a multiple of 128, dim of 64), on the tensor
//      cores: split_w3 writes W_r as three bf16 terms whose sum is W_r
//      exactly; router_scores_tc multiplies x by all three with tcgen05 MMAs
//      (exact products) and adds each k-block's partial into fp32 registers,
//      with a deterministic split over dim when there are too few tiles to
//      fill the GPU.
//  1b. otherwise router_scores, tiled fp32 FMA on the CUDA cores with the
//      same kind of split.  The excerpt scores in fp32.
//  2. router_select: one warp per token; sums the split partials in a fixed
//     order, applies sigmoid/softmax and the bias, picks groups and experts
//     with warp-shuffle arg-max rounds and writes gates, indices and the
//     smallest decision gap.
#include <cuda_bf16.h>
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "moe_router.h"
#include "route.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using route::SC_BM;
using route::SC_BN;
using route::SC_BK;
using route::SC_THREADS;
using route::SelectArgs;
constexpr int SEL_WARPS = 8;

// z_part[split][t][e] = sum over this split's columns d of x[t,d] * w[e,d].
template <typename XT>
__global__ void __launch_bounds__(SC_THREADS) router_scores(const XT *__restrict__ x,
                                                            const float *__restrict__ w,
                                                            float *__restrict__ z_part, int T,
                                                            int E, int D, int cols_per_split) {
  __shared__ float xs[SC_BK][SC_BM + 4];
  __shared__ float ws[SC_BK][SC_BN + 4];
  route::scores_tile(x, w, z_part, T, E, D, cols_per_split, blockIdx.x * SC_BM,
                     blockIdx.y * SC_BN, blockIdx.z, xs, ws);
}

// One warp per token.  Shared memory per warp: s[E] and c[E].
__global__ void __launch_bounds__(SEL_WARPS * 32) router_select(SelectArgs a) {
  extern __shared__ float sel_smem[];
  const int warp = threadIdx.x / 32;
  const int t = blockIdx.x * SEL_WARPS + warp;
  if (t >= a.T) return;
  float *s = sel_smem + (size_t)warp * 2 * a.E;
  route::select_token(a, t, s, s + a.E);
}

// ------------------------------------------------ tensor-core scores (bf16 x)
//
// z = x W_r^T with x in bf16 (exact in fp32) and W_r in fp32: W_r is split
// once per call into three bf16 matrices with W_r = hi + mid + lo exactly
// (each term holds the next 8 significant bits; the remainders are exact in
// fp32), and z = x hi^T + x mid^T + x lo^T runs as three tcgen05 bf16 MMAs
// per k-step into one fp32 TMEM accumulator.  The products are exact, so z
// carries only fp32 accumulation error, as an fp32 dot product would.

__global__ void __launch_bounds__(256) split_w3(const float *__restrict__ w, __nv_bfloat16 *w3,
                                                int64_t n) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = w[i];
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  w3[i] = hi;
  w3[n + i] = mid;
  w3[2 * n + i] = __float2bfloat16_rn(r2);
}

namespace tcr {

constexpr int BK = 64, BM = 128, THREADS = 192, EPI_WARPS = 4;
constexpr int A_BYTES = BM * BK * 2;  // one of the three weight terms
constexpr int NCHUNK = 3;             // TMEM buffers for per-k-block partial sums

struct Params {
  int T, E, nsplit, kb_per_split, KB, mt, nt;
  float *z_part;  // [nsplit][T][E]
  int32_t *status;
  int64_t timeout_ns;
};

template <int BN, int STAGES>
struct Layout {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = 3 * A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // full, empty, chunk_full, chunk_empty, drain
  static constexpr int MISC_OFF = BAR_OFF + (2 * STAGES + 2 * NCHUNK + 1) * 8;
  static constexpr size_t SMEM = 1024 + MISC_OFF + 16 + 4 * STAGES;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(NCHUNK * BN <= 512, "TMEM chunk buffers");
};

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, int64_t limit_ns) {
  const uint64_t t0 = sm100::globaltimer_ns();
  while (!sm100::mbar_try_wait(bar, parity))
    if ((int64_t)(sm100::globaltimer_ns() - t0) > limit_ns) break;
}

// Tensor cores add in fp32 with a rounding that drifts with the number of
// additions into one accumulator, so the MMAs of each k-block (x times the
// three weight terms, 64 columns of dim) go into a fresh TMEM buffer and the
// epilogue warps add that partial into fp32 running sums in registers:
// every accumulation chain stays a dozen additions long.
//
// tile -> (split, token tile, expert tile); expert tiles innermost so the
// CTAs sharing an x tile run together
template <int BN, int STAGES>
__global__ void __launch_bounds__(THREADS, 1)
    router_scores_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                     const Params p) {
  using L = Layout<BN, STAGES>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
  uint64_t *empty = full + STAGES;
  uint64_t *cfull = empty + STAGES;
  uint64_t *cempty = cfull + NCHUNK;
  uint64_t *drain = cempty + NCHUNK;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 4);
  volatile int *pending = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 16);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      pending[s] = -1;
    }
    for (int c = 0; c < NCHUNK; ++c) {
      mbar_init(cfull + c, 1);
      mbar_init(cempty + c, EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.nsplit * p.nt * p.mt;

  auto decode = [&](int tile, int &split, int &n0, int &m0, int &kb0, int &kb1, int &nvalid) {
    const int mt = tile % p.mt;
    const int rest = tile / p.mt;
    const int nt = rest % p.nt;
    split = rest / p.nt;
    m0 = mt * BM;
    n0 = nt * BN;
    nvalid = min(BN, p.T - n0);
    kb0 = split * p.kb_per_split;
    kb1 = min(p.KB, kb0 + p.kb_per_split);
  };

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_last();  // the weight terms are re-read per token tile
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        int split, n0, m0, kb0, kb1, nvalid;
        decode(tile, split, n0, m0, kb0, kb1, nvalid);
        const int nbox = (nvalid + 31) / 32;
        const uint32_t bytes = (uint32_t)(3 * A_BYTES + nbox * 32 * BK * 2);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full + stage, bytes);
          pending[stage] = (int)phase;
          uint8_t *dst = sm + stage * L::STAGE_BYTES;
          for (int t3 = 0; t3 < 3; ++t3)
            tma_load_2d_hint(&tmW, dst + t3 * A_BYTES, full + stage, kb * BK, t3 * p.E + m0,
                             pol_w);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(&tmX, dst + 3 * A_BYTES + i * 32 * BK * 2, full + stage, kb * BK,
                        n0 + i * 32);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, c = 0;
      uint32_t phase = 0, cphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        int split, n0, m0, kb0, kb1, nvalid;
        decode(tile, split, n0, m0, kb0, kb1, nvalid);
        const uint32_t idesc = idesc_bf16_f32(BM, (nvalid + 15) & ~15);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bounded(cempty + c, cphase ^ 1u, abort_flag, p.timeout_ns, p.status) ||
              !wait_bounded(full + stage, phase, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          pending[stage] = -1;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(c * BN);
          const uint32_t a_addr = smem_u32(sm + stage * L::STAGE_BYTES);
          const uint32_t b_addr = a_addr + 3 * A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
            for (int t3 = 0; t3 < 3; ++t3)
              mma_bf16(d_tmem, sdesc_sw128(a_addr + t3 * A_BYTES + kk * 32),
                       sdesc_sw128(b_addr + kk * 32), idesc, (kk > 0 || t3 > 0) ? 1u : 0u);
          mma_commit(empty + stage);
          mma_commit(cfull + c);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++c == NCHUNK) {
            c = 0;
            cphase ^= 1u;
          }
        }
      }
      if (!ok) {
        mma_commit(drain);
        drain_wait(drain, 0, p.timeout_ns);
      }
    }
  } else {
    // epilogue: running fp32 sums of the per-k-block partials; lane = expert,
    // the 128 columns (tokens) of the tile in four groups of 32
    const int q = warp & 3;
    int c = 0;
    uint32_t cphase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int split, n0, m0, kb0, kb1, nvalid;
      decode(tile, split, n0, m0, kb0, kb1, nvalid);
      float run[BN];
#pragma unroll
      for (int j = 0; j < BN; ++j) run[j] = 0.f;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(cfull + c, cphase, abort_flag, p.timeout_ns, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * BN);
#pragma unroll
        for (int g = 0; g < BN / 32; ++g) {
          if (g * 32 < nvalid) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + (uint32_t)(g * 32), v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) run[g * 32 + j] += __uint_as_float(v[j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(cempty + c);
        if (++c == NCHUNK) {
          c = 0;
          cphase ^= 1u;
        }
      }
      if (!ok) break;
      float *out = p.z_part + (size_t)split * p.T * p.E;
      const int e = m0 + q * 32 + lane;
#pragma unroll
      for (int j = 0; j < BN; ++j)
        if (j < nvalid) out[(size_t)(n0 + j) * p.E + e] = run[j];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag)
    for (int s = 0; s < STAGES; ++s)
      if (pending[s] >= 0) drain_wait(full + s, (uint32_t)pending[s], p.timeout_ns);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

}  // namespace tcr

constexpr int TC_BN = 128, TC_STAGES = 3;

bool tc_router(const moe_cfg *c, moe_dtype x_dt) {
  return x_dt == MOE_BF16 && c->n_routed % tcr::BM == 0 && c->dim % tcr::BK == 0;
}

struct TcPlan {
  int mt, nt, nsplit, kb_per_split, KB;
};

TcPlan plan_tc(const moe_cfg *c, int64_t T) {
  TcPlan p;
  p.KB = c->dim / tcr::BK;
  p.mt = c->n_routed / tcr::BM;
  p.nt = (int)((T + TC_BN - 1) / TC_BN);
  const int tiles = p.mt * p.nt;
  // splits of dim: the count with the least estimated time on the B200's
  // 148 SMs -- waves of tiles times k-blocks per tile at about 1 us each
  // (64 KB of operands per k-block and SM), plus writing and reading back
  // each split's fp32 partial sums at about 6.5 TB/s; ties go to fewer
  // splits
  constexpr int SMS = 148;
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int ns = 1; ns <= p.KB; ++ns) {
    const int kbps = (p.KB + ns - 1) / ns;
    const int n = (p.KB + kbps - 1) / kbps;
    if (n != ns) continue;  // the same split as a smaller count
    const int64_t waves = ((int64_t)tiles * n + SMS - 1) / SMS;
    const int64_t cost = waves * kbps * 1000 + (int64_t)n * T * c->n_routed * 8 / 6500;
    if (cost < best_cost) {
      best_cost = cost;
      best = n;
    }
  }
  p.kb_per_split = (p.KB + best - 1) / best;
  p.nsplit = best;
  return p;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

size_t tc_ws_bytes(const moe_cfg *c, int64_t T) {
  if (c->n_routed % tcr::BM != 0 || c->dim % tcr::BK != 0) return 0;  // CUDA-core path only
  const TcPlan p = plan_tc(c, T);
  return align_up((size_t)3 * c->n_routed * c->dim * 2, 1024) +
         align_up((size_t)p.nsplit * T * c->n_routed * 4, 256);
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
  const size_t simt = align_up((size_t)p.nsplit * (size_t)T * cfg->n_routed * sizeof(float), 256);
  const size_t tc = tc_ws_bytes(cfg, T);
  return simt > tc ? simt : tc;
}

namespace moe {
namespace {

// bytes of the three-term bf16 split of W_r (0 when the tensor-core scores do
// not apply to this configuration)
size_t split_bytes(const moe_cfg *c) {
  if (c->n_routed % tcr::BM != 0 || c->dim % tcr::BK != 0) return 0;
  return (size_t)3 * c->n_routed * c->dim * 2;
}

moe_status enqueue_split(const moe_cfg *cfg, const float *w_r, __nv_bfloat16 *w3,
                         cudaStream_t s) {
  const int64_t nw = (int64_t)cfg->n_routed * cfg->dim;
  split_w3<<<(unsigned)((nw + 255) / 256), 256, 0, s>>>(w_r, w3, nw);
  return launch_status();
}

// The forward behind both entry points; w_split is the prepared split of W_r
// or NULL (then it is written into the workspace first).
moe_status router_forward(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                          const float *w_r, const void *w_split, const float *bias,
                          float *weights, int32_t *indices, float *sel_gap, void *ws,
                          size_t ws_bytes, int32_t *dev_status, cudaStream_t s) {
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

  float *z_part = static_cast<float *>(ws);
  int nsplit;
  if (tc_router(cfg, x_dt) && T >= 32) {
    const TcPlan tp = plan_tc(cfg, T);
    const __nv_bfloat16 *w3 = static_cast<const __nv_bfloat16 *>(w_split);
    z_part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                       align_up(split_bytes(cfg), 1024));
    if (!w3) {
      __nv_bfloat16 *w3ws = static_cast<__nv_bfloat16 *>(ws);
      if ((st = enqueue_split(cfg, w_r, w3ws, s)) != MOE_OK) return st;
      w3 = w3ws;
    }
    CUtensorMap mw, mx;
    if (!make_tmap_bf16(&mw, w3, (uint64_t)3 * cfg->n_routed, cfg->dim, tcr::BM) ||
        !make_tmap_bf16(&mx, x, (uint64_t)T, cfg->dim, 32))
      return MOE_ERR_CUDA;
    tcr::Params pp;
    pp.T = (int)T;
    pp.E = cfg->n_routed;
    pp.nsplit = tp.nsplit;
    pp.kb_per_split = tp.kb_per_split;
    pp.KB = tp.KB;
    pp.mt = tp.mt;
    pp.nt = tp.nt;
    pp.z_part = z_part;
    pp.status = dev_status;
    pp.timeout_ns = 1000000000LL;
    using L = tcr::Layout<TC_BN, TC_STAGES>;
    auto kern = tcr::router_scores_tc<TC_BN, TC_STAGES>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    const int total = tp.nsplit * tp.nt * tp.mt;
    const int nsm = sm_count();
    if (nsm <= 0) return MOE_ERR_CUDA;
    kern<<<total < nsm ? total : nsm, tcr::THREADS, L::SMEM, s>>>(mw, mx, pp);
    if ((st = launch_status()) != MOE_OK) return st;
    nsplit = tp.nsplit;
  } else {
    const Plan p = plan_scores(cfg, T);
    nsplit = p.nsplit;
    dim3 grid((unsigned)((T + SC_BM - 1) / SC_BM),
              (unsigned)((cfg->n_routed + SC_BN - 1) / SC_BN), (unsigned)p.nsplit);
    if (x_dt == MOE_BF16)
      router_scores<__nv_bfloat16><<<grid, SC_THREADS, 0, s>>>(
          static_cast<const __nv_bfloat16 *>(x), w_r, z_part, (int)T, cfg->n_routed, cfg->dim,
          p.cols_per_split);
    else
      router_scores<float><<<grid, SC_THREADS, 0, s>>>(static_cast<const float *>(x), w_r,
                                                       z_part, (int)T, cfg->n_routed, cfg->dim,
                                                       p.cols_per_split);
    if ((st = launch_status()) != MOE_OK) return st;
  }

  SelectArgs a;
  a.z_part = z_part;
  a.nsplit = nsplit;
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
  return launch_status();
}

}  // namespace
}  // namespace moe

MOE_EXPORT size_t moe_router_prepare_size(const moe_cfg *cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return split_bytes(cfg);
}

MOE_EXPORT moe_status moe_router_prepare(const moe_cfg *cfg, const float *w_r, void *prep,
                                         size_t prep_bytes, moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (!w_r || !prep) return MOE_ERR_INVALID;
  const size_t need = split_bytes(cfg);
  if (need == 0) return MOE_ERR_UNSUPPORTED;
  if (prep_bytes < need) return MOE_ERR_WORKSPACE;
  return enqueue_split(cfg, w_r, static_cast<__nv_bfloat16 *>(prep), as_stream(stream));
}

MOE_EXPORT moe_status moe_router_forward(const moe_cfg *cfg, int64_t T, const void *x,
                                         moe_dtype x_dt, const float *w_r, const float *bias,
                                         float *weights, int32_t *indices, float *sel_gap,
                                         void *ws, size_t ws_bytes, int32_t *dev_status,
                                         moe_stream_t stream) {
  return router_forward(cfg, T, x, x_dt, w_r, nullptr, bias, weights, indices, sel_gap, ws,
                        ws_bytes, dev_status, as_stream(stream));
}

MOE_EXPORT moe_status moe_router_forward_prepared(const moe_cfg *cfg, int64_t T, const void *x,
                                                  moe_dtype x_dt, const float *w_r,
                                                  const void *prep, const float *bias,
                                                  float *weights, int32_t *indices,
                                                  float *sel_gap, void *ws, size_t ws_bytes,
                                                  int32_t *dev_status, moe_stream_t stream) {
  if (!prep) return MOE_ERR_INVALID;
  return router_forward(cfg, T, x, x_dt, w_r, prep, bias, weights, indices, sel_gap, ws,
                        ws_bytes, dev_status, as_stream(stream));
}
