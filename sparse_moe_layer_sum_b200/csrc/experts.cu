// moe_experts: routed experts and the shared expert as grouped SwiGLU GEMMs.
//
// Expert body: w2(silu(w1 x) * w3 x), three bias-free matrices -- the reading
// of Expert(dim, moe_inter_dim) in the moe-init excerpt of "DeepSeek-V3.2-Exp
// · Mixture of experts" that matches that page's per-expert count of
// 3 * 7168 * 2048 parameters.  The shared expert runs on every token.
//
// Tensor-core path (bf16 activations; bf16 or e4m3 weights), sm_100a:
//   gather_rows   X_perm[p] = x[sorted_token[p]] (expert-contiguous rows),
//                 followed by the T rows of x for the shared expert
//                 (gather_rows_f16 converts them to fp16 for e4m3 weights).
//   GEMM1         h = silu(X W1^T) * (X W3^T), bf16 out (fp16 with e4m3)
//   GEMM2         o = h W2^T, fp32 out, or gate * o added into y
// Both GEMMs are one persistent, warp-specialised kernel template
// (tc_expert_gemm): warp 0 issues TMA loads into a shared-memory ring, one
// thread of warp 1 issues tcgen05.mma into TMEM, four or eight epilogue
// warps drain TMEM with tcgen05.ld, and with e4m3 weights eight converter
// warps expand each code tile into the fp16 tile the MMA reads.
//
// The operands are swapped relative to the usual token-major GEMM: the 128
// rows of an MMA (M) per SM are weight rows and the MMA's N is the expert's
// tokens.  N is a run-time field of the instruction descriptor, so a tile
// spends MMA work only on the tokens its expert really has (rounded up to
// 16) -- from 1 token per expert at decode to 256 at prefill -- and each
// weight byte is streamed from HBM once per token tile.  Prefill tiles run on
// SM pairs (cta_group::2, M = 256).  In the first matmul each SM of a pair
// holds 128 rows of W1 and the same 128 rows of W3 in two accumulators (AT =
// 2), so a thread holds both SwiGLU halves of its feature; at decode a
// 128-row tile holds 64 rows of each and the epilogue pairs the warps that
// hold them (AT = 1).  In the second matmul each SM of a pair holds two
// 128-row blocks of W2 (AT = 2), whose single accumulator the epilogue reads
// in register batches and hands back before its last stores; the weighted
// scatter adds 16-byte vectors into y after a 4 x 4 transpose in each quad
// of lanes.
//
// FP8 x FP8 path (e4m3 weights and activations, act_e4m3): quant_rows_e4m3
// quantises the expert rows of x and later h (one scale per row), and
// tc_fp8_gemm runs both matmuls as e4m3 x e4m3 MMAs whose per-k-block partial
// sums eight promotion warps scale by the weight block's scale and add in
// fp32 registers; two helper warps build the scatter's gate lists and finish
// half of each tile's sums from shared memory.
//
// CUDA-core path: any other dtype combination (the fp32 configuration) runs
// on simt_gemm1 / simt_gemm2 in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include "common.cuh"
#include "moe_experts.h"
#include "dispatch_dev.cuh"
#include "route.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------------ tiling

// Per group g (routed experts 0..E-1, then the shared expert): its row count
// n_g, split into ntt_g token tiles of tile_base[g] rows (a multiple of 16,
// at most rows_max) and ft feature tiles; tile_start[g] is the exclusive
// prefix of ntt_g * ft over the groups and tile_start[G] the total.
struct Tiling {
  int rows_max;
  int ft;
  int32_t *tile_start;  // [G + 1]
  int32_t *tile_base;   // [G]
};

__device__ __forceinline__ void group_tiles(int n, int rows_max, int &base, int &ntt) {
  if (n <= 0) {
    base = 16;
    ntt = 0;
    return;
  }
  const int ntt0 = (n + rows_max - 1) / rows_max;
  base = ((n + ntt0 - 1) / ntt0 + 15) / 16 * 16;
  ntt = (n + base - 1) / base;
}

// The part of the experts' work one call runs: routed experts [e0, e1) and
// the shared expert on tokens [st0, st1).  A single-GPU call runs all of it;
// an expert-parallel rank runs its own experts and its slice of the tokens.
struct Shard {
  int e0, e1, st0, st1;
};

// Rows of group g in this call: an expert's tokens when it is one of the
// call's experts, else none; the shared expert's token slice.
__device__ __forceinline__ int group_rows(int g, const int32_t *off, int E, const Shard &sh) {
  if (g < E) return g >= sh.e0 && g < sh.e1 ? off[g + 1] - off[g] : 0;
  return sh.st1 - sh.st0;
}

// One warp: lane l owns a contiguous run of groups.
__device__ __forceinline__ void prep_tiles_warp(const int32_t *__restrict__ offsets, int E, int G,
                                                Shard sh, Tiling t0, Tiling t1) {
  const int lane = threadIdx.x % 32;
  const int per = (G + 31) / 32;
  const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
  for (int which = 0; which < 2; ++which) {
    const Tiling tl = which == 0 ? t0 : t1;
    if (!tl.tile_start) continue;
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      const int n = group_rows(g, offsets, E, sh);
      int base, ntt;
      group_tiles(n, tl.rows_max, base, ntt);
      tl.tile_base[g] = base;
      local += ntt * tl.ft;
    }
    int inc = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    int run = inc - local;
    for (int g = g0; g < g1; ++g) {
      const int n = group_rows(g, offsets, E, sh);
      int base, ntt;
      group_tiles(n, tl.rows_max, base, ntt);
      tl.tile_start[g] = run;
      run += ntt * tl.ft;
    }
    if (lane == 31) tl.tile_start[G] = inc;
  }
}

__global__ void __launch_bounds__(32) prep_tiles(const int32_t *__restrict__ offsets, int E,
                                                 int G, Shard sh, Tiling t0, Tiling t1) {
  prep_tiles_warp(offsets, E, G, sh, t0, t1);
}

// g: group (routed expert, then the shared expert); wg: its index in the
// call's weight tensors (the call's experts e0.. first, then the shared one);
// tok0: first token of a shared-expert tile.
struct Tile {
  int g, wg, ft, tt, ntt, n0, nvalid, rowbase, tok0;
};

// First k-block of a tile.  Tiles that run at the same time share operands
// (the feature tiles of one expert read the same token rows; the token tiles
// of one expert read the same weight rows); starting them at different
// k-blocks spreads those concurrent reads over different L2 lines instead of
// sending every SM to the same lines at once.
__device__ __forceinline__ int k_rotation(const Tile &t, int KB) { return (t.ft * 7 + t.tt * 5) % KB; }

// rowbase: first row of the group in the expert-contiguous activation
// buffers (routed: offsets[g]; shared: after the T*k routed rows).
__device__ __forceinline__ Tile decode_tile(int tile, const int32_t *tstart, const int32_t *tbase,
                                            const int32_t *off, int G, int E, int T,
                                            int rows_routed, const Shard &sh) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tstart[mid] <= tile)
      lo = mid;
    else
      hi = mid;
  }
  Tile t;
  t.g = lo;
  t.wg = lo < E ? lo - sh.e0 : (sh.e1 - sh.e0) + (lo - E);
  const int n = group_rows(lo, off, E, sh);
  const int base = tbase[lo];
  const int ntt = (n + base - 1) / base;
  const int local = tile - tstart[lo];
  t.ft = local / ntt;
  t.tt = local - t.ft * ntt;
  t.ntt = ntt;
  t.n0 = t.tt * base;
  t.nvalid = min(base, n - t.n0);
  t.rowbase = lo < E ? off[lo] : rows_routed + (lo - E) * T + sh.st0;
  t.tok0 = sh.st0 + t.n0;
  return t;
}

// ------------------------------------------------------------------ gather

// X_perm[p] = x[sorted_token[p]] for p < rows_routed, then x itself for the
// shared expert's rows.  One warp per row, 16-byte vectors.
// Whether row p of the expert-contiguous buffers belongs to this call's share
// (every row when the call is not sharded: off == NULL).
__device__ __forceinline__ bool row_in_shard(int row, int rows_routed, int T,
                                             const int32_t *off, const Shard &sh) {
  if (!off) return true;
  if (row < rows_routed) return row >= off[sh.e0] && row < off[sh.e1];
  const int t = (row - rows_routed) % T;
  return t >= sh.st0 && t < sh.st1;
}

__global__ void __launch_bounds__(256) gather_rows(const uint4 *__restrict__ x,
                                                   const int32_t *__restrict__ sorted_token,
                                                   uint4 *__restrict__ xp, int rows_routed,
                                                   int rows_total, int T, int vec_per_row,
                                                   const int32_t *off, Shard sh) {
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) / 32);
  const int lane = threadIdx.x % 32;
  if (row >= rows_total || !row_in_shard(row, rows_routed, T, off, sh)) return;
  const int src = row < rows_routed ? sorted_token[row] : (row - rows_routed) % T;
  const uint4 *s = x + (size_t)src * vec_per_row;
  uint4 *d = xp + (size_t)row * vec_per_row;
  // four 16-byte loads in flight per lane before their stores
  int v = lane;
  for (; v + 96 < vec_per_row; v += 128) {
    const uint4 a = __ldg(s + v), b = __ldg(s + v + 32), c = __ldg(s + v + 64), e = __ldg(s + v + 96);
    d[v] = a;
    d[v + 32] = b;
    d[v + 64] = c;
    d[v + 96] = e;
  }
  for (; v < vec_per_row; v += 32) d[v] = __ldg(s + v);
}

// The same rows converted to fp16 (the e4m3 path computes in fp16; bf16 values
// in the fp16 normal range convert exactly).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  const __half2 h = __float22half2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v)));
  return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(256) gather_rows_f16(const uint4 *__restrict__ x,
                                                       const int32_t *__restrict__ sorted_token,
                                                       uint4 *__restrict__ xp, int rows_routed,
                                                       int rows_total, int T, int vec_per_row,
                                                       const int32_t *off, Shard sh) {
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) / 32);
  const int lane = threadIdx.x % 32;
  if (row >= rows_total || !row_in_shard(row, rows_routed, T, off, sh)) return;
  const int src = row < rows_routed ? sorted_token[row] : (row - rows_routed) % T;
  const uint4 *s = x + (size_t)src * vec_per_row;
  uint4 *d = xp + (size_t)row * vec_per_row;
  // 8 values per 16-byte vector, two vectors in flight per lane
  int v = lane;
  for (; v + 32 < vec_per_row; v += 64) {
    const uint4 a = __ldg(s + v), b = __ldg(s + v + 32);
    d[v] = make_uint4(bf16x2_to_f16x2(a.x), bf16x2_to_f16x2(a.y), bf16x2_to_f16x2(a.z),
                      bf16x2_to_f16x2(a.w));
    d[v + 32] = make_uint4(bf16x2_to_f16x2(b.x), bf16x2_to_f16x2(b.y), bf16x2_to_f16x2(b.z),
                           bf16x2_to_f16x2(b.w));
  }
  for (; v < vec_per_row; v += 32) {
    const uint4 a = __ldg(s + v);
    d[v] = make_uint4(bf16x2_to_f16x2(a.x), bf16x2_to_f16x2(a.y), bf16x2_to_f16x2(a.z),
                      bf16x2_to_f16x2(a.w));
  }
}

// ------------------------------------------------------- tensor-core GEMMs

namespace tc {

constexpr int BK = 64;                 // K elements per ring stage (128 bytes bf16)
constexpr int BM = 128;                // MMA M per SM: weight rows of one weight tile
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
// warp 0 issues TMA loads, warp 1 MMAs, warps 2 .. 1 + epi_warps(AT) run the
// epilogue; with e4m3 weights the CONV_WARPS warps after them expand the
// weight tiles
#ifndef MOE_TC_CONV_WARPS
#define MOE_TC_CONV_WARPS 8
#endif
constexpr int CONV_WARPS = MOE_TC_CONV_WARPS;
// e4m3 path: the block scales are taken times 2^8 when the codes are expanded
// (keeping scale and products in the fp16 normal range) and the accumulator is
// multiplied by 2^-8 in the epilogue -- both exact powers of two
constexpr float F8_SCALE_UP = 256.0f, F8_SCALE_DOWN = 1.0f / 256.0f;
// epilogue warps: four (one per TMEM lane quarter), or eight when a CTA holds
// two weight tiles (two warps per lane quarter, alternating column chunks)
__host__ __device__ constexpr int epi_warps(int at) { return at == 2 ? 8 : 4; }
__host__ __device__ constexpr int threads_of(bool f8, int at) {
  return 32 * (2 + epi_warps(at) + (f8 ? CONV_WARPS : 0));
}
constexpr int XB_STRIDE = 17;          // exchange buffer row stride (floats)

struct Params {
  const int32_t *tile_start;
  const int32_t *tile_base;
  const int32_t *offsets;
  int E, G, T;
  int KB;           // K blocks of 64
  int I, D;
  int rows_routed;  // T * k
  void *out;        // GEMM1: h [rows, I] bf16; GEMM2: out_perm [T*k, D] fp32
  float *out_shared;
  int32_t *status;
  int64_t timeout_ns;
  // MODE 3 (second GEMM with the weighted scatter into y)
  const int32_t *sorted_token;
  const int32_t *indices;  // [T, k]
  const float *weights;    // [T, k]
  int k;
  float *y;                // [T, D], zeroed before the launch
  // e4m3 weights: fp32 scales of 128 x 128 blocks, [G, rows/128, cols/128]
  const float *sA0, *sA1;  // GEMM1: w1, w3; second GEMM: w2 (sA1 unused)
  // FP8 x FP8 path: the activation rows' scales, one per row
  const float *sX;
  Shard sh;
};

// CG = CTA group: 1 = one SM per tile; 2 = an SM pair per tile (cta_group::2),
// where each CTA holds 128 weight rows and half of the token tile.
// AT = weight tiles of 128 rows per CTA and stage.  AT = 1: one tile (GEMM1:
// 64 rows of w1 over the same 64 rows of w3, so the SwiGLU halves meet in
// different TMEM lanes).  AT = 2: two tiles, each with its own accumulator and
// the same token rows (GEMM1: 128 rows of w1 and the same 128 rows of w3, so a
// thread holds both halves of its features; GEMM2: two blocks of 128 rows of
// w2), which halves the token bytes each weight byte is paired with.
// F8: the weights arrive as e4m3 tiles (A8, 64 bytes per row) that the
// converter warps expand into the bf16 tile the MMA reads.
template <int MODE, int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
struct Layout {
  static constexpr int EPI = epi_warps(AT);
  static constexpr int NT = threads_of(F8, AT);
  static constexpr int B_ROWS = BN_MAX / CG;  // token rows one CTA holds per stage
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int A_ALL = AT * A_BYTES;  // all weight tiles of a stage
  static constexpr int A8_BYTES = F8 ? AT * BM * BK : 0;
  static constexpr int A8_OFF = A_ALL + B_BYTES;  // within a stage
  static constexpr int STAGE_BYTES = A_ALL + B_BYTES + A8_BYTES;
  // TMA parts of a stage's weights: GEMM1 always loads w1 and w3; rows per part
  static constexpr int NPARTS = MODE == 1 ? 2 : AT;
  static constexpr int PART_ROWS = MODE == 1 && AT == 1 ? 64 : BM;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // full, empty, [a8_full, converted], acc_full x2, acc_empty x2, drain,
  // list_full x2, list_empty x2
  static constexpr int NBARS = (F8 ? 4 : 2) * STAGES + 9;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int MISC_BYTES = 16 + 8 * STAGES;
  static constexpr int XBUF_OFF = (MISC_OFF + MISC_BYTES + 127) / 128 * 128;
  // an epilogue warp's token columns are chunks of 32, CSTEP apart
  static constexpr int CSTEP = 32 * (EPI / 4);
  // GEMM1 with AT = 1: SwiGLU exchange buffers; MODE 3: two (token, gate)
  // lists of a tile's columns, used by alternate tiles
  static constexpr int XBUF_BYTES =
      MODE == 1 ? (AT == 1 ? 2 * 2 * 32 * XB_STRIDE * 4 : 0) : MODE == 3 ? 2 * BN_MAX * 8 : 0;
  static constexpr int TAB_OFF = XBUF_OFF + XBUF_BYTES;
  // TMEM: AT accumulators of BN_MAX columns per tile, double-buffered when
  // two tiles' worth fits in the 512 columns
  static constexpr int ACC_COLS = AT * BN_MAX;
  static constexpr int NBUF = 2 * ACC_COLS <= 512 ? 2 : 1;
  static constexpr uint32_t TMEM_COLS =
      NBUF * ACC_COLS <= 32 ? 32 : NBUF * ACC_COLS <= 64 ? 64 : NBUF * ACC_COLS <= 128 ? 128
                                 : NBUF * ACC_COLS <= 256 ? 256 : 512;
  // weight rows one tile covers (per pair): GEMM1 features (each with a row
  // of w1 and of w3), GEMM2 rows of w2
  static constexpr int FEAT = (MODE == 1 ? (AT == 1 ? 64 : BM) : AT * BM) * CG;
  static size_t smem_bytes(int G, int E) {
    return 1024 + TAB_OFF + sizeof(int32_t) * (size_t)((G + 1) + G + (E + 1));
  }
  static_assert(CG == 1 || CG == 2, "CTA group");
  static_assert(AT == 1 || AT == 2, "weight tiles per CTA");
  static_assert(NBUF * ACC_COLS <= 512, "TMEM columns");
  static_assert(BN_MAX % 16 == 0 && BN_MAX >= 16 && BN_MAX <= 256, "MMA N range");
  static_assert(BOXN % 16 == 0 && B_ROWS % BOXN == 0, "B box rows");
};

// silu(a) * u for the tensor-core epilogues, whose h is rounded to bf16 (or
// fp16) right after: the hardware exp2 and reciprocal used here are within a
// few parts in 1e6 of the exact value for the |a| that occur, far inside that
// rounding, at a third of the instructions of the IEEE-exact forms
__device__ __forceinline__ float swiglu_h(float a, float u) {
  return __fdividef(a, 1.0f + __expf(-a)) * u;
}

// L2 priority of the token rows a matmul streams (the expert-ordered x rows
// in the first, h in the second): 0 evict-first, 1 normal, 2 evict-last.
// The rows of an expert are re-read by its feature tiles, which run at about
// the same time, and are dead afterwards.
#ifndef MOE_TOKEN_L2_UP
#define MOE_TOKEN_L2_UP 2
#endif
#ifndef MOE_TOKEN_L2_DOWN
#define MOE_TOKEN_L2_DOWN 2
#endif
__device__ __forceinline__ uint64_t token_policy(bool up) {
  const int k = up ? MOE_TOKEN_L2_UP : MOE_TOKEN_L2_DOWN;
  return k == 0 ? sm100::policy_evict_first()
                : k == 1 ? sm100::policy_evict_normal() : sm100::policy_evict_last();
}

// Waits for a barrier phase with a time limit but ignores the abort flag;
// used only to drain copies already in flight before the CTA exits.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, int64_t limit_ns) {
  const uint64_t t0 = sm100::globaltimer_ns();
  while (!sm100::mbar_try_wait(bar, parity)) {
    if ((int64_t)(sm100::globaltimer_ns() - t0) > limit_ns) break;
  }
}

__device__ __forceinline__ void sleep_ns(int64_t ns) {
  const uint64_t t0 = sm100::globaltimer_ns();
  while ((int64_t)(sm100::globaltimer_ns() - t0) < ns) {
  }
}

// The body of the expert GEMM kernel, over the shared memory `sm` (1024-byte
// aligned).  Warps beyond the variant's roles (in a larger block that runs
// it as one phase) take no part but the block-wide barriers.  A CTA that will
// allocate tensor memory again later (a later phase) passes last_alloc =
// false, so that it keeps its right to allocate.
template <int MODE, int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
__device__ __forceinline__ void gemm_body(const CUtensorMap &tmA0, const CUtensorMap &tmA1,
                                          const CUtensorMap &tmB, const Params &p, uint8_t *sm,
                                          bool last_alloc = true) {
  using L = Layout<MODE, CG, AT, BN_MAX, BOXN, STAGES, F8>;
  using namespace sm100;
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
  uint64_t *empty = full + STAGES;
  uint64_t *a8full = empty + STAGES;                 // F8 only
  uint64_t *conv = a8full + (F8 ? STAGES : 0);       // F8 only
  uint64_t *accf = conv + (F8 ? STAGES : 0);
  uint64_t *acce = accf + 2;
  uint64_t *drain = acce + 2;
  uint64_t *lfull = drain + 1;   // MODE 3: a tile's token list written
  uint64_t *lempty = lfull + 2;  // MODE 3: a tile's token list read
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 4);
  volatile int *pending = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 16);
  volatile int *pend8 = pending + STAGES;  // e4m3 loads in flight (F8)
  float *xbuf = reinterpret_cast<float *>(sm + L::XBUF_OFF);
  int32_t *s_tstart = reinterpret_cast<int32_t *>(sm + L::TAB_OFF);
  int32_t *s_tbase = s_tstart + p.G + 1;
  int32_t *s_off = s_tbase + p.G;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // this CTA's rank in its pair, the tile-unit (pair or CTA) index and count
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int unit = CG == 2 ? (int)cluster_id_x() : (int)blockIdx.x;
  const int nunits = CG == 2 ? (int)cluster_count_x() : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      pending[s] = -1;
      pend8[s] = -1;
      if (F8) {
        mbar_init(a8full + s, 1);
        mbar_init(conv + s, CONV_WARPS * CG);
      }
    }
    mbar_init(accf + 0, 1);
    mbar_init(accf + 1, 1);
    mbar_init(acce + 0, L::EPI * CG);
    mbar_init(acce + 1, L::EPI * CG);
    mbar_init(drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(lfull + b, L::EPI);
      mbar_init(lempty + b, L::EPI);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    if (MODE == 1) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  const int NT = blockDim.x;
  for (int i = threadIdx.x; i <= p.G; i += NT) s_tstart[i] = p.tile_start[i];
  for (int i = threadIdx.x; i < p.G; i += NT) s_tbase[i] = p.tile_base[i];
  for (int i = threadIdx.x; i <= p.E; i += NT) s_off[i] = p.offsets[i];
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
      if (last_alloc) tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, L::TMEM_COLS);
      if (last_alloc) tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // the pair's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tstart[p.G];

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      // weights: kept at normal L2 priority when the expert has more than one
      // token tile, so that its token tiles, which run at about the same time
      // on neighbouring units, share them in L2; in the second matmul an
      // expert with a single token tile loads them evict-first, because the
      // fp32 sums it scatters into y need L2 more
      const uint64_t pol_normal = policy_evict_normal();
      const uint64_t pol_first = MODE == 1 ? pol_normal : policy_evict_first();
      const uint64_t pol_x = token_policy(MODE == 1);  // re-read per feature tile
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += nunits) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        const uint64_t pol_w = t.ntt > 1 ? pol_normal : pol_first;
        const int nmma = (t.nvalid + 15) & ~15;
        const int brows = nmma / CG;  // this CTA's share of the token rows
        const int b0 = t.rowbase + t.n0 + (int)rank * brows;
        // first weight row of this CTA's part 0; part i of GEMM2 lies
        // i * 128 * CG rows further, GEMM1's part 1 is w3 at the same rows
        const int arow = MODE == 1 ? t.wg * p.I + t.ft * L::FEAT + (int)rank * L::PART_ROWS
                                   : t.wg * p.D + t.ft * L::FEAT + (int)rank * BM;
        const int nbox = (brows + BOXN - 1) / BOXN;
        // with e4m3 weights the full barrier counts only the token rows; the
        // weight tile arrives on this CTA's own a8_full barrier
        const uint32_t bytes = (uint32_t)((F8 ? 0 : L::A_ALL) + nbox * BOXN * BK * 2);
        const int k0 = k_rotation(t, p.KB);
        for (int i = 0; i < p.KB; ++i) {
          const int kb = k0 + i < p.KB ? k0 + i : k0 + i - p.KB;
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          // the leader's full barrier counts the bytes of both CTAs
          if (leader) mbar_arrive_expect_tx(full + stage, bytes * CG);
          pending[stage] = (int)phase;
          uint8_t *a_dst = sm + stage * L::STAGE_BYTES;
          uint8_t *b_dst = a_dst + L::A_ALL;
          if (F8) {
            uint8_t *a8 = a_dst + L::A8_OFF;
            mbar_arrive_expect_tx(a8full + stage, L::A8_BYTES);
            pend8[stage] = (int)phase;
#pragma unroll
            for (int i = 0; i < L::NPARTS; ++i)
              tma_load_2d_hint(MODE == 1 && i == 1 ? &tmA1 : &tmA0,
                               a8 + i * (L::A8_BYTES / L::NPARTS), a8full + stage, kb * BK,
                               arow + (MODE == 1 ? 0 : i * BM * CG), pol_w);
            if (CG == 2) {
              const uint32_t fb = mapa_shared(smem_u32(full + stage), 0);
              for (int i = 0; i < nbox; ++i)
                tma_load_2d_pair(&tmB, b_dst + i * BOXN * BK * 2, fb, kb * BK, b0 + i * BOXN, pol_x);
            } else {
              for (int i = 0; i < nbox; ++i)
                tma_load_2d_hint(&tmB, b_dst + i * BOXN * BK * 2, full + stage, kb * BK,
                                 b0 + i * BOXN, pol_x);
            }
          } else if (CG == 2) {
            const uint32_t fb = mapa_shared(smem_u32(full + stage), 0);
#pragma unroll
            for (int i = 0; i < L::NPARTS; ++i)
              tma_load_2d_pair(MODE == 1 && i == 1 ? &tmA1 : &tmA0,
                               a_dst + i * (L::A_ALL / L::NPARTS), fb, kb * BK,
                               arow + (MODE == 1 ? 0 : i * BM * CG), pol_w);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d_pair(&tmB, b_dst + i * BOXN * BK * 2, fb, kb * BK, b0 + i * BOXN, pol_x);
          } else {
#pragma unroll
            for (int i = 0; i < L::NPARTS; ++i)
              tma_load_2d_hint(MODE == 1 && i == 1 ? &tmA1 : &tmA0,
                               a_dst + i * (L::A_ALL / L::NPARTS), full + stage, kb * BK,
                               arow + (MODE == 1 ? 0 : i * BM * CG), pol_w);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d_hint(&tmB, b_dst + i * BOXN * BK * 2, full + stage, kb * BK,
                               b0 + i * BOXN, pol_x);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------ MMA issuer
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += nunits) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        if (!wait_bounded(acce + acc, acc_phase ^ 1u, abort_flag, p.timeout_ns, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * L::ACC_COLS);
        const int nmma = (t.nvalid + 15) & ~15;
        const uint32_t idesc = F8 ? idesc_f16_f32(BM * CG, nmma) : idesc_bf16_f32(BM * CG, nmma);
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!wait_bounded(full + stage, phase, abort_flag, p.timeout_ns, p.status) ||
              (F8 && !wait_bounded(conv + stage, phase, abort_flag, p.timeout_ns, p.status))) {
            ok = false;
            break;
          }
          pending[stage] = -1;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm + stage * L::STAGE_BYTES);
          const uint32_t b_addr = a_addr + L::A_ALL;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(b_addr + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
#pragma unroll
            for (int a = 0; a < AT; ++a) {
              const uint64_t ad = sdesc_sw128(a_addr + a * A_BYTES + kk * 32);
              if (CG == 2)
                mma_bf16_pair(d_tmem + a * BN_MAX, ad, bd, idesc, accum);
              else
                mma_bf16(d_tmem + a * BN_MAX, ad, bd, idesc, accum);
            }
          }
          if (CG == 2)
            mma_commit_pair_mc(empty + stage, 0x3);
          else
            mma_commit(empty + stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 2)
          mma_commit_pair_mc(accf + acc, 0x3);
        else
          mma_commit(accf + acc);
        if (++acc == L::NBUF) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        // make sure no MMA is still writing TMEM before it is freed
        if (CG == 2)
          mma_commit_pair(drain);
        else
          mma_commit(drain);
        drain_wait(drain, 0, p.timeout_ns);
      }
    }
  } else if (warp >= 2 + L::EPI) {
    if (F8) {
      // ------------------------------------------------ e4m3 -> f16 converter
      // A8 row r (64 codes) becomes A row r (64 fp16) in the 128-byte swizzled
      // layout: 16-byte chunk c of row r lands at chunk c ^ (r % 8).  A code
      // converts to fp16 exactly; it is then multiplied by 2^8 times the fp32
      // scale of its 128 x 128 block (rounded once to fp16).  On this path
      // the token rows and h are fp16 as well.
      const int ct = threadIdx.x - 32 * (2 + L::EPI);  // 0 .. 32 * CONV_WARPS - 1
      const int rows_w = MODE == 1 ? p.I : p.D;            // rows of one expert's matrix
      const int cols_w = MODE == 1 ? p.D : p.I;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += nunits) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        // scale rows of part 0 and part 1 (GEMM1: w1 and w3 at the same
        // rows; GEMM2 with two parts: 128 * CG rows apart)
        const int r0 = t.ft * L::FEAT + (int)rank * L::PART_ROWS;
        const size_t srow = ((size_t)t.wg * (rows_w / 128) + r0 / 128) * (cols_w / 128);
        const size_t srow1 =
            MODE != 1 && AT == 2 ? srow + (size_t)CG * (cols_w / 128) : srow;
        const float *sc1 = MODE == 1 ? p.sA1 : p.sA0;
        const int k0 = k_rotation(t, p.KB);
        // the block scales of the next k-block are loaded while this one's
        // codes are awaited and expanded, keeping their latency off the path
        float n0 = p.sA0[srow + k0 / 2], n1 = L::NPARTS == 2 ? sc1[srow1 + k0 / 2] : 0.0f;
        for (int i = 0; i < p.KB; ++i) {
          const int kn = k0 + i + 1 < p.KB ? k0 + i + 1 : k0 + i + 1 - p.KB;
          const float c0 = n0, c1 = n1;
          if (i + 1 < p.KB) {
            n0 = p.sA0[srow + kn / 2];
            if (L::NPARTS == 2) n1 = sc1[srow1 + kn / 2];
          }
          if (!wait_bounded(a8full + stage, phase, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          pend8[stage] = -1;
          const uint32_t s0 = f16x2_splat(c0 * F8_SCALE_UP);
          const uint32_t s1 = L::NPARTS == 2 ? f16x2_splat(c1 * F8_SCALE_UP) : s0;
          const uint8_t *a8 = sm + stage * L::STAGE_BYTES + L::A8_OFF;
          uint8_t *a16 = sm + stage * L::STAGE_BYTES;
          if (AT == 2) {
            // two weight tiles per stage: each step turns 16 codes (one
            // 16-byte load) into two 16-byte chunks (2c, 2c + 1) of the row
#pragma unroll
            for (int it = 0; it < AT * BM * 4 / (32 * CONV_WARPS); ++it) {
              const int idx = ct + it * 32 * CONV_WARPS;
              const int r = idx >> 2, c = idx & 3;  // rows of all parts lie back to back
              const uint32_t sc = r >= L::PART_ROWS ? s1 : s0;
              const uint4 q = *reinterpret_cast<const uint4 *>(a8 + r * 64 + c * 16);
              uint4 o0, o1;
              o0.x = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.x & 0xffffu)), sc);
              o0.y = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.x >> 16)), sc);
              o0.z = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.y & 0xffffu)), sc);
              o0.w = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.y >> 16)), sc);
              o1.x = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.z & 0xffffu)), sc);
              o1.y = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.z >> 16)), sc);
              o1.z = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.w & 0xffffu)), sc);
              o1.w = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.w >> 16)), sc);
              *reinterpret_cast<uint4 *>(a16 + r * 128 + (((2 * c) ^ (r & 7)) << 4)) = o0;
              *reinterpret_cast<uint4 *>(a16 + r * 128 + (((2 * c + 1) ^ (r & 7)) << 4)) = o1;
            }
          } else {
            // one tile: 8 codes (one 8-byte load) per 16-byte chunk c
#pragma unroll 4
            for (int it = 0; it < AT * BM * 8 / (32 * CONV_WARPS); ++it) {
              const int idx = ct + it * 32 * CONV_WARPS;
              const int r = idx >> 3, c = idx & 7;
              const uint32_t sc = r >= L::PART_ROWS ? s1 : s0;
              const uint2 q = *reinterpret_cast<const uint2 *>(a8 + r * 64 + c * 8);
              uint4 o;
              o.x = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.x & 0xffffu)), sc);
              o.y = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.x >> 16)), sc);
              o.z = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.y & 0xffffu)), sc);
              o.w = f16x2_mul(e4m3x2_to_f16x2((uint16_t)(q.y >> 16)), sc);
              *reinterpret_cast<uint4 *>(a16 + r * 128 + ((c ^ (r & 7)) << 4)) = o;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (CG == 2)
              mbar_arrive_cluster(mapa_shared(smem_u32(conv + stage), 0));  // the leader's barrier
            else
              mbar_arrive(conv + stage);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    // with eight epilogue warps, the two warps of a lane quarter take
    // alternate 32-column chunks
    const int half = (warp - 2) >> 2;
    constexpr int CSTEP = L::CSTEP;
    const float acc_scale = F8 ? F8_SCALE_DOWN : 1.0f;
    int acc = 0;
    uint32_t acc_phase = 0;
    // MODE 3: the tile's token and gate of each column (gate 1 for the shared
    // expert), in one of two lists that alternate between tiles; every
    // epilogue warp writes a share of it before waiting for the accumulator
    // and reads all of it in the stores
    int32_t *s_tok = nullptr;
    float *s_gate = nullptr;
    int ntile = 0;
    for (int tile = unit; tile < total; tile += nunits, ++ntile) {
      const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
      if (MODE == 3) {
        const int lb = ntile & 1;
        const uint32_t lph = (uint32_t)(ntile >> 1) & 1u;
        s_tok = reinterpret_cast<int32_t *>(xbuf) + lb * 2 * BN_MAX;
        s_gate = reinterpret_cast<float *>(s_tok + BN_MAX);
        // the list's previous tile has been read by every epilogue warp
        if (!wait_bounded(lempty + lb, lph ^ 1u, abort_flag, p.timeout_ns, p.status)) break;
        // this warp's columns, all loads issued together
        constexpr int PER = (BN_MAX + 32 * L::EPI - 1) / (32 * L::EPI);
        int tok[PER], pos[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = ((warp - 2) + i * L::EPI) * 32 + lane;
          tok[i] = c >= t.nvalid ? -1 : t.g < p.E ? p.sorted_token[t.rowbase + t.n0 + c] : t.tok0 + c;
          pos[i] = -1;
        }
        if (t.g < p.E) {
          for (int jj = 0; jj < p.k; ++jj)
#pragma unroll
            for (int i = 0; i < PER; ++i)
              if (tok[i] >= 0 && p.indices[(size_t)tok[i] * p.k + jj] == t.g) pos[i] = jj;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = ((warp - 2) + i * L::EPI) * 32 + lane;
          if (tok[i] >= 0) {
            s_tok[c] = tok[i];
            s_gate[c] = pos[i] >= 0 ? p.weights[(size_t)tok[i] * p.k + pos[i]] : 1.0f;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(lfull + lb);
        if (!wait_bounded(lfull + lb, lph, abort_flag, p.timeout_ns, p.status)) break;
      }
      if (!wait_bounded(accf + acc, acc_phase, abort_flag, p.timeout_ns, p.status)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * L::ACC_COLS);
      // hands the accumulator back to the MMA once this warp has read it
      bool released = false;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2)
            mbar_arrive_cluster(mapa_shared(smem_u32(acce + acc), 0));  // the leader's barrier
          else
            mbar_arrive(acce + acc);
        }
        released = true;
      };
      if (MODE == 2 || MODE == 3) {
        // lanes are output features d, columns are tokens; MODE 3 adds
        // gate * o into y with fp32 reductions, MODE 2 writes per-slot rows
        float *out = nullptr;
        size_t row0 = 0;
        if (MODE == 2 && t.g < p.E) {
          out = static_cast<float *>(p.out);
          row0 = (size_t)t.rowbase + t.n0;
        } else if (MODE == 2) {
          out = p.out_shared;
          row0 = (size_t)(t.g - p.E) * p.T + t.tok0;
        }
        // the 32 columns from c0 of accumulator a, read into v
        auto store = [&](int a, int c0, const uint32_t *v) {
          const int d = t.ft * L::FEAT + a * BM * CG + (int)rank * BM + q * 32 + lane;
          if (MODE == 3) {
            // 16-byte fp32 reductions: a lane holds one d for 32 tokens, so
            // each quad of lanes transposes its 4 x 4 blocks (4 d by 4
            // tokens) in two shuffle rounds and lane t of a quad adds 4
            // consecutive d of token 4u + t -- a quarter of the reductions
            const int t4 = lane & 3, hi = t4 >> 1, lo = t4 & 1;
            float *yq = p.y + (d - (lane & 3));
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              // M[r][s]: d of lane (lane & ~3) + r, token c0 + 4u + s
              const float m0 = s_gate[c0 + 4 * u + 0] * (__uint_as_float(v[4 * u + 0]) * acc_scale);
              const float m1 = s_gate[c0 + 4 * u + 1] * (__uint_as_float(v[4 * u + 1]) * acc_scale);
              const float m2 = s_gate[c0 + 4 * u + 2] * (__uint_as_float(v[4 * u + 2]) * acc_scale);
              const float m3 = s_gate[c0 + 4 * u + 3] * (__uint_as_float(v[4 * u + 3]) * acc_scale);
              const float y0 = __shfl_xor_sync(0xffffffffu, hi ? m0 : m2, 2);
              const float y1 = __shfl_xor_sync(0xffffffffu, hi ? m1 : m3, 2);
              const float b0 = hi ? y0 : m0, b1 = hi ? y1 : m1;
              const float b2 = hi ? m2 : y0, b3 = hi ? m3 : y1;
              const float z0 = __shfl_xor_sync(0xffffffffu, lo ? b0 : b1, 1);
              const float z1 = __shfl_xor_sync(0xffffffffu, lo ? b2 : b3, 1);
              const float o0 = lo ? b1 : b0, o1 = lo ? b3 : b2;
              const int c = c0 + 4 * u + t4;
              if (c < t.nvalid)
                red_add_v4_f32(yq + (size_t)s_tok[c] * p.D, lo ? z0 : o0, lo ? o0 : z0,
                               lo ? z1 : o1, lo ? o1 : z1);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < t.nvalid) out[(row0 + c0 + j) * p.D + d] = __uint_as_float(v[j]) * acc_scale;
          }
        };
        if (L::NBUF == 1) {
          // single-buffered accumulator: this warp's chunks are read in
          // batches of up to NB (32 registers each) and the accumulator goes
          // back to the MMA right after the last batch's reads, so that the
          // stores of that batch overlap the next tile's MMAs
          constexpr int NB = F8 ? 2 : 4;  // the converter warps leave fewer registers
          const int nch = t.nvalid > half * 32 ? (t.nvalid - half * 32 + CSTEP - 1) / CSTEP : 0;
          const int nall = AT * nch;
          for (int b0 = 0; b0 < nall; b0 += NB) {
            uint32_t v[NB][32];
#pragma unroll
            for (int u = 0; u < NB; ++u)
              if (b0 + u < nall) {
                const int a = (b0 + u) / nch, c0 = half * 32 + ((b0 + u) % nch) * CSTEP;
                tmem_ld_32x32b_x32(tb + (uint32_t)(a * BN_MAX + c0), v[u]);
              }
            tmem_wait_ld();
            if (b0 + NB >= nall) release();
#pragma unroll
            for (int u = 0; u < NB; ++u)
              if (b0 + u < nall) store((b0 + u) / nch, half * 32 + ((b0 + u) % nch) * CSTEP, v[u]);
          }
        } else {
#pragma unroll
          for (int a = 0; a < AT; ++a)
            for (int c0 = half * 32; c0 < t.nvalid; c0 += CSTEP) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(tb + (uint32_t)(a * BN_MAX + c0), v);
              tmem_wait_ld();
              store(a, c0, v);
            }
        }
      } else if (AT == 2) {
        // lanes are features; the w1.x accumulator (a) and the w3.x one (u)
        // sit BN_MAX columns apart in the same lanes
        // the accumulator is single-buffered here, so each warp releases it
        // right after its last TMEM read, before that chunk's arithmetic
        const int f = t.ft * L::FEAT + (int)rank * BM + q * 32 + lane;
        const size_t row0 = (size_t)t.rowbase + t.n0;
        for (int c0 = half * 32; c0 < t.nvalid; c0 += CSTEP) {
          uint32_t va[32], vu[32];
          tmem_ld_32x32b_x32(tb + (uint32_t)c0, va);
          tmem_ld_32x32b_x32(tb + (uint32_t)(BN_MAX + c0), vu);
          tmem_wait_ld();
          if (c0 + CSTEP >= t.nvalid) release();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float h = swiglu_h(__uint_as_float(va[j]) * acc_scale,
                                     __uint_as_float(vu[j]) * acc_scale);
            if (c0 + j < t.nvalid) {
              if (F8)  // fp16 h: the second matmul's operand on the e4m3 path
                reinterpret_cast<__half *>(p.out)[(row0 + c0 + j) * p.I + f] = __float2half_rn(h);
              else
                static_cast<bf16 *>(p.out)[(row0 + c0 + j) * p.I + f] = __float2bfloat16_rn(h);
            }
          }
        }
      } else {
        // lanes 0-63 hold w1.x (a), lanes 64-127 hold w3.x (u) for the same
        // 64 features; warps q and q+2 pair up through shared memory, each
        // finishing half of the 32 columns of a chunk
        const int pr = q & 1;
        const bool is_a = q < 2;
        float *buf_a = xbuf + pr * 2 * 32 * XB_STRIDE;  // a, columns 16-31 of the chunk
        float *buf_u = buf_a + 32 * XB_STRIDE;          // u, columns 0-15 of the chunk
        bf16 *out = static_cast<bf16 *>(p.out);
        const int f = t.ft * L::FEAT + (int)rank * 64 + pr * 32 + lane;
        const size_t row0 = (size_t)t.rowbase + t.n0;
        for (int c0 = 0; c0 < t.nvalid; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tb + (uint32_t)c0, v);
          tmem_wait_ld();
          float *mine = is_a ? buf_a : buf_u;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            mine[lane * XB_STRIDE + j] = __uint_as_float(is_a ? v[16 + j] : v[j]);
          named_bar_sync(1 + pr, 64);
          const float *other = is_a ? buf_u : buf_a;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = is_a ? j : 16 + j;
            const float a = (is_a ? __uint_as_float(v[j]) : other[lane * XB_STRIDE + j]) * acc_scale;
            const float u = (is_a ? other[lane * XB_STRIDE + j] : __uint_as_float(v[16 + j])) * acc_scale;
            const float h = swiglu_h(a, u);
            if (c0 + col < t.nvalid) {
              if (F8)  // fp16 h: the second matmul's operand on the e4m3 path
                reinterpret_cast<__half *>(out)[(row0 + c0 + col) * p.I + f] = __float2half_rn(h);
              else
                out[(row0 + c0 + col) * p.I + f] = __float2bfloat16_rn(h);
            }
          }
          named_bar_sync(1 + pr, 64);
        }
      }
      if (!released) release();
      if (MODE == 3) {
        __syncwarp();  // this warp's reads of the list are done
        if (lane == 0) mbar_arrive(lempty + (ntile & 1));
      }
      if (++acc == L::NBUF) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // a stalled pipeline stopped early: let copies already issued land.  The
    // leader's full barriers count both CTAs' copies; the other CTA of a pair
    // cannot wait on them and just allows its copies time to land.
    if (F8)  // the e4m3 tiles land on this CTA's own barriers
      for (int s = 0; s < STAGES; ++s)
        if (pend8[s] >= 0) drain_wait(a8full + s, (uint32_t)pend8[s], p.timeout_ns);
    if (leader) {
      for (int s = 0; s < STAGES; ++s)
        if (pending[s] >= 0) drain_wait(full + s, (uint32_t)pending[s], p.timeout_ns);
    } else {
      sleep_ns(200000);
    }
  }
  __syncthreads();
  if (CG == 2) cluster_sync();  // neither CTA leaves while the other may touch its memory
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

template <int MODE, int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
__global__ void __launch_bounds__(threads_of(F8, AT), 1)
    tc_expert_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  gemm_body<MODE, CG, AT, BN_MAX, BOXN, STAGES, F8>(tmA0, tmA1, tmB, p, sm);
}

// single-CTA self-test of the bounded wait: nothing ever arrives
__global__ void selftest_wait_kernel(int64_t limit_ns, int32_t *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = sm100::wait_bounded(&bar, 0, &abort_flag, limit_ns, status);
    (void)ok;
  }
}

}  // namespace tc

// ------------------------------------------------ FP8 x FP8 (e4m3 activations)
//
// The optional path for e4m3 weights on which the activations are quantised
// to e4m3 as well, so that the matmuls run as e4m3 x e4m3 tensor-core MMAs
// (kind::f8f6f4, twice the bf16 rate).  The weights carry fp32 scales per
// 128 x 128 block, the activation rows one fp32 scale per row.  A k-block of
// 128 is one 128-byte swizzle row of e4m3, so every k-block's partial sum is
// scaled by one weight scale per CTA (its 128 weight rows lie in one scale
// block), and the token's scale factors out of the whole sum:
//   acc[m, n] = s_x[n] * sum_kb  s_w[kb] * (sum_{k in kb} q_w[m, k] q_x[n, k])
// The MMAs of a k-block write a fresh TMEM partial (two buffers alternate)
// and eight promotion warps fold it into fp32 running sums in registers with
// one warp-uniform scale; s_x is applied once per tile.

// Rows of a bf16 matrix [*, K] quantised to e4m3 with one scale per row:
// scale = amax / 448 (IEEE division), r = 1 / scale (IEEE reciprocal),
// code = e4m3(v * r), rounded to nearest even and saturated; an all-zero row
// has scale 0 and codes 0.  With GATHER, output row p < rows_routed is token
// sorted_token[p] and row rows_routed + t is token t (the shared expert's
// rows); otherwise row p is source row p.  Codes go to q [rows, K]
// row-major, scales to sc [rows].  One warp per row: a pass for the row's
// amax, a second (from L1/L2) for the codes, four values per lane and step.
template <bool GATHER>
__global__ void __launch_bounds__(256) quant_rows_e4m3(const uint2 *__restrict__ src,
                                                       const int32_t *__restrict__ sorted_token,
                                                       uint32_t *__restrict__ q,
                                                       float *__restrict__ sc, int rows_routed,
                                                       int rows_total, int T, int K,
                                                       const int32_t *off, Shard sh) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows_total) return;
  if (!row_in_shard(row, rows_routed, T, off, sh)) return;
  const int srow = !GATHER ? row : row < rows_routed ? sorted_token[row] : row - rows_routed;
  const uint2 *s = src + (size_t)srow * (K / 4);
  uint32_t *d = q + (size_t)row * (K / 4);
  const int n4 = K / 4;  // groups of four values in the row
  float m = 0.0f;
  for (int i = lane; i < n4; i += 32) {
    const uint2 v = __ldg(s + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(v.x << 16)), fabsf(__uint_as_float(v.x & 0xffff0000u))),
                       fmaxf(fabsf(__uint_as_float(v.y << 16)), fabsf(__uint_as_float(v.y & 0xffff0000u)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float scale = m / 448.0f;
  const float r = scale > 0.0f ? __frcp_rn(scale) : 0.0f;
  for (int i = lane; i < n4; i += 32) {
    uint32_t packed = 0;
    if (scale > 0.0f) {
      const uint2 v = __ldg(s + i);
      const float f0 = __uint_as_float(v.x << 16), f1 = __uint_as_float(v.x & 0xffff0000u);
      const float f2 = __uint_as_float(v.y << 16), f3 = __uint_as_float(v.y & 0xffff0000u);
      packed = (uint32_t)sm100::f32x2_to_e4m3x2(__fmul_rn(f0, r), __fmul_rn(f1, r)) |
               ((uint32_t)sm100::f32x2_to_e4m3x2(__fmul_rn(f2, r), __fmul_rn(f3, r)) << 16);
    }
    d[i] = packed;
  }
  if (lane == 0) sc[row] = scale;
}

// The same quantiser for K % 8 == 0 with 16-byte rows (8 values per lane and
// step, 8 codes per store): a row of up to 2048 values is read once into
// registers and quantised from there; longer rows take the two passes, four
// 16-byte loads in flight per lane.  Same arithmetic, bit for bit.
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float amax8(const uint4 &v) {
  return fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))),
                     fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))),
               fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))),
                     fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
}
__device__ __forceinline__ uint2 codes8(const uint4 &v, float r) {
  auto c2 = [&](uint32_t w) {
    return (uint32_t)sm100::f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w), r), __fmul_rn(bf16_hi(w), r));
  };
  return make_uint2(c2(v.x) | (c2(v.y) << 16), c2(v.z) | (c2(v.w) << 16));
}

template <bool GATHER>
__global__ void __launch_bounds__(256) quant_rows_e4m3_v8(const uint4 *__restrict__ src,
                                                          const int32_t *__restrict__ sorted_token,
                                                          uint2 *__restrict__ q,
                                                          float *__restrict__ sc, int rows_routed,
                                                          int rows_total, int T, int K,
                                                          const int32_t *off, Shard sh) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows_total) return;
  if (!row_in_shard(row, rows_routed, T, off, sh)) return;
  const int srow = !GATHER ? row : row < rows_routed ? sorted_token[row] : row - rows_routed;
  const uint4 *s = src + (size_t)srow * (K / 8);
  uint2 *d = q + (size_t)row * (K / 8);
  const int n8 = K / 8;  // groups of eight values in the row
  float m = 0.0f;
  if (n8 <= 32 * 8) {
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < n8) v[j] = __ldg(s + lane + 32 * j);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < n8) m = fmaxf(m, amax8(v[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float scale = m / 448.0f;
    const float r = scale > 0.0f ? __frcp_rn(scale) : 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < n8) d[lane + 32 * j] = scale > 0.0f ? codes8(v[j], r) : make_uint2(0, 0);
    if (lane == 0) sc[row] = scale;
    return;
  }
  int i = lane;
  for (; i + 96 < n8; i += 128) {
    const uint4 a = __ldg(s + i), b = __ldg(s + i + 32), c = __ldg(s + i + 64), e = __ldg(s + i + 96);
    m = fmaxf(m, fmaxf(fmaxf(amax8(a), amax8(b)), fmaxf(amax8(c), amax8(e))));
  }
  for (; i < n8; i += 32) m = fmaxf(m, amax8(__ldg(s + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float scale = m / 448.0f;
  const float r = scale > 0.0f ? __frcp_rn(scale) : 0.0f;
  i = lane;
  for (; i + 96 < n8; i += 128) {
    const uint4 a = __ldg(s + i), b = __ldg(s + i + 32), c = __ldg(s + i + 64), e = __ldg(s + i + 96);
    d[i] = scale > 0.0f ? codes8(a, r) : make_uint2(0, 0);
    d[i + 32] = scale > 0.0f ? codes8(b, r) : make_uint2(0, 0);
    d[i + 64] = scale > 0.0f ? codes8(c, r) : make_uint2(0, 0);
    d[i + 96] = scale > 0.0f ? codes8(e, r) : make_uint2(0, 0);
  }
  for (; i < n8; i += 32) d[i] = scale > 0.0f ? codes8(__ldg(s + i), r) : make_uint2(0, 0);
  if (lane == 0) sc[row] = scale;
}

namespace f8 {

using tc::drain_wait;
using tc::sleep_ns;
using tc::swiglu_h;
using tc::token_policy;

constexpr int BK = 128;                // K per stage: one 128-byte swizzle row of e4m3
constexpr int BM = 128;                // weight rows per CTA
constexpr int BN_MAX = 256;            // token rows per tile (per SM pair)
constexpr int BOXN = 32;               // token rows per TMA box
constexpr int EPI = 8;                 // promotion / epilogue warps (two per TMEM lane quarter)
// warpgroup 0: warp 0 TMA, warp 1 MMA, warps 2-3 idle; warpgroups 1-2: the
// promotion / epilogue warps.  A thread's registers are split unevenly with
// setmaxnreg: the block launches with REG_LAUNCH per thread (the most that
// three warps per SM sub-partition allow), warpgroup 0 gives all but
// REG_LOW back and the two epilogue warpgroups take REG_HIGH, which holds
// their fp32 running sums (128 per thread) without spilling.  The shares
// add up to the launch's total: 4 * 56 + 8 * 224 = 12 * 168 (per warp, x32).
constexpr int EPI0 = 4;                // first epilogue warp
constexpr int NT = 32 * (EPI0 + EPI);
constexpr int REG_LAUNCH = 168, REG_LOW = 56, REG_HIGH = 224;
static_assert(4 * REG_LOW + EPI * REG_HIGH == (NT / 32) * REG_LAUNCH, "register split");
constexpr int A_BYTES = BM * BK;       // 16 KB
constexpr int B_ROWS = BN_MAX / 2;     // token rows one CTA holds
constexpr int B_BYTES = B_ROWS * BK;   // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NPBUF = 2;               // TMEM partial-sum buffers of BN_MAX columns
constexpr int CHUNKS = BN_MAX / 32 / 2;  // 32-column chunks per promotion warp
constexpr int XB_STRIDE = 17;
// chunks 0 .. SCH-1 of each promotion warp's sums (token columns 0-127 of a
// tile) are handed to the two helper warps through shared memory, which
// finish them while the next tile's k-loop runs: the SwiGLU and h in the
// first matmul, the reductions into y in the second with the scatter
constexpr int SCH = 2;
__host__ __device__ constexpr bool staged(int mode) { return mode == 1 || mode == 3; }
template <int MODE, int STAGES>
struct Layout {
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // full, empty per stage; partial full, partial empty per buffer; drain;
  // list full, list empty per token list; staged sums full, empty
  static constexpr int NBARS = 2 * STAGES + 2 * NPBUF + 1 + 4 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int MISC_BYTES = 16 + 4 * STAGES;  // TMEM slot, abort flag, pending loads
  static constexpr int SC_OFF = (MISC_OFF + MISC_BYTES + 127) / 128 * 128;
  static constexpr int SC_BYTES = EPI * CHUNKS * 32 * 4;  // the tile's token scales, per warp
  static constexpr int XBUF_OFF = SC_OFF + SC_BYTES;
  // SwiGLU exchange of the four warp pairs (first matmul), or two (token,
  // gate) lists used by alternate tiles (second matmul with the scatter)
  static constexpr int XBUF_BYTES = MODE == 1 ? 4 * 2 * 32 * XB_STRIDE * 4 : 2 * BN_MAX * 8;
  // staged sums (scatter): [promotion warp][chunk < SCH][token column][d]
  static constexpr int STG_OFF = XBUF_OFF + XBUF_BYTES;
  static constexpr int STG_BYTES = staged(MODE) ? EPI * SCH * 32 * 32 * 4 : 0;
  static constexpr int TAB_OFF = STG_OFF + STG_BYTES;
  static size_t smem_bytes(int G, int E) {
    return 1024 + TAB_OFF + sizeof(int32_t) * (size_t)((G + 1) + G + (E + 1));
  }
  static_assert(2 * BN_MAX * 8 <= XBUF_BYTES, "token lists");
  static_assert(NPBUF * BN_MAX <= 512, "TMEM columns");
  static_assert(SCH <= CHUNKS, "staged chunks");
};

// MODE 1: h = silu(x w1^T) * (x w3^T), bf16 out (the pair's 256 weight rows
// per tile are 64 rows of w1 over the same 64 rows of w3 in each CTA: 128
// features).  MODE 2: o = h w2^T, fp32 per-slot outputs.  MODE 3: gate * o
// added into y.  Warp 0 issues TMA loads, one thread of warp 1 the MMAs,
// warps 2-9 promote the partial sums and run the epilogue.
template <int MODE, int STAGES>
__global__ void __launch_bounds__(NT, 1)
    tc_fp8_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB, const tc::Params p) {
  using L = Layout<MODE, STAGES>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + L::BAR_OFF);
  uint64_t *empty = full + STAGES;
  uint64_t *pfull = empty + STAGES;
  uint64_t *pempty = pfull + NPBUF;
  uint64_t *drain = pempty + NPBUF;
  uint64_t *lfull = drain + 1;   // MODE 3: a tile's token list written
  uint64_t *lempty = lfull + 2;  // MODE 3: a tile's token list read
  uint64_t *sfull = lempty + 2;  // MODES 1, 3: a tile's staged sums written
  uint64_t *sempty = sfull + 1;  // MODES 1, 3: the staged sums finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC_OFF);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 4);
  volatile int *pending = reinterpret_cast<volatile int *>(sm + L::MISC_OFF + 16);
  float *s_comb = reinterpret_cast<float *>(sm + L::SC_OFF);
  float *xbuf = reinterpret_cast<float *>(sm + L::XBUF_OFF);
  int32_t *s_tstart = reinterpret_cast<int32_t *>(sm + L::TAB_OFF);
  int32_t *s_tbase = s_tstart + p.G + 1;
  int32_t *s_off = s_tbase + p.G;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int unit = (int)cluster_id_x();
  const int nunits = (int)cluster_count_x();
  const int KB = p.KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      pending[s] = -1;
    }
    for (int b = 0; b < NPBUF; ++b) {
      mbar_init(pfull + b, 1);
      mbar_init(pempty + b, EPI * 2);
    }
    mbar_init(drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(lfull + b, 2);          // the two helper warps
      mbar_init(lempty + b, EPI + 2);   // the epilogue and helper warps
    }
    mbar_init(sfull, EPI);
    mbar_init(sempty, 2);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    if (MODE == 1) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  for (int i = threadIdx.x; i <= p.G; i += NT) s_tstart[i] = p.tile_start[i];
  for (int i = threadIdx.x; i < p.G; i += NT) s_tbase[i] = p.tile_base[i];
  for (int i = threadIdx.x; i <= p.E; i += NT) s_off[i] = p.offsets[i];
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tstart[p.G];

  if (warp < EPI0) {
    // warpgroup 0 as a whole gives registers back, then splits into roles
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_LOW));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------- TMA producer
      // weights at normal L2 priority when their expert has several token
      // tiles (which then share them in L2), else evict-first in the second
      // matmul, whose scattered fp32 sums need L2 more; token rows evict-last
      const uint64_t pol_normal = policy_evict_normal();
      const uint64_t pol_first = MODE == 1 ? pol_normal : policy_evict_first();
      const uint64_t pol_x = token_policy(MODE == 1);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += nunits) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        const uint64_t pol_w = t.ntt > 1 ? pol_normal : pol_first;
        const int nmma = (t.nvalid + 15) & ~15;
        const int brows = nmma / 2;
        const int b0 = t.rowbase + t.n0 + (int)rank * brows;
        const int arow = MODE == 1 ? t.wg * p.I + t.ft * 128 + (int)rank * 64
                                   : t.wg * p.D + t.ft * 256 + (int)rank * BM;
        const int nbox = (brows + BOXN - 1) / BOXN;
        const uint32_t bytes = (uint32_t)(A_BYTES + nbox * BOXN * BK);
        const int k0 = k_rotation(t, KB);
        for (int i = 0; i < KB; ++i) {
          const int kb = k0 + i < KB ? k0 + i : k0 + i - KB;
          if (!wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          // the leader's full barrier counts the bytes of both CTAs
          if (leader) mbar_arrive_expect_tx(full + stage, bytes * 2);
          pending[stage] = (int)phase;
          uint8_t *a_dst = sm + stage * STAGE_BYTES;
          uint8_t *b_dst = a_dst + A_BYTES;
          const uint32_t fb = mapa_shared(smem_u32(full + stage), 0);
          if (MODE == 1) {
            tma_load_2d_pair(&tmA0, a_dst, fb, kb * BK, arow, pol_w);
            tma_load_2d_pair(&tmA1, a_dst + A_BYTES / 2, fb, kb * BK, arow, pol_w);
          } else {
            tma_load_2d_pair(&tmA0, a_dst, fb, kb * BK, arow, pol_w);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(&tmB, b_dst + b * BOXN * BK, fb, kb * BK, b0 + b * BOXN, pol_x);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    } else if (warp == 1 && lane == 0 && leader) {
      // ------------------------------------------------------ MMA issuer
      int stage = 0, pb = 0;
      uint32_t phase = 0, pphase = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += nunits) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        const int nmma = (t.nvalid + 15) & ~15;
        const uint32_t idesc = idesc_e4m3_f32(2 * BM, nmma);
        for (int i = 0; i < KB; ++i) {
          if (!wait_bounded(pempty + pb, pphase ^ 1u, abort_flag, p.timeout_ns, p.status) ||
              !wait_bounded(full + stage, phase, abort_flag, p.timeout_ns, p.status)) {
            ok = false;
            break;
          }
          pending[stage] = -1;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
          const uint32_t d_tmem = tmem_base + (uint32_t)(pb * BN_MAX);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_f8_pair(d_tmem, sdesc_sw128(a_addr + kk * 32), sdesc_sw128(b_addr + kk * 32), idesc,
                        kk != 0 ? 1u : 0u);
          mma_commit_pair_mc(empty + stage, 0x3);
          mma_commit_pair_mc(pfull + pb, 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++pb == NPBUF) {
            pb = 0;
            pphase ^= 1u;
          }
        }
      }
      if (!ok) {
        // make sure no MMA is still writing TMEM before it is freed
        mma_commit_pair(drain);
        drain_wait(drain, 0, p.timeout_ns);
      }
    } else if (MODE == 1 && warp >= 2) {
      // ----------------------------------------------------- helper warps
      // the staged sums of each tile (columns 0-127): a = w1.x in TMEM rows
      // 0-63 and u = w3.x in rows 64-127 of the same 64 features meet here;
      // h = silu(a) * u in bf16.  Lane l takes features 2l, 2l + 1 (4-byte
      // stores, 128 bytes per token row and warp), the two warps alternate
      // token columns.
      const int hw = warp - 2;
      const float *stg = reinterpret_cast<const float *>(sm + L::STG_OFF);
      const int qa = lane >> 4;             // TMEM lane quarter of the two a rows
      const int fl = (2 * lane) & 31;        // their lane within the quarter
      bf16 *out = static_cast<bf16 *>(p.out);
      int ntile = 0;
      for (int tile = unit; tile < total; tile += nunits, ++ntile) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        const int row0 = t.rowbase + t.n0;
        __nv_bfloat162 *orow =
            reinterpret_cast<__nv_bfloat162 *>(out + t.ft * 128 + (int)rank * 64 + 2 * lane);
        if (!wait_bounded(sfull, (uint32_t)ntile & 1u, abort_flag, p.timeout_ns, p.status)) break;
        const int ncol = t.nvalid < 128 ? t.nvalid : 128;
        for (int c = hw; c < ncol; c += 2) {
          // column c: warp half (c / 32) % 2, chunk c / 64, element c % 32
          const int h2 = (c >> 5) & 1, jc = c >> 6, e = c & 31;
          const float2 a = *reinterpret_cast<const float2 *>(
              stg + ((size_t)((qa + 4 * h2) * SCH + jc) * 32 + e) * 32 + fl);
          const float2 u = *reinterpret_cast<const float2 *>(
              stg + ((size_t)((qa + 2 + 4 * h2) * SCH + jc) * 32 + e) * 32 + fl);
          orow[(size_t)(row0 + c) * (p.I / 2)] =
              __floats2bfloat162_rn(swiglu_h(a.x, u.x), swiglu_h(a.y, u.y));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty);
      }
    } else if (MODE == 3 && warp >= 2) {
      // ----------------------------------------------------- helper warps
      // per tile: the (token, gate) list for the scatter into y (gate 1 for
      // the shared expert), written into one of two lists that alternate
      // between tiles well before the tile's end; then, once the promotion
      // warps have staged their first SCH chunks of the tile's sums (gate
      // applied), those sums are added into y with 16-byte reductions while
      // the next tile's k-loop runs
      const int hw = warp - 2;          // 0, 1
      const int bt = threadIdx.x - 64;  // 0 .. 63
      const float *stg = reinterpret_cast<const float *>(sm + L::STG_OFF);
      int ntile = 0;
      for (int tile = unit; tile < total; tile += nunits, ++ntile) {
        const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
        const int lb = ntile & 1;
        const uint32_t lph = (uint32_t)(ntile >> 1) & 1u;
        int32_t *s_tok = reinterpret_cast<int32_t *>(xbuf) + lb * 2 * BN_MAX;
        float *s_gate = reinterpret_cast<float *>(s_tok + BN_MAX);
        // every reader is done with this list's previous tile
        if (!wait_bounded(lempty + lb, lph ^ 1u, abort_flag, p.timeout_ns, p.status)) break;
        constexpr int PER = BN_MAX / 64;
        int tok[PER], pos[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = bt + 64 * i;
          tok[i] = c >= t.nvalid ? -1 : t.g < p.E ? p.sorted_token[t.rowbase + t.n0 + c] : t.tok0 + c;
          pos[i] = -1;
        }
        if (t.g < p.E) {
          for (int jj = 0; jj < p.k; ++jj)
#pragma unroll
            for (int i = 0; i < PER; ++i)
              if (tok[i] >= 0 && p.indices[(size_t)tok[i] * p.k + jj] == t.g) pos[i] = jj;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int c = bt + 64 * i;
          if (tok[i] >= 0) {
            s_tok[c] = tok[i];
            s_gate[c] = pos[i] >= 0 ? p.weights[(size_t)tok[i] * p.k + pos[i]] : 1.0f;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(lfull + lb);
        // the tile's staged sums: unit u = promotion warp u / SCH, its chunk
        // u % SCH; this warp takes every other unit.  Lane l adds 4
        // consecutive d (l % 8) of token column l / 8 + 4 eb.
        if (!wait_bounded(sfull, (uint32_t)ntile & 1u, abort_flag, p.timeout_ns, p.status)) break;
        const int i4 = lane & 7, es = lane >> 3;
        for (int u = hw; u < EPI * SCH; u += 2) {
          const int w = u / SCH, jc = u % SCH;
          const int c0 = (2 * jc + (w >> 2)) * 32;
          if (c0 >= t.nvalid) continue;
          float *yq = p.y + t.ft * 256 + (int)rank * BM + (w & 3) * 32 + 4 * i4;
          const float *src = stg + (size_t)u * 32 * 32;
#pragma unroll 4
          for (int eb = 0; eb < 8; ++eb) {
            const int e = 4 * eb + es;
            if (c0 + e < t.nvalid) {
              const float4 v = *reinterpret_cast<const float4 *>(src + e * 32 + 4 * i4);
              red_add_v4_f32(yq + (size_t)s_tok[c0 + e] * p.D, v.x, v.y, v.z, v.w);
            }
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(sempty);
          mbar_arrive(lempty + lb);
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_HIGH));
    // ------------------------------------------- promotion and epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - EPI0) >> 2;  // the two warps of a quarter take alternate chunks
    float *comb = s_comb + (warp - EPI0) * CHUNKS * 32;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    int pb = 0;
    uint32_t pphase = 0;
    bool ok = true;
    int ntile = 0;
    for (int tile = unit; ok && tile < total; tile += nunits, ++ntile) {
      const Tile t = decode_tile(tile, s_tstart, s_tbase, s_off, p.G, p.E, p.T, p.rows_routed, p.sh);
      const int row0 = t.rowbase + t.n0;
      // weight scales of this CTA's rows, one per k-block
      const float *sw;
      if (MODE == 1)
        sw = (q < 2 ? p.sA0 : p.sA1) + ((size_t)t.wg * (p.I / 128) + t.ft) * KB;
      else
        sw = p.sA0 + ((size_t)t.wg * (p.D / 128) + t.ft * 2 + (int)rank) * KB;
      // each lane's token scales, which the tile's end needs, are fetched now
      // so that their latency passes during the k-loop
      float sxr[CHUNKS];
#pragma unroll
      for (int j = 0; j < CHUNKS; ++j) {
        const int c = (2 * j + half) * 32 + lane;
        sxr[j] = c < t.nvalid ? __ldg(p.sX + row0 + c) : 0.0f;
      }
      // MODE 3: this tile's (token, gate) list, written by the list builders
      const int lb = ntile & 1;
      const uint32_t lph = (uint32_t)(ntile >> 1) & 1u;
      const int32_t *s_tok = reinterpret_cast<const int32_t *>(xbuf) + lb * 2 * BN_MAX;
      const float *s_gate = reinterpret_cast<const float *>(s_tok + BN_MAX);
      // running sums: this lane's row, the warp's columns
      float acc[CHUNKS][32];
#pragma unroll
      for (int j = 0; j < CHUNKS; ++j)
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[j][e] = 0.0f;
#define ACC(j, e) acc[j][e]
      const int k0 = k_rotation(t, KB);
      // the weight scale of each k-block, fetched one k-block ahead of its use
      float nw = __ldg(sw + k0);
      for (int i = 0; i < KB; ++i) {
        const float cw = nw;
        if (i + 1 < KB) nw = __ldg(sw + (k0 + i + 1 < KB ? k0 + i + 1 : k0 + i + 1 - KB));
        if (!wait_bounded(pfull + pb, pphase, abort_flag, p.timeout_ns, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // acc += s_w[kb] * partial: a chunk's 32 columns per TMEM load, with
        // the (warp-uniform) weight scale
#pragma unroll
        for (int j = 0; j < CHUNKS; ++j) {
          const int c0 = (2 * j + half) * 32;
          if (c0 >= t.nvalid) continue;
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + (uint32_t)(pb * BN_MAX + c0), v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[j][e] = fmaf(__uint_as_float(v[e]), cw, acc[j][e]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(pempty + pb), 0));
        if (++pb == NPBUF) {
          pb = 0;
          pphase ^= 1u;
        }
      }
      if (!ok) break;
      // times each token's activation scale (one per row, the same for every
      // k-block) -- and, for the scatter, its gate -- handed from the lane
      // that holds it to all lanes through this warp's shared-memory slots
      if (MODE == 3 && !wait_bounded(lfull + lb, lph, abort_flag, p.timeout_ns, p.status)) break;
#pragma unroll
      for (int j = 0; j < CHUNKS; ++j)
        comb[j * 32 + lane] = MODE == 3 ? sxr[j] * s_gate[(2 * j + half) * 32 + lane] : sxr[j];
      __syncwarp();
#pragma unroll
      for (int j = 0; j < CHUNKS; ++j)
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[j][e] *= comb[j * 32 + e];
      __syncwarp();

      if (staged(MODE)) {
        // the first SCH chunks go to the helper warps through shared memory,
        // once they are done with the previous tile's
        if (!wait_bounded(sempty, ((uint32_t)ntile & 1u) ^ 1u, abort_flag, p.timeout_ns, p.status))
          break;
        float *stg = reinterpret_cast<float *>(sm + L::STG_OFF) + (size_t)(warp - EPI0) * SCH * 32 * 32;
#pragma unroll
        for (int j = 0; j < SCH; ++j) {
          const int c0 = (2 * j + half) * 32;
          if (c0 >= t.nvalid) continue;
#pragma unroll
          for (int e = 0; e < 32; ++e) stg[(j * 32 + e) * 32 + lane] = ACC(j, e);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sfull);
      }

      if (MODE == 1) {
        // lanes 0-63 of the CTA hold w1.x (a), lanes 64-127 w3.x (u) of the
        // same 64 features; for the chunks not staged, warps q and q+2 of
        // one half pair up through shared memory, each finishing 16 of the
        // 32 columns of a chunk
        const int pr = q & 1;
        const bool is_a = q < 2;
        float *buf_a = xbuf + (pr + 2 * half) * 2 * 32 * XB_STRIDE;
        float *buf_u = buf_a + 32 * XB_STRIDE;
        const int bar = 1 + pr + 2 * half;
        const int f = t.ft * 128 + (int)rank * 64 + pr * 32 + lane;
        bf16 *out = static_cast<bf16 *>(p.out);
#pragma unroll
        for (int j = SCH; j < CHUNKS; ++j) {
          const int c0 = (2 * j + half) * 32;
          if (c0 >= t.nvalid) continue;
          float *mine = is_a ? buf_a : buf_u;
#pragma unroll
          for (int e = 0; e < 16; ++e) mine[lane * XB_STRIDE + e] = is_a ? ACC(j, 16 + e) : ACC(j, e);
          named_bar_sync(bar, 64);
          const float *other = is_a ? buf_u : buf_a;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = is_a ? e : 16 + e;
            const float a = is_a ? ACC(j, e) : other[lane * XB_STRIDE + e];
            const float u = is_a ? other[lane * XB_STRIDE + e] : ACC(j, 16 + e);
            if (c0 + col < t.nvalid)
              out[(size_t)(row0 + c0 + col) * p.I + f] = __float2bfloat16_rn(swiglu_h(a, u));
          }
          named_bar_sync(bar, 64);
        }
      } else if (MODE == 2) {
        float *out;
        size_t r0;
        if (t.g < p.E) {
          out = static_cast<float *>(p.out);
          r0 = (size_t)row0;
        } else {
          out = p.out_shared;
          r0 = (size_t)(t.g - p.E) * p.T + t.tok0;
        }
        const int d = t.ft * 256 + (int)rank * BM + q * 32 + lane;
#pragma unroll
        for (int j = 0; j < CHUNKS; ++j) {
          const int c0 = (2 * j + half) * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c0 + e < t.nvalid) out[(r0 + c0 + e) * p.D + d] = ACC(j, e);
        }
      } else {
        // weighted scatter into y (the sums already carry the gate, 1 for
        // the shared expert).  The first SCH chunks go to the helper warps
        // through shared memory, which add them into y during the next
        // tile's k-loop;
        // the rest are added here, while the MMA waits, with 16-byte fp32
        // reductions: a lane holds one d for 32 tokens, so each quad of
        // lanes transposes its 4 x 4 blocks (4 d by 4 tokens) with two
        // shuffle rounds and lane t of a quad adds 4 consecutive d of token
        // 4u + t -- a quarter of the reductions of one per element.
        const int t4 = lane & 3, hi = t4 >> 1, lo = t4 & 1;
        float *yrow = p.y + t.ft * 256 + (int)rank * BM + q * 32 + (lane & ~3);
#pragma unroll
        for (int j = SCH; j < CHUNKS; ++j) {
          const int c0 = (2 * j + half) * 32;
          if (c0 >= t.nvalid) continue;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            // M[r][s]: d = (lane & ~3) + r of the quarter, token c0 + 4u + s;
            // this lane holds row r = t4
            const float a0 = ACC(j, 4 * u + 0), a1 = ACC(j, 4 * u + 1);
            const float a2 = ACC(j, 4 * u + 2), a3 = ACC(j, 4 * u + 3);
            // round 1 (lanes t, t ^ 2): b[2 rr + cc] = M[lo + 2 rr][2 hi + cc]
            const float y0 = __shfl_xor_sync(0xffffffffu, hi ? a0 : a2, 2);
            const float y1 = __shfl_xor_sync(0xffffffffu, hi ? a1 : a3, 2);
            const float b0 = hi ? y0 : a0, b1 = hi ? y1 : a1;
            const float b2 = hi ? a2 : y0, b3 = hi ? a3 : y1;
            // round 2 (lanes t, t ^ 1): column t4 of all four rows
            const float z0 = __shfl_xor_sync(0xffffffffu, lo ? b0 : b1, 1);
            const float z1 = __shfl_xor_sync(0xffffffffu, lo ? b2 : b3, 1);
            const float o0 = lo ? b1 : b0, o1 = lo ? b3 : b2;
            const int c = c0 + 4 * u + t4;
            if (c < t.nvalid)
              red_add_v4_f32(yrow + (size_t)s_tok[c] * p.D, lo ? z0 : o0, lo ? o0 : z0,
                             lo ? z1 : o1, lo ? o1 : z1);
          }
        }
        __syncwarp();  // this warp's reads of the list are done
        if (lane == 0) mbar_arrive(lempty + lb);
      }
    }
  }
#undef ACC
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // a stalled pipeline stopped early: let copies already issued land (the
    // leader's full barriers count both CTAs' copies)
    if (leader) {
      for (int s = 0; s < STAGES; ++s)
        if (pending[s] >= 0) drain_wait(full + s, (uint32_t)pending[s], p.timeout_ns);
    } else {
      sleep_ns(200000);
    }
  }
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace f8

// ------------------------------------------------ fused decode block
//
// The whole block for a decode-sized batch in one persistent, cooperative
// launch (one CTA per SM): the router (fp32 FMA scores, then the selection),
// the token grouping and both tile tables, the row gather, the first matmul
// and the second with the weighted scatter into y, as phases separated by
// grid-wide barriers.  Each phase runs the same device code as the separate
// kernels; the launch gaps between them go away.  Every barrier wait is
// bounded: a CTA that waits too long records MOE_ERR_TIMEOUT and returns.

namespace fused {

constexpr int THREADS = 256;  // the router's tile shape; the GEMM phases use six warps of it

struct Args {
  const __nv_bfloat16 *x;  // [T, D]
  const float *w_r;        // [E, D]
  float *z_part;           // [nsplit, T, E]
  int nsplit, cols_per_split;
  route::SelectArgs sel;   // the selection's inputs and outputs
  int32_t *chunk_hist;     // [nchunks, E]
  int nchunks;
  int32_t *counts, *offsets, *sorted_token, *slot_of;
  Tiling t1, t2;           // the two matmuls' tile tables
  Shard sh;
  uint4 *xperm;            // expert-contiguous rows of x
  float *y;                // [T, D]
  int32_t *status;
  unsigned *bar;           // grid barrier: arrivals, generation (zero at launch)
  int64_t timeout_ns;
  int T, D, E, G, k, rows_routed, rows_total;
};

// All CTAs meet; false (after recording MOE_ERR_TIMEOUT) when this CTA gave
// up waiting.  Thread 0 arrives on the arrival counter and waits for the
// generation to move on; the last to arrive resets the counter and moves it.
__device__ __forceinline__ bool grid_sync(const Args &a, int *flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    volatile unsigned *gen = a.bar + 1;
    __threadfence();
    const unsigned g = *gen;
    if (atomicAdd(a.bar, 1u) == gridDim.x - 1) {
      atomicExch(a.bar, 0u);
      __threadfence();
      atomicAdd(a.bar + 1, 1u);
    } else {
      const uint64_t t0 = sm100::globaltimer_ns();
      while (*gen == g) {
        if ((int64_t)(sm100::globaltimer_ns() - t0) > a.timeout_ns) {
          set_status(a.status, MOE_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(100);
      }
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(THREADS, 1)
    decode_block(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW3,
                 const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW2,
                 const __grid_constant__ CUtensorMap tmH, const Args a, const tc::Params p1,
                 const tc::Params p2) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_flag;
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x / 32;
  const int nwarps = gridDim.x * (THREADS / 32);
  const int gwarp = blockIdx.x * (THREADS / 32) + warp;
  const int T = a.T, E = a.E, D = a.D;

  // 1. y = 0; router scores z = x W_r^T in tiles of 64 tokens x 64 experts
  //    x one split of dim
  {
    float4 *y4 = reinterpret_cast<float4 *>(a.y);
    const size_t n4 = (size_t)T * D / 4;
    for (size_t i = (size_t)blockIdx.x * THREADS + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * THREADS)
      y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto xs = reinterpret_cast<float(*)[route::SC_BM + 4]>(sm);
    auto ws = reinterpret_cast<float(*)[route::SC_BN + 4]>(
        sm + route::SC_BK * (route::SC_BM + 4) * sizeof(float));
    const int mt = (T + route::SC_BM - 1) / route::SC_BM;
    const int nt = (E + route::SC_BN - 1) / route::SC_BN;
    const int ntiles = mt * nt * a.nsplit;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int split = tile / (mt * nt), r = tile - split * (mt * nt);
      route::scores_tile(a.x, a.w_r, a.z_part, T, E, D, a.cols_per_split,
                         (r / nt) * route::SC_BM, (r % nt) * route::SC_BN, split, xs, ws);
      __syncthreads();
    }
  }
  if (!grid_sync(a, &s_flag)) return;

  // 2. selection: one warp per token
  {
    float *s = reinterpret_cast<float *>(sm) + (size_t)warp * 2 * E;
    for (int t = gwarp; t < T; t += nwarps) route::select_token(a.sel, t, s, s + E);
  }
  if (!grid_sync(a, &s_flag)) return;

  // 3. the grouping and both tile tables (one CTA)
  if (blockIdx.x == 0) {
    int32_t *h = reinterpret_cast<int32_t *>(sm);
    int32_t *wt = h + E;
    int32_t *base = wt + 32;
    for (int c = 0; c < a.nchunks; ++c) {
      grouping::hist_chunk(a.sel.indices, T, a.k, E, c, a.chunk_hist, a.status, h);
      __syncthreads();
    }
    grouping::scan_chunks(a.chunk_hist, a.nchunks, E, a.counts, a.offsets, wt);
    __syncthreads();
    if (warp == 0)
      for (int c = 0; c < a.nchunks; ++c)
        grouping::scatter_chunk(a.sel.indices, T, a.k, E, c, a.chunk_hist, a.offsets,
                                a.sorted_token, a.slot_of, base);
    __syncthreads();
    if (warp == 1) prep_tiles_warp(a.offsets, E, a.G, a.sh, a.t1, a.t2);
  }
  if (!grid_sync(a, &s_flag)) return;

  // 4. the expert-contiguous rows (one warp per row), then made visible to
  //    the TMA loads of the next phase
  {
    const int vec = D * 2 / 16;
    const uint4 *x4 = reinterpret_cast<const uint4 *>(a.x);
    const int lane = threadIdx.x % 32;
    for (int row = gwarp; row < a.rows_total; row += nwarps) {
      const int src = row < a.rows_routed ? a.sorted_token[row] : row - a.rows_routed;
      const uint4 *s = x4 + (size_t)src * vec;
      uint4 *d = a.xperm + (size_t)row * vec;
      for (int v = lane; v < vec; v += 32) d[v] = __ldg(s + v);
    }
    sm100::fence_proxy_async_global();
  }
  if (!grid_sync(a, &s_flag)) return;
  sm100::fence_proxy_async_global();  // (the reading side of the same ordering)

  // 5. first matmul + SwiGLU (h is then made visible to the next TMA loads);
  //    this CTA allocates tensor memory again in phase 6, so it keeps the
  //    right to allocate
  tc::gemm_body<1, 1, 1, BN, 32, STAGES, false>(tmW1, tmW3, tmX, p1, sm, false);
  sm100::fence_proxy_async_global();
  if (!grid_sync(a, &s_flag)) return;
  sm100::fence_proxy_async_global();

  // 6. second matmul, gate times output added into y
  tc::gemm_body<3, 1, 1, BN, 32, STAGES, false>(tmW2, tmW2, tmH, p2, sm, true);
}

}  // namespace fused

// ----------------------------------------------------------- CUDA-core path

__device__ __forceinline__ float ld_f(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_f(const bf16 *p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float ld_f(const __nv_fp8_e4m3 *p, size_t i) { return float(p[i]); }

// element (r, c) of group g's [rows, cols] matrix, with the 128 x 128 block
// scale for e4m3 weights
template <typename WT>
__device__ __forceinline__ float w_at(const WT *w, const float *scale, int g, int r, int c,
                                      int rows, int cols) {
  const float v = ld_f(w, ((size_t)g * rows + r) * cols + c);
  if (scale) {
    const int sr = rows / 128, sc = cols / 128;
    return v * scale[((size_t)g * sr + r / 128) * sc + c / 128];
  }
  return v;
}

constexpr int ST = 32;  // CUDA-core tile: 32 rows x 32 features

struct SimtArgs {
  const int32_t *tile_start, *tile_base, *offsets, *sorted_token;
  int E, G, T, D, I, rows_routed, act_bf16;
  float *h;  // [rows, I] fp32 (values rounded to bf16 when act_bf16)
  float *out_perm, *out_shared;
  // weighted scatter into y instead of out_perm / out_shared (when y != NULL)
  const int32_t *indices;
  const float *weights;
  int k;
  float *y;
  Shard sh;
};

template <typename XT, typename WT>
__global__ void __launch_bounds__(256) simt_gemm1(const XT *__restrict__ x, const WT *w1,
                                                  const WT *w3, const float *s1, const float *s3,
                                                  SimtArgs a) {
  __shared__ float xs[ST][ST + 1], as_[ST][ST + 1], us[ST][ST + 1];
  __shared__ int tok[ST];
  const int tile = blockIdx.x;
  if (tile >= a.tile_start[a.G]) return;
  const Tile t = decode_tile(tile, a.tile_start, a.tile_base, a.offsets, a.G, a.E, a.T,
                             a.rows_routed, a.sh);
  if (threadIdx.x < ST) {
    const int r = threadIdx.x;
    tok[r] = r < t.nvalid ? (t.g < a.E ? a.sorted_token[t.rowbase + t.n0 + r] : t.tok0 + r) : -1;
  }
  const int r = threadIdx.x / 8, fq = (threadIdx.x % 8) * 4;
  float acc_a[4] = {0.f, 0.f, 0.f, 0.f}, acc_u[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < a.D; k0 += ST) {
    __syncthreads();
    for (int i = threadIdx.x; i < ST * ST; i += 256) {
      const int rr = i / ST, kk = i % ST, kd = k0 + kk;
      xs[rr][kk] = (tok[rr] >= 0 && kd < a.D) ? ld_f(x, (size_t)tok[rr] * a.D + kd) : 0.f;
      const int f = t.ft * ST + rr;
      const bool in = f < a.I && kd < a.D;
      as_[rr][kk] = in ? w_at(w1, s1, t.wg, f, kd, a.I, a.D) : 0.f;
      us[rr][kk] = in ? w_at(w3, s3, t.wg, f, kd, a.I, a.D) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < ST; ++kk) {
      const float xv = xs[r][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc_a[j] = fmaf(xv, as_[fq + j][kk], acc_a[j]);
        acc_u[j] = fmaf(xv, us[fq + j][kk], acc_u[j]);
      }
    }
  }
  if (r < t.nvalid) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = t.ft * ST + fq + j;
      if (f >= a.I) continue;
      float h = acc_a[j] / (1.0f + expf(-acc_a[j])) * acc_u[j];
      if (a.act_bf16) h = __bfloat162float(__float2bfloat16_rn(h));
      a.h[((size_t)t.rowbase + t.n0 + r) * a.I + f] = h;
    }
  }
}

template <typename WT>
__global__ void __launch_bounds__(256) simt_gemm2(const WT *w2, const float *s2, SimtArgs a) {
  __shared__ float hs[ST][ST + 1], ws[ST][ST + 1];
  const int tile = blockIdx.x;
  if (tile >= a.tile_start[a.G]) return;
  const Tile t = decode_tile(tile, a.tile_start, a.tile_base, a.offsets, a.G, a.E, a.T,
                             a.rows_routed, a.sh);
  const int r = threadIdx.x / 8, dq = (threadIdx.x % 8) * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < a.I; k0 += ST) {
    __syncthreads();
    for (int i = threadIdx.x; i < ST * ST; i += 256) {
      const int rr = i / ST, kk = i % ST, ki = k0 + kk;
      hs[rr][kk] = (rr < t.nvalid && ki < a.I)
                       ? a.h[((size_t)t.rowbase + t.n0 + rr) * a.I + ki]
                       : 0.f;
      const int d = t.ft * ST + rr;
      ws[rr][kk] = (d < a.D && ki < a.I) ? w_at(w2, s2, t.wg, d, ki, a.D, a.I) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < ST; ++kk) {
      const float hv = hs[r][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = fmaf(hv, ws[dq + j][kk], acc[j]);
    }
  }
  if (r < t.nvalid) {
    if (a.y) {
      int tok = t.tok0 + r;
      float gate = 1.0f;
      if (t.g < a.E) {
        tok = a.sorted_token[t.rowbase + t.n0 + r];
        for (int jj = 0; jj < a.k; ++jj)
          if (a.indices[(size_t)tok * a.k + jj] == t.g) gate = a.weights[(size_t)tok * a.k + jj];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = t.ft * ST + dq + j;
        if (d < a.D) atomicAdd(a.y + (size_t)tok * a.D + d, gate * acc[j]);
      }
      return;
    }
    float *out;
    size_t row;
    if (t.g < a.E) {
      out = a.out_perm;
      row = (size_t)t.rowbase + t.n0 + r;
    } else {
      out = a.out_shared;
      row = (size_t)(t.g - a.E) * a.T + t.tok0 + r;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = t.ft * ST + dq + j;
      if (d < a.D) out[row * a.D + d] = acc[j];
    }
  }
}

// -------------------------------------------------------------- host side

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

// 2-D row-major [rows, cols] matrix of `elem` bytes, box of box_rows rows x
// box_cols columns, 128-byte swizzle (box_cols * elem must be 128) unless
// `plain` (rows of the box stored back to back, as the e4m3 tiles are).
bool make_tmap(CUtensorMap *m, const void *base, CUtensorMapDataType dt, size_t elem,
               uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
               bool plain = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {cols, rows};
  cuuint64_t gstride[1] = {cols * elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            plain ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

struct WsLayout {
  size_t tab, xperm, h, total;
  int64_t rows_pad;
  // FP8 x FP8 path (e4m3 weights): e4m3 codes and per-row scales of the
  // expert rows (xq, xs) and of h (hq, hs), and h in bf16 (hb)
  size_t xq, xs, hb, hq, hs;
};

constexpr int ROW_PAD = 256;  // spare rows so a TMA box never starts past a buffer

bool tc_path(const moe_cfg *c, moe_dtype x_dt, moe_dtype w_dt) {
  return x_dt == MOE_BF16 && (w_dt == MOE_BF16 || w_dt == MOE_E4M3) && c->dim % 128 == 0 &&
         c->inter % 128 == 0;
}

WsLayout ws_layout(const moe_cfg *c, int64_t T, moe_dtype x_dt, moe_dtype w_dt) {
  WsLayout l;
  const int64_t G = c->n_routed + c->n_shared;
  l.rows_pad = T * c->topk + T * c->n_shared + ROW_PAD;
  l.tab = 0;
  size_t off = align_up(sizeof(int32_t) * (size_t)(4 * G + 4), 1024);
  const bool tc = tc_path(c, x_dt, w_dt);
  l.xperm = off;
  if (tc) off = align_up(off + (size_t)l.rows_pad * c->dim * 2, 1024);
  l.h = off;
  off = align_up(off + (size_t)l.rows_pad * c->inter * (tc ? 2 : 4), 1024);
  l.total = off;
  l.xq = l.xs = l.hb = l.hq = l.hs = 0;
  if (tc && w_dt == MOE_E4M3) {
    size_t o = align_up(sizeof(int32_t) * (size_t)(4 * G + 4), 1024);
    const size_t rp = (size_t)l.rows_pad;
    l.xq = o;
    o = align_up(o + rp * c->dim, 1024);
    l.xs = o;
    o = align_up(o + rp * 4, 1024);
    l.hb = o;
    o = align_up(o + rp * c->inter * 2, 1024);
    l.hq = o;
    o = align_up(o + rp * c->inter, 1024);
    l.hs = o;
    o = align_up(o + rp * 4, 1024);
    if (o > l.total) l.total = o;
  }
  return l;
}

template <int MODE, int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
moe_status launch_tc(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                     const tc::Params &p, cudaStream_t s) {
  using L = tc::Layout<MODE, CG, AT, BN_MAX, BOXN, STAGES, F8>;
  auto kern = tc::tc_expert_gemm<MODE, CG, AT, BN_MAX, BOXN, STAGES, F8>;
  const size_t smem_max = 232448;
  if (L::smem_bytes(p.G, p.E) > smem_max) return MOE_ERR_UNSUPPORTED;
  const size_t smem = L::smem_bytes(p.G, p.E);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  const int nsm = sm_count();
  if (nsm < 2) return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(L::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.gridDim = dim3(nsm);
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one persistent pair per co-resident SM pair
    int pairs = nsm / 2;
    cfg.gridDim = dim3(2 * pairs);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) == cudaSuccess && active > 0 &&
        active < pairs)
      pairs = active;
    cfg.gridDim = dim3(2 * pairs);
  }
  if (cudaLaunchKernelEx(&cfg, kern, a0, a1, b, p) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_status();
}

// MOE_ERR_CUDA for a failed runtime call; with MOE_DEBUG set in the
// environment the call site and the runtime's error name go to stderr.
moe_status cuda_fail(const char *where, cudaError_t e) {
  if (getenv("MOE_DEBUG"))
    fprintf(stderr, "moe_experts: %s: %s\n", where, cudaGetErrorName(e));
  return MOE_ERR_CUDA;
}

moe_status checked_launch(const char *where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail(where, e);
}

template <int MODE, int STAGES>
moe_status launch_fp8(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                      const tc::Params &p, cudaStream_t s) {
  using L = f8::Layout<MODE, STAGES>;
  auto kern = f8::tc_fp8_gemm<MODE, STAGES>;
  const size_t smem = L::smem_bytes(p.G, p.E);
  if (smem > 232448) return MOE_ERR_UNSUPPORTED;
  cudaError_t e = cudaGetLastError();  // nothing earlier may be reported as this launch's
  if (e != cudaSuccess) return cuda_fail("before the FP8 GEMM", e);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_fail("FP8 GEMM shared memory", e);
  const int nsm = sm_count();
  if (nsm < 2) return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(f8::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one persistent pair per co-resident SM pair
  int pairs = nsm / 2;
  cfg.gridDim = dim3(2 * pairs);
  int active = 0;
  e = cudaOccupancyMaxActiveClusters(&active, kern, &cfg);
  if (e != cudaSuccess) {
    cudaGetLastError();  // not sticky: the launch below decides
    if (getenv("MOE_DEBUG")) cuda_fail("FP8 GEMM occupancy query", e);
  } else if (active > 0 && active < pairs) {
    pairs = active;
  }
  cfg.gridDim = dim3(2 * pairs);
  e = cudaLaunchKernelEx(&cfg, kern, a0, a1, b, p);
  if (e != cudaSuccess) return cuda_fail("FP8 GEMM launch", e);
  return checked_launch("FP8 GEMM launch");
}

// Optional profiling events (caller-owned cudaEvent_t), recorded on the call's
// stream around the kernels of the experts: [0] before the gather, [1] before
// GEMM1, [2] after GEMM1, [3] before GEMM2, [4] after GEMM2.
cudaEvent_t g_prof[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
int g_nprof = 0;

void prof(int i, cudaStream_t s) {
  if (i < g_nprof && g_prof[i]) cudaEventRecord(g_prof[i], s);
}

struct Job {
  const moe_cfg *c;
  int64_t T;
  const void *x;
  moe_dtype x_dt;
  const moe_expert_weights *w;
  const int32_t *offsets;
  const int32_t *sorted_token;
  float *out_perm;
  float *out_shared;
  // weighted scatter into y (moe_experts_forward_combine); y == NULL otherwise
  const int32_t *indices;
  const float *weights;
  float *y;
  uint8_t *ws;
  WsLayout l;
  int32_t *status;
  cudaStream_t s;

  int E() const { return c->n_routed; }
  int G() const { return c->n_routed + c->n_shared; }
  // the call's share of the work (all of it unless expert-parallel) and
  // whether it is a strict part (then rows outside it are skipped)
  Shard sh;
  bool sharded;
  int wgroups() const { return (sh.e1 - sh.e0) + c->n_shared; }  // groups in the weight tensors
  const int32_t *shard_off() const { return sharded ? offsets : nullptr; }
  int rows_routed() const { return (int)(T * c->topk); }
  int rows_total() const { return (int)(T * c->topk + T * c->n_shared); }
  int32_t *tab() const { return reinterpret_cast<int32_t *>(ws + l.tab); }
};

tc::Params tc_params(const Job &j) {
  tc::Params p;
  p.offsets = j.offsets;
  p.E = j.E();
  p.G = j.G();
  p.T = (int)j.T;
  p.I = j.c->inter;
  p.D = j.c->dim;
  p.rows_routed = j.rows_routed();
  p.out_shared = j.out_shared;
  p.status = j.status;
  p.timeout_ns = 1000000000LL;
  p.sorted_token = j.sorted_token;
  p.indices = j.indices;
  p.weights = j.weights;
  p.k = j.c->topk;
  p.y = j.y;
  p.sA0 = nullptr;
  p.sA1 = nullptr;
  p.sX = nullptr;
  p.sh = j.sh;
  return p;
}

// Weight tensor map: bf16 tiles in the 128-byte swizzled layout the MMA reads,
// or e4m3 tiles stored plainly (64 bytes per row) for the converter warps.
bool weight_tmap(CUtensorMap *m, const void *w, bool f8, uint64_t rows, uint64_t cols,
                 uint32_t box_rows) {
  if (f8) return make_tmap(m, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, cols, box_rows, 64, true);
  return make_tmap(m, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box_rows, 64);
}

template <int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
moe_status tc_up(const Job &j) {
  using L = tc::Layout<1, CG, AT, BN_MAX, BOXN, STAGES, F8>;
  const int G = j.G(), D = j.c->dim, I = j.c->inter;
  int32_t *tab = j.tab();
  Tiling t1{BN_MAX, I / L::FEAT, tab, tab + (G + 1)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t1, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  bf16 *xperm = reinterpret_cast<bf16 *>(j.ws + j.l.xperm);
  bf16 *h = reinterpret_cast<bf16 *>(j.ws + j.l.h);
  prof(0, j.s);
  const int64_t threads = (int64_t)j.rows_total() * 32;
  if (F8)
    gather_rows_f16<<<(unsigned)((threads + 255) / 256), 256, 0, j.s>>>(
        static_cast<const uint4 *>(j.x), j.sorted_token, reinterpret_cast<uint4 *>(xperm),
        j.rows_routed(), j.rows_total(), (int)j.T, D * 2 / 16, j.shard_off(), j.sh);
  else
    gather_rows<<<(unsigned)((threads + 255) / 256), 256, 0, j.s>>>(
        static_cast<const uint4 *>(j.x), j.sorted_token, reinterpret_cast<uint4 *>(xperm),
        j.rows_routed(), j.rows_total(), (int)j.T, D * 2 / 16, j.shard_off(), j.sh);
  if ((st = launch_status()) != MOE_OK) return st;
  CUtensorMap mw1, mw3, mx;
  const CUtensorMapDataType BF = F8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!weight_tmap(&mw1, j.w->w1, F8, (uint64_t)j.wgroups() * I, D, L::PART_ROWS) ||
      !weight_tmap(&mw3, j.w->w3, F8, (uint64_t)j.wgroups() * I, D, L::PART_ROWS) ||
      !make_tmap(&mx, xperm, BF, 2, (uint64_t)j.l.rows_pad, D, BOXN, 64))
    return MOE_ERR_CUDA;
  tc::Params p = tc_params(j);
  p.tile_start = t1.tile_start;
  p.tile_base = t1.tile_base;
  p.KB = D / tc::BK;
  p.out = h;
  p.sA0 = j.w->s1;
  p.sA1 = j.w->s3;
  prof(1, j.s);
  st = launch_tc<1, CG, AT, BN_MAX, BOXN, STAGES, F8>(mw1, mw3, mx, p, j.s);
  prof(2, j.s);
  return st;
}

template <int CG, int AT, int BN_MAX, int BOXN, int STAGES, bool F8>
moe_status tc_down(const Job &j) {
  using L = tc::Layout<3, CG, AT, BN_MAX, BOXN, STAGES, F8>;
  const int G = j.G(), D = j.c->dim, I = j.c->inter;
  int32_t *tab = j.tab();
  Tiling t2{BN_MAX, D / L::FEAT, tab + (2 * G + 1), tab + (3 * G + 2)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t2, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  bf16 *h = reinterpret_cast<bf16 *>(j.ws + j.l.h);
  CUtensorMap mw2, mh;
  const CUtensorMapDataType BF = F8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!weight_tmap(&mw2, j.w->w2, F8, (uint64_t)j.wgroups() * D, I, tc::BM) ||
      !make_tmap(&mh, h, BF, 2, (uint64_t)j.l.rows_pad, I, BOXN, 64))
    return MOE_ERR_CUDA;
  tc::Params p = tc_params(j);
  p.tile_start = t2.tile_start;
  p.tile_base = t2.tile_base;
  p.KB = I / tc::BK;
  p.out = j.out_perm;
  p.sA0 = j.w->s2;
  p.sA1 = j.w->s2;
  prof(3, j.s);
  if (j.y)
    st = launch_tc<3, CG, AT, BN_MAX, BOXN, STAGES, F8>(mw2, mw2, mh, p, j.s);
  else
    st = launch_tc<2, CG, AT, BN_MAX, BOXN, STAGES, F8>(mw2, mw2, mh, p, j.s);
  prof(4, j.s);
  return st;
}

// ring depth of the FP8 x FP8 GEMMs: 32 KB per stage (16 KB of weight codes,
// 128 token rows of 128 codes)
#ifndef MOE_F8_STAGES
#define MOE_F8_STAGES 6
#endif
// the first matmul and the scatter variant give 64 KB to their staged sums:
// four stages
#ifndef MOE_F8_STAGES_STAGED
#define MOE_F8_STAGES_STAGED 4
#endif

bool e4m3_tmap(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tmap(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, cols, box_rows, 128);
}

moe_status quantise_rows(const Job &j, const void *src, bool gather, size_t q_off, size_t s_off,
                         int K) {
  const int rows = j.rows_total();
  const unsigned grid = (unsigned)((rows + 7) / 8);
  // K is a multiple of 128 on this path: 16-byte rows
  uint2 *q = reinterpret_cast<uint2 *>(j.ws + q_off);
  float *sc = reinterpret_cast<float *>(j.ws + s_off);
  if (gather)
    quant_rows_e4m3_v8<true><<<grid, 256, 0, j.s>>>(static_cast<const uint4 *>(src),
                                                    j.sorted_token, q, sc, j.rows_routed(), rows,
                                                    (int)j.T, K, j.shard_off(), j.sh);
  else
    quant_rows_e4m3_v8<false><<<grid, 256, 0, j.s>>>(static_cast<const uint4 *>(src), nullptr, q,
                                                     sc, j.rows_routed(), rows, (int)j.T, K,
                                                     j.shard_off(), j.sh);
  return checked_launch("e4m3 row quantiser");
}

moe_status fp8_up(const Job &j) {
  const int G = j.G(), D = j.c->dim, I = j.c->inter;
  int32_t *tab = j.tab();
  Tiling t1{f8::BN_MAX, I / 128, tab, tab + (G + 1)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t1, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  prof(0, j.s);
  if ((st = quantise_rows(j, j.x, true, j.l.xq, j.l.xs, D)) != MOE_OK) return st;
  CUtensorMap mw1, mw3, mx;
  if (!e4m3_tmap(&mw1, j.w->w1, (uint64_t)j.wgroups() * I, D, 64) ||
      !e4m3_tmap(&mw3, j.w->w3, (uint64_t)j.wgroups() * I, D, 64) ||
      !e4m3_tmap(&mx, j.ws + j.l.xq, (uint64_t)j.l.rows_pad, D, f8::BOXN))
    return cuda_fail("FP8 first matmul tensor maps", cudaErrorInvalidValue);
  tc::Params p = tc_params(j);
  p.tile_start = t1.tile_start;
  p.tile_base = t1.tile_base;
  p.KB = D / f8::BK;
  p.out = j.ws + j.l.hb;
  p.sA0 = j.w->s1;
  p.sA1 = j.w->s3;
  p.sX = reinterpret_cast<const float *>(j.ws + j.l.xs);
  prof(1, j.s);
  st = launch_fp8<1, MOE_F8_STAGES_STAGED>(mw1, mw3, mx, p, j.s);
  prof(2, j.s);
  if (st != MOE_OK) return st;
  // h (bf16) to e4m3 codes and scales for the second matmul
  return quantise_rows(j, j.ws + j.l.hb, false, j.l.hq, j.l.hs, I);
}

moe_status fp8_down(const Job &j) {
  const int G = j.G(), D = j.c->dim, I = j.c->inter;
  int32_t *tab = j.tab();
  Tiling t2{f8::BN_MAX, D / 256, tab + (2 * G + 1), tab + (3 * G + 2)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t2, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  CUtensorMap mw2, mh;
  if (!e4m3_tmap(&mw2, j.w->w2, (uint64_t)j.wgroups() * D, I, f8::BM) ||
      !e4m3_tmap(&mh, j.ws + j.l.hq, (uint64_t)j.l.rows_pad, I, f8::BOXN))
    return cuda_fail("FP8 second matmul tensor maps", cudaErrorInvalidValue);
  tc::Params p = tc_params(j);
  p.tile_start = t2.tile_start;
  p.tile_base = t2.tile_base;
  p.KB = I / f8::BK;
  p.out = j.out_perm;
  p.sA0 = j.w->s2;
  p.sA1 = j.w->s2;
  p.sX = reinterpret_cast<const float *>(j.ws + j.l.hs);
  prof(3, j.s);
  if (j.y)
    st = launch_fp8<3, MOE_F8_STAGES_STAGED>(mw2, mw2, mh, p, j.s);
  else
    st = launch_fp8<2, MOE_F8_STAGES>(mw2, mw2, mh, p, j.s);
  prof(4, j.s);
  return st;
}

SimtArgs simt_args(const Job &j, const Tiling &t) {
  SimtArgs a;
  a.offsets = j.offsets;
  a.sorted_token = j.sorted_token;
  a.E = j.E();
  a.G = j.G();
  a.T = (int)j.T;
  a.D = j.c->dim;
  a.I = j.c->inter;
  a.rows_routed = j.rows_routed();
  a.act_bf16 = j.x_dt == MOE_BF16;
  a.h = reinterpret_cast<float *>(j.ws + j.l.h);
  a.out_perm = j.out_perm;
  a.out_shared = j.out_shared;
  a.tile_start = t.tile_start;
  a.tile_base = t.tile_base;
  a.indices = j.indices;
  a.weights = j.weights;
  a.k = j.c->topk;
  a.y = j.y;
  a.sh = j.sh;
  return a;
}

// upper bound on CUDA-core tiles: sum over groups of ceil(n_g / 16) times feature tiles
int64_t simt_tile_bound(const Job &j, int ft) { return ((int64_t)j.rows_total() / 16 + j.G()) * ft; }

template <typename XT, typename WT>
moe_status simt_up(const Job &j) {
  const int G = j.G();
  int32_t *tab = j.tab();
  Tiling t1{ST, (j.c->inter + ST - 1) / ST, tab, tab + (G + 1)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t1, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  const SimtArgs a = simt_args(j, t1);
  const bool e4 = j.w->w_dt == MOE_E4M3;
  prof(0, j.s);
  prof(1, j.s);
  simt_gemm1<XT, WT><<<(unsigned)simt_tile_bound(j, t1.ft), 256, 0, j.s>>>(
      static_cast<const XT *>(j.x), static_cast<const WT *>(j.w->w1),
      static_cast<const WT *>(j.w->w3), e4 ? j.w->s1 : nullptr, e4 ? j.w->s3 : nullptr, a);
  st = launch_status();
  prof(2, j.s);
  return st;
}

template <typename WT>
moe_status simt_down(const Job &j) {
  const int G = j.G();
  int32_t *tab = j.tab();
  Tiling t2{ST, (j.c->dim + ST - 1) / ST, tab + (2 * G + 1), tab + (3 * G + 2)};
  Tiling none{0, 0, nullptr, nullptr};
  prep_tiles<<<1, 32, 0, j.s>>>(j.offsets, j.E(), G, j.sh, t2, none);
  moe_status st = launch_status();
  if (st != MOE_OK) return st;
  const SimtArgs a = simt_args(j, t2);
  prof(3, j.s);
  simt_gemm2<WT><<<(unsigned)simt_tile_bound(j, t2.ft), 256, 0, j.s>>>(
      static_cast<const WT *>(j.w->w2), j.w->w_dt == MOE_E4M3 ? j.w->s2 : nullptr, a);
  st = launch_status();
  prof(4, j.s);
  return st;
}

template <typename XT>
moe_status simt_up_x(const Job &j) {
  switch (j.w->w_dt) {
    case MOE_F32: return simt_up<XT, float>(j);
    case MOE_BF16: return simt_up<XT, bf16>(j);
    case MOE_E4M3: return simt_up<XT, __nv_fp8_e4m3>(j);
  }
  return MOE_ERR_UNSUPPORTED;
}

moe_status simt_down_w(const Job &j) {
  switch (j.w->w_dt) {
    case MOE_F32: return simt_down<float>(j);
    case MOE_BF16: return simt_down<bf16>(j);
    case MOE_E4M3: return simt_down<__nv_fp8_e4m3>(j);
  }
  return MOE_ERR_UNSUPPORTED;
}

// Tile shapes of the two instantiations (compile-time tunables).
#ifndef MOE_TC_PREFILL_BN
#define MOE_TC_PREFILL_BN 256
#endif
// weight tiles per SM in the first matmul (two: w1 and w3 in accumulators of
// their own, half the token bytes per weight byte) and in the second (two
// blocks of w2 rows, for the same reason, their single accumulator handed
// back before the last stores of each tile)
#ifndef MOE_TC_PREFILL_AT_UP
#define MOE_TC_PREFILL_AT_UP 2
#endif
#ifndef MOE_TC_PREFILL_AT_DOWN
#define MOE_TC_PREFILL_AT_DOWN 2
#endif
#ifndef MOE_TC_PREFILL_AT_DOWN_F8
#define MOE_TC_PREFILL_AT_DOWN_F8 2
#endif
#ifndef MOE_TC_PREFILL_CG
#define MOE_TC_PREFILL_CG 2
#endif
#ifndef MOE_TC_DECODE_BN
#define MOE_TC_DECODE_BN 32
#endif
#ifndef MOE_TC_DECODE_STAGES
#define MOE_TC_DECODE_STAGES 10
#endif
constexpr int PF_BN = MOE_TC_PREFILL_BN;
constexpr int PF_AT_UP = MOE_TC_PREFILL_AT_UP;
constexpr int pf_at_down(bool f8) { return f8 ? MOE_TC_PREFILL_AT_DOWN_F8 : MOE_TC_PREFILL_AT_DOWN; }
// ring depth filling about 200 KB of shared memory: a stage holds AT 16 KB
// weight tiles, PF_BN / 2 token rows of 128 bytes and, with e4m3 weights, AT
// 8 KB code tiles
constexpr int pf_stages(int at, bool f8) { return 200 * 1024 / (at * (f8 ? 24576 : 16384) + PF_BN * 64); }
constexpr int DC_BN = MOE_TC_DECODE_BN, DC_ST = MOE_TC_DECODE_STAGES;

// few rows per expert (decode): one SM per tile, narrow token tiles and a deep
// ring so that enough weight bytes are in flight; otherwise SM pairs with
// token tiles of up to PF_BN rows, each SM holding half of them
bool decode_variant(const Job &j) { return j.T * j.c->topk <= (int64_t)16 * j.c->n_routed; }

// an SM pair per tile (cta_group::2) covers 64 * 2 * PF_AT_UP features of
// w1/w3, and 256 rows of w2 per weight tile
bool pair_up_ok(const Job &j) {
  return MOE_TC_PREFILL_CG == 2 && j.c->inter % (128 * PF_AT_UP) == 0;
}
bool pair_down_ok(const Job &j, int at) { return MOE_TC_PREFILL_CG == 2 && j.c->dim % (256 * at) == 0; }

// e4m3 weights add 8 KB of codes per weight tile and stage; the ring depths
// shrink to fit shared memory, and half as many weight bytes need to be in
// flight.
template <bool F8>
moe_status run_up_t(const Job &j) {
  if (decode_variant(j)) return tc_up<1, 1, DC_BN, 32, F8 ? 7 : DC_ST, F8>(j);
  if (pair_up_ok(j)) return tc_up<2, PF_AT_UP, PF_BN, 32, pf_stages(PF_AT_UP, F8), F8>(j);
  return tc_up<1, 1, 256, 32, F8 ? 3 : 4, F8>(j);
}

template <bool F8>
moe_status run_down_t(const Job &j) {
  if (decode_variant(j)) return tc_down<1, 1, DC_BN, 32, F8 ? 7 : DC_ST, F8>(j);
  constexpr int AT = pf_at_down(F8);
  if (pair_down_ok(j, AT)) return tc_down<2, AT, PF_BN, 32, pf_stages(AT, F8), F8>(j);
  if (AT != 1 && pair_down_ok(j, 1)) return tc_down<2, 1, PF_BN, 32, pf_stages(1, F8), F8>(j);
  return tc_down<1, 1, 256, 32, F8 ? 3 : 4, F8>(j);
}

moe_status run_up(const Job &j) {
  if (j.w->act_e4m3) return fp8_up(j);
  if (tc_path(j.c, j.x_dt, j.w->w_dt))
    return j.w->w_dt == MOE_E4M3 ? run_up_t<true>(j) : run_up_t<false>(j);
  return j.x_dt == MOE_BF16 ? simt_up_x<bf16>(j) : simt_up_x<float>(j);
}

moe_status run_down(const Job &j) {
  if (j.w->act_e4m3) return fp8_down(j);
  if (tc_path(j.c, j.x_dt, j.w->w_dt))
    return j.w->w_dt == MOE_E4M3 ? run_down_t<true>(j) : run_down_t<false>(j);
  return simt_down_w(j);
}

// Checks shared by the entry points; fills the job on success.
moe_status make_job(Job &j, const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                    const moe_expert_weights *w, const int32_t *offsets,
                    const int32_t *sorted_token, float *out_perm, float *out_shared, void *ws,
                    size_t ws_bytes, int32_t *dev_status, moe_stream_t stream, bool need_up,
                    bool need_down) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || (T * (int64_t)cfg->topk + T) >= ((int64_t)1 << 31)) return MOE_ERR_INVALID;
  if (!w || !w->w1 || !w->w3 || !w->w2 || !offsets || !ws) return MOE_ERR_INVALID;
  if (need_up && (!x || !sorted_token)) return MOE_ERR_INVALID;
  if (need_down && !out_perm) return MOE_ERR_INVALID;
  if (cfg->n_shared > 1) return MOE_ERR_UNSUPPORTED;
  if (need_down && cfg->n_shared == 1 && !out_shared) return MOE_ERR_INVALID;
  if (x_dt != MOE_F32 && x_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (w->w_dt != MOE_F32 && w->w_dt != MOE_BF16 && w->w_dt != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (w->w_dt == MOE_E4M3) {
    if (!w->s1 || !w->s3 || !w->s2) return MOE_ERR_INVALID;
    if (cfg->dim % 128 != 0 || cfg->inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  }
  if (w->act_e4m3 != 0 && w->act_e4m3 != 1) return MOE_ERR_INVALID;
  if (w->act_e4m3 && (w->w_dt != MOE_E4M3 || x_dt != MOE_BF16 || cfg->dim % 256 != 0 ||
                      cfg->inter % 128 != 0))
    return MOE_ERR_UNSUPPORTED;
  j.l = ws_layout(cfg, T, x_dt, w->w_dt);
  if (ws_bytes < j.l.total) return MOE_ERR_WORKSPACE;
  j.c = cfg;
  j.T = T;
  j.x = x;
  j.x_dt = x_dt;
  j.w = w;
  j.offsets = offsets;
  j.sorted_token = sorted_token;
  j.out_perm = out_perm;
  j.out_shared = out_shared;
  j.indices = nullptr;
  j.weights = nullptr;
  j.y = nullptr;
  j.ws = static_cast<uint8_t *>(ws);
  j.status = dev_status;
  j.sh = Shard{0, cfg->n_routed, 0, (int)T};
  j.sharded = false;
  j.s = as_stream(stream);
  return MOE_OK;
}

// ------------------------------------------------ fused decode block (host)

struct DecodePlan {
  int nsplit, cols_per_split, nchunks;
  size_t z_off, hist_off, ex_off, total;
  WsLayout l;
};

// Workspace of the fused decode launch: the grid barrier's two words, the
// router's split partial scores (sized for the most splits, dim / 256), the
// grouping's chunk histograms, then the experts' workspace.
DecodePlan decode_plan(const moe_cfg *c, int64_t T, int grid) {
  DecodePlan d;
  const int mt = (int)((T + route::SC_BM - 1) / route::SC_BM);
  const int nt = (c->n_routed + route::SC_BN - 1) / route::SC_BN;
  const int max_split = c->dim / 256 > 1 ? c->dim / 256 : 1;
  int ns = grid > 0 ? (grid + mt * nt - 1) / (mt * nt) : 1;
  ns = ns < 1 ? 1 : (ns > max_split ? max_split : ns);
  int cps = (c->dim + ns - 1) / ns;
  cps = (cps + route::SC_BK - 1) / route::SC_BK * route::SC_BK;
  d.nsplit = (c->dim + cps - 1) / cps;
  d.cols_per_split = cps;
  d.nchunks = (int)((T + grouping::CHUNK_TOKENS - 1) / grouping::CHUNK_TOKENS);
  if (d.nchunks < 1) d.nchunks = 1;
  d.z_off = 256;
  d.hist_off = align_up(d.z_off + (size_t)max_split * T * c->n_routed * 4, 256);
  d.ex_off = align_up(d.hist_off + (size_t)d.nchunks * c->n_routed * 4, 1024);
  d.l = ws_layout(c, T, MOE_BF16, MOE_BF16);
  d.total = d.ex_off + d.l.total;
  return d;
}

// the decode tile shape of the expert GEMMs (one SM per tile)
template <int BN, int STAGES>
moe_status launch_decode_block(const Job &j, const DecodePlan &pl, const float *w_r,
                               const float *bias, float *weights, int32_t *indices,
                               float *sel_gap, int32_t *counts, int32_t *slot_of) {
  using L1 = tc::Layout<1, 1, 1, BN, 32, STAGES, false>;
  using L3 = tc::Layout<3, 1, 1, BN, 32, STAGES, false>;
  const moe_cfg *c = j.c;
  const int G = j.G(), D = c->dim, I = c->inter, E = c->n_routed;
  const int nsm = sm_count();
  if (nsm < 1) return MOE_ERR_CUDA;
  int32_t *tab = j.tab();
  Tiling t1{BN, I / L1::FEAT, tab, tab + (G + 1)};
  Tiling t2{BN, D / L3::FEAT, tab + (2 * G + 1), tab + (3 * G + 2)};
  bf16 *xperm = reinterpret_cast<bf16 *>(j.ws + j.l.xperm);
  bf16 *h = reinterpret_cast<bf16 *>(j.ws + j.l.h);
  CUtensorMap mw1, mw3, mx, mw2, mh;
  if (!weight_tmap(&mw1, j.w->w1, false, (uint64_t)G * I, D, L1::PART_ROWS) ||
      !weight_tmap(&mw3, j.w->w3, false, (uint64_t)G * I, D, L1::PART_ROWS) ||
      !make_tmap(&mx, xperm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)j.l.rows_pad, D, 32,
                 64) ||
      !weight_tmap(&mw2, j.w->w2, false, (uint64_t)G * D, I, tc::BM) ||
      !make_tmap(&mh, h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)j.l.rows_pad, I, 32, 64))
    return cuda_fail("fused decode tensor maps", cudaErrorInvalidValue);
  tc::Params p1 = tc_params(j);
  p1.tile_start = t1.tile_start;
  p1.tile_base = t1.tile_base;
  p1.KB = D / tc::BK;
  p1.out = h;
  tc::Params p2 = tc_params(j);
  p2.tile_start = t2.tile_start;
  p2.tile_base = t2.tile_base;
  p2.KB = I / tc::BK;
  p2.out = nullptr;

  fused::Args a;
  uint8_t *ws = static_cast<uint8_t *>(j.ws) - pl.ex_off;  // the whole workspace
  a.x = static_cast<const __nv_bfloat16 *>(j.x);
  a.w_r = w_r;
  a.z_part = reinterpret_cast<float *>(ws + pl.z_off);
  a.nsplit = pl.nsplit;
  a.cols_per_split = pl.cols_per_split;
  a.sel.z_part = a.z_part;
  a.sel.nsplit = pl.nsplit;
  a.sel.bias = c->has_bias ? bias : nullptr;
  a.sel.weights = weights;
  a.sel.indices = indices;
  a.sel.sel_gap = sel_gap;
  a.sel.T = (int)j.T;
  a.sel.E = E;
  a.sel.G = c->n_groups;
  a.sel.Gk = c->topk_groups;
  a.sel.k = c->topk;
  a.sel.route_scale = c->route_scale;
  a.sel.softmax = c->score_func == MOE_SCORE_SOFTMAX;
  a.chunk_hist = reinterpret_cast<int32_t *>(ws + pl.hist_off);
  a.nchunks = pl.nchunks;
  a.counts = counts;
  a.offsets = const_cast<int32_t *>(j.offsets);
  a.sorted_token = const_cast<int32_t *>(j.sorted_token);
  a.slot_of = slot_of;
  a.t1 = t1;
  a.t2 = t2;
  a.sh = j.sh;
  a.xperm = reinterpret_cast<uint4 *>(xperm);
  a.y = j.y;
  a.status = j.status;
  a.bar = reinterpret_cast<unsigned *>(ws);
  a.timeout_ns = 1000000000LL;
  a.T = (int)j.T;
  a.D = D;
  a.E = E;
  a.G = G;
  a.k = c->topk;
  a.rows_routed = j.rows_routed();
  a.rows_total = j.rows_total();

  size_t smem = L1::smem_bytes(G, E);
  if (L3::smem_bytes(G, E) > smem) smem = L3::smem_bytes(G, E);
  const size_t sel_smem = 1024 + (size_t)(fused::THREADS / 32) * 2 * E * sizeof(float);
  if (sel_smem > smem) smem = sel_smem;
  if (smem > 232448 - 16) return MOE_ERR_UNSUPPORTED;
  auto kern = fused::decode_block<BN, STAGES>;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("before the fused decode launch", e);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_fail("fused decode shared memory", e);
  e = cudaMemsetAsync(a.bar, 0, 2 * sizeof(unsigned), j.s);
  if (e != cudaSuccess) return cuda_fail("fused decode barrier reset", e);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barriers need it
  attr[0].val.cooperative = 1;
  cfg.gridDim = dim3(nsm);
  cfg.blockDim = dim3(fused::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = j.s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mw1, mw3, mx, mw2, mh, a, p1, p2);
  if (e != cudaSuccess) return cuda_fail("fused decode launch", e);
  return checked_launch("fused decode launch");
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_EXPORT size_t moe_experts_workspace_size(const moe_cfg *cfg, int64_t T, moe_dtype x_dt,
                                             moe_dtype w_dt) {
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  return ws_layout(cfg, T, x_dt, w_dt).total;
}

MOE_EXPORT moe_status moe_experts_up(const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt,
                                     const moe_expert_weights *w, const int32_t *offsets,
                                     const int32_t *sorted_token, void *ws, size_t ws_bytes,
                                     int32_t *dev_status, moe_stream_t stream) {
  Job j;
  moe_status st = make_job(j, cfg, T, x, x_dt, w, offsets, sorted_token, nullptr, nullptr, ws,
                           ws_bytes, dev_status, stream, true, false);
  if (st != MOE_OK || T == 0) return st;
  return run_up(j);
}

MOE_EXPORT moe_status moe_experts_down(const moe_cfg *cfg, int64_t T, moe_dtype x_dt,
                                       const moe_expert_weights *w, const int32_t *offsets,
                                       float *out_perm, float *out_shared, void *ws,
                                       size_t ws_bytes, int32_t *dev_status,
                                       moe_stream_t stream) {
  Job j;
  moe_status st = make_job(j, cfg, T, nullptr, x_dt, w, offsets, nullptr, out_perm, out_shared,
                           ws, ws_bytes, dev_status, stream, false, true);
  if (st != MOE_OK || T == 0) return st;
  return run_down(j);
}

MOE_EXPORT moe_status moe_experts_forward(const moe_cfg *cfg, int64_t T, const void *x,
                                          moe_dtype x_dt, const moe_expert_weights *w,
                                          const int32_t *offsets, const int32_t *sorted_token,
                                          float *out_perm, float *out_shared, void *ws,
                                          size_t ws_bytes, int32_t *dev_status,
                                          moe_stream_t stream) {
  Job j;
  moe_status st = make_job(j, cfg, T, x, x_dt, w, offsets, sorted_token, out_perm, out_shared,
                           ws, ws_bytes, dev_status, stream, true, true);
  if (st != MOE_OK || T == 0) return st;
  if ((st = run_up(j)) != MOE_OK) return st;
  return run_down(j);
}

MOE_EXPORT moe_status moe_experts_forward_combine(const moe_cfg *cfg, int64_t T, const void *x,
                                                  moe_dtype x_dt, const moe_expert_weights *w,
                                                  const int32_t *offsets,
                                                  const int32_t *sorted_token,
                                                  const int32_t *indices, const float *weights,
                                                  float *y, void *ws, size_t ws_bytes,
                                                  int32_t *dev_status, moe_stream_t stream) {
  Job j;
  // out_perm / out_shared are not used on this path; y stands in for the checks
  moe_status st = make_job(j, cfg, T, x, x_dt, w, offsets, sorted_token, y, y, ws, ws_bytes,
                           dev_status, stream, true, true);
  if (st != MOE_OK || T == 0) return st;
  if (!indices || !weights || !y) return MOE_ERR_INVALID;
  // the scatter adds 16-byte vectors into y
  if ((reinterpret_cast<uintptr_t>(y) & 15u) != 0) return MOE_ERR_INVALID;
  j.out_perm = nullptr;
  j.out_shared = nullptr;
  j.indices = indices;
  j.weights = weights;
  j.y = y;
  if (cudaMemsetAsync(y, 0, (size_t)T * cfg->dim * sizeof(float), j.s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((st = run_up(j)) != MOE_OK) return st;
  return run_down(j);
}

// The rank's share of the expert work (host only; no device call).
static moe_status ep_plan(const moe_cfg *cfg, int64_t T, const moe_ep_shard *shard, Shard *out) {
  if (check_cfg(cfg) != MOE_OK || !shard || T < 0) return MOE_ERR_INVALID;
  const int W = shard->world, r = shard->rank;
  if (W < 1 || r < 0 || r >= W) return MOE_ERR_INVALID;
  if (cfg->n_routed % W != 0) return MOE_ERR_UNSUPPORTED;
  const int per = cfg->n_routed / W;
  out->e0 = r * per;
  out->e1 = (r + 1) * per;
  out->st0 = (int)(T * r / W);
  out->st1 = (int)(T * (r + 1) / W);
  return MOE_OK;
}

MOE_EXPORT moe_status moe_ep_plan(const moe_cfg *cfg, int64_t T, const moe_ep_shard *shard,
                                  int32_t *out) {
  if (!out) return MOE_ERR_INVALID;
  Shard sh;
  const moe_status st = ep_plan(cfg, T, shard, &sh);
  if (st != MOE_OK) return st;
  out[0] = sh.e0;
  out[1] = sh.e1;
  out[2] = sh.st0;
  out[3] = sh.st1;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_experts_forward_combine_ep(
    const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt, const moe_expert_weights *w,
    const moe_ep_shard *shard, const int32_t *offsets, const int32_t *sorted_token,
    const int32_t *indices, const float *weights, float *y, void *ws, size_t ws_bytes,
    int32_t *dev_status, moe_stream_t stream) {
  Job j;
  moe_status st = make_job(j, cfg, T, x, x_dt, w, offsets, sorted_token, y, y, ws, ws_bytes,
                           dev_status, stream, true, true);
  if (st != MOE_OK) return st;
  Shard sh;
  if ((st = ep_plan(cfg, T, shard, &sh)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!indices || !weights || !y) return MOE_ERR_INVALID;
  // the scatter adds 16-byte vectors into y
  if ((reinterpret_cast<uintptr_t>(y) & 15u) != 0) return MOE_ERR_INVALID;
  j.out_perm = nullptr;
  j.out_shared = nullptr;
  j.indices = indices;
  j.weights = weights;
  j.y = y;
  j.sh = sh;
  j.sharded = shard->world > 1;
  if (cudaMemsetAsync(y, 0, (size_t)T * cfg->dim * sizeof(float), j.s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((st = run_up(j)) != MOE_OK) return st;
  return run_down(j);
}

MOE_EXPORT moe_status moe_quantize_e4m3_rows(const void *src, int64_t rows, int32_t K,
                                             uint8_t *q, float *scales, moe_stream_t stream) {
  if (rows < 0 || rows >= ((int64_t)1 << 31) || K <= 0 || K % 4 != 0) return MOE_ERR_INVALID;
  if (rows == 0) return MOE_OK;
  if (!src || !q || !scales) return MOE_ERR_INVALID;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (K % 8 == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(q) & 7u) == 0)
    quant_rows_e4m3_v8<false><<<grid, 256, 0, as_stream(stream)>>>(
        static_cast<const uint4 *>(src), nullptr, reinterpret_cast<uint2 *>(q), scales, 0,
        (int)rows, 1, K, nullptr, Shard{0, 0, 0, 0});
  else
    quant_rows_e4m3<false><<<grid, 256, 0, as_stream(stream)>>>(
        static_cast<const uint2 *>(src), nullptr, reinterpret_cast<uint32_t *>(q), scales, 0,
        (int)rows, 1, K, nullptr, Shard{0, 0, 0, 0});
  return launch_status();
}

MOE_EXPORT size_t moe_block_decode_workspace_size(const moe_cfg *cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  return decode_plan(cfg, T, 0).total;
}

MOE_EXPORT moe_status moe_block_forward_decode(
    const moe_cfg *cfg, int64_t T, const void *x, moe_dtype x_dt, const float *w_r,
    const float *bias, const moe_expert_weights *w, float *weights, int32_t *indices,
    float *sel_gap, int32_t *counts, int32_t *offsets, int32_t *sorted_token, int32_t *slot_of,
    float *y, void *ws, size_t ws_bytes, int32_t *dev_status, moe_stream_t stream) {
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID;
  if (!w) return MOE_ERR_INVALID;
  if (x_dt != MOE_BF16 || w->w_dt != MOE_BF16 || w->act_e4m3) return MOE_ERR_UNSUPPORTED;
  if (cfg->n_shared != 1 || cfg->n_routed > 256 || cfg->n_groups > 32 || cfg->topk > 32 ||
      cfg->dim % 128 != 0 || cfg->inter % 128 != 0)
    return MOE_ERR_UNSUPPORTED;
  // the decode regime: at most 16 rows per expert on average
  if (T * cfg->topk > (int64_t)16 * cfg->n_routed) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!x || !w_r || !weights || !indices || !counts || !offsets || !sorted_token || !slot_of ||
      !y || !ws || (cfg->has_bias && !bias))
    return MOE_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(y) & 15u) != 0) return MOE_ERR_INVALID;  // 16-byte reductions
  const DecodePlan pl = decode_plan(cfg, T, sm_count());
  if (ws_bytes < decode_plan(cfg, T, 0).total) return MOE_ERR_WORKSPACE;
  Job j;
  st = make_job(j, cfg, T, x, x_dt, w, offsets, sorted_token, y, y, static_cast<uint8_t *>(ws) + pl.ex_off,
                ws_bytes - pl.ex_off, dev_status, stream, true, true);
  if (st != MOE_OK) return st;
  j.out_perm = nullptr;
  j.out_shared = nullptr;
  j.indices = indices;
  j.weights = weights;
  j.y = y;
  return launch_decode_block<DC_BN, DC_ST>(j, pl, w_r, bias, weights, indices, sel_gap, counts,
                                           slot_of);
}

MOE_EXPORT moe_status moe_experts_set_profile_events(void *const *events, int32_t n) {
  if (n < 0 || n > 5 || (n > 0 && !events)) return MOE_ERR_INVALID;
  for (int i = 0; i < 5; ++i) g_prof[i] = i < n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  g_nprof = n;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_experts_selftest_wait(int64_t limit_ns, int32_t *dev_status,
                                                moe_stream_t stream) {
  if (limit_ns <= 0 || limit_ns > 2000000000LL || !dev_status) return MOE_ERR_INVALID;
  tc::selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns, dev_status);
  return launch_status();
}
