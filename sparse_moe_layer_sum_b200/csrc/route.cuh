// The router's arithmetic as device functions, shared by the moe_router
// kernels and the fused decode kernel of moe_experts:
//  * scores_tile: z = x W_r^T for one tile of tokens x experts over one split
//    of dim, fp32 FMAs in a fixed order (split partials are summed in split
//    order by select_token);
//  * select_token: for one token, s = sigmoid(z) (or softmax), c = s + bias,
//    the group scores (sum of the top two, or the top one without a bias),
//    the kept groups, the top-k experts among them (descending, ties to the
//    lower index), the gates (unbiased s, renormalised for sigmoid, times
//    route_scale) and the smallest decision gap.
// Page "DeepSeek-V3.2-Exp · Router": the four equations under "All 4 steps"
// and the gate-forward code excerpt under "Code".
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

namespace moe {
namespace {
namespace route {

constexpr int SC_BM = 64, SC_BN = 64, SC_BK = 16, SC_THREADS = 256;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// z_part[split][t][e] = sum over this split's columns d of x[t,d] * w[e,d].
// One tile (tokens m0.., experts n0.., split `split` of the columns) for
// SC_THREADS threads (threadIdx.x < SC_THREADS); xs and ws are shared-memory
// staging of SC_BK x (64 + 4) floats each.
template <typename XT>
__device__ __forceinline__ void scores_tile(const XT *__restrict__ x, const float *__restrict__ w,
                                            float *__restrict__ z_part, int T, int E, int D,
                                            int cols_per_split, int m0, int n0, int split,
                                            float (*xs)[SC_BM + 4], float (*ws)[SC_BN + 4]) {
  const int kbeg = split * cols_per_split;
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
  float *out = z_part + (size_t)split * T * E;
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

// An unsigned key with the order of the float v (larger v, larger key; -0
// taken as +0, as the float comparison does; no NaN), and back.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// warp_argmax on keys: the largest key, ties to the lowest index, in every
// lane; two warp reductions instead of five shuffle rounds of two values.
__device__ __forceinline__ void warp_argmax_key(uint32_t &key, int &i) {
  const uint32_t mk = __reduce_max_sync(0xffffffffu, key);
  i = (int)__reduce_min_sync(0xffffffffu, key == mk ? (uint32_t)i : 0xffffffffu);
  key = mk;
}

// Token t's selection by one warp with at most 8 experts per lane (E <= 256),
// each lane's scores in registers.  The same arithmetic, in the same order,
// and the same decisions (ties to the lower index) as the general form
// below; s is the warp's shared-memory row of E scores (for the gates).
__device__ __forceinline__ void select_token_e256(const SelectArgs &a, int t, float *s) {
  const int lane = threadIdx.x % 32;
  const int E = a.E;
  const float NEG_INF = -INFINITY;
  const uint32_t KEY_NEG_INF = order_key(NEG_INF);

  // z: split partials summed in split order, four splits' loads in flight
  float z[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) z[m] = 0.f;
  {
    const float *zt = a.z_part + (size_t)t * E;
    const size_t ps = (size_t)a.T * E;
    int p = 0;
    for (; p + 4 <= a.nsplit; p += 4) {
      float v[4][8];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int m = 0; m < 8; ++m)
          v[q][m] = lane + 32 * m < E ? zt[(p + q) * ps + lane + 32 * m] : 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int m = 0; m < 8; ++m) z[m] += v[q][m];
    }
    for (; p < a.nsplit; ++p)
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (lane + 32 * m < E) z[m] += zt[p * ps + lane + 32 * m];
  }
  // s = sigmoid(z) (or softmax), c = s + b
  float sr[8], cr[8];
  if (a.softmax) {
    float zmax = NEG_INF;
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (lane + 32 * m < E) zmax = fmaxf(zmax, z[m]);
    zmax = warp_max(zmax);
    float part = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (lane + 32 * m < E) {
        sr[m] = expf(z[m] - zmax);
        part += sr[m];
      }
    const float tot = warp_sum(part);
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (lane + 32 * m < E) sr[m] = sr[m] / tot;
  } else {
#pragma unroll
    for (int m = 0; m < 8; ++m)
      if (lane + 32 * m < E) sr[m] = 1.0f / (1.0f + expf(-z[m]));
  }
#pragma unroll
  for (int m = 0; m < 8; ++m)
    if (lane + 32 * m < E) {
      const int e = lane + 32 * m;
      cr[m] = a.bias ? sr[m] + a.bias[e] : sr[m];
      s[e] = sr[m];
    } else {
      cr[m] = NEG_INF;
    }

  // group selection
  const int P = E / a.G;
  float gap = INFINITY;
  uint32_t kept = 0xffffffffu;
  if (a.G > 1) {
    float gs = NEG_INF;  // lane q < G: the score of group q
    if (P == 32) {
      // group q is experts 32 q .. 32 q + 31: element q of every lane.  The
      // largest and (with a bias) the second largest, one instance of the
      // largest left out; their sum in that order
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= a.G) break;
        const uint32_t kq = order_key(cr[q]);
        const uint32_t k1 = __reduce_max_sync(0xffffffffu, kq);
        float g = key_value(k1);
        if (a.bias) {
          const uint32_t l1 = __reduce_min_sync(0xffffffffu, kq == k1 ? (uint32_t)lane : 32u);
          const uint32_t k2 = __reduce_max_sync(0xffffffffu, lane == (int)l1 ? 0u : kq);
          g = g + key_value(k2);
        }
        if (lane == q) gs = g;
      }
    } else {
      // a lane per group scans its P experts (as the general form)
      float *c = s + E;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (lane + 32 * m < E) c[lane + 32 * m] = cr[m];
      __syncwarp();
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
    }
    kept = 0;
    float prev = 0.f;
    const int rounds = a.Gk < a.G ? a.Gk + 1 : a.Gk;
    for (int r = 0; r < rounds; ++r) {
      const bool open = lane < a.G && !((kept >> lane) & 1u);
      uint32_t k = open ? order_key(gs) : KEY_NEG_INF;
      int i = open ? lane : 0x7fffffff;
      warp_argmax_key(k, i);
      const float v = key_value(k);
      if (r < a.Gk) {
        kept |= 1u << i;
        prev = v;
      } else {
        gap = fminf(gap, prev - v);  // last kept group minus best dropped group
      }
    }
  }

  // expert selection over the kept groups: k arg-max rounds plus one for
  // the first expert left out
  uint32_t ck[8];  // keys of the candidates (-inf outside the kept groups)
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int e = lane + 32 * m;
    ck[m] = e < E && ((kept >> (e / P)) & 1u) ? order_key(cr[m]) : KEY_NEG_INF;
  }
  uint32_t taken = 0;  // bit m: expert lane + 32 m already chosen
  float prev_v = 0.f;
  int chosen_i = 0;
  const int rounds = a.k < E ? a.k + 1 : a.k;
  for (int r = 0; r < rounds; ++r) {
    uint32_t k = KEY_NEG_INF;
    int i = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e = lane + 32 * m;
      if (e >= E || ((taken >> m) & 1u)) continue;
      if (ck[m] > k || (ck[m] == k && e < i)) {
        k = ck[m];
        i = e;
      }
    }
    warp_argmax_key(k, i);
    const float v = key_value(k);
    if (r < a.k) {
      if (i % 32 == lane) taken |= 1u << (i / 32);
      if (r > 0) gap = fminf(gap, prev_v - v);  // consecutive chosen experts
      prev_v = v;
      if (lane == r) chosen_i = i;
    } else {
      gap = fminf(gap, prev_v - v);  // k-th chosen minus first left out
    }
  }
  __syncwarp();

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

// The general form (any E up to 1024): s and c are the warp's shared-memory
// rows of E floats (the scores and the biased scores).
__device__ __forceinline__ void select_token_general(const SelectArgs &a, int t, float *s,
                                                     float *c) {
  const int lane = threadIdx.x % 32;
  const int E = a.E;
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

// Token t's selection by one warp; s and c are that warp's shared-memory
// rows of E floats.
__device__ __forceinline__ void select_token(const SelectArgs &a, int t, float *s, float *c) {
  if (a.E <= 256)
    select_token_e256(a, t, s);
  else
    select_token_general(a, t, s, c);
}

}  // namespace route
}  // namespace
}  // namespace moe
