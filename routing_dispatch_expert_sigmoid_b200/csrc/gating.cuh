// Per-token gating shared by the gating kernel (K2) and the fused small-batch
// routing kernel: the specified fp32 sigmoid, the (key, index) ordering and
// the selection of k_t experts with their combine weights for one token, run
// by one warp.  Constants and the arithmetic are described in gating.cu.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace gating {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float spec_expf(float z) {
  const float kLog2e = 1.44269502162933349609375f;   // 0x3FB8AA3B
  const float kLn2Hi = 0.693115234375f;              // 2839 / 4096 = 0x3F317000
  const float kLn2Lo = 3.19461832987144589424133e-05f; // 0x3805FDF4
  const float kC7 = 1.98412701138295233249664e-04f;  // 1/5040 -> 0x39500D01
  const float kC6 = 1.38888892251998186111450e-03f;  // 1/720  -> 0x3AB60B61
  const float kC5 = 8.33333376795053482055664e-03f;  // 1/120  -> 0x3C088889
  const float kC4 = 4.16666679084300994873047e-02f;  // 1/24   -> 0x3D2AAAAB
  const float kC3 = 1.66666671633720397949219e-01f;  // 1/6    -> 0x3E2AAAAB
  z = z > 87.0f ? 87.0f : z;
  z = z < -87.0f ? -87.0f : z;
  const float n = rintf(__fmul_rn(z, kLog2e));
  float r = __fmaf_rn(-n, kLn2Hi, z);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = kC7;
  p = __fmaf_rn(p, r, kC6);
  p = __fmaf_rn(p, r, kC5);
  p = __fmaf_rn(p, r, kC4);
  p = __fmaf_rn(p, r, kC3);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ni = static_cast<int>(n);
  return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float spec_sigmoidf(float z) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, spec_expf(-z)));
}

// Selection keys as unsigned integers in the fp32 order of the keys, -0 and
// +0 equal (both rank as +0).  0 is below every key and stands for "no
// candidate" (a negative NaN that would map there is moved up to 1).
__device__ __forceinline__ uint32_t order_key(float k) {
  uint32_t b = __float_as_uint(k);
  if (b == 0x80000000u) b = 0u;
  const uint32_t u = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return u ? u : 1u;
}

// The warp's best candidate: lane candidates (ordered key u, index i; u == 0
// for none) are ranked by larger key, then lower index.  Two warp reductions
// (the largest key, then the lowest index holding it).  -1 if no lane has a
// candidate.
__device__ __forceinline__ int warp_best(uint32_t u, int i) {
  const uint32_t top = __reduce_max_sync(kFull, u);
  if (top == 0u) return -1;
  return __reduce_min_sync(kFull, u == top ? i : 0x7fffffff);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}

struct GatingArgs {
  const float *logits;
  const float *sel_bias;
  const int32_t *k_per_token;
  int32_t *topk_idx;
  float *topk_w;
  int T, E, k_max, mode, n_groups, topk_groups, group_score_topk;
  float routed_scale;
  uint32_t *err;
};

// One warp chooses token t's experts and weights from its logits row `l`
// (E fp32 values) and writes topk_idx/topk_w[t, :]; `s_u` is E floats of
// this warp's shared memory (sigmoid mode only).
template <int NPL>
__device__ __forceinline__ void gate_token(const GatingArgs &g, int t, const float *l, float *s_u) {
  const int lane = threadIdx.x % 32;
  const int E = g.E;

  float key[NPL], val[NPL];  // val: logit (softmax modes) or sigmoid score
  uint32_t ku[NPL];          // key[i] as an ordered integer
  uint32_t alive = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = i * 32 + lane;
    key[i] = -INFINITY;
    val[i] = 0.f;
    if (e < E) {
      const float v = l[e];
      alive |= 1u << i;
      if (g.mode == MOE_SIGMOID_GROUPED) {
        const float s = spec_sigmoidf(v);
        val[i] = s;
        key[i] = __fadd_rn(s, g.sel_bias ? g.sel_bias[e] : 0.0f);
      } else {
        val[i] = v;
        key[i] = v;
      }
    }
    ku[i] = order_key(key[i]);
  }

  int kt = g.k_per_token ? g.k_per_token[t] : g.k_max;
  if (kt < 1 || kt > g.k_max) {
    if (lane == 0) raise_error(g.err, kErrRouting);
    kt = kt < 1 ? 1 : g.k_max;
  }

  if (g.mode == MOE_SIGMOID_GROUPED) {
    const int gsz = E / g.n_groups, m = g.group_score_topk;
    uint32_t gu = 0;  // lane g: group g's score, ordered (0: no group)
    if (gsz == 32) {
      // Group gi is register gi across the 32 lanes (experts 32*gi + lane):
      // its m largest biased scores come out of m rounds of warp reductions,
      // largest first, equal scores in lane (expert) order, and are added in
      // that order.
#pragma unroll
      for (int gi = 0; gi < NPL; ++gi) {
        if (gi < g.n_groups) {
          uint32_t taken = 0;
          float sc = 0.f;
          for (int j = 0; j < m; ++j) {
            const uint32_t u = ((taken >> lane) & 1u) ? 0u : ku[gi];
            const uint32_t top = __reduce_max_sync(kFull, u);
            const int w = __reduce_min_sync(kFull, u == top ? lane : 32);
            taken |= 1u << w;
            const float v = __shfl_sync(kFull, key[gi], w);
            sc = j == 0 ? v : __fadd_rn(sc, v);
          }
          if (lane == gi) gu = order_key(sc);
        }
      }
    } else {
      // Lane g sums, in descending order, the group_score_topk largest
      // biased scores of group g (from a copy of the scores in shared memory).
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) s_u[e] = key[i];
      }
      __syncwarp();
      if (lane < g.n_groups) {
        float top[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) top[q] = -INFINITY;
        for (int e = lane * gsz; e < (lane + 1) * gsz; ++e) {
          float v = s_u[e];
          // insert v into the descending list top[0..m-1]
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (q < m && v > top[q]) {
              const float tmp = top[q];
              top[q] = v;
              v = tmp;
            }
          }
        }
        float sc = top[0];
#pragma unroll
        for (int q = 1; q < 8; ++q)
          if (q < m) sc = __fadd_rn(sc, top[q]);
        gu = order_key(sc);
      }
    }
    // then keep the topk_groups best groups
    uint32_t kept_groups = 0;
    for (int r = 0; r < g.topk_groups; ++r) {
      const int win = warp_best(gu, lane);
      if (win < 0) break;
      kept_groups |= 1u << win;
      if (win == lane) gu = 0;
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = i * 32 + lane;
      if (e < E && !((kept_groups >> (e / gsz)) & 1u)) alive &= ~(1u << i);
    }
  }

  // k_t rounds of warp argmax; lane j keeps slot j.
  int my_idx = -1;
  float my_val = 0.f;
  if constexpr (NPL >= 8) {
    // Wide rows: each lane keeps its kCache best alive candidates in order
    // (larger key first, lower index among equals).  A round compares the
    // lanes' heads; the winning lane drops its head, and a lane whose cache
    // runs dry while candidates remain refills it from the rest.  The heads
    // are always the lanes' best remaining candidates, so the winners and
    // their order are those of scanning every candidate each round, for
    // a quarter of the scans.
    constexpr int kCache = 4;
    uint32_t cu[kCache];
    int ci[kCache];
    float cv[kCache];
    uint32_t pool = alive;  // alive candidates not yet in the cache
    auto fill = [&]() {
#pragma unroll
      for (int q = 0; q < kCache; ++q) {
        uint32_t bu = 0;
        int bi = 0;
        float bv = 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          if (((pool >> i) & 1u) && ku[i] > bu) {
            bu = ku[i];
            bi = i;
            bv = val[i];
          }
        }
        cu[q] = bu;
        ci[q] = bi;
        cv[q] = bv;
        if (bu) pool &= ~(1u << bi);
      }
    };
    fill();
    for (int j = 0; j < kt; ++j) {
      const int win = warp_best(cu[0], cu[0] ? ci[0] * 32 + lane : 0x7fffffff);
      if (win < 0) break;  // fewer candidates than k_t (rejected on the host)
      const int owner = win & 31;
      const float v = __shfl_sync(kFull, cv[0], owner);
      if (lane == owner) {
#pragma unroll
        for (int q = 0; q + 1 < kCache; ++q) {
          cu[q] = cu[q + 1];
          ci[q] = ci[q + 1];
          cv[q] = cv[q + 1];
        }
        cu[kCache - 1] = 0;
      }
      if (lane == j) {
        my_idx = win;
        my_val = v;
      }
      const bool dry = cu[0] == 0 && pool != 0;
      if (__any_sync(kFull, dry) && dry) fill();
    }
  } else {
    for (int j = 0; j < kt; ++j) {
      uint32_t bu = 0;  // this lane's best alive candidate (the lowest i among equals)
      int bi = 0x7fffffff;
      float bv = 0.f;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if (((alive >> i) & 1u) && ku[i] > bu) {
          bu = ku[i];
          bi = i * 32 + lane;
          bv = val[i];
        }
      }
      const int win = warp_best(bu, bi);
      if (win < 0) break;  // fewer candidates than k_t (rejected on the host)
      const int owner = win & 31;
      const float v = __shfl_sync(kFull, bv, owner);
      if (lane == owner) alive &= ~(1u << (win >> 5));
      if (lane == j) {
        my_idx = win;
        my_val = v;
      }
    }
  }

  // Weights.
  float w = 0.f;
  const bool mine = lane < kt;
  if (g.mode == MOE_TOPK_SOFTMAX) {
    const float top = __shfl_sync(kFull, my_val, 0);
    const float ex = mine ? expf(my_val - top) : 0.f;
    w = ex / warp_sum(ex);
  } else if (g.mode == MOE_SOFTMAX_TOPK_RENORM) {
    const float top = __shfl_sync(kFull, my_val, 0);  // the largest logit of the row
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (i * 32 + lane < E) z += expf(l[i * 32 + lane] - top);
    z = warp_sum(z);
    const float p = mine ? expf(my_val - top) / z : 0.f;
    w = p / warp_sum(p);
  } else {
    const float s = mine ? my_val : 0.f;
    w = g.routed_scale * s / warp_sum(s);
  }
  if (lane < g.k_max) {
    g.topk_idx[(size_t)t * g.k_max + lane] = mine ? my_idx : -1;
    g.topk_w[(size_t)t * g.k_max + lane] = mine ? w : 0.f;
  }
}

}  // namespace gating
}  // namespace moe
