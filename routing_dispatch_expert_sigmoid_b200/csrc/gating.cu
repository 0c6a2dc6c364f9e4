// K2 -- gating: per token, choose k_t experts and their combine weights.
//
// "Paralelismo experto para el servicio MoE", "Buceo profundo" and FAQ: each
// token keeps its top-k experts; "Expert Parallelism: MoE 模型的并行切分",
// section 12 question 2: outputs are combined weighted by the router weight;
// "MoE-Prism" summary, section 2.B: the routing budget k is a per-request
// runtime control (k_per_token).  Sigmoid scores with a selection bias and
// group-limited routing follow the DeepSeek-V3-shaped workload specification.
//
// One warp per token.  Lane l holds experts l, l+32, l+64, ... (NPL of them),
// so the logits row is read with coalesced 128-byte transactions.  Each of
// the k_t selection rounds is a lane-local scan plus a 5-step butterfly
// argmax over (key, index) pairs: larger key wins, equal keys go to the lower
// index.  Group scores (sigmoid mode) are computed one group per lane from a
// per-warp copy of the biased scores in shared memory.
//
// The sigmoid is the specified fp32 function: Cody & Waite additive range
// reduction, degree-7 Taylor polynomial of e^r by Horner's rule with one
// fused multiply-add per step, scaling by 2^n through the exponent field,
// sigma(z) = 1 / (1 + e^-z) with an IEEE division.  Every operation is an
// explicitly rounded intrinsic so the compiler cannot contract or reorder it,
// and the result is bit-identical to any IEEE implementation of the same
// sequence.  Constants (derived from their definitions):
//   log2(e) rounded to binary32; ln 2 rounded to 12 significant bits
//   (2839/4096, so n * hi is exact); the binary32 rounding of
//   ln 2 - 2839/4096; and 1/k! rounded to binary32 for k = 2..7.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

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

// Is candidate (k1, i1) ranked ahead of (k0, i0)?
__device__ __forceinline__ bool ahead(float k1, int i1, float k0, int i0) {
  return k1 > k0 || (k1 == k0 && i1 < i0);
}

__device__ __forceinline__ void warp_argmax(float &key, int &idx) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float ok = __shfl_xor_sync(kFull, key, off);
    int oi = __shfl_xor_sync(kFull, idx, off);
    if (ahead(ok, oi, key, idx)) {
      key = ok;
      idx = oi;
    }
  }
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

constexpr int kWarpsPerBlock = 4;

template <int NPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_gating(GatingArgs g) {
  extern __shared__ float s_u_all[];  // [kWarpsPerBlock][E], sigmoid mode only
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kWarpsPerBlock + warp;
  if (t >= g.T) return;  // whole warp leaves together
  const int E = g.E;
  const float *l = g.logits + (size_t)t * E;

  float key[NPL], val[NPL];  // val: logit (softmax modes) or sigmoid score
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
  }

  int kt = g.k_per_token ? g.k_per_token[t] : g.k_max;
  if (kt < 1 || kt > g.k_max) {
    if (lane == 0) raise_error(g.err, kErrRouting);
    kt = kt < 1 ? 1 : g.k_max;
  }

  if (g.mode == MOE_SIGMOID_GROUPED) {
    // Group scores: lane g sums, in descending order, the group_score_topk
    // largest biased scores of group g; then keep the topk_groups best groups.
    float *s_u = s_u_all + warp * E;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = i * 32 + lane;
      if (e < E) s_u[e] = key[i];
    }
    __syncwarp();
    const int gsz = E / g.n_groups, m = g.group_score_topk;
    float gscore = -INFINITY;
    int gidx = 0x7fffffff;
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
      gscore = sc;
      gidx = lane;
    }
    uint32_t kept_groups = 0;
    for (int r = 0; r < g.topk_groups; ++r) {
      float bk = gscore;
      int bi = gidx;
      warp_argmax(bk, bi);
      kept_groups |= 1u << bi;
      if (bi == lane) {
        gscore = -INFINITY;
        gidx = 0x7fffffff;
      }
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
  for (int j = 0; j < kt; ++j) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
    float bv = 0.f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (((alive >> i) & 1u) && (key[i] > bk || bi == 0x7fffffff)) {
        bk = key[i];
        bi = i * 32 + lane;
        bv = val[i];
      }
    }
    warp_argmax(bk, bi);
    if (bi == 0x7fffffff) break;  // fewer candidates than k_t (rejected on the host)
    const int owner = bi & 31;
    const float v = __shfl_sync(kFull, bv, owner);
    if (lane == owner) alive &= ~(1u << (bi >> 5));
    if (lane == j) {
      my_idx = bi;
      my_val = v;
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

template <int NPL>
cudaError_t run(const GatingArgs &a, cudaStream_t s) {
  const int blocks = (a.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const size_t smem =
      a.mode == MOE_SIGMOID_GROUPED ? sizeof(float) * kWarpsPerBlock * (size_t)a.E : 0;
  k_gating<NPL><<<blocks, kWarpsPerBlock * 32, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gating(const moe_config &c, const float *logits, const float *sel_bias,
                          const int32_t *k_per_token, int32_t *topk_idx, float *topk_w,
                          uint32_t *err, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  GatingArgs a{logits,  sel_bias, k_per_token, topk_idx,      topk_w,
               c.T,     c.E,      c.k_max,     c.gating,      c.n_groups,
               c.topk_groups,     c.group_score_topk, c.routed_scale, err};
  const int npl = (c.E + 31) / 32;
  if (npl <= 1) return run<1>(a, s);
  if (npl <= 2) return run<2>(a, s);
  if (npl <= 4) return run<4>(a, s);
  if (npl <= 8) return run<8>(a, s);
  if (npl <= 16) return run<16>(a, s);
  return run<32>(a, s);
}

}  // namespace moe
