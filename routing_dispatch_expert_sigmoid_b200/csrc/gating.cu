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
#include "gating.cuh"

namespace moe {
namespace {

using gating::GatingArgs;

constexpr int kWarpsPerBlock = 4;

template <int NPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_gating(GatingArgs g) {
  grid_dependency();  // the previous grid is complete; the next may launch
  extern __shared__ float s_u_all[];  // [kWarpsPerBlock][E], sigmoid mode only
  const int warp = threadIdx.x / 32;
  const int t = blockIdx.x * kWarpsPerBlock + warp;
  if (t >= g.T) return;  // whole warp leaves together
  gating::gate_token<NPL>(g, t, g.logits + (size_t)t * g.E, s_u_all + warp * g.E);
}

template <int NPL>
cudaError_t run(const GatingArgs &a, cudaStream_t s) {
  const int blocks = (a.T + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const size_t smem =
      a.mode == MOE_SIGMOID_GROUPED ? sizeof(float) * kWarpsPerBlock * (size_t)a.E : 0;
  launch_k(k_gating<NPL>, blocks, kWarpsPerBlock * 32, smem, s, a);
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
