// K8 at decode size -- the shared expert split along K.
//
// "LLM MoE Expert Parallel 生产实战", section 5: DeepSeek-V3 adds one always-on
// shared expert to the routed ones; every token runs it.  Its FFN is a plain
// SwiGLU of the T token rows:
//   h = silu(x . Ws1) * (x . Ws3),   y_sh = h . Ws2.
// With a decode-sized batch (T <= 256 rows: one or two 128-row tiles) the
// two projections make too few output tiles to stream the weights with the
// whole GPU (16 tiles of 128 columns for a 2048-wide expert).  Both are then
// split along K: split s of a projection multiplies the rows by weight rows
// s*K/S .. (s+1)*K/S-1 and writes fp32 partial sums [S][T][N]; the SwiGLU
// kernel below adds the up projection's S partial sums of the gate and of the
// up operand in split order before the activation, and the combine adds the
// down projection's partial sums (one part when the down projection has
// enough tiles unsplit).
#include <stdlib.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kTargetCtas = 148;  // one wave of CTAs on a B200

int env_disabled() {
  const char *env = getenv("MOE_SHARED_SPLIT");
  return env && env[0] == '0';
}

// Largest divisor s of kb (the number of 64-deep K blocks) with
// s * tiles <= kTargetCtas, at most 16.
int pick_splits(int kb, long long tiles) {
  int best = 1;
  for (int s = 1; s <= 16 && s <= kb; ++s)
    if (kb % s == 0 && s * tiles <= kTargetCtas) best = s;
  return best;
}

__global__ void __launch_bounds__(256)
    k_swiglu_parts(const float4 *__restrict__ gate, const float4 *__restrict__ up, int parts,
                   long long n4, uint2 *__restrict__ h) {
  grid_dependency();  // the previous grid is complete; the next may launch
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    float4 a = gate[i], b = up[i];
    for (int s = 1; s < parts; ++s) {
      const float4 ga = gate[(size_t)s * n4 + i], ub = up[(size_t)s * n4 + i];
      a.x += ga.x;
      a.y += ga.y;
      a.z += ga.z;
      a.w += ga.w;
      b.x += ub.x;
      b.y += ub.y;
      b.z += ub.z;
      b.w += ub.w;
    }
    // the same SiLU as the grouped GEMM's SwiGLU epilogue
    const float v0 = silu_times(a.x, b.x);
    const float v1 = silu_times(a.y, b.y);
    const float v2 = silu_times(a.z, b.z);
    const float v3 = silu_times(a.w, b.w);
    __nv_bfloat162 p01 = __floats2bfloat162_rn(v0, v1), p23 = __floats2bfloat162_rn(v2, v3);
    h[i] = make_uint2(*reinterpret_cast<uint32_t *>(&p01), *reinterpret_cast<uint32_t *>(&p23));
  }
}

}  // namespace

SharedSplitPlan shared_split_plan(const moe_config &c) {
  SharedSplitPlan p;
  if (c.f_shared <= 0 || c.dtype != MOE_BF16 || env_disabled()) return p;
  const long long row_tiles = (c.T + 127) / 128;
  if (row_tiles > 2 || c.d % 64 || c.f_shared % 64) return p;
  // 256-column output tiles: each CTA reads its slice of x once for 256
  // columns (narrower tiles would re-read it from L2 once per 64 columns)
  const int bn = 256;
  const long long up_tiles = row_tiles * ((c.f_shared + bn - 1) / bn);
  const long long dn_tiles = row_tiles * ((c.d + bn - 1) / bn);
  p.s_up = pick_splits(c.d / 64, up_tiles);
  p.s_down = pick_splits(c.f_shared / 64, dn_tiles);
  p.use = p.s_up >= 2;
  return p;
}

size_t shared_split_bytes(const moe_config &c) {
  const SharedSplitPlan p = shared_split_plan(c);
  if (!p.use) return 0;
  size_t b = 2 * (size_t)p.s_up * c.T * c.f_shared * sizeof(float);
  if (p.s_down > 1) b += (size_t)p.s_down * c.T * c.d * sizeof(float);
  return b;
}

cudaError_t launch_shared_split(const moe_config &c, const SharedSplitPlan &p, bool fp8,
                                const void *x, const void *W1, const void *W3, const void *W2,
                                const float *s1, const float *s3, const float *s2, void *h,
                                float *y_sh, void *scratch, const float **shared_y,
                                int *shared_parts, uint32_t *err, cudaStream_t s) {
  float *pg = static_cast<float *>(scratch);
  float *pu = pg + (size_t)p.s_up * c.T * c.f_shared;
  float *pd = pu + (size_t)p.s_up * c.T * c.f_shared;
  cudaError_t e;
  e = launch_gemm_split(fp8, c.T, c.d, c.f_shared, p.s_up, x, W1, s1, pg, err, s);
  if (e != cudaSuccess) return e;
  e = launch_gemm_split(fp8, c.T, c.d, c.f_shared, p.s_up, x, W3, s3, pu, err, s);
  if (e != cudaSuccess) return e;
  const long long n4 = (long long)c.T * c.f_shared / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 4 * kTargetCtas) blocks = 4 * kTargetCtas;
  launch_k(k_swiglu_parts, (int)blocks, 256, 0, s, reinterpret_cast<const float4 *>(pg),
                                              reinterpret_cast<const float4 *>(pu), p.s_up, n4,
                                              static_cast<uint2 *>(h));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  float *yd = p.s_down > 1 ? pd : y_sh;
  e = launch_gemm_split(fp8, c.T, c.f_shared, c.d, p.s_down, h, W2, s2, yd, err, s);
  if (e != cudaSuccess) return e;
  *shared_y = yd;
  *shared_parts = p.s_down;
  return cudaSuccess;
}

}  // namespace moe
