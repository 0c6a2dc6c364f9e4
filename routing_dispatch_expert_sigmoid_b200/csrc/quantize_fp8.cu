// FP8 weight preparation: per output column of each expert matrix, an fp32
// scale and e4m3 codes, stored K-contiguous for the GEMMs.
//
// "LLM MoE Expert Parallel 生产实战", section 5: DeepSeek-V3 is served with
// fp8 quantisation; section 10: the router head must not be disturbed by it,
// so only the experts' matrices are quantised.  For W [G, K, N] (bf16):
//   scale[g, n] = max_k |W[g, k, n]| / 448      (fp32 division; 1 if all zero)
//   Wq[g, n, k] = e4m3(W[g, k, n] / scale[g, n]) (fp32 quotient, round to
//                                                 nearest even, saturating)
// 448 is the largest finite e4m3 magnitude, so each column's largest weight
// takes the largest code.  The conversion is the hardware's rounding
// conversion (cvt with .satfinite) through cuda_fp8.h.  The codes are the
// transpose of W: the K codes of one output column are contiguous, which is
// the order in which the GEMMs widen them (one column per converter thread).
//
// A block takes 32 columns of one group: 8 threads per column find the
// column maxima, then 32 x 32 tiles of W pass through shared memory so that
// both the reads of W (along N) and the writes of Wq (along K) are whole
// rows.  It runs once per weight set, off the hot path.
#include <cuda_fp8.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kCols = 32;

__global__ void __launch_bounds__(256)
    k_quantize_fp8(const __nv_bfloat16 *__restrict__ W, int K, int N, uint8_t *__restrict__ Wq,
                   float *__restrict__ scale) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ float s_max[8][kCols];
  __shared__ float s_scale[kCols];
  __shared__ uint8_t s_tile[kCols][kCols + 4];  // [n][k]
  const int g = blockIdx.y, n0 = blockIdx.x * kCols;
  const int tx = threadIdx.x % kCols, ty = threadIdx.x / kCols;  // ty: 0..7
  const __nv_bfloat16 *Wg = W + (size_t)g * K * N;
  const int n = n0 + tx;
  float amax = 0.0f;
  if (n < N)
    for (int k = ty; k < K; k += 8) {
      const float a = fabsf(__bfloat162float(Wg[(size_t)k * N + n]));
      if (a > amax) amax = a;  // NaN never wins
    }
  s_max[ty][tx] = amax;
  __syncthreads();
  if (ty == 0) {
    float m = s_max[0][tx];
    for (int i = 1; i < 8; ++i) m = s_max[i][tx] > m ? s_max[i][tx] : m;
    const float s = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
    s_scale[tx] = s;
    if (n < N) scale[(size_t)g * N + n] = s;
  }
  __syncthreads();
  uint8_t *Qg = Wq + (size_t)g * N * K;
  for (int k0 = 0; k0 < K; k0 += kCols) {
    // load and quantise a 32 (k) x 32 (n) tile: thread (tx, ty) takes n0+tx, k0+ty+8i
    for (int i = ty; i < kCols; i += 8) {
      const int k = k0 + i;
      uint8_t code = 0;
      if (k < K && n < N) {
        const float q = __fdiv_rn(__bfloat162float(Wg[(size_t)k * N + n]), s_scale[tx]);
        code = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
      }
      s_tile[tx][i] = code;
    }
    __syncthreads();
    // write it transposed: thread (tx, ty) writes Wq[n0+ty+8i][k0+tx]
    for (int i = ty; i < kCols; i += 8) {
      const int nn = n0 + i, k = k0 + tx;
      if (nn < N && k < K) Qg[(size_t)nn * K + k] = s_tile[i][tx];
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(int G, int K, int N, const void *W, uint8_t *Wq, float *scale,
                                cudaStream_t s) {
  if ((long long)G * K * N == 0) return cudaSuccess;
  const dim3 grid((N + kCols - 1) / kCols, G);
  launch_k(k_quantize_fp8, grid, 256, 0, s, static_cast<const __nv_bfloat16 *>(W), K, N, Wq, scale);
  return cudaGetLastError();
}

}  // namespace moe
