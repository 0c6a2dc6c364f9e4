// FP8 weight preparation: per output column of each expert matrix, an fp32
// scale and e4m3 codes.
//
// "LLM MoE Expert Parallel 生产实战", section 5: DeepSeek-V3 is served with
// fp8 quantisation; section 10: the router head must not be disturbed by it,
// so only the experts' matrices are quantised.  For W [G, K, N] (bf16):
//   scale[g, n] = max_k |W[g, k, n]| / 448      (fp32 division; 1 if all zero)
//   Wq[g, k, n] = e4m3(W[g, k, n] / scale[g, n]) (fp32 quotient, round to
//                                                 nearest even, saturating)
// 448 is the largest finite e4m3 magnitude, so each column's largest weight
// takes the largest code.  The conversion is the hardware's rounding
// conversion (cvt with .satfinite) through cuda_fp8.h.
//
// One thread per column: a first pass over K for the maximum, a second to
// write the codes.  Threads of a block take consecutive columns, so every
// pass reads and writes whole rows of W and Wq.  It runs once per weight
// set, off the hot path.
#include <cuda_fp8.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256)
    k_quantize_fp8(const __nv_bfloat16 *__restrict__ W, int K, int N, uint8_t *__restrict__ Wq,
                   float *__restrict__ scale) {
  const int g = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const size_t base = (size_t)g * K * N + n;
  float amax = 0.0f;
  for (int k = 0; k < K; ++k) {
    const float a = fabsf(__bfloat162float(W[base + (size_t)k * N]));
    if (a > amax) amax = a;  // NaN never wins
  }
  const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  scale[(size_t)g * N + n] = s;
  for (int k = 0; k < K; ++k) {
    const float q = __fdiv_rn(__bfloat162float(W[base + (size_t)k * N]), s);
    Wq[base + (size_t)k * N] = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(int G, int K, int N, const void *W, uint8_t *Wq, float *scale,
                                cudaStream_t s) {
  if ((long long)G * K * N == 0) return cudaSuccess;
  const dim3 grid((N + 255) / 256, G);
  k_quantize_fp8<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(W), K, N, Wq, scale);
  return cudaGetLastError();
}

}  // namespace moe
