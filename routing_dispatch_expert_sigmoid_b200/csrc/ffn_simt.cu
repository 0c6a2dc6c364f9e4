// K9 -- fp32 grouped SwiGLU FFN on the CUDA cores, for layers stored in fp32.
//
// "LLM MoE Expert Parallel 生产实战", section "为什么 MoE 推理会慢在'最热专家'",
// step 3: every expert runs its FFN on the rows routed to it.  Rows of group
// g are offsets[g]..offsets[g+1]-1 (the expert-contiguous layout of the
// dispatch step).  fp32 tensors have no bf16 tensor-core path; the fp32
// workload is the small correctness configuration, so a tiled fp32 FMA GEMM
// (64 x 64 tiles, 4 x 4 outputs per thread) is enough.
//   pass 1 (swiglu): h[r, n] = silu(sum_k A[r,k] W1[g,k,n]) * (sum_k A[r,k] W3[g,k,n])
//   pass 2 (plain):  y[r, n] = sum_k h[r,k] W2[g,k,n]
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <bool SWIGLU>
__global__ void __launch_bounds__(256)
    k_ffn_f32(const float *__restrict__ A, const float *__restrict__ B1,
              const float *__restrict__ B3, float *__restrict__ C, const int32_t *offsets,
              int fixed_rows, int K, int N) {
  __shared__ float as[BK][BM + 4];
  __shared__ float b1s[BK][BN];
  __shared__ float b3s[SWIGLU ? BK : 1][BN];
  const int g = blockIdx.z;
  const int r0 = offsets ? offsets[g] : 0;
  const int rows = offsets ? offsets[g + 1] - r0 : fixed_rows;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  if (m0 >= rows) return;
  const float *Bg1 = B1 + (size_t)g * K * N;
  const float *Bg3 = SWIGLU ? B3 + (size_t)g * K * N : nullptr;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc1[4][4], acc3[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc1[i][j] = acc3[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const int m = m0 + r, k = k0 + kk;
      as[kk][r] = (m < rows && k < K) ? A[(size_t)(r0 + m) * K + k] : 0.f;
    }
    for (int i = tid; i < BK * BN; i += 256) {
      const int kk = i / BN, c = i % BN;
      const int k = k0 + kk, n = n0 + c;
      const bool in = k < K && n < N;
      b1s[kk][c] = in ? Bg1[(size_t)k * N + n] : 0.f;
      if (SWIGLU) b3s[kk][c] = in ? Bg3[(size_t)k * N + n] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b1[4], b3[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = as[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b1[j] = b1s[kk][tx * 4 + j];
        if (SWIGLU) b3[j] = b3s[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
          if (SWIGLU) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc1[i][j];
      if (SWIGLU) v = (v / (1.0f + expf(-v))) * acc3[i][j];
      C[(size_t)(r0 + m) * N + n] = v;
    }
  }
}

}  // namespace

cudaError_t launch_ffn_simt_f32(int rows_cap, int d, int f, int G, const int32_t *offsets,
                                int fixed_rows, const float *x_perm, const float *W1,
                                const float *W3, const float *W2, float *h, float *y,
                                cudaStream_t s) {
  // A group never holds more rows than the buffer, so rows_cap bounds the M grid.
  const int max_rows = offsets ? rows_cap : fixed_rows;
  if (max_rows == 0 || G == 0) return cudaSuccess;
  dim3 g1((f + BN - 1) / BN, (max_rows + BM - 1) / BM, G);
  k_ffn_f32<true><<<g1, 256, 0, s>>>(x_perm, W1, W3, h, offsets, fixed_rows, d, f);
  dim3 g2((d + BN - 1) / BN, (max_rows + BM - 1) / BM, G);
  k_ffn_f32<false><<<g2, 256, 0, s>>>(h, W2, nullptr, y, offsets, fixed_rows, f, d);
  return cudaGetLastError();
}

}  // namespace moe
