// K9 -- fp32 grouped SwiGLU FFN on the CUDA cores, for layers stored in fp32.
//
// "LLM MoE Expert Parallel 生产实战", section "为什么 MoE 推理会慢在'最热专家'",
// step 3: every expert runs its FFN on the rows routed to it.  Rows of group
// g are offsets[g]..offsets[g+1]-1 (the expert-contiguous layout of the
// dispatch step).  fp32 tensors have no bf16 tensor-core path; the fp32
// workload is the small correctness configuration, so a tiled fp32 FMA GEMM
// is enough.
//   pass 1 (swiglu): h[r, n] = silu(sum_k A[r,k] W1[g,k,n]) * (sum_k A[r,k] W3[g,k,n])
//   pass 2 (plain):  y[r, n] = sum_k h[r,k] W2[g,k,n]
#include "moe_internal.cuh"

namespace moe {
namespace {

// 32 x 32 output tiles (2 x 2 per thread) so that the few rows of a small
// layer still spread over the SMs; the next K slice is loaded into registers
// while the current one is multiplied from shared memory.
constexpr int BM = 32, BN = 32, BK = 32;
constexpr int kPer = BM * BK / 256;  // elements of a tile each thread loads (4)

template <bool SWIGLU>
__global__ void __launch_bounds__(256)
    k_ffn_f32(const float *__restrict__ A, const float *__restrict__ B1,
              const float *__restrict__ B3, float *__restrict__ C, const int32_t *offsets,
              int fixed_rows, int K, int N) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ float as[BK][BM + 1];
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
  float ra[kPer], rb1[kPer], rb3[kPer];
  // element i of this thread's share: A (row i*8 + tid/32, k tid%32), B (k i*8 + tid/32, col tid%32)
  auto load = [&](int k0) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = i * 8 + tid / 32, kk = tid % 32;
      const int m = m0 + r, k = k0 + kk;
      ra[i] = (m < rows && k < K) ? A[(size_t)(r0 + m) * K + k] : 0.f;
      const int kb = k0 + r, n = n0 + kk;
      const bool in = kb < K && n < N;
      rb1[i] = in ? Bg1[(size_t)kb * N + n] : 0.f;
      if (SWIGLU) rb3[i] = in ? Bg3[(size_t)kb * N + n] : 0.f;
    }
  };
  float acc1[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, acc3[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  load(0);
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = i * 8 + tid / 32, kk = tid % 32;
      as[kk][r] = ra[i];
      b1s[r][kk] = rb1[i];
      if (SWIGLU) b3s[r][kk] = rb3[i];
    }
    __syncthreads();
    if (k0 + BK < K) load(k0 + BK);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float a0 = as[kk][ty * 2], a1 = as[kk][ty * 2 + 1];
      const float b0 = b1s[kk][tx * 2], b1 = b1s[kk][tx * 2 + 1];
      acc1[0][0] = fmaf(a0, b0, acc1[0][0]);
      acc1[0][1] = fmaf(a0, b1, acc1[0][1]);
      acc1[1][0] = fmaf(a1, b0, acc1[1][0]);
      acc1[1][1] = fmaf(a1, b1, acc1[1][1]);
      if (SWIGLU) {
        const float c0 = b3s[kk][tx * 2], c1 = b3s[kk][tx * 2 + 1];
        acc3[0][0] = fmaf(a0, c0, acc3[0][0]);
        acc3[0][1] = fmaf(a0, c1, acc3[0][1]);
        acc3[1][0] = fmaf(a1, c0, acc3[1][0]);
        acc3[1][1] = fmaf(a1, c1, acc3[1][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int m = m0 + ty * 2 + i;
    if (m >= rows) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = n0 + tx * 2 + j;
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
  launch_k(k_ffn_f32<true>, g1, 256, 0, s, x_perm, W1, W3, h, offsets, fixed_rows, d, f);
  dim3 g2((d + BN - 1) / BN, (max_rows + BM - 1) / BM, G);
  launch_k(k_ffn_f32<false>, g2, 256, 0, s, h, W2, nullptr, y, offsets, fixed_rows, f, d);
  return cudaGetLastError();
}

}  // namespace moe
