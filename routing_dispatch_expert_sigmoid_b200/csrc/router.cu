// K1 -- router GEMM: logits[T,E] = x[T,d] . Wr[d,E] (+ logit_bias[E]), fp32.
//
// "Paralelismo experto para el servicio MoE", section "Buceo profundo": a
// router scores the experts of every token.  The scores feed an integer
// decision (top-k), and the logits must match a fp64 reference within 1e-4 of
// their RMS, so accumulation is plain fp32 FMA on the CUDA cores (no TF32).
//
// Tiling: a CTA computes a BM x BN tile of logits with 256 threads, each
// owning TM x TN outputs; x and Wr tiles of BK along d are staged through
// shared memory (x transposed so a thread's TM rows are one broadcast read).
// The expert tile width BN follows E so that small-E layers do not waste
// lanes on empty columns.  Short batches with at most 16 experts take one
// warp per token instead.
#include "moe_internal.cuh"

namespace moe {
namespace {

template <typename T, int BM, int BN, int BK, int TM, int TN>
__global__ void __launch_bounds__(256) k_router(const T *__restrict__ x, const T *__restrict__ Wr,
                                                const float *__restrict__ bias,
                                                float *__restrict__ logits, int Tn, int d, int E) {
  grid_dependency();  // the previous grid is complete; the next may launch
  static_assert((BM / TM) * (BN / TN) == 256, "256 threads");
  __shared__ float xs[BK][BM + 4];
  __shared__ float ws[BK][BN];
  const int t0 = blockIdx.x * BM, e0 = blockIdx.y * BN;
  const int tid = threadIdx.x;
  const int tx = tid % (BN / TN), ty = tid / (BN / TN);
  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      int r = i / BK, kk = i % BK;
      int t = t0 + r, k = k0 + kk;
      xs[kk][r] = (t < Tn && k < d) ? to_f32(x[(size_t)t * d + k]) : 0.f;
    }
    for (int i = tid; i < BK * BN; i += 256) {
      int kk = i / BN, c = i % BN;
      int k = k0 + kk, e = e0 + c;
      ws[kk][c] = (k < d && e < E) ? to_f32(Wr[(size_t)k * E + e]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[TM], b[TN];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = xs[kk][ty * TM + i];
#pragma unroll
      for (int j = 0; j < TN; ++j) b[j] = ws[kk][tx * TN + j];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    int t = t0 + ty * TM + i;
    if (t >= Tn) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      int e = e0 + tx * TN + j;
      if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
    }
  }
}

// Short batches with few experts: one warp per token, lane l accumulating
// the products of K positions l, l+32, ... for every expert, then a
// butterfly sum across the warp (a fixed order).  The tiled kernel above
// would give a 256-token batch only four CTAs.
template <typename T, int EMAX>
__global__ void __launch_bounds__(256)
    k_router_warp(const T *__restrict__ x, const T *__restrict__ Wr, const float *__restrict__ bias,
                  float *__restrict__ logits, int Tn, int d, int E) {
  grid_dependency();  // the previous grid is complete; the next may launch
  const int t = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (t >= Tn) return;  // whole warp leaves together
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
  const T *xr = x + (size_t)t * d;
#pragma unroll 4
  for (int k = lane; k < d; k += 32) {
    const float xv = to_f32(xr[k]);
    const T *w = Wr + (size_t)k * E;
#pragma unroll
    for (int e = 0; e < EMAX; ++e)
      if (e < E) acc[e] = fmaf(xv, to_f32(w[e]), acc[e]);
  }
  float mine = 0.f;
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    float v = acc[e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == e) mine = v;
  }
  if (lane < E) logits[(size_t)t * E + lane] = mine + (bias ? bias[lane] : 0.f);
}

template <typename T, int EMAX>
cudaError_t run_warp(const moe_config &c, const void *x, const void *Wr, const float *bias,
                     float *logits, cudaStream_t s) {
  launch_k(k_router_warp<T, EMAX>, (c.T + 7) / 8, 256, 0, s,
      static_cast<const T *>(x), static_cast<const T *>(Wr), bias, logits, c.T, c.d, c.E);
  return cudaGetLastError();
}

template <typename T, int BM, int BN, int BK, int TM, int TN>
cudaError_t run(const moe_config &c, const void *x, const void *Wr, const float *bias,
                float *logits, cudaStream_t s) {
  dim3 grid((c.T + BM - 1) / BM, (c.E + BN - 1) / BN);
  launch_k(k_router<T, BM, BN, BK, TM, TN>, grid, 256, 0, s,
      static_cast<const T *>(x), static_cast<const T *>(Wr), bias, logits, c.T, c.d, c.E);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_tile(const moe_config &c, const void *x, const void *Wr, const float *bias,
                          float *logits, cudaStream_t s) {
  if (c.T <= 2048 && c.E <= 8) return run_warp<T, 8>(c, x, Wr, bias, logits, s);
  if (c.T <= 2048 && c.E <= 16) return run_warp<T, 16>(c, x, Wr, bias, logits, s);
  if (c.E <= 8) return run<T, 64, 8, 32, 2, 1>(c, x, Wr, bias, logits, s);
  if (c.E <= 16) return run<T, 64, 16, 32, 2, 2>(c, x, Wr, bias, logits, s);
  if (c.E <= 32) return run<T, 64, 32, 32, 2, 4>(c, x, Wr, bias, logits, s);
  return run<T, 64, 64, 16, 4, 4>(c, x, Wr, bias, logits, s);
}

}  // namespace

cudaError_t launch_router(const moe_config &c, const void *x, const void *Wr,
                          const float *logit_bias, float *logits, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  if (c.dtype == MOE_F32) return dispatch_tile<float>(c, x, Wr, logit_bias, logits, s);
  return dispatch_tile<__nv_bfloat16>(c, x, Wr, logit_bias, logits, s);
}

}  // namespace moe
