// Internal declarations shared by the CUDA translation units of libmoe.so.
// Nothing here is part of the public ABI (include/moe.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Device error flags (bit positions documented with moe_check_errors).
enum : uint32_t {
  kErrIndex = 1u,    // a gather/scatter index out of range
  kErrWait = 2u,     // a pipeline wait hit its time limit
  kErrRouting = 4u,  // an expert index or k_t out of range
};

// Address of this device's error word (a file-scope __device__ variable of
// moe_api.cu), looked up once per device.
uint32_t *device_error_word();

// SwiGLU's elementwise step, silu(g) * u = g / (1 + e^-g) * u, with the fast
// reciprocal division (at most 2 ulp; h is rounded to bf16 right after).  For
// g below about -87 the denominator exceeds 2^126 and the quotient is 0, the
// limit of silu there.
__device__ __forceinline__ float silu_times(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ void raise_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

// ---- programmatic dependent launch ----------------------------------------
// Every kernel of the library starts with grid_dependency(): it waits until
// the grid launched before it on the stream has finished and its memory is
// visible (an immediate return when the kernel was launched without the
// programmatic-serialization attribute), then allows the grid launched after
// it to start its launch and prologue.  So a kernel never reads or writes
// memory before its predecessor is complete, whichever way it was launched,
// and launch_k can overlap one kernel's launch with the previous one's tail.
__device__ __forceinline__ void grid_dependency() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Whether launch_k sets the programmatic-serialization attribute
// (MOE_PDL=0: plain stream order).
bool pdl_enabled();

// kernel<<<grid, block, smem, s>>>(args...), with programmatic stream
// serialization when pdl_enabled().  Returns the launch's status.
template <typename... Params, typename... Args>
cudaError_t launch_k(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, Args &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

// ---- element access -------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---- launchers (host) -----------------------------------------------------
// Every launcher enqueues on `stream` and returns the cudaGetLastError() of its
// launches.  Shapes have been validated by the ABI layer before the call.

// K1: logits[T,E] = x[T,d] . Wr[d,E] (+ bias) in fp32 (SIMT, full fp32 FMA).
cudaError_t launch_router(const moe_config &c, const void *x, const void *Wr,
                          const float *logit_bias, float *logits, cudaStream_t s);

// K2: gating, one warp per token.
cudaError_t launch_gating(const moe_config &c, const float *logits, const float *sel_bias,
                          const int32_t *k_per_token, int32_t *topk_idx, float *topk_w,
                          uint32_t *err, cudaStream_t s);

// K3: histogram, capacity, prefix sum, stable ranks.  `scratch` holds
// capacity_scratch_bytes(c) bytes.
size_t capacity_scratch_bytes(const moe_config &c);
cudaError_t launch_capacity(const moe_config &c, const int32_t *topk_idx, int32_t *counts,
                            int32_t *kept, int32_t *offsets, int32_t *slot_row,
                            int32_t *row_src, int32_t *n_dropped, void *scratch, uint32_t *err,
                            cudaStream_t s);

// K4: x_perm[r] = x[row_src[r] / k_max] for r < offsets[E].
// The dispatch walked by token (x rows read once; moe_layer, long batches).
cudaError_t launch_dispatch_by_token(const moe_config &c, const void *x,
                                     const int32_t *slot_row, void *x_perm, uint32_t *err,
                                     cudaStream_t s);
cudaError_t launch_dispatch(const moe_config &c, const void *x, const int32_t *offsets,
                            const int32_t *row_src, void *x_perm, uint32_t *err, cudaStream_t s);

// K7: out[t] = sum_j w[t,j] y_perm[slot_row[t,j]] (+ shared[t]); y_perm and
// shared are fp32, out is in the layer dtype.  topk_w == nullptr: the rows
// already carry their gate weights (applied by the down projection).
// shared_y: shared_parts fp32 blocks [T, d] (partial sums of the shared
// expert, added in order), or nullptr.  yexp (bf16 layers): y_perm holds
// y16 rows with these block exponents [rows, ceil(d / 32)] instead of fp32.
cudaError_t launch_combine(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                           const float *topk_w, const void *shared_y, void *out, uint32_t *err,
                           cudaStream_t s, int shared_parts = 1, const int8_t *yexp = nullptr);

// K9: fp32 SIMT grouped SwiGLU FFN (fp32 layers).  h: [rows_cap, f] fp32.
cudaError_t launch_ffn_simt_f32(int rows_cap, int d, int f, int G, const int32_t *offsets,
                                int fixed_rows, const float *x_perm, const float *W1,
                                const float *W3, const float *W2, float *h, float *y,
                                cudaStream_t s);

// K5/K6: tcgen05 grouped GEMMs (bf16 in, fp32 accumulate).
//   swiglu: out[r, :] = silu(A[r].B1[g]) * (A[r].B3[g])  bf16 out   (B*: [G, K, N])
//   plain:  out[r, :] = A[r].B1[g]                       fp32 out
// Rows of group g are offsets[g]..offsets[g+1]-1 of A (rows_cap rows, K
// columns); offsets == nullptr means one group of fixed_rows rows.  With
// row_src (swiglu only, when grouped_gemm_can_gather says so), row r of A is
// row row_src[r] / k_max of A itself ([a_rows, K], the token rows): the
// dispatch gather is fused into the GEMM's loads.
bool grouped_gemm_can_gather(bool swiglu, int rows_cap, int G, const int32_t *offsets,
                             int fixed_rows);
// row_w (plain only): output row r is multiplied by row_w[w_row_src[r]], the
// gate weight of the slot it serves (the combine then only sums).
// yexp (plain only, engines other than swap-AB: grouped_gemm_y16_out):
// out receives the compact y16 form of the rows, see launch_grouped_gemm_mixed.
cudaError_t launch_grouped_gemm_bf16(bool swiglu, int rows_cap, int K, int N, int G,
                                     const int32_t *offsets, int fixed_rows, const void *A,
                                     const void *B1, const void *B3, void *out, uint32_t *err,
                                     cudaStream_t s, const int32_t *row_src = nullptr,
                                     int k_max = 1, int a_rows = 0,
                                     const float *row_w = nullptr,
                                     const int32_t *w_row_src = nullptr,
                                     int8_t *yexp = nullptr);
// Whether the down projection of this shape can write y16 rows.
bool grouped_gemm_y16_out(int rows_cap, int G, const int32_t *offsets, int fixed_rows, int N);

// K5/K6 with fp8 weights: B1, B3 are e4m3 codes [G, K, N] (N % 16 == 0) with
// per-column fp32 scales s1, s3 [G, N] (16-byte aligned); the codes are
// widened to bf16 in shared memory and the scales applied in the epilogue.
// Output types as for launch_grouped_gemm_bf16.
cudaError_t launch_grouped_gemm_fp8(bool swiglu, int rows_cap, int K, int N, int G,
                                    const int32_t *offsets, int fixed_rows, const void *A,
                                    const void *B1, const void *B3, const float *s1,
                                    const float *s3, void *out, uint32_t *err, cudaStream_t s,
                                    const float *row_w = nullptr,
                                    const int32_t *w_row_src = nullptr);

// K5/K6 for ragged routed groups (grouped_gemm_mixed.cu): each group's full
// 128-row chunks on ordinary tiles and its remainder on a swap-AB tile, in
// one launch.  Operands and outputs as for launch_grouped_gemm_bf16.
// yexp (plain only): when given, out receives the compact y16 form of the
// fp32 rows (fp16 values, one power-of-two exponent per 32-column block in
// yexp [rows_cap, ceil(N / 32)]; see tcgen05_common.cuh).
// row_src (swiglu only): row r of A is row row_src[r] / k_max of A itself
// ([a_rows, K], the token rows), fetched with cp.async by the kernel -- the
// dispatch copy fused into the up projection.
cudaError_t launch_grouped_gemm_mixed(bool swiglu, int rows_cap, int K, int N, int G,
                                      const int32_t *offsets, const void *A, const void *B1,
                                      const void *B3, void *out, uint32_t *err, cudaStream_t s,
                                      const float *row_w = nullptr,
                                      const int32_t *w_row_src = nullptr,
                                      int8_t *yexp = nullptr, const int32_t *row_src = nullptr,
                                      int k_max = 1, int a_rows = 0);

// K5/K6 with fp8 weights on tcgen05.mma kind::f8f6f4 (grouped_gemm_f8.cu):
// decode-sized routed groups.  The activations come as two e4m3 planes with a
// power-of-two scale per row (launch_split_planes): planes [2 * rows_cap, K],
// plane q's row r at q * rows_cap + r; row_scale [rows_cap].  B1, B3: e4m3
// codes [G, N, K] with column scales s1, s3 [G, N].  Output types as for
// launch_grouped_gemm_bf16.
cudaError_t launch_grouped_gemm_f8(bool swiglu, int rows_cap, int K, int N, int G,
                                   const int32_t *offsets, const uint8_t *planes,
                                   const float *row_scale, const void *B1, const void *B3,
                                   const float *s1, const float *s3, void *out, uint32_t *err,
                                   cudaStream_t s, const float *row_w = nullptr,
                                   const int32_t *w_row_src = nullptr);
// Bytes of the two planes of rows_cap rows of K values.
size_t fp8_planes_bytes(int rows_cap, int K);
// Rows r < (*n_rows, or fixed_rows when n_rows is nullptr) of the bf16 rows
// src [., K] -- with row_src, token row row_src[r] / k_max (< src_rows) of
// them -- into planes and row scales (K % 16 == 0).
cudaError_t launch_split_planes(const void *src, const int32_t *n_rows, int fixed_rows,
                                const int32_t *row_src, int k_max, int src_rows, int rows_cap,
                                int K, uint8_t *planes, float *row_scale, uint32_t *err,
                                cudaStream_t s);

// Expert parallelism (expert_parallel.cu): the exchange plan of one rank
// from the counts of all ranks C [n_ranks][E], the dispatch of its kept rows
// into the owners' receive buffers, and the return of its experts' outputs to
// the sources' y_back buffers (fp32 rows).
cudaError_t launch_ep_plan(const int32_t *C, int n_ranks, int E, int rank, int32_t *recv_offsets,
                           int32_t *send_base, cudaStream_t s);
cudaError_t launch_ep_dispatch(const moe_config &c, int n_ranks, void *const *recv_rows,
                               const void *x, const int32_t *offsets, const int32_t *row_src,
                               const int32_t *topk_idx, const int32_t *send_base, uint32_t *err,
                               cudaStream_t s);
cudaError_t launch_ep_return(const moe_config &c, int n_ranks, int rank, const int32_t *C,
                             float *const *y_back, const float *y_recv,
                             const int32_t *recv_offsets, uint32_t *err, cudaStream_t s);

// Per-column e4m3 quantisation of bf16 weights W [G, K, N]: scale[g, n] =
// max_k |W| / 448 (1 for an all-zero column), Wq = e4m3(W / scale), rounded
// to nearest even with saturation.
cudaError_t launch_quantize_fp8(int G, int K, int N, const void *W, uint8_t *Wq, float *scale,
                                cudaStream_t s);

// K1 on the tensor cores (bf16 layers with E % 8 == 0): logits[T,E] =
// x[T,d] . Wr[d,E] (+ bias), fp32 accumulation in tensor memory, fp32 out.
cudaError_t launch_router_tc(int T, int d, int E, const void *x, const void *Wr,
                             const float *bias, float *logits, uint32_t *err, cudaStream_t s);

// K1 split along K: partials[g][T][E] = x[:, g*k_split ..] . Wr[g*k_split .., :]
// for g < S (k_split a multiple of 64; the last slice may run past d).  The
// first thread of block 0 sets *clear to zero.
cudaError_t launch_router_split(int T, int d, int E, int S, int k_split, const void *x,
                                const void *Wr, float *partials, int32_t *clear, uint32_t *err,
                                cudaStream_t s);

// Split-K GEMM of one group of T rows (bf16 A [T, K]): out [S][T][N] fp32,
// split s over K columns s*K/S .. (s+1)*K/S-1 (K a multiple of 64*S).  B is
// [K, N] bf16, or with fp8 the e4m3 codes [N, K] and column scales [N].
cudaError_t launch_gemm_split(bool fp8, int T, int K, int N, int S, const void *A, const void *B,
                              const float *scale, float *out, uint32_t *err, cudaStream_t s);

// The shared expert of a decode-sized batch, split along K (shared_expert.cu).
struct SharedSplitPlan {
  bool use = false;
  int s_up = 1, s_down = 1;
};
SharedSplitPlan shared_split_plan(const moe_config &c);
// Scratch for the partial sums (0 without a plan).
size_t shared_split_bytes(const moe_config &c);
// h: [T, f_shared] bf16; y_sh: [T, d] fp32.  On return *shared_y / *shared_parts
// describe the partial sums the combine adds.
cudaError_t launch_shared_split(const moe_config &c, const SharedSplitPlan &p, bool fp8,
                                const void *x, const void *W1, const void *W3, const void *W2,
                                const float *s1, const float *s3, const float *s2, void *h,
                                float *y_sh, void *scratch, const float **shared_y,
                                int *shared_parts, uint32_t *err, cudaStream_t s);

// Routing of small batches (decode): split-K router, then one kernel that
// sums the partials, gates and ranks (see route_small.cu).  The plan depends
// on the layer's shape only.
struct SmallRoutePlan {
  bool use = false;
  int S = 0, k_split = 0;
  size_t partial_bytes = 0, scratch_bytes = 0;
};
SmallRoutePlan small_route_plan(const moe_config &c);
// Scratch of the routing step: the small-batch plan's, else the capacity step's.
size_t route_scratch_bytes(const moe_config &c);
cudaError_t launch_route_small(const moe_config &c, const SmallRoutePlan &plan, const void *x,
                               const void *Wr, const float *logit_bias, const float *sel_bias,
                               const int32_t *k_per_token, const moe_route_out &o, void *scratch,
                               uint32_t *err, cudaStream_t s);

}  // namespace moe
