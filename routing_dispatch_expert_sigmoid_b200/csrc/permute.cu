// K4 dispatch and K7 combine: the local (single-GPU) form of the two exchange
// steps of an MoE layer.
//
// "Expert Parallelism: MoE 模型的并行切分", section 12 question 2: dispatch
// copies each token's hidden state once per selected expert; combine returns
// the k outputs to the token's position and sums them weighted by the router
// weight.  Section 3 and "LLM MoE Expert Parallel 生产实战" (steps 2 and 4)
// describe the same two steps as all-to-alls across GPUs; here both sides are
// on one GPU, so they are a gather into expert-contiguous rows and a weighted
// gather back.
//
// Both kernels are HBM-bound row copies with 16-byte vector loads and stores
// (rows of d*s bytes, d*s a multiple of 16); a warp takes a chunk of one row
// (dispatch) or of one token's output (combine) at a time.  The number of rows R lives on the device
// (offsets[E]); a fixed grid strides over the row space and stops at R.
#include <cuda_fp16.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ uint4 ldg_nc(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Work items are (row, chunk of 32 x VPL 16-byte vectors): a lane issues its
// VPL loads before its stores, and the token index of the warp's next item
// is loaded before the current item's rows, so each item costs about one
// memory round trip.  4 KB chunks (VPL = 8), or 2 KB for small batches so
// that their few rows still spread over the GPU.
template <int VPL>
__global__ void __launch_bounds__(256)
    k_dispatch(const uint4 *__restrict__ x, const int32_t *__restrict__ offsets,
               const int32_t *__restrict__ row_src, uint4 *__restrict__ x_perm, int E,
               int k_max, int T, int rows_cap, int row_vecs, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  int R = offsets[E];
  if (R > rows_cap || R < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrIndex);
    R = R < 0 ? 0 : rows_cap;
  }
  constexpr int kChunkVecs = 32 * VPL;
  const int lane = threadIdx.x % 32;
  const int chunks = (row_vecs + kChunkVecs - 1) / kChunkVecs;
  const long long items = (long long)R * chunks;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  long long it = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  int a_next = it < items ? row_src[it / chunks] : 0;
  for (; it < items; it += warps) {
    const int row = (int)(it / chunks), ch = (int)(it % chunks);
    const int a = a_next;
    if (it + warps < items) a_next = row_src[(it + warps) / chunks];
    const int t = a / k_max;
    if (a < 0 || t >= T) {
      if (lane == 0) raise_error(err, kErrIndex);
      continue;
    }
    const uint4 *src = x + (size_t)t * row_vecs;
    uint4 *dst = x_perm + (size_t)row * row_vecs;
    const int v0 = ch * kChunkVecs + lane;
    uint4 u[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) u[i] = ldg_nc(src + v0 + 32 * i);
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) dst[v0 + 32 * i] = u[i];
  }
}

// The same copy walked by token: a warp reads a token's row once and stores
// it to each of the token's kept rows (slot_row[t, j] >= 0).  For long
// batches the rows of x are then read from HBM once: walked by destination
// row, each token row is fetched k_t times, and the x_perm stores push it
// out of L2 between the fetches.
template <int VPL>
__global__ void __launch_bounds__(256)
    k_dispatch_tok(const uint4 *__restrict__ x, const int32_t *__restrict__ slot_row,
                   uint4 *__restrict__ x_perm, int T, int k_max, int rows_cap, int row_vecs,
                   uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  constexpr int kChunkVecs = 32 * VPL;
  const int lane = threadIdx.x % 32;
  const int warps = gridDim.x * (blockDim.x / 32);
  for (int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; t < T; t += warps) {
    int my_row = -1;  // lane j: the destination of slot j
    if (lane < k_max) my_row = slot_row[(size_t)t * k_max + lane];
    if (my_row >= rows_cap || my_row < -1) {
      raise_error(err, kErrIndex);
      my_row = -1;
    }
    const unsigned live = __ballot_sync(0xffffffffu, my_row >= 0);
    const uint4 *src = x + (size_t)t * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += kChunkVecs) {
      uint4 u[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int v = c0 + lane + 32 * i;
        if (v < row_vecs) u[i] = ldg_nc(src + v);
      }
      for (unsigned m = live; m; m &= m - 1) {
        const int j = __ffs(m) - 1;
        uint4 *dst = x_perm + (size_t)__shfl_sync(0xffffffffu, my_row, j) * row_vecs;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int v = c0 + lane + 32 * i;
          if (v < row_vecs) dst[v] = u[i];
        }
      }
    }
  }
}

// 16 bytes of T as fp32 values.
template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const uint4 &u, float *f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 store(const float *f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static uint4 store(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// y and shared_y are fp32 rows (Q 16-byte vectors per output vector); out
// rows are T (row_vecs vectors of Vec<T>::N values).  Work items are (token,
// 32 consecutive output vectors): lane l of the item's warp owns one output
// vector and sums the token's kept slots for it in slot order.
// KB: slots whose rows are loaded before they are summed (k_max rounded up
// to 2, 4 or 8, so that top-2 layers keep their registers few).
template <typename T, int KB>
__global__ void __launch_bounds__(256)
    k_combine(const uint4 *__restrict__ y, const int32_t *__restrict__ slot_row,
              const float *__restrict__ topk_w, const uint4 *__restrict__ shared_y,
              int shared_parts, uint4 *__restrict__ out, int Tn, int k_max, int rows_cap,
              int row_vecs, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  constexpr int N = Vec<T>::N;  // output values per 16-byte vector
  constexpr int Q = N / 4;      // fp32 input vectors per output vector
  __shared__ int32_t s_row[8][32];
  __shared__ float s_w[8][32];
  const int lane = threadIdx.x % 32, wib = threadIdx.x / 32;
  const int chunks = (row_vecs + 31) / 32;
  const long long items = (long long)Tn * chunks;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  const size_t in_vecs = (size_t)row_vecs * Q;  // fp32 vectors per row
  // The token's slots of the warp's next item are loaded while the current
  // item's rows are summed.
  long long it = (long long)blockIdx.x * (blockDim.x / 32) + wib;
  int next_row = -1;
  float next_w = 0.f;
  if (it < items && lane < k_max) {
    const size_t at = (size_t)(it / chunks) * k_max + lane;
    next_row = slot_row[at];
    next_w = topk_w ? topk_w[at] : 1.0f;  // fmaf(1, y, acc) = y + acc
  }
  for (; it < items; it += warps) {
    const int t = (int)(it / chunks), ch = (int)(it % chunks);
    int my_row = next_row;
    const float my_w = next_w;
    if (it + warps < items && lane < k_max) {
      const size_t at = (size_t)((it + warps) / chunks) * k_max + lane;
      next_row = slot_row[at];
      next_w = topk_w ? topk_w[at] : 1.0f;
    }
    if (my_row >= rows_cap) {
      raise_error(err, kErrIndex);
      my_row = -1;
    }
    const unsigned live = __ballot_sync(0xffffffffu, my_row >= 0);
    const int n_live = __popc(live);
    if (my_row >= 0) {  // compact the kept slots, in slot order
      const int pos = __popc(live & ((1u << lane) - 1u));
      s_row[wib][pos] = my_row;
      s_w[wib][pos] = my_w;
    }
    __syncwarp();
    const int v = ch * 32 + lane;
    if (v < row_vecs) {
      float acc[N];
      if (shared_y) {
#pragma unroll
        for (int q = 0; q < Q; ++q)
          Vec<float>::load(ldg_nc(shared_y + (size_t)t * in_vecs + (size_t)v * Q + q), acc + 4 * q);
        for (int sp = 1; sp < shared_parts; ++sp) {  // further partial sums, in order
          const uint4 *part = shared_y + (size_t)sp * Tn * in_vecs + (size_t)t * in_vecs;
#pragma unroll
          for (int q = 0; q < Q; ++q) {
            float f[4];
            Vec<float>::load(ldg_nc(part + (size_t)v * Q + q), f);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[4 * q + i] += f[i];
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < N; ++i) acc[i] = 0.f;
      }
      for (int j0 = 0; j0 < n_live; j0 += KB) {
        uint4 u[KB][Q];
#pragma unroll
        for (int j = 0; j < KB; ++j)  // issue the loads before the FMAs
          if (j0 + j < n_live) {
            const uint4 *src = y + (size_t)s_row[wib][j0 + j] * in_vecs + (size_t)v * Q;
#pragma unroll
            for (int q = 0; q < Q; ++q) u[j][q] = ldg_nc(src + q);
          }
#pragma unroll
        for (int j = 0; j < KB; ++j) {
          if (j0 + j < n_live) {
            const float wj = s_w[wib][j0 + j];
            float f[N];
#pragma unroll
            for (int q = 0; q < Q; ++q) Vec<float>::load(u[j][q], f + 4 * q);
#pragma unroll
            for (int i = 0; i < N; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
          }
        }
      }
      out[(size_t)t * row_vecs + v] = Vec<T>::store(acc);
    }
    __syncwarp();
  }
}

// The same combine on y16 rows (fp16 values, one power-of-two exponent per
// 32-column block, written by the down projection): value = y16 * 2^e.  The
// bf16 output vector of a lane spans 8 columns of one block, so each slot
// costs one 16-byte load and one exponent byte; the exponent is folded into
// the slot's weight (w * 2^e is exact).  A lane owns VPL output vectors
// (work items of 32 VPL vectors), so that a top-2 layer still has a few
// loads in flight per lane.
// At least two CTAs (16 warps) per SM: left alone the compiler gives the
// kernel over 160 registers, one CTA per SM, and the y16 reads half the
// loads in flight they need (Qwen3-shaped combine 0.20 vs 0.13 ms).  SH =
// false leaves out the shared expert's partial sums: the registers that
// frees hold more row loads in flight (top-2 with four vectors per lane:
// Mixtral-shaped combine 0.065 -> 0.050 ms; top-8 with two vectors, no
// spills: Qwen3-shaped 0.123 -> 0.107 ms).  With a shared expert its partial
// sums are read after the first batch of rows is issued (one vector per lane).
template <int KB, int VPL, typename Idx, bool SH = true>
__global__ void __launch_bounds__(256, 2)
    k_combine_y16(const uint4 *__restrict__ y, const int8_t *__restrict__ yexp, int nblk,
                  const int32_t *__restrict__ slot_row, const float *__restrict__ topk_w,
                  const uint4 *__restrict__ shared_y, int shared_parts, uint4 *__restrict__ out,
                  int Tn, int k_max, int rows_cap, int row_vecs, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ int32_t s_row[8][32];
  __shared__ float s_w[8][32];
  const int lane = threadIdx.x % 32, wib = threadIdx.x / 32;
  constexpr int kItemVecs = 32 * VPL;
  const int chunks = (row_vecs + kItemVecs - 1) / kItemVecs;
  // Idx: int when the work items fit (no 64-bit divisions in the loop)
  const Idx items = (Idx)Tn * chunks;
  const Idx warps = (Idx)gridDim.x * (blockDim.x / 32);
  const size_t sh_vecs = (size_t)row_vecs * 2;  // fp32 vectors per shared row
  Idx it = (Idx)blockIdx.x * (blockDim.x / 32) + wib;
  int next_row = -1;
  float next_w = 0.f;
  if (it < items && lane < k_max) {
    const size_t at = (size_t)(it / chunks) * k_max + lane;
    next_row = slot_row[at];
    next_w = topk_w ? topk_w[at] : 1.0f;
  }
  for (; it < items; it += warps) {
    const int t = (int)(it / chunks), ch = (int)(it % chunks);
    int my_row = next_row;
    const float my_w = next_w;
    if (it + warps < items && lane < k_max) {
      const size_t at = (size_t)((it + warps) / chunks) * k_max + lane;
      next_row = slot_row[at];
      next_w = topk_w ? topk_w[at] : 1.0f;
    }
    if (my_row >= rows_cap) {
      raise_error(err, kErrIndex);
      my_row = -1;
    }
    const unsigned live = __ballot_sync(0xffffffffu, my_row >= 0);
    const int n_live = __popc(live);
    if (my_row >= 0) {  // compact the kept slots, in slot order
      const int pos = __popc(live & ((1u << lane) - 1u));
      s_row[wib][pos] = my_row;
      s_w[wib][pos] = my_w;
    }
    __syncwarp();
    const int v0 = ch * kItemVecs + lane;  // this lane's vectors: v0 + 32 i
    float acc[VPL][8];
#pragma unroll
    for (int i = 0; i < VPL; ++i)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[i][q] = 0.f;
    // The shared expert's partial sums go into acc first, but they are read
    // after the first batch of rows has been issued, so the two sets of
    // loads are in flight together.
    bool sh_pending = SH && shared_y != nullptr;
    for (int j0 = 0; j0 < n_live || sh_pending; j0 += KB) {
      uint4 u[KB][VPL];
      int e[KB][VPL];
#pragma unroll
      for (int j = 0; j < KB; ++j)  // issue the loads before the FMAs
        if (j0 + j < n_live) {
          const int r = s_row[wib][j0 + j];
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            const int v = v0 + 32 * i;
            if (v < row_vecs) {
              u[j][i] = ldg_nc(y + (size_t)r * row_vecs + v);
              e[j][i] = __ldg(yexp + (size_t)r * nblk + (v >> 2));  // 8 columns per vector
            }
          }
        }
      if (SH && sh_pending) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int v = v0 + 32 * i;
          if (v < row_vecs) {
            for (int sp = 0; sp < shared_parts; ++sp) {  // partial sums, in order
              const uint4 *part = shared_y + (size_t)sp * Tn * sh_vecs + (size_t)t * sh_vecs;
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                float f[4];
                Vec<float>::load(ldg_nc(part + (size_t)v * 2 + q), f);
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][4 * q + c] += f[c];
              }
            }
          }
        }
        sh_pending = false;
      }
#pragma unroll
      for (int j = 0; j < KB; ++j) {
        if (j0 + j < n_live) {
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            if (v0 + 32 * i < row_vecs) {
              const float wj = s_w[wib][j0 + j] * __int_as_float((e[j][i] + 127) << 23);
              const uint32_t hw[4] = {u[j][i].x, u[j][i].y, u[j][i].z, u[j][i].w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hw[q]));
                // one packed fp32 FMA for the pair (each half rounded as fmaf)
                const float2 s2 = __ffma2_rn(make_float2(wj, wj), f,
                                             make_float2(acc[i][2 * q], acc[i][2 * q + 1]));
                acc[i][2 * q] = s2.x;
                acc[i][2 * q + 1] = s2.y;
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = v0 + 32 * i;
      if (v < row_vecs) out[(size_t)t * row_vecs + v] = Vec<__nv_bfloat16>::store(acc[i]);
    }
    __syncwarp();
  }
}

int grid_for(long long warps_needed) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (warps_needed + 7) / 8;
  const long long cap = (long long)sms * 8;
  return (int)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace

cudaError_t launch_dispatch_by_token(const moe_config &c, const void *x,
                                     const int32_t *slot_row, void *x_perm, uint32_t *err,
                                     cudaStream_t s) {
  const int esz = c.dtype == MOE_F32 ? 4 : 2;
  const int rows_cap = c.T * c.k_max;
  if (rows_cap == 0) return cudaSuccess;
  const int row_vecs = c.d * esz / 16;
  launch_k(k_dispatch_tok<8>, grid_for(c.T), 256, 0, s, static_cast<const uint4 *>(x), slot_row,
                                                  static_cast<uint4 *>(x_perm), c.T, c.k_max,
                                                  rows_cap, row_vecs, err);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const moe_config &c, const void *x, const int32_t *offsets,
                            const int32_t *row_src, void *x_perm, uint32_t *err,
                            cudaStream_t s) {
  const int esz = c.dtype == MOE_F32 ? 4 : 2;
  const int rows_cap = c.T * c.k_max;
  if (rows_cap == 0) return cudaSuccess;
  const int row_vecs = c.d * esz / 16;
  const auto *xs = static_cast<const uint4 *>(x);
  auto *xp = static_cast<uint4 *>(x_perm);
  if ((long long)rows_cap * row_vecs * 16 <= (16ll << 20)) {  // at most 16 MB of rows
    const long long items = (long long)rows_cap * ((row_vecs + 127) / 128);
    launch_k(k_dispatch<4>, grid_for(items), 256, 0, s, xs, offsets, row_src, xp, c.E, c.k_max, c.T,
                                                  rows_cap, row_vecs, err);
  } else {
    const long long items = (long long)rows_cap * ((row_vecs + 255) / 256);
    launch_k(k_dispatch<8>, grid_for(items), 256, 0, s, xs, offsets, row_src, xp, c.E, c.k_max, c.T,
                                                  rows_cap, row_vecs, err);
  }
  return cudaGetLastError();
}

namespace {

template <typename T, int KB>
cudaError_t run_combine(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                        const float *topk_w, const void *shared_y, void *out, uint32_t *err,
                        cudaStream_t s, int shared_parts, int grid, int row_vecs) {
  launch_k(k_combine<T, KB>, grid, 256, 0, s, 
      static_cast<const uint4 *>(y_perm), slot_row, topk_w, static_cast<const uint4 *>(shared_y),
      shared_parts, static_cast<uint4 *>(out), c.T, c.k_max, c.T * c.k_max, row_vecs, err);
  return cudaGetLastError();
}

template <typename T>
cudaError_t combine_k(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                      const float *topk_w, const void *shared_y, void *out, uint32_t *err,
                      cudaStream_t s, int shared_parts, int grid, int row_vecs) {
  if (c.k_max <= 2)
    return run_combine<T, 2>(c, y_perm, slot_row, topk_w, shared_y, out, err, s, shared_parts,
                             grid, row_vecs);
  if (c.k_max <= 4)
    return run_combine<T, 4>(c, y_perm, slot_row, topk_w, shared_y, out, err, s, shared_parts,
                             grid, row_vecs);
  return run_combine<T, 8>(c, y_perm, slot_row, topk_w, shared_y, out, err, s, shared_parts,
                           grid, row_vecs);
}

}  // namespace

cudaError_t launch_combine(const moe_config &c, const void *y_perm, const int32_t *slot_row,
                           const float *topk_w, const void *shared_y, void *out, uint32_t *err,
                           cudaStream_t s, int shared_parts, const int8_t *yexp) {
  if (c.T == 0) return cudaSuccess;
  const int esz = c.dtype == MOE_F32 ? 4 : 2;
  const int row_vecs = c.d * esz / 16;
  const int grid = grid_for((long long)c.T * ((row_vecs + 31) / 32));
  if (yexp) {  // y16 rows (bf16 layers only)
    if (c.dtype != MOE_BF16) return cudaErrorInvalidValue;
    const auto *y = static_cast<const uint4 *>(y_perm);
    const auto *sh = static_cast<const uint4 *>(shared_y);
    auto *o = static_cast<uint4 *>(out);
    const int nblk = (c.d + 31) / 32, rows_cap = c.T * c.k_max;
    // 32-bit item indices unless T x chunks (plus a grid's worth of warps)
    // could pass 2^31
    const bool narrow = (long long)c.T * ((row_vecs + 31) / 32) + 148LL * 64 < (1LL << 31);
    auto launch = [&](auto kernel, int g) {
      launch_k(kernel, g, 256, 0, s, y, yexp, nblk, slot_row, topk_w, sh, shared_parts, o, c.T, c.k_max,
                               rows_cap, row_vecs, err);
    };
    // MOE_COMBINE_VPL=1: one 16-byte vector per lane per row (two for top-2)
    const char *cv = getenv("MOE_COMBINE_VPL");
    const bool one = cv && cv[0] == '1';
    if (c.k_max <= 2) {
      if (narrow && !sh && !one)  // four vectors per lane: items of 128 vectors
        launch(k_combine_y16<2, 4, int, false>,
               grid_for((long long)c.T * ((row_vecs + 127) / 128)));
      else if (narrow)  // two vectors per lane: items of 64 vectors
        launch(k_combine_y16<2, 2, int>, grid_for((long long)c.T * ((row_vecs + 63) / 64)));
      else
        launch(k_combine_y16<2, 2, long long>,
               grid_for((long long)c.T * ((row_vecs + 63) / 64)));
    } else if (c.k_max <= 4) {
      if (narrow)
        launch(k_combine_y16<4, 1, int>, grid);
      else
        launch(k_combine_y16<4, 1, long long>, grid);
    } else if (narrow && !one && !sh) {
      // two vectors per lane (twice the loads in flight per warp): 6% faster
      // on the Qwen3- and GPT-OSS-shaped layers than one
      launch(k_combine_y16<8, 2, int, false>, grid_for((long long)c.T * ((row_vecs + 63) / 64)));
    } else if (narrow) {
      // with a shared expert one vector per lane: the partial sums' registers
      // leave no room for two without spills (DeepSeek-V3-shaped prefill
      // combine 0.136 -> 0.122 ms with the shared loads overlapped)
      launch(k_combine_y16<8, 1, int>, grid);
    } else {
      launch(k_combine_y16<8, 1, long long>, grid);
    }
    return cudaGetLastError();
  }
  if (c.dtype == MOE_F32)
    return combine_k<float>(c, y_perm, slot_row, topk_w, shared_y, out, err, s, shared_parts,
                            grid, row_vecs);
  return combine_k<__nv_bfloat16>(c, y_perm, slot_row, topk_w, shared_y, out, err, s,
                                  shared_parts, grid, row_vecs);
}

}  // namespace moe
