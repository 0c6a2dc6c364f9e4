// Expert parallelism: the exchange steps of an MoE layer whose experts are
// split over ranks.
//
// "Expert Parallelism: MoE 模型的并行切分" (SGLang learning notes), section 3
// (the all-to-all dispatch and combine around the local expert compute) and
// section 8 (an 8-rank placement of the experts), and "LLM MoE Expert Parallel
// 生产实战", steps 2 and 4 (send every token to the ranks of its experts,
// bring the results back and combine them).  Rank r owns experts
// [r*E/n, (r+1)*E/n).  Given the kept-row counts of every rank, C[s][e], the
// layout of the exchange is fixed, so every rank can compute where its rows go
// and where returned rows land without asking anyone:
//   receive layout of rank r: its experts in ascending order, inside an
//   expert the source ranks in ascending order, inside a source the source's
//   own row order;
//   send base of rank s for expert e (owner r): the rows of r's experts
//   before e, plus the rows of e from sources before s;
//   a received row p of rank r (expert e, source s, i-th of s's rows of e)
//   returns to row  sum_{e' < e} C[s][e'] + i  of s's own layout.
// The dispatch and return kernels store each row straight into the
// destination rank's buffer (a peer pointer over NVLink, or one GPU's memory
// when the ranks are emulated there): 16-byte vector copies, no staging.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = 256;

__device__ __forceinline__ uint4 ldg_nc16(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One block: recv_offsets [E_loc + 1] and send_base [E] of this rank.
__global__ void __launch_bounds__(kPlanThreads)
    k_ep_plan(const int32_t *__restrict__ C, int n_ranks, int E, int rank,
              int32_t *__restrict__ recv_offsets, int32_t *__restrict__ send_base) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ int32_t s_tot[1024];  // rows of expert e over all sources
  const int e_loc = E / n_ranks;
  for (int e = threadIdx.x; e < E; e += kPlanThreads) {
    int t = 0;
    for (int s = 0; s < n_ranks; ++s) t += C[(size_t)s * E + e];
    s_tot[e] = t;
  }
  __syncthreads();
  // per owner, an exclusive scan of s_tot over its experts (n_ranks scans of
  // e_loc values; e_loc <= 1024): thread 0..n_ranks-1, one owner each
  if (threadIdx.x < n_ranks) {
    const int r = threadIdx.x, e0 = r * e_loc;
    int run = 0;
    for (int j = 0; j < e_loc; ++j) {
      const int e = e0 + j;
      int before = 0;
      for (int s = 0; s < rank; ++s) before += C[(size_t)s * E + e];
      send_base[e] = run + before;
      if (r == rank) recv_offsets[j] = run;
      run += s_tot[e];
    }
    if (r == rank) recv_offsets[e_loc] = run;
  }
}

// Dispatch: row r < offsets[E] of this rank's layout (slot row_src[r], expert
// e = topk_idx[slot]) -> row send_base[e] + r - offsets[e] of the owner's
// receive buffer.  A warp copies a chunk of 32 x VPL 16-byte vectors.
struct PeerRows {
  uint4 *rows[MOE_EP_MAX_RANKS];
};

template <int VPL>
__global__ void __launch_bounds__(256)
    k_ep_dispatch(const uint4 *__restrict__ x, const int32_t *__restrict__ offsets,
                  const int32_t *__restrict__ row_src, const int32_t *__restrict__ topk_idx,
                  const int32_t *__restrict__ send_base, PeerRows dst, int n_ranks, int E,
                  int k_max, int T, int rows_cap, int recv_cap, int row_vecs, uint32_t *err) {
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
  const int e_loc = E / n_ranks;
  for (long long it = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; it < items;
       it += warps) {
    const int r = (int)(it / chunks), ch = (int)(it % chunks);
    const int a = row_src[r];
    const int t = a / k_max;
    const int e = (a >= 0 && a < rows_cap) ? topk_idx[a] : -1;
    const int owner = e >= 0 ? e / e_loc : -1;
    const int pos = e >= 0 ? send_base[e] + r - offsets[e] : -1;
    if (a < 0 || t >= T || e < 0 || e >= E || owner >= n_ranks || pos < 0 || pos >= recv_cap) {
      if (lane == 0) raise_error(err, kErrIndex);
      continue;
    }
    const uint4 *src = x + (size_t)t * row_vecs;
    uint4 *out = dst.rows[owner] + (size_t)pos * row_vecs;
    const int v0 = ch * kChunkVecs + lane;
    uint4 u[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) u[i] = ldg_nc16(src + v0 + 32 * i);
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) out[v0 + 32 * i] = u[i];
  }
}

// Return: received row p < recv_offsets[E_loc] of this rank (local expert j,
// the i-th row of source s) -> row (rows of s's experts before e) + i of
// s's y_back.  Each block first turns C into the tables it needs: for every
// source s and local expert j, the start of s's rows of e inside the receive
// block of e, and the row in s's own layout where s's rows of e begin.
struct PeerY {
  float *rows[MOE_EP_MAX_RANKS];
};

template <int VPL>
__global__ void __launch_bounds__(256)
    k_ep_return(const uint4 *__restrict__ y, const int32_t *__restrict__ recv_offsets,
                const int32_t *__restrict__ C, PeerY dst, int n_ranks, int E, int rank,
                int src_cap, int recv_cap, int row_vecs, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  extern __shared__ int32_t s_tab[];
  const int e_loc = E / n_ranks, e0 = rank * e_loc;
  int32_t *s_in = s_tab;                         // [e_loc][n_ranks + 1]: source starts in e's block
  int32_t *s_row = s_tab + e_loc * (n_ranks + 1);  // [n_ranks][e_loc]: first row in s's layout
  for (int j = threadIdx.x; j < e_loc; j += blockDim.x) {
    int run = 0;
    for (int s = 0; s < n_ranks; ++s) {
      s_in[j * (n_ranks + 1) + s] = run;
      run += C[(size_t)s * E + e0 + j];
    }
    s_in[j * (n_ranks + 1) + n_ranks] = run;
  }
  for (int s = threadIdx.x; s < n_ranks; s += blockDim.x) {
    int before = 0;
    for (int e = 0; e < e0; ++e) before += C[(size_t)s * E + e];
    for (int j = 0; j < e_loc; ++j) {
      s_row[s * e_loc + j] = before;
      before += C[(size_t)s * E + e0 + j];
    }
  }
  __syncthreads();
  int R = recv_offsets[e_loc];
  if (R > recv_cap || R < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrIndex);
    R = R < 0 ? 0 : recv_cap;
  }
  constexpr int kChunkVecs = 32 * VPL;
  const int lane = threadIdx.x % 32;
  const int chunks = (row_vecs + kChunkVecs - 1) / kChunkVecs;
  const long long items = (long long)R * chunks;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long it = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; it < items;
       it += warps) {
    const int p = (int)(it / chunks), ch = (int)(it % chunks);
    int lo = 0, hi = e_loc - 1;  // local expert: largest j with recv_offsets[j] <= p
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (recv_offsets[mid] <= p)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int j = lo, q = p - recv_offsets[j];
    int s = 0;
    while (s + 1 < n_ranks && s_in[j * (n_ranks + 1) + s + 1] <= q) ++s;
    const int row = s_row[s * e_loc + j] + q - s_in[j * (n_ranks + 1) + s];
    if (q < 0 || row < 0 || row >= src_cap) {
      if (lane == 0) raise_error(err, kErrIndex);
      continue;
    }
    const uint4 *src = y + (size_t)p * row_vecs;
    uint4 *out = reinterpret_cast<uint4 *>(dst.rows[s]) + (size_t)row * row_vecs;
    const int v0 = ch * kChunkVecs + lane;
    uint4 u[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) u[i] = ldg_nc16(src + v0 + 32 * i);
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (v0 + 32 * i < row_vecs) out[v0 + 32 * i] = u[i];
  }
}

int ep_grid(long long warps_needed) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (warps_needed + 7) / 8;
  const long long cap = (long long)sms * 8;
  return (int)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace

cudaError_t launch_ep_plan(const int32_t *C, int n_ranks, int E, int rank, int32_t *recv_offsets,
                           int32_t *send_base, cudaStream_t s) {
  k_ep_plan<<<1, kPlanThreads, 0, s>>>(C, n_ranks, E, rank, recv_offsets, send_base);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const moe_config &c, int n_ranks, void *const *recv_rows,
                               const void *x, const int32_t *offsets, const int32_t *row_src,
                               const int32_t *topk_idx, const int32_t *send_base, uint32_t *err,
                               cudaStream_t s) {
  const int esz = c.dtype == MOE_F32 ? 4 : 2;
  const int rows_cap = c.T * c.k_max;
  const int row_vecs = c.d * esz / 16;
  PeerRows dst{};
  for (int r = 0; r < n_ranks; ++r) dst.rows[r] = static_cast<uint4 *>(recv_rows[r]);
  const long long items = (long long)rows_cap * ((row_vecs + 255) / 256);
  k_ep_dispatch<8><<<ep_grid(items), 256, 0, s>>>(
      static_cast<const uint4 *>(x), offsets, row_src, topk_idx, send_base, dst, n_ranks, c.E,
      c.k_max, c.T, rows_cap, n_ranks * rows_cap, row_vecs, err);
  return cudaGetLastError();
}

cudaError_t launch_ep_return(const moe_config &c, int n_ranks, int rank, const int32_t *C,
                             float *const *y_back, const float *y_recv,
                             const int32_t *recv_offsets, uint32_t *err, cudaStream_t s) {
  const int rows_cap = c.T * c.k_max;
  const int row_vecs = c.d * 4 / 16;  // fp32 rows
  PeerY dst{};
  for (int r = 0; r < n_ranks; ++r) dst.rows[r] = y_back[r];
  const int e_loc = c.E / n_ranks;
  const size_t smem = sizeof(int32_t) * ((size_t)e_loc * (n_ranks + 1) + (size_t)n_ranks * e_loc);
  const long long items = (long long)n_ranks * rows_cap * ((row_vecs + 255) / 256);
  k_ep_return<8><<<ep_grid(items), 256, smem, s>>>(
      reinterpret_cast<const uint4 *>(y_recv), recv_offsets, C, dst, n_ranks, c.E, rank, rows_cap,
      n_ranks * rows_cap, row_vecs, err);
  return cudaGetLastError();
}

}  // namespace moe
