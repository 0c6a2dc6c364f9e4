// K3 -- per-expert histogram, capacity, prefix sum and stable dispatch ranks.
//
// "Paralelismo experto para el servicio MoE", section "Información técnica"
// and FAQ: a per-expert capacity bounds the tokens an expert takes; the rest
// are dropped.  "Expert Parallelism: MoE 模型的并行切分", section 4 ("Token
// sorting") and question 4 (no padding): tokens bound for the same expert are
// grouped together, in a ragged (unpadded) layout.
//
// Slots a = t*k_max + j are admitted per expert in (t, j) order; the first C
// of each expert are kept.  Positions are decided without atomics, so the
// layout is deterministic and equals a stable sort of the kept slots by
// expert:
//   K3a  one CTA per chunk of kChunk slots: per-chunk expert histogram
//        (shared-memory atomics; counts do not depend on order);
//   K3b  one CTA per 32 experts: per expert, exclusive scan of the chunk
//        histograms (the chunk's first rank; each expert's chunks split into
//        ranges summed by separate warps) and its total; the last CTA to
//        finish (an atomic ticket only picks which one) computes
//        C = ceil(cf * sum k_t / E) in double, kept = min(count, C),
//        offsets = exclusive scan of kept, drops;
//   K3c  one CTA per chunk, eight warps of 128 slots each: a warp counts its
//        slots per expert, the counts give each warp's first rank per
//        expert, then each warp walks its slots 32 at a time in order; lanes
//        with the same expert find each other with __match_any_sync and rank
//        themselves by lane order on top of the warp's running count.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kChunk = 1024;

int num_chunks(const moe_config &c) {
  const long long slots = (long long)c.T * c.k_max;
  return (int)((slots + kChunk - 1) / kChunk);
}

__global__ void __launch_bounds__(256) k_hist(const int32_t *__restrict__ idx, long long n_slots,
                                              int E, int32_t *__restrict__ chunk_counts,
                                              int32_t *__restrict__ ticket, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  extern __shared__ int32_t cnt[];
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0;  // the scan's ticket
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const long long a0 = (long long)blockIdx.x * kChunk;
  const long long a1 = min(a0 + kChunk, n_slots);
  bool bad = false;
  for (long long a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
    const int e = idx[a];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else if (e != -1)
      bad = true;
  }
  if (bad) raise_error(err, kErrRouting);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

constexpr int kScanThreads = 1024;
constexpr int kScanBatch = 16;    // chunk histograms loaded before they are summed
constexpr int kScanExperts = 32;  // experts per CTA: lane = expert, warp = chunk range

// One CTA per 32 experts.  Expert e's chunks are split into 32 contiguous
// ranges, one warp each (lane = expert, so a warp's loads are one 128-byte
// row of a chunk histogram): the ranges are summed, each thread takes the sum
// of the earlier ranges as its base and writes its chunks' bases; the last
// range's end is the expert's count.  The CTA that finishes last (a ticket,
// zeroed by the histogram kernel) then computes, for all experts, the
// capacity, kept counts, offsets and drops.
__global__ void __launch_bounds__(kScanThreads)
    k_scan(const int32_t *__restrict__ chunk_counts, int n_chunks, int E, double cf,
           int32_t *__restrict__ chunk_base, int32_t *__restrict__ counts,
           int32_t *__restrict__ kept, int32_t *__restrict__ offsets,
           int32_t *__restrict__ n_dropped, int32_t *__restrict__ cap_out,
           int32_t *__restrict__ ticket) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ long long s_part[kScanThreads / 32];
  __shared__ long long s_total;
  __shared__ int32_t s_sum[32][kScanExperts + 1];  // [range][expert] range sums
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  {
    const int e = blockIdx.x * kScanExperts + lane;
    const bool ev = e < E;
    const int per = (n_chunks + 31) / 32;
    const int c0 = min(warp * per, n_chunks), c1 = min(c0 + per, n_chunks);
    int sum = 0;
    for (int c = c0; c < c1; c += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        v[i] = ev && c + i < c1 ? chunk_counts[(size_t)(c + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) sum += v[i];
    }
    s_sum[warp][lane] = sum;
    __syncthreads();
    int run = 0;
    for (int q = 0; q < warp; ++q) run += s_sum[q][lane];
    for (int c = c0; c < c1; c += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        v[i] = ev && c + i < c1 ? chunk_counts[(size_t)(c + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        if (c + i < c1) {
          if (ev) chunk_base[(size_t)(c + i) * E + e] = run;
          run += v[i];
        }
    }
    if (warp == 31 && ev) counts[e] = run;
  }
  if (gridDim.x > 1) {
    __threadfence();  // this CTA's counts before its ticket
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();  // every other CTA's counts are visible past its ticket
  }
  __syncthreads();
  long long my = 0;
  if (tid < E) my = __ldcg(counts + tid);
  // block sum of counts = sum over tokens of k_t
  long long v = my;
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) s_part[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = s_part[lane];
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if (lane == 0) s_total = w;
  }
  __syncthreads();
  const long long sum_k = s_total;
  long long C = -1;
  if (cf > 0.0) C = (long long)ceil(cf * (double)sum_k / (double)E);
  int k = 0;
  if (tid < E) {
    k = (int)my;
    if (C >= 0 && k > C) k = (int)C;
    kept[tid] = k;
  }
  // exclusive scan of kept over experts
  int incl = k;
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  __syncthreads();
  if (lane == 31) s_part[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = s_part[lane];
    long long winc = w;
    for (int off = 1; off < 32; off <<= 1) {
      long long o = __shfl_up_sync(0xffffffffu, winc, off);
      if (lane >= off) winc += o;
    }
    s_part[lane] = winc - w;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = (int)s_part[warp] + incl - k;
  if (tid < E) offsets[tid] = excl;
  if (tid == E - 1) {
    offsets[E] = excl + k;
    n_dropped[0] = (int32_t)(sum_k - (excl + k));
    cap_out[0] = C < 0 ? -1 : (C > 0x7fffffffLL ? 0x7fffffff : (int32_t)C);
  }
}

// kRankWarps warps per chunk, warp w walking slots [w 128, (w+1) 128) of it:
// each warp first counts its own slots per expert, the counts become each
// warp's first rank per expert (the chunk's base plus the earlier warps'
// counts), then every warp walks its 128 slots in order.  The ranks are the
// same as one warp walking the whole chunk; the walk is 4 steps instead of 32.
constexpr int kRankWarps = kChunk / 128;

__global__ void __launch_bounds__(32 * kRankWarps)
    k_rank(const int32_t *__restrict__ idx, long long n_slots, int E,
           const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ offsets,
           const int32_t *__restrict__ cap, int32_t *__restrict__ slot_row,
           int32_t *__restrict__ row_src) {
  grid_dependency();  // the previous grid is complete; the next may launch
  extern __shared__ int32_t s_rank[];  // run[kRankWarps][E] (running ranks), off[E] (first row)
  int32_t *off = s_rank + kRankWarps * E;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int32_t *run = s_rank + warp * E;
  const long long a0 = (long long)blockIdx.x * kChunk + warp * 128;
  const long long a1 = min((long long)blockIdx.x * kChunk + kChunk, n_slots);
  int ev[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long a = a0 + 32 * i + lane;
    ev[i] = a < a1 ? idx[a] : -1;
  }
  for (int i = threadIdx.x; i < kRankWarps * E; i += blockDim.x) s_rank[i] = 0;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (ev[i] >= 0 && ev[i] < E) atomicAdd(&run[ev[i]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int base = chunk_base[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kRankWarps; ++w) {
      const int c = s_rank[w * E + e];
      s_rank[w * E + e] = base;
      base += c;
    }
    off[e] = offsets[e];
  }
  const int C = cap[0];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long a = a0 + 32 * i + lane;
    const bool valid = a < a1;
    const int e = ev[i];
    const bool real = valid && e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, real ? e : E + lane);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int start = real ? run[e] : 0;
    __syncwarp();
    if (real) {
      const int rho = start + before;
      if (lane == 31 - __clz(peers)) run[e] = start + __popc(peers);
      if (C >= 0 && rho >= C) {
        slot_row[a] = -1;
      } else {
        const int row = off[e] + rho;
        slot_row[a] = row;
        row_src[row] = (int32_t)a;
      }
    } else if (valid) {
      slot_row[a] = -1;
    }
    __syncwarp();
  }
}

}  // namespace

size_t capacity_scratch_bytes(const moe_config &c) {
  // chunk_counts + chunk_base (n_chunks x E each) + capacity word, 256-byte aligned
  const size_t n = (size_t)num_chunks(c) * c.E;
  return ((2 * n * sizeof(int32_t) + 255) / 256) * 256 + 256;
}

cudaError_t launch_capacity(const moe_config &c, const int32_t *topk_idx, int32_t *counts,
                            int32_t *kept, int32_t *offsets, int32_t *slot_row,
                            int32_t *row_src, int32_t *n_dropped, void *scratch, uint32_t *err,
                            cudaStream_t s) {
  const int nch = num_chunks(c);
  const long long slots = (long long)c.T * c.k_max;
  const size_t n = (size_t)nch * c.E;
  int32_t *chunk_counts = static_cast<int32_t *>(scratch);
  int32_t *chunk_base = chunk_counts + n;
  int32_t *cap = reinterpret_cast<int32_t *>(static_cast<char *>(scratch) +
                                             ((2 * n * sizeof(int32_t) + 255) / 256) * 256);
  const size_t eb = sizeof(int32_t) * (size_t)c.E;
  int32_t *ticket = cap + 1;  // in the scratch's last 256 bytes, with the capacity word
  if (nch > 0) launch_k(k_hist, nch, 256, eb, s, topk_idx, slots, c.E, chunk_counts, ticket, err);
  // one CTA when there is no histogram kernel to zero the ticket
  const int scan_ctas = nch > 0 ? (c.E + kScanExperts - 1) / kScanExperts : 1;
  launch_k(k_scan, scan_ctas, kScanThreads, 0, s, chunk_counts, nch, c.E, (double)c.capacity_factor,
                                            chunk_base, counts, kept, offsets, n_dropped, cap,
                                            ticket);
  if (nch > 0)
    launch_k(k_rank, nch, 32 * kRankWarps, (kRankWarps + 1) * eb, s, topk_idx, slots, c.E, chunk_base,
                                                                offsets, cap, slot_row, row_src);
  return cudaGetLastError();
}

}  // namespace moe
