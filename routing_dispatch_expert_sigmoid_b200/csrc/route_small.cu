// K1-K3 for small batches (decode): the router on the tensor cores with K
// split across CTAs, then ONE kernel that sums the partial logits, gates every
// token and, in whichever CTA finishes last, does the histogram, capacity,
// prefix sum and stable ranks of the whole batch.
//
// The operations are those of the three routing kernels ("Paralelismo experto
// para el servicio MoE", sections "Buceo profundo" and "Información técnica":
// a router scores the experts, each token keeps its top-k, a per-expert
// capacity bounds what an expert takes; "Expert Parallelism: MoE 模型的并行切分",
// section 4: the kept rows are grouped by expert).  Only the schedule
// differs: a decode batch of up to 128 tokens is too small to fill the GPU
// with one tile per CTA, so
//   * the router GEMM x[T,d] . Wr[d,E] runs as S independent K slices (the
//     grouped GEMM's split-K mode), each writing fp32 partial logits
//     [S][T][E]; S is a function of the layer's shape alone;
//   * k_route_small: one warp per token adds the S partials (then the logit
//     bias) in a fixed order, stores the logits row and gates the token; each
//     CTA then takes a ticket, and the CTA holding the last ticket ranks all
//     T*k_max slots in shared memory.  No CTA waits for another: the ticket
//     only decides which CTA continues.
// The result is deterministic and, given the same logits, bit-identical to
// the separate kernels (same gating code; same capacity arithmetic).
#include <math.h>
#include <stdlib.h>

#include "gating.cuh"

namespace moe {
namespace {

constexpr int kWarps = 4;                   // tokens per CTA, one warp each
constexpr int kSmallMaxT = 128;             // largest batch taking this path
constexpr size_t kPartialBudget = 768u << 10;  // fp32 partial logits, bytes
constexpr int kSplitTarget = 148;           // CTAs to aim for (SMs of a B200)
constexpr int kBK = 64;                     // K per pipeline stage of the GEMM
constexpr int kBN = 64;                     // output columns per GEMM tile
constexpr int kBatch = 8;                   // slices loaded per step (columns of <= 16)

struct SmallArgs {
  gating::GatingArgs g;  // g.logits is the row this kernel writes
  float *logits;
  const float *partials;  // [S][T][E]
  int S;
  const float *logit_bias;
  int32_t *ticket;
  int32_t *counts, *kept, *offsets, *slot_row, *row_src, *n_dropped;
  double cf;
};

// The last CTA: per-expert counts, capacity, kept, offsets and the stable
// rank of every slot, for n = T*k_max slots with kWarps warps.  Warp w takes
// slots [w*seg, (w+1)*seg) and starts each expert's rank at that expert's
// count in the earlier segments.
__device__ void rank_slots(const SmallArgs &a, int32_t *smem) {
  const int E = a.g.E, n = a.g.T * a.g.k_max;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int32_t *s_idx = smem;                 // [n]
  int32_t *s_base = s_idx + n;           // [kWarps][E]: segment counts, then running ranks
  int32_t *s_cnt = s_base + kWarps * E;  // [E]: kept
  int32_t *s_off = s_cnt + E;            // [E]
  __shared__ long long s_red[kWarps];
  __shared__ int s_wsum[kWarps];

  bool bad = false;
  for (int i = tid; i < n; i += kWarps * 32) {
    int e = __ldcg(a.g.topk_idx + i);
    if (e != -1 && (e < 0 || e >= E)) {
      bad = true;
      e = -1;
    }
    s_idx[i] = e;
  }
  for (int i = tid; i < kWarps * E; i += kWarps * 32) s_base[i] = 0;
  if (bad) raise_error(a.g.err, kErrRouting);
  __syncthreads();
  const int seg = (n + kWarps - 1) / kWarps;
  const int a0 = min(warp * seg, n), a1 = min(a0 + seg, n);
  for (int i = a0 + lane; i < a1; i += 32) {
    const int e = s_idx[i];
    if (e >= 0) atomicAdd(&s_base[warp * E + e], 1);
  }
  __syncthreads();
  long long my = 0;
  for (int e = tid; e < E; e += kWarps * 32) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int v = s_base[w * E + e];
      s_base[w * E + e] = run;
      run += v;
    }
    s_cnt[e] = run;
    a.counts[e] = run;
    my += run;
  }
  for (int off = 16; off > 0; off >>= 1) my += __shfl_xor_sync(0xffffffffu, my, off);
  if (lane == 0) s_red[warp] = my;
  __syncthreads();
  long long sum_k = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) sum_k += s_red[w];
  long long C = -1;
  if (a.cf > 0.0) C = (long long)ceil(a.cf * (double)sum_k / (double)E);

  // kept = min(count, C); offsets = exclusive scan of kept.  Thread tid owns
  // experts [tid*per, tid*per + per).
  const int per = (E + kWarps * 32 - 1) / (kWarps * 32);
  const int e0 = min(tid * per, E), e1 = min(e0 + per, E);
  int local = 0;
  for (int e = e0; e < e1; ++e) {
    int k = s_cnt[e];
    if (C >= 0 && k > C) k = (int)C;
    s_cnt[e] = k;
    a.kept[e] = k;
    local += k;
  }
  int incl = local;
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int run = incl - local;
  for (int w = 0; w < warp; ++w) run += s_wsum[w];
  for (int e = e0; e < e1; ++e) {
    s_off[e] = run;
    a.offsets[e] = run;
    run += s_cnt[e];
  }
  if (tid == kWarps * 32 - 1) {
    a.offsets[E] = run;  // the last thread's running sum is the total kept
    a.n_dropped[0] = (int32_t)(sum_k - run);
  }
  __syncthreads();

  // Stable ranks: lanes with the same expert find each other with
  // __match_any_sync and order themselves by lane on top of the running rank.
  for (int base = a0; base < a1; base += 32) {
    const int i = base + lane;
    const bool valid = i < a1;
    const int e = valid ? s_idx[i] : -1;
    const bool real = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, real ? e : E + lane);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int start = real ? s_base[warp * E + e] : 0;
    __syncwarp();
    if (real) {
      const int rho = start + before;
      if (lane == 31 - __clz(peers)) s_base[warp * E + e] = start + __popc(peers);
      if (C >= 0 && rho >= C) {
        a.slot_row[i] = -1;
      } else {
        const int row = s_off[e] + rho;
        a.slot_row[i] = row;
        a.row_src[row] = i;
      }
    } else if (valid) {
      a.slot_row[i] = -1;
    }
    __syncwarp();
  }
}

template <int NPL>
__global__ void __launch_bounds__(kWarps * 32) k_route_small(SmallArgs a) {
  grid_dependency();  // the previous grid is complete; the next may launch
  extern __shared__ int32_t s_dyn[];
  __shared__ int s_last;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int T = a.g.T, E = a.g.E;
  const int t = blockIdx.x * kWarps + warp;
  if (t < T) {
    float *row = a.logits + (size_t)t * E;
    const float *pt = a.partials + (size_t)t * E;
    const size_t slab = (size_t)T * E;
    const int S = a.S;
    if (NPL == 1 && E <= 16) {
      // 32/E lanes share a column: lane l sums slices l/E, l/E + 32/E, ...
      // of column l % E, then the column's lanes are added in lane order.
      const int lpc = 32 / E, e = lane % E, sub = lane / E;
      float v = 0.f;
      for (int s0 = sub; s0 < S; s0 += kBatch * lpc) {
        float b[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)  // clamped address: every load is issued
          b[j] = pt[(size_t)min(s0 + j * lpc, S - 1) * slab + e];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (s0 + j * lpc < S) v += b[j];
      }
      float tot = __shfl_sync(0xffffffffu, v, e);
      for (int q = 1; q < lpc; ++q) tot += __shfl_sync(0xffffffffu, v, e + q * E);
      if (lane < E) row[e] = a.logit_bias ? tot + a.logit_bias[e] : tot;
    } else {
      // lane l owns columns l, l+32, ...: per step, kSteps slices x NPL
      // columns of independent loads, added in slice order per column
      constexpr int kSteps = NPL >= 16 ? 1 : 16 / NPL;
      float acc[NPL];
#pragma unroll
      for (int i = 0; i < NPL; ++i) acc[i] = 0.f;
      for (int s0 = 0; s0 < S; s0 += kSteps) {
        float b[kSteps][NPL];
#pragma unroll
        for (int j = 0; j < kSteps; ++j)
#pragma unroll
          for (int i = 0; i < NPL; ++i)
            b[j][i] = pt[(size_t)min(s0 + j, S - 1) * slab + min(i * 32 + lane, E - 1)];
#pragma unroll
        for (int j = 0; j < kSteps; ++j)
#pragma unroll
          for (int i = 0; i < NPL; ++i)
            if (s0 + j < S) acc[i] += b[j][i];
      }
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) row[e] = a.logit_bias ? acc[i] + a.logit_bias[e] : acc[i];
      }
    }
    __syncwarp();  // a lane reads back only its own entries; this orders the warp
    gating::gate_token<NPL>(a.g, t, row, reinterpret_cast<float *>(s_dyn) + warp * E);
  }
  __threadfence();  // every thread's topk_idx stores before the CTA's ticket
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(a.ticket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();  // every other CTA's stores are visible past its ticket
  rank_slots(a, s_dyn);
}

template <int NPL>
cudaError_t run(const SmallArgs &a, size_t smem, cudaStream_t s) {
  const int blocks = (a.g.T + kWarps - 1) / kWarps;
  launch_k(k_route_small<NPL>, blocks, kWarps * 32, smem, s, a);
  return cudaGetLastError();
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

SmallRoutePlan small_route_plan(const moe_config &c) {
  // MOE_SMALL_ROUTE=0 keeps decode batches on the separate routing kernels
  static const bool enabled = [] {
    const char *v = getenv("MOE_SMALL_ROUTE");
    return !(v && v[0] == '0');
  }();
  SmallRoutePlan p;
  if (!enabled) return p;
  if (c.dtype != MOE_BF16 || c.E % 8 != 0 || c.T < 1 || c.T > kSmallMaxT) return p;
  const int num_kb = (c.d + kBK - 1) / kBK;
  const int n_tiles = (c.E + kBN - 1) / kBN;
  long long S = kSplitTarget / n_tiles;
  const long long by_budget = (long long)(kPartialBudget / (sizeof(float) * (size_t)c.T * c.E));
  if (S > by_budget) S = by_budget;
  if (S > num_kb) S = num_kb;
  if (S < 1) S = 1;
  const int kb_per = (int)((num_kb + S - 1) / S);
  p.use = true;
  p.S = (num_kb + kb_per - 1) / kb_per;  // no empty slice
  p.k_split = kb_per * kBK;
  p.partial_bytes = up256(sizeof(float) * (size_t)p.S * c.T * c.E);
  p.scratch_bytes = p.partial_bytes + 256;  // + the ticket word
  return p;
}

size_t route_scratch_bytes(const moe_config &c) {
  const SmallRoutePlan p = small_route_plan(c);
  return p.use ? p.scratch_bytes : capacity_scratch_bytes(c);
}

cudaError_t launch_route_small(const moe_config &c, const SmallRoutePlan &plan, const void *x,
                               const void *Wr, const float *logit_bias, const float *sel_bias,
                               const int32_t *k_per_token, const moe_route_out &o, void *scratch,
                               uint32_t *err, cudaStream_t s) {
  float *partials = static_cast<float *>(scratch);
  int32_t *ticket =
      reinterpret_cast<int32_t *>(static_cast<char *>(scratch) + plan.partial_bytes);
  cudaError_t e = launch_router_split(c.T, c.d, c.E, plan.S, plan.k_split, x, Wr, partials,
                                      ticket, err, s);
  if (e != cudaSuccess) return e;
  SmallArgs a{};
  a.g = gating::GatingArgs{o.logits,      sel_bias, k_per_token, o.topk_idx,
                           o.topk_w,      c.T,      c.E,         c.k_max,
                           c.gating,      c.n_groups, c.topk_groups, c.group_score_topk,
                           c.routed_scale, err};
  a.logits = o.logits;
  a.partials = partials;
  a.S = plan.S;
  a.logit_bias = logit_bias;
  a.ticket = ticket;
  a.counts = o.counts;
  a.kept = o.kept;
  a.offsets = o.offsets;
  a.slot_row = o.slot_row;
  a.row_src = o.row_src;
  a.n_dropped = o.n_dropped;
  a.cf = (double)c.capacity_factor;
  // shared memory: the larger of the gating buffers and the ranking tables
  const size_t n = (size_t)c.T * c.k_max;
  const size_t gate_b = sizeof(float) * kWarps * (size_t)c.E;
  const size_t rank_b = sizeof(int32_t) * (n + (size_t)(kWarps + 2) * c.E);
  const size_t smem = gate_b > rank_b ? gate_b : rank_b;
  const int npl = (c.E + 31) / 32;
  if (npl <= 1) return run<1>(a, smem, s);
  if (npl <= 2) return run<2>(a, smem, s);
  if (npl <= 4) return run<4>(a, smem, s);
  if (npl <= 8) return run<8>(a, smem, s);
  if (npl <= 16) return run<16>(a, smem, s);
  return run<32>(a, smem, s);
}

}  // namespace moe
