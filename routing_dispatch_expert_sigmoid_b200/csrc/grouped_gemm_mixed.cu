// K5/K6 for ragged groups: full row tiles and swap-AB remainder tiles in one
// persistent launch.
//
// "MoE-Prism" (section 2.A) splits experts into fine-grained sub-experts, and
// "Paralelismo experto para el servicio MoE" (FAQ) notes that expert loads
// are data-dependent: most groups of such a layer hold a few rows, a few
// hold thousands.  A grouped GEMM made of 128-row tiles pays a whole tile of
// tensor work for every group's last, partial tile -- for a group of 2 rows,
// 64 times the useful work -- and those tiles also stream the group's
// weights from HBM on their own.  Here every group is cut into its full
// 128-row chunks, computed as usual (rows = the MMA's M, weights = N), and
// its remainder (1..127 rows), computed swap-AB (weights = M, 128 output
// columns per MMA; rows = N, rounded up to 16).  Both kinds of tile are
// dealt from one list to the same persistent CTAs, so the weight-streaming
// remainder tiles of small groups run alongside the compute-bound tiles of
// large ones instead of in a phase of their own.
//
// The two kinds share one shared-memory stage layout: 16 KB of rows (a
// 128 x 64 tile of A, or up to four 32-row boxes of the remainder) and 32 KB
// of weights (four 64 x 64 MN-major spans: gate and up 128 columns each for
// the up projection, 256 columns for the down projection), and one tensor
// memory layout (two 256-column accumulators).  What differs is the MMA's
// operand order and descriptors and the epilogue's orientation (lane = row
// for full tiles; lane = column, transposed through shared memory, for
// remainder tiles).
//   SWIGLU: h[r, n] = silu(A[r].W1[g][:, n]) * (A[r].W3[g][:, n])   bf16 out
//   PLAIN:  y[r, n] = A[r].W1[g][:, n]                             fp32 out
// Warp 0 issues TMA, warp 1 allocates tensor memory and issues tcgen05.mma,
// warps 2-5 drain the accumulators.  Every mbarrier wait is bounded.  No TMA
// multicast.
#include "tcgen05_common.cuh"

namespace moe {
namespace tc {
namespace {

template <bool SWIGLU>
struct ShapeMixed {
  static constexpr int BN = SWIGLU ? 128 : 256;            // output columns per tile
  static constexpr uint32_t kABytes = BM * BK * 2;         // 16 KB: A tile or remainder rows
  static constexpr uint32_t kSpanBytes = BK * 128;         // 8 KB: 64 K-rows x 64 columns
  static constexpr uint32_t kBBytes = 4 * kSpanBytes;      // 32 KB of weights
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 4;
  static constexpr uint32_t kAccCols = 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kHalf = 128;                   // second swap accumulator
  static constexpr uint32_t kRowBoxBytes = 32 * BK * 2;    // 4 KB: 32 remainder rows
  // full tiles: M = 128 rows, N = 256 (gate | up, or 256 output columns)
  static constexpr uint32_t kIdescFull = instr_desc(BM, 256);
  static constexpr uint32_t kStageRowWords = 36;
  static constexpr uint32_t kEpiBytes = 4 * 32 * kStageRowWords * 4;  // 18 KB
  static constexpr int kBars = 2 * kStages + 5;
  static constexpr size_t kSmemFixed = 1024 + kStages * kStageBytes + 256 + kEpiBytes;
  static_assert(kStageBytes % 1024 == 0, "swizzled tiles on 1024-byte boundaries");
};

// kind::f16 descriptor of a remainder tile: fp32 accumulator, bf16 A and B,
// A (the weights) MN-major, B (the rows) K-major.
__device__ __forceinline__ uint32_t instr_desc_rem(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

struct ParamsMixed {
  const int32_t *offsets;  // [G+1]
  int G, rows_cap, K, N;
  void *out;               // SWIGLU: bf16 [rows_cap, N]; PLAIN: fp32 [rows_cap, N], or y16
  const float *row_w;      // PLAIN: output row r times row_w[w_row_src[r]], or nullptr
  const int32_t *w_row_src;
  uint32_t *err;
  uint64_t wait_limit_ns;
  int8_t *yexp;            // PLAIN: non-null -> out is y16 rows with these block exponents
  int nblk;                // exponents per row: ceil(N / 32)
  // GATHER: row r of A is row row_src[r] / k_max (< a_count) of a_rows [a_count, K]
  const void *a_rows;
  const int32_t *row_src;
  int k_max, a_count;
  int l2_hints;  // L2 eviction hints on the TMA loads (rows kept, weights streamed)
  int lists;     // bit 0: the heavy list, bit 1: the light list
  int phased;    // 1: every heavy tile before the first light one
  int light_evict_first;  // evict-first hint on the light tiles' weights only
};

// A tile of the list: group g, column tile n, and either a full chunk (rows
// row0 .. row0+127) or the group's remainder (nr rows from row0).
struct TileRef {
  int g, n, row0, nr;
  bool full;
};

// GATHER (up projection): the rows of A are token rows of x, row r being
// x[row_src[r] / k_max] -- the dispatch copy fused into the GEMM.  Four more
// warps (6-9) fetch them with cp.async (16 bytes per thread, 8 threads per
// 128-byte row segment) into the 128-byte-swizzled layout the MMA reads, wait
// for their copies, make them visible to the tensor cores (proxy fence) and
// arrive on the stage's "full" barrier, which also counts the weights' TMA
// bytes.  x is read from L2: it is T rows, each needed by its k_t experts.
constexpr int kGatherLag = 2;  // stages a gather warp keeps in flight before it signals

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Deal variants of the tile lists, from the environment: MOE_MIXED_SPLIT=1
// runs the heavy and the light list as two launches, MOE_MIXED_PHASED=1 deals
// every heavy tile before the light ones, MOE_MIXED_LIGHT_EVICT=1 marks the
// light tiles' weights evict-first in L2.
struct MixedOptions {
  int split, phased, light_evict_first;
};
inline MixedOptions mixed_options() {
  auto on = [](const char *name) {
    const char *v = getenv(name);
    return (v && v[0] == '1') ? 1 : 0;
  };
  return {on("MOE_MIXED_SPLIT"), on("MOE_MIXED_PHASED"), on("MOE_MIXED_LIGHT_EVICT")};
}

template <bool SWIGLU, bool GATHER>
__global__ void __launch_bounds__(GATHER ? kThreads + 128 : kThreads, 1)
    k_grouped_gemm_mixed(const __grid_constant__ CUtensorMap tmA,   // rows, 128-row box
                         const __grid_constant__ CUtensorMap tmX,   // rows, 32-row box
                         const __grid_constant__ CUtensorMap tmW1,  // [G, K, N]
                         const __grid_constant__ CUtensorMap tmW3, const ParamsMixed p) {
  grid_dependency();  // the previous grid is complete; the next may launch
  using S = ShapeMixed<SWIGLU>;
  constexpr int kCta = GATHER ? kThreads + 128 : kThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + S::kStages * S::kStageBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + S::kBars);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  float *s_epi = reinterpret_cast<float *>(ring + S::kStages * S::kStageBytes + 256);
  int32_t *s_off =
      reinterpret_cast<int32_t *>(ring + S::kStages * S::kStageBytes + 256 + S::kEpiBytes);
  int32_t *s_tstart = s_off + (p.G + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S::kStages);
  const uint32_t accf0 = smem_addr(bars + 2 * S::kStages);
  const uint32_t acce0 = smem_addr(bars + 2 * S::kStages + 2);
  const uint32_t drain = smem_addr(bars + 2 * S::kStages + 4);
  const Ctl ctl{abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      // the weights' arrive.expect_tx, plus one arrival per gather warp
      mbar_init(full0 + 8 * s, GATHER ? 5 : 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW1);
    if (SWIGLU) prefetch_tmap(&tmW3);
  }
  // Group table: row offsets, then two tile lists, each an exclusive scan of
  // per-group tile counts:
  //   heavy: groups of at least 128 rows -- their full chunks and remainder,
  //          chunks fastest within a column tile (CTAs running together share
  //          the weight tile, L2 serves all but the first read);
  //   light: groups of 1..127 rows -- one remainder tile per column tile.
  // The deal merges the two lists evenly (tile t is light when the count of
  // light tiles among the first t+1 tiles, round-down of (t+1) L / total,
  // steps up), so every wave mixes compute-bound heavy tiles with light tiles
  // that mostly stream their group's weights, instead of running those
  // phases one after the other.
  bool bad = false;
  for (int g = threadIdx.x; g <= p.G; g += kCta) {
    const int v = p.offsets[g];
    s_off[g] = v;
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  int32_t *s_lstart = s_tstart + (p.G + 1);
  const int n_tiles = (p.N + S::BN - 1) / S::BN;
  for (int g = threadIdx.x; g < p.G; g += kCta) {
    const int rows = s_off[g + 1] - s_off[g];
    if (rows < 0) bad = true;
    s_tstart[g] = ((p.lists & 1) && rows >= BM) ? ((rows + BM - 1) / BM) * n_tiles : 0;
    s_lstart[g] = ((p.lists & 2) && rows > 0 && rows < BM) ? n_tiles : 0;
  }
  if (bad) {
    *abort_flag = 1;
    raise_error(p.err, kErrIndex);
  }
  __syncthreads();
  if (warp == 0 || warp == 1) {  // in-place exclusive scans, 32 groups per step
    int32_t *sc = warp == 0 ? s_tstart : s_lstart;
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      const int v = g < p.G ? sc[g] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < p.G) sc[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sc[p.G] = carry;
  }
  if (warp == 1) tmem_relinquish();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_heavy = s_tstart[p.G], n_light = s_lstart[p.G];
  const int total = *abort_flag ? 0 : n_heavy + n_light;
  const int num_kb = (p.K + BK - 1) / BK;

  // largest g with start[g] <= idx (a group with tiles: an empty group shares
  // its start with the next one)
  auto find_group = [&](const int32_t *start, int idx) {
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start[mid] <= idx)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  };
  auto tile_ref = [&](int tile) {
    TileRef t;
    long long l0, l1;
    if (p.phased) {  // heavy tiles 0 .. n_heavy-1, then the light ones
      l0 = tile < n_heavy ? 0 : tile - n_heavy;
      l1 = tile < n_heavy ? 0 : l0 + 1;
    } else {
      l0 = (long long)tile * n_light / total;
      l1 = (long long)(tile + 1) * n_light / total;
    }
    if (l1 > l0) {  // light: the whole group, column tile n
      const int li = (int)l0;
      t.g = find_group(s_lstart, li);
      t.n = li - s_lstart[t.g];
      t.row0 = s_off[t.g];
      t.nr = s_off[t.g + 1] - s_off[t.g];
    } else {  // heavy: chunk m of column tile n
      const int hi = tile - (int)l0;
      t.g = find_group(s_tstart, hi);
      const int rows = s_off[t.g + 1] - s_off[t.g];
      const int chunks = (rows + BM - 1) / BM;
      const int local = hi - s_tstart[t.g];
      t.n = local / chunks;
      const int m = local - t.n * chunks;
      t.row0 = s_off[t.g] + m * BM;
      t.nr = min(BM, rows - m * BM);
    }
    t.full = t.nr == BM;
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0, issued_parity = 0, issued_mask = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileRef t = tile_ref(tile);
        const bool light = !t.full && s_off[t.g + 1] - s_off[t.g] < BM;
        const bool hint_w = p.l2_hints || (p.light_evict_first && light);
        const int nq = t.full ? 0 : (t.nr + 31) / 32;  // remainder: 32-row boxes
        const uint32_t bytes =
            (GATHER ? 0u : (t.full ? S::kABytes : nq * S::kRowBoxBytes)) + S::kBBytes;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait(empty0 + 8 * s, ph ^ 1, ctl)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          const uint32_t fb = full0 + 8 * s;
          mbar_expect_tx(fb, bytes);
          if (GATHER) {
            // the rows come from the gather warps
          } else if (t.full) {
            if (p.l2_hints)
              tma_load_2d_hint(st, &tmA, fb, kb * BK, t.row0, pol_keep);
            else
              tma_load_2d(st, &tmA, fb, kb * BK, t.row0);
          } else {
            for (int q = 0; q < nq; ++q) {
              if (p.l2_hints)
                tma_load_2d_hint(st + q * S::kRowBoxBytes, &tmX, fb, kb * BK, t.row0 + 32 * q,
                                 pol_keep);
              else
                tma_load_2d(st + q * S::kRowBoxBytes, &tmX, fb, kb * BK, t.row0 + 32 * q);
            }
          }
          // weights: four 64-column spans (gate 0-1 and up 2-3, or 256 columns)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const CUtensorMap *m = (SWIGLU && j >= 2) ? &tmW3 : &tmW1;
            const int col = SWIGLU ? t.n * S::BN + (j & 1) * 64 : t.n * S::BN + j * 64;
            if (hint_w)
              tma_load_3d_hint(st + S::kABytes + j * S::kSpanBytes, m, fb, col, kb * BK, t.g,
                               pol_stream);
            else
              tma_load_3d(st + S::kABytes + j * S::kSpanBytes, m, fb, col, kb * BK, t.g);
          }
          issued_mask |= 1u << s;
          issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
          if (++s == S::kStages) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {  // stopped early: let the copies already issued land first
        for (int q = 0; q < S::kStages; ++q)
          if ((issued_mask >> q) & 1u) wait_drain(full0 + 8 * q, (issued_parity >> q) & 1u, p.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, buf = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true, any = false;
      // Shared-memory descriptors of stage 0; the address field counts 16-byte
      // units in bits 0-13 and every stage lies below 256 KB, so stage s, K
      // step kk and weight span j are plain additions to it.  A remainder
      // tile issues eight small MMAs per k-block, so the issuing thread's own
      // instruction count per MMA sets its pace.
      //   rows: K-major 128-byte rows, 8-row groups 1024 B apart, K step 32 B
      //   weights: MN-major 64-column spans kSpanBytes apart (LBO), 8-row K
      //   groups 1024 B apart (SBO), K step 16 rows = 2048 B
      const uint64_t rows_d0 = smem_desc(smem_addr(ring), 16, 1024);
      const uint64_t w_d0 = smem_desc(smem_addr(ring) + S::kABytes, S::kSpanBytes, 1024);
      constexpr uint32_t kStageStep = S::kStageBytes >> 4, kRowK = 32 >> 4, kWK = 2048 >> 4;
      constexpr uint32_t kW3 = (2 * S::kSpanBytes) >> 4;  // spans 2-3: the second 128 columns
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileRef t = tile_ref(tile);
        const uint32_t idesc_rem = instr_desc_rem((t.nr + 15) & ~15);
        if (!wait(acce0 + 8 * buf, acc_ph ^ 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * S::kAccCols;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait(full0 + 8 * s, ph, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t rd = rows_d0 + s * kStageStep, wd = w_d0 + s * kStageStep;
          const uint32_t acc0 = kb != 0;
          if (t.full) {  // rows as A (M = 128), weights as B (N = 256)
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma(d_tmem, rd + kk * kRowK, wd + kk * kWK, S::kIdescFull, kk ? 1u : acc0);
          } else {  // weights as A (two MMAs of 128 columns), rows as B
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t acc = kk ? 1u : acc0;
              umma(d_tmem, wd + kk * kWK, rd + kk * kRowK, idesc_rem, acc);
              umma(d_tmem + S::kHalf, wd + kW3 + kk * kWK, rd + kk * kRowK, idesc_rem, acc);
            }
          }
          any = true;
          umma_commit(empty0 + 8 * s);
          if (++s == S::kStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * buf);
        buf ^= 1;
        if (buf == 0) acc_ph ^= 1;
      }
      if (!ok && any) {  // stopped early: wait for the MMAs in flight
        umma_commit(drain);
        wait_drain(drain, 0, p.err);
      }
    }
    __syncwarp();
  } else if (GATHER && warp >= 6) {
    // ------------------------------------------------------------ row gather
    // Warp gw fetches rows 32*gw .. 32*gw+31 of the tile: instruction k moves
    // rows 32*gw + 4k + lane/8, 16-byte chunk lane%8 of the k-block's 128-byte
    // row segment, into slot chunk ^ (row % 8) (the 128-byte swizzle).  A
    // stage is signalled kGatherLag stages later, once its copies have landed.
    const int gw = warp - 6, c = lane & 7;
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(p.a_rows);
    int s = 0, n_issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileRef t = tile_ref(tile);
      int tok[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = gw * 32 + 4 * k + (lane >> 3);
        tok[k] = -1;
        if (i < t.nr) {
          const int a = p.row_src[t.row0 + i];
          const int tk = a / p.k_max;
          if (a >= 0 && tk < p.a_count)
            tok[k] = tk;
          else if (c == 0)
            raise_error(p.err, kErrIndex);
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        int okw = 1;
        if (lane == 0) okw = wait(empty0 + 8 * s, ph ^ 1, ctl) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) {
          ok = false;
          break;
        }
        const uint32_t st = smem_addr(ring + s * S::kStageBytes);
        const int kcol = kb * BK + c * 8;  // first K element of this lane's chunk
        const uint32_t nbytes = kcol < p.K ? 16u : 0u;  // past K: zeros
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (tok[k] < 0) continue;
          const int i = gw * 32 + 4 * k + (lane >> 3);
          const __nv_bfloat16 *src = x + (size_t)tok[k] * p.K + (nbytes ? kcol : 0);
          cp_async_16(st + i * 128 + ((c ^ (i & 7)) << 4), src, nbytes);
        }
        cp_async_commit();
        if (++n_issued > kGatherLag) {  // the stage issued kGatherLag stages ago
          cp_async_wait<kGatherLag>();
          fence_proxy_async_shared();
          __syncwarp();
          const int sd = (s - kGatherLag + S::kStages) % S::kStages;
          if (lane == 0) mbar_arrive(full0 + 8 * sd);
        }
        if (++s == S::kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    cp_async_wait<0>();  // every copy has landed before the CTA moves on
    if (ok) {  // signal the stages still pending
      fence_proxy_async_shared();
      __syncwarp();
      for (int q = (n_issued < kGatherLag ? n_issued : kGatherLag); q >= 1; --q) {
        const int sd = (s - q + S::kStages) % S::kStages;
        if (lane == 0) mbar_arrive(full0 + 8 * sd);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    int buf = 0;
    uint32_t acc_ph = 0;
    float *stg = s_epi + (warp - 2) * 32 * S::kStageRowWords;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileRef t = tile_ref(tile);
      int ready = 0;
      if (lane == 0) ready = wait(accf0 + 8 * buf, acc_ph, ctl) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + buf * S::kAccCols + ((uint32_t)(quarter * 32) << 16);
      if (t.full) {
        // lane = row: rows row0 + 32*quarter .. of the chunk, 32 columns at a time
        const int row0 = t.row0 + quarter * 32;
        // one 32-column chunk of this warp's 32 rows, from registers to memory
        auto store_chunk = [&](float(&v)[32], int c) {
          const int col = t.n * S::BN + c;
          if (SWIGLU) {  // h: bf16, a staged row is 16 words
            uint32_t *st = reinterpret_cast<uint32_t *>(stg);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
                w[i] = *reinterpret_cast<uint32_t *>(&b2);
              }
              *reinterpret_cast<uint4 *>(st + lane * S::kStageRowWords + 4 * q) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // 8 rows x 64 bytes per instruction
              const int r = i * 8 + (lane >> 2), q = lane & 3;
              const int grow = row0 + r, gcol = col + q * 8;
              const uint4 val =
                  *reinterpret_cast<const uint4 *>(st + r * S::kStageRowWords + 4 * q);
              if (gcol < p.N)
                *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                           (size_t)grow * p.N + gcol) = val;
            }
          } else if (p.yexp) {  // y16: fp16 rows, one exponent per 32-column block
            if (p.row_w) {
              const float wr = p.row_w[p.w_row_src[row0 + lane]];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= wr;
            }
            store_y16_lane_rows(v, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords, lane,
                                row0, row0 + 32, col, p.N, p.out, p.yexp, p.nblk);
          } else {  // y: fp32, a staged row is 32 words
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4 *>(stg + lane * S::kStageRowWords + 4 * q) =
                  make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {  // 4 rows x 128 bytes per instruction
              const int r = i * 4 + (lane >> 3), q = lane & 7;
              const int grow = row0 + r, gcol = col + q * 4;
              float4 o = *reinterpret_cast<const float4 *>(stg + r * S::kStageRowWords + 4 * q);
              if (gcol < p.N) {
                if (p.row_w) {  // the slot's gate weight, applied here instead of in combine
                  const float wr = p.row_w[p.w_row_src[grow]];
                  o.x *= wr;
                  o.y *= wr;
                  o.z *= wr;
                  o.w *= wr;
                }
                *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (size_t)grow * p.N +
                                            gcol) = o;
              }
            }
          }
          __syncwarp();  // the next chunk overwrites the staging buffer
        };
        // two chunks per wait for tensor memory: gate and up of the same
        // columns, or two neighbouring column chunks of the plain product
#pragma unroll 1
        for (int c = 0; c < S::BN; c += SWIGLU ? 32 : 64) {
          float v[32], u[32];
          if (SWIGLU) {
            tmem_ld32x2(tb + c, tb + S::BN + c, v, u);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = silu_times(v[i], u[i]);
            store_chunk(v, c);
          } else {
            tmem_ld32x2(tb + c, tb + c + 32, v, u);
            if (p.yexp) {  // y16: both blocks of a row in one 128-byte segment
              if (p.row_w) {
                const float wr = p.row_w[p.w_row_src[row0 + lane]];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  v[i] *= wr;
                  u[i] *= wr;
                }
              }
              store_y16_lane_rows2(v, u, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords,
                                   lane, row0, row0 + 32, t.n * S::BN + c, p.N, p.out, p.yexp,
                                   p.nblk);
            } else {
              store_chunk(v, c);
              store_chunk(u, c + 32);
            }
          }
        }
      } else {
        // lane = output column (32*quarter .. of each 128-column half), TMEM
        // column = row of the remainder
        for (int h = 0; h < (SWIGLU ? 1 : 2); ++h) {
          const int col0 = t.n * S::BN + h * 128 + quarter * 32;
#pragma unroll 1
          for (int j0 = 0; j0 < t.nr; j0 += 32) {
            float v[32], u[32];  // v[j] = out[row j0 + j][col0 + lane]
            if (SWIGLU)
              tmem_ld32x2(tb + h * S::kHalf + j0, tb + S::kHalf + j0, v, u);
            else
              tmem_ld32(tb + h * S::kHalf + j0, v);
            if (SWIGLU) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = silu_times(v[i], u[i]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[j * S::kStageRowWords + lane] = v[j];
            __syncwarp();
            if (SWIGLU) {  // bf16 rows: 8 lanes x 8 bytes, 4 rows per step
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int j = i * 4 + (lane >> 3), q = lane & 7;
                const int grow = t.row0 + j0 + j, gcol = col0 + q * 4;
                const float4 f =
                    *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
                if (j0 + j < t.nr && gcol < p.N) {
                  __nv_bfloat162 lo = __floats2bfloat162_rn(f.x, f.y);
                  __nv_bfloat162 hi = __floats2bfloat162_rn(f.z, f.w);
                  uint2 w;
                  w.x = *reinterpret_cast<uint32_t *>(&lo);
                  w.y = *reinterpret_cast<uint32_t *>(&hi);
                  *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                             (size_t)grow * p.N + gcol) = w;
                }
              }
            } else if (p.yexp) {
              store_y16_staged(stg, S::kStageRowWords, lane, t.row0 + j0, t.nr - j0, col0, p.N,
                               p.out, p.yexp, p.nblk, p.row_w, p.w_row_src);
            } else {  // fp32 rows: 8 lanes x 16 bytes, 4 rows per step
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int j = i * 4 + (lane >> 3), q = lane & 7;
                const int grow = t.row0 + j0 + j, gcol = col0 + q * 4;
                float4 o =
                    *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
                if (j0 + j < t.nr && gcol < p.N) {
                  if (p.row_w) {
                    const float wr = p.row_w[p.w_row_src[grow]];
                    o.x *= wr;
                    o.y *= wr;
                    o.z *= wr;
                    o.w *= wr;
                  }
                  *reinterpret_cast<float4 *>(static_cast<float *>(p.out) +
                                              (size_t)grow * p.N + gcol) = o;
                }
              }
            }
            __syncwarp();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
      buf ^= 1;
      if (buf == 0) acc_ph ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// 2-D map over rows [rows, K] bf16 (K contiguous), box 64 (K) x box_rows,
// 128-byte swizzle.
bool make_map_rows_m(CUtensorMap *m, const void *A, int rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(A), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the weights [G, K, N] bf16 (N contiguous), box 64 (N) x 64 (K)
// x 1, 128-byte swizzle.
bool make_map_w_m(CUtensorMap *m, const void *B, int G, int K, int N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)K * N * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)BK, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(B), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SWIGLU, bool GATHER>
cudaError_t launch_mixed(int rows_cap, int K, int N, int G, const int32_t *offsets,
                         const void *A, const void *B1, const void *B3, void *out,
                         const float *row_w, const int32_t *w_row_src, uint32_t *err,
                         cudaStream_t s, int8_t *yexp, const int32_t *row_src, int k_max,
                         int a_count) {
  using S = ShapeMixed<SWIGLU>;
  constexpr int kCta = GATHER ? kThreads + 128 : kThreads;
  CUtensorMap ma, mx, mw1, mw3;
  // with GATHER the row maps are not read; they describe the token rows
  const int map_rows = GATHER ? a_count : rows_cap;
  if (!make_map_rows_m(&ma, A, map_rows, K, BM) || !make_map_rows_m(&mx, A, map_rows, K, 32) ||
      !make_map_w_m(&mw1, B1, G, K, N) || !make_map_w_m(&mw3, SWIGLU ? B3 : B1, G, K, N))
    return cudaErrorInvalidValue;
  // group tables: row offsets, heavy and light tile starts
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 3 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_mixed<SWIGLU, GATHER>,
                                    S::kSmemFixed + sizeof(int32_t) * 3 * (kMaxGroups + 1)))
    return e;
  const MixedOptions o = mixed_options();
  ParamsMixed p{offsets, G,   rows_cap, K, N, out, row_w, w_row_src, err,
                pipeline_wait_limit_ns(), yexp, (N + 31) / 32, A, row_src, k_max, a_count,
                l2_hints_enabled(), 3, o.phased, o.light_evict_first};
  const long long max_tiles = (long long)((rows_cap + BM - 1) / BM + G) *
                              ((N + S::BN - 1) / S::BN);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  if (!o.split) {
    launch_k(k_grouped_gemm_mixed<SWIGLU, GATHER>, grid, kCta, smem, s, ma, mx, mw1, mw3, p);
    return cudaGetLastError();
  }
  for (int lists = 1; lists <= 2; ++lists) {  // heavy groups, then light ones
    p.lists = lists;
    launch_k(k_grouped_gemm_mixed<SWIGLU, GATHER>, grid, kCta, smem, s, ma, mx, mw1, mw3, p);
    if (cudaError_t e = cudaGetLastError()) return e;
  }
  return cudaSuccess;
}

}  // namespace
}  // namespace tc

cudaError_t launch_grouped_gemm_mixed(bool swiglu, int rows_cap, int K, int N, int G,
                                      const int32_t *offsets, const void *A, const void *B1,
                                      const void *B3, void *out, uint32_t *err, cudaStream_t s,
                                      const float *row_w, const int32_t *w_row_src,
                                      int8_t *yexp, const int32_t *row_src, int k_max,
                                      int a_rows) {
  if (rows_cap <= 0) return cudaSuccess;
  if (!offsets || G <= 0 || G > tc::kMaxGroups) return cudaErrorInvalidValue;
  if ((row_w || yexp) && swiglu) return cudaErrorInvalidValue;  // down projection only
  if (row_src && (!swiglu || k_max < 1 || a_rows < 1)) return cudaErrorInvalidValue;
  if (row_src)
    return tc::launch_mixed<true, true>(rows_cap, K, N, G, offsets, A, B1, B3, out, nullptr,
                                        nullptr, err, s, nullptr, row_src, k_max, a_rows);
  return swiglu ? tc::launch_mixed<true, false>(rows_cap, K, N, G, offsets, A, B1, B3, out,
                                                nullptr, nullptr, err, s, nullptr, nullptr, 1, 0)
                : tc::launch_mixed<false, false>(rows_cap, K, N, G, offsets, A, B1, B1, out, row_w,
                                                 w_row_src, err, s, yexp, nullptr, 1, 0);
}

}  // namespace moe
