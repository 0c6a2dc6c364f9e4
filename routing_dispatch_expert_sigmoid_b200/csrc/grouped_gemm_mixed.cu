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
};

// A tile of the list: group g, column tile n, and either a full chunk (rows
// row0 .. row0+127) or the group's remainder (nr rows from row0).
struct TileRef {
  int g, n, row0, nr;
  bool full;
};

template <bool SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_mixed(const __grid_constant__ CUtensorMap tmA,   // rows, 128-row box
                         const __grid_constant__ CUtensorMap tmX,   // rows, 32-row box
                         const __grid_constant__ CUtensorMap tmW1,  // [G, K, N]
                         const __grid_constant__ CUtensorMap tmW3, const ParamsMixed p) {
  using S = ShapeMixed<SWIGLU>;
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
      mbar_init(full0 + 8 * s, 1);
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
  // Group table: row offsets and tile starts (chunks = ceil(rows / 128) per
  // column tile), checked against the buffer size.
  bool bad = false;
  for (int g = threadIdx.x; g <= p.G; g += kThreads) {
    const int v = p.offsets[g];
    s_off[g] = v;
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  const int n_tiles = (p.N + S::BN - 1) / S::BN;
  for (int g = threadIdx.x; g < p.G; g += kThreads) {
    const int rows = s_off[g + 1] - s_off[g];
    if (rows < 0) bad = true;
    s_tstart[g] = rows > 0 ? ((rows + BM - 1) / BM) * n_tiles : 0;
  }
  if (bad) {
    *abort_flag = 1;
    raise_error(p.err, kErrIndex);
  }
  __syncthreads();
  if (warp == 0) {  // in-place exclusive scan, 32 groups per step
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      const int v = g < p.G ? s_tstart[g] : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < p.G) s_tstart[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_tstart[p.G] = carry;
  }
  if (warp == 1) tmem_relinquish();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = *abort_flag ? 0 : s_tstart[p.G];
  const int num_kb = (p.K + BK - 1) / BK;

  // tile -> (group, column tile, chunk), chunks fastest: CTAs running at the
  // same time share a weight tile
  auto tile_ref = [&](int tile) {
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= tile)
        lo = mid;
      else
        hi = mid - 1;
    }
    TileRef t;
    t.g = lo;
    const int rows = s_off[lo + 1] - s_off[lo];
    const int chunks = (rows + BM - 1) / BM;
    const int local = tile - s_tstart[lo];
    t.n = local / chunks;
    const int m = local - t.n * chunks;
    t.row0 = s_off[lo] + m * BM;
    t.nr = min(BM, rows - m * BM);
    t.full = t.nr == BM;
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued_parity = 0, issued_mask = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileRef t = tile_ref(tile);
        const int nq = t.full ? 0 : (t.nr + 31) / 32;  // remainder: 32-row boxes
        const uint32_t bytes = (t.full ? S::kABytes : nq * S::kRowBoxBytes) + S::kBBytes;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait(empty0 + 8 * s, ph ^ 1, ctl)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          const uint32_t fb = full0 + 8 * s;
          mbar_expect_tx(fb, bytes);
          if (t.full) {
            tma_load_2d(st, &tmA, fb, kb * BK, t.row0);
          } else {
            for (int q = 0; q < nq; ++q)
              tma_load_2d(st + q * S::kRowBoxBytes, &tmX, fb, kb * BK, t.row0 + 32 * q);
          }
          // weights: four 64-column spans (gate 0-1 and up 2-3, or 256 columns)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const CUtensorMap *m = (SWIGLU && j >= 2) ? &tmW3 : &tmW1;
            const int col = SWIGLU ? t.n * S::BN + (j & 1) * 64 : t.n * S::BN + j * 64;
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
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          const uint32_t wt = st + S::kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            // rows: K-major 128-byte rows, 8-row groups 1024 B apart, K step 32 B
            const uint64_t rd = smem_desc(st + kk * 32, 16, 1024);
            if (t.full) {
              // weights as B: MN-major, 64-column spans kSpanBytes apart (LBO),
              // 8-row K groups 1024 B apart (SBO); K step 16 rows = 2048 B
              const uint64_t bd = smem_desc(wt + kk * 2048, S::kSpanBytes, 1024);
              umma(d_tmem, rd, bd, S::kIdescFull, acc);
            } else {
              // weights as A (128 columns = spans 0-1, and spans 2-3), rows as B
              const uint64_t w0 = smem_desc(wt + kk * 2048, S::kSpanBytes, 1024);
              const uint64_t w1 = smem_desc(wt + 2 * S::kSpanBytes + kk * 2048, S::kSpanBytes, 1024);
              umma(d_tmem, w0, rd, idesc_rem, acc);
              umma(d_tmem + S::kHalf, w1, rd, idesc_rem, acc);
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
#pragma unroll 1
        for (int c = 0; c < S::BN; c += 32) {
          float v[32];
          tmem_ld32(tb + c, v);
          if (SWIGLU) {
            float u[32];
            tmem_ld32(tb + S::BN + c, u);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = (v[i] / (1.0f + __expf(-v[i]))) * u[i];
          }
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
        }
      } else {
        // lane = output column (32*quarter .. of each 128-column half), TMEM
        // column = row of the remainder
        for (int h = 0; h < (SWIGLU ? 1 : 2); ++h) {
          const int col0 = t.n * S::BN + h * 128 + quarter * 32;
#pragma unroll 1
          for (int j0 = 0; j0 < t.nr; j0 += 32) {
            float v[32];
            tmem_ld32(tb + h * S::kHalf + j0, v);  // v[j] = out[row j0 + j][col0 + lane]
            if (SWIGLU) {
              float u[32];
              tmem_ld32(tb + S::kHalf + j0, u);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = (v[i] / (1.0f + __expf(-v[i]))) * u[i];
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

template <bool SWIGLU>
cudaError_t launch_mixed(int rows_cap, int K, int N, int G, const int32_t *offsets,
                         const void *A, const void *B1, const void *B3, void *out,
                         const float *row_w, const int32_t *w_row_src, uint32_t *err,
                         cudaStream_t s, int8_t *yexp) {
  using S = ShapeMixed<SWIGLU>;
  CUtensorMap ma, mx, mw1, mw3;
  if (!make_map_rows_m(&ma, A, rows_cap, K, BM) || !make_map_rows_m(&mx, A, rows_cap, K, 32) ||
      !make_map_w_m(&mw1, B1, G, K, N) || !make_map_w_m(&mw3, SWIGLU ? B3 : B1, G, K, N))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_mixed<SWIGLU>,
                                    S::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  ParamsMixed p{offsets, G,   rows_cap, K, N, out, row_w, w_row_src, err,
                pipeline_wait_limit_ns(), yexp, (N + 31) / 32};
  const long long max_tiles = (long long)((rows_cap + BM - 1) / BM + G) *
                              ((N + S::BN - 1) / S::BN);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  k_grouped_gemm_mixed<SWIGLU><<<grid, kThreads, smem, s>>>(ma, mx, mw1, mw3, p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

cudaError_t launch_grouped_gemm_mixed(bool swiglu, int rows_cap, int K, int N, int G,
                                      const int32_t *offsets, const void *A, const void *B1,
                                      const void *B3, void *out, uint32_t *err, cudaStream_t s,
                                      const float *row_w, const int32_t *w_row_src,
                                      int8_t *yexp) {
  if (rows_cap <= 0) return cudaSuccess;
  if (!offsets || G <= 0 || G > tc::kMaxGroups) return cudaErrorInvalidValue;
  if ((row_w || yexp) && swiglu) return cudaErrorInvalidValue;  // down projection only
  return swiglu ? tc::launch_mixed<true>(rows_cap, K, N, G, offsets, A, B1, B3, out, nullptr,
                                         nullptr, err, s, nullptr)
                : tc::launch_mixed<false>(rows_cap, K, N, G, offsets, A, B1, B1, out, row_w,
                                          w_row_src, err, s, yexp);
}

}  // namespace moe
