// K5/K6 on fp8 expert weights for decode-sized groups: tcgen05.mma kind::f8f6f4.
//
// "LLM MoE Expert Parallel 生产实战", section 5 serves DeepSeek-V3 with fp8
// quantisation, and section 10 asks that it leave the router head alone: the
// experts' matrices are e4m3 codes with one fp32 scale per output column
// (include/moe.h), everything else stays bf16.  At decode size a layer is a
// stream of expert weights, so halving their bytes halves its time -- if the
// weights reach the tensor cores without per-weight work on the SM.  Here they
// do: TMA brings the codes from HBM into shared memory and the MMA reads them
// there as its e4m3 A operand.
//
// The activations (x rows for the up projection, h rows for the down
// projection) are bf16.  The MMA's other operand must be an 8-bit float too,
// so each activation row is split into two e4m3 planes with one power-of-two
// scale per row (k_split_planes below):
//   s = 2^k, the smallest with max|v| / s <= 448, so max|v| / s is in (224, 448]
//   q0 = e4m3(v / s),  q1 = e4m3(v / s - q0)           (round to nearest even)
// v / s is exact (a power-of-two scaling of a bf16 value).  A bf16 value has 8
// significant bits: q0 keeps the top 4 (the remainder v/s - q0 is exact in
// fp32, an integer multiple of v/s's last bit no larger than 8 of them), and
// q1 holds that remainder exactly whenever its last bit is at least 2^-9, the
// smallest e4m3 step -- for every element with |v| >= s / 4, i.e. within
// 2^9.8 of the row's largest magnitude.  Smaller elements keep an absolute
// error of at most 2^-10 s < 2^-17.8 max|v|.  The tensor cores multiply e4m3
// by e4m3 exactly and accumulate in fp32; the epilogue multiplies by the
// column scale and the row scale.  So the fp8 layer computes with the same
// bf16 activations as the bf16 layer, up to those tiniest elements.
//
// Engine: swap-AB, like the bf16 decode engine -- the weights are the MMA's M
// operand (128 output columns), a group's rows its N operand (up to kQRows
// per tile, N = rows rounded up to 16).  One CTA per SM, persistent, 192
// threads, warp-specialised:
//   warp 0     TMA producer: per k-block of 128 K, two code tiles (128 columns
//              x 128 bytes, 128-byte swizzle) and the tile's rows of both
//              planes (16-row boxes, as many as the tile has rows);
//   warp 1     allocates tensor memory; one thread issues tcgen05.mma
//              kind::f8f6f4 (M=128, K=32), one per plane and code tile per
//              K step, into two accumulators (up projection: gate and up of
//              the same 128 columns; down projection: two 128-column halves
//              of a 256-column tile);
//   warps 2-5  epilogue: tcgen05.ld (lane = output column, TMEM column =
//              row), scales, SiLU-gate product for the up projection,
//              transposed through shared memory into row-major h (bf16) or
//              y (fp32).
// Every mbarrier wait is bounded like those of the bf16 engines.  No TMA
// multicast.
#include <cuda_fp8.h>

#include "tcgen05_common.cuh"

namespace moe {
namespace tc {
namespace {

constexpr int kQK = 128;    // K per stage: one 128-byte swizzle span of e4m3
constexpr int kQRows = 32;  // rows per tile (the MMA's N, at most)
constexpr int kPlanes = 2;
constexpr int kRowBoxQ = 16;  // rows per TMA box of a plane

template <bool SWIGLU>
struct ShapeF8 {
  static constexpr int kCols = 128;                       // columns per code tile (MMA M)
  static constexpr int kTileCols = SWIGLU ? 128 : 256;    // output columns per tile
  static constexpr uint32_t kCodeBytes = kCols * kQK;     // 16 KB
  static constexpr uint32_t kPlaneBytes = kQRows * kQK;   // 4 KB: the tile's rows of one plane
  static constexpr uint32_t kStageBytes = 2 * kCodeBytes + kPlanes * kPlaneBytes;  // 40 KB
  // A decode-sized layer streams every weight once, so the pace is set by the
  // bytes each SM keeps in flight: five stages hold 160 KB of codes.
  static constexpr int kStages = 5;
  static constexpr uint32_t kRingBytes = kStages * kStageBytes;
  // an accumulator per code span, each 2 * kQRows columns: the hi plane's
  // rows in the first kQRows, the lo plane's in the next (one MMA covers both
  // planes, which lie one after the other in shared memory)
  static constexpr uint32_t kAccCols = 4 * kQRows;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;     // double-buffered: 256
  static constexpr uint32_t kStageRowWords = 36;
  static constexpr uint32_t kEpiBytes = 4 * 32 * kStageRowWords * 4;  // 18 KB
  static constexpr int kBars = 2 * kStages + 5;
  static constexpr size_t kSmemFixed = 1024 + kRingBytes + 256 + kEpiBytes;
  static_assert(kStageBytes % 1024 == 0 && kPlaneBytes % 1024 == 0,
                "swizzled tiles start on 1024-byte boundaries");
  static_assert(kBars * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");
  static_assert(kQRows % 32 == 0 && kQRows <= 256, "MMA N");
  static_assert(kSmemFixed + 4 * 1025 <= 232448, "shared memory of a CTA");
};

// kind::f8f6f4 instruction descriptor: fp32 accumulator (bits 4-5 = 1), A and
// B e4m3 (format code 0 at bits 7-9 and 10-12), both K-major (bits 15, 16
// clear), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t instr_desc_f8(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}


// D[tmem] (+)= A[smem] * B[smem], e4m3 inputs, fp32 accumulation.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct ParamsF8 {
  const int32_t *offsets;  // [G+1]: rows of group g are offsets[g] .. offsets[g+1]-1
  int G, rows_cap, K, N;
  void *out;               // SWIGLU: h bf16 [rows_cap, N]; PLAIN: y fp32 [rows_cap, N]
  const float *scale1;     // column scales [G, N] of B1 (and of B3: scale3)
  const float *scale3;
  const float *row_scale;  // [rows_cap]: the planes' power-of-two row scales
  const float *row_w;      // PLAIN: output row r times row_w[w_row_src[r]], or nullptr
  const int32_t *w_row_src;
  uint32_t *err;
  uint64_t wait_limit_ns;
  int prefetch;  // k-blocks of codes prefetched into L2 ahead of their loads (0: none)
  int kstagger;  // rotate each CTA's k-block order (MOE_F8_KSTAGGER=1)
};

template <bool SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_f8(const __grid_constant__ CUtensorMap tmP,   // planes [2*rows_cap, K]
                      const __grid_constant__ CUtensorMap tmW1,  // codes [G, N, K]
                      const __grid_constant__ CUtensorMap tmW3, const ParamsF8 p) {
  grid_dependency();  // the previous grid is complete; the next may launch
  using S = ShapeF8<SWIGLU>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + S::kRingBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + S::kBars);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  float *s_epi = reinterpret_cast<float *>(ring + S::kRingBytes + 256);
  // the tile starts live in shared memory; the row offsets are read from
  // global memory (L1-cached): five stages leave no room for both tables
  int32_t *s_tstart = reinterpret_cast<int32_t *>(ring + S::kRingBytes + 256 + S::kEpiBytes);
  const int32_t *s_off = p.offsets;

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
    prefetch_tmap(&tmP);
    prefetch_tmap(&tmW1);
    if (SWIGLU) prefetch_tmap(&tmW3);
  }
  // Tile starts, from the row offsets checked against the buffer size.
  bool bad = false;
  for (int g = threadIdx.x; g <= p.G; g += kThreads) {
    const int v = p.offsets[g];
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  const int col_tiles = (p.N + S::kTileCols - 1) / S::kTileCols;
  for (int g = threadIdx.x; g < p.G; g += kThreads) {
    const int rows = s_off[g + 1] - s_off[g];
    if (rows < 0) bad = true;
    s_tstart[g] = rows > 0 ? ((rows + kQRows - 1) / kQRows) * col_tiles : 0;
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
  const int num_kb = (p.K + kQK - 1) / kQK;
  // p.kstagger: each CTA walks the k-blocks of its tiles from its own
  // starting block (the MMAs accumulate the same products in a rotated
  // order), so that the CTAs streaming at the same time read codes at
  // different offsets of their rows instead of all at the same one
  const int kstart = p.kstagger ? (int)((blockIdx.x * 37u) % (unsigned)num_kb) : 0;

  // tile -> (group g, column tile c, row tile r); rows fastest, so CTAs running
  // at the same time share a weight tile
  auto tile_coords = [&](int tile, int &g, int &c, int &row0, int &nr) {
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= tile)
        lo = mid;
      else
        hi = mid - 1;
    }
    g = lo;
    const int rows = s_off[g + 1] - s_off[g];
    const int rt = (rows + kQRows - 1) / kQRows;
    const int local = tile - s_tstart[g];
    c = local / rt;
    const int r = local - c * rt;
    row0 = s_off[g] + r * kQRows;
    nr = min(kQRows, rows - r * kQRows);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued_parity = 0, issued_mask = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int g, c, row0, nr;
        tile_coords(tile, g, c, row0, nr);
        const int nq = (nr + kRowBoxQ - 1) / kRowBoxQ;  // plane boxes per plane
        const uint32_t bytes = 2 * S::kCodeBytes + kPlanes * nq * kRowBoxQ * kQK;
        const int col_a = c * S::kTileCols, col_b = SWIGLU ? col_a : col_a + 128;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait(empty0 + 8 * s, ph ^ 1, ctl)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          const uint32_t fb = full0 + 8 * s;
          if (p.prefetch > 0) {  // the k-block p.prefetch ahead (the first ones too)
            for (int q = kb == 0 ? 0 : p.prefetch; q <= p.prefetch; ++q) {
              if (kb + q >= num_kb) break;
              const int kp = (kb + q + kstart) % num_kb;
              tma_prefetch_3d(&tmW1, kp * kQK, col_a, g);
              tma_prefetch_3d(SWIGLU ? &tmW3 : &tmW1, kp * kQK, col_b, g);
            }
          }
          mbar_expect_tx(fb, bytes);
          // the k-blocks of a tile in a rotated order (kq), see p.kstagger
          const int kq = kb + kstart < num_kb ? kb + kstart : kb + kstart - num_kb;
          // codes [G, N, K]: coordinates (k, n, group)
          tma_load_3d(st, &tmW1, fb, kq * kQK, col_a, g);
          tma_load_3d(st + S::kCodeBytes, SWIGLU ? &tmW3 : &tmW1, fb, kq * kQK, col_b, g);
          // planes [2*rows_cap, K]: plane q's row r at q*rows_cap + r
          for (int q = 0; q < kPlanes; ++q)
            for (int b = 0; b < nq; ++b)
              tma_load_2d(st + 2 * S::kCodeBytes + q * S::kPlaneBytes + b * kRowBoxQ * kQK, &tmP,
                          fb, kq * kQK, q * p.rows_cap + row0 + b * kRowBoxQ);
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
      // Every operand K-major, 128-byte rows, 8-row groups 1024 B apart; a K
      // step of 32 e4m3 values is 32 bytes.  The descriptor of stage 0's
      // first code span plus offsets (16-byte units, all below 256 KB) gives
      // every operand, so the issuing thread spends about one instruction per
      // address.
      const uint64_t st_d0 = smem_desc(smem_addr(ring), 16, 1024);
      constexpr uint32_t kStageStep = S::kStageBytes >> 4, kK = 32 >> 4;
      constexpr uint32_t kSpan1 = S::kCodeBytes >> 4, kPlanesAt = (2 * S::kCodeBytes) >> 4;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int g, c, row0, nr;
        tile_coords(tile, g, c, row0, nr);
        // N: the hi plane's kQRows rows, then the lo plane's rows (nr rounded
        // up to 16); hi-plane rows beyond nr only touch accumulator columns
        // the epilogue never reads
        const uint32_t idesc = instr_desc_f8(S::kCols, kQRows + ((nr + 15) & ~15));
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
          const uint64_t sd = st_d0 + s * kStageStep;
          const uint32_t acc0 = kb != 0;
#pragma unroll
          for (int kk = 0; kk < kQK / 32; ++kk) {
            const uint32_t acc = kk ? 1u : acc0;
            umma_f8(d_tmem, sd + kk * kK, sd + kPlanesAt + kk * kK, idesc, acc);
            umma_f8(d_tmem + 2 * kQRows, sd + kSpan1 + kk * kK, sd + kPlanesAt + kk * kK, idesc,
                    acc);
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
    // TMEM lane = output column (this warp: columns 32*quarter .. of each
    // 128-column operand), TMEM column = row of the tile.
    const int quarter = warp & 3;
    int buf = 0;
    uint32_t acc_ph = 0;
    float *stg = s_epi + (warp - 2) * 32 * S::kStageRowWords;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, c, row0, nr;
      tile_coords(tile, g, c, row0, nr);
      int ready = 0;
      if (lane == 0) ready = wait(accf0 + 8 * buf, acc_ph, ctl) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + buf * S::kAccCols + ((uint32_t)(quarter * 32) << 16);
      // PLAIN: two 128-column halves, each its own accumulator; SWIGLU: one
      // pass over gate (accumulator 0) and up (accumulator 1)
      for (int h = 0; h < (SWIGLU ? 1 : 2); ++h) {
        const int col0 = c * S::kTileCols + h * 128 + quarter * 32;  // this warp's columns
        const int col = col0 + lane;                                 // this lane's column
        float sc1 = 0.f, sc3 = 0.f;
        if (col < p.N) {
          sc1 = p.scale1[(size_t)g * p.N + col];
          if (SWIGLU) sc3 = p.scale3[(size_t)g * p.N + col];
        }
#pragma unroll 1
        for (int j0 = 0; j0 < nr; j0 += 32) {
          // the row scales of rows j0 .. j0+31 of the tile, one per lane
          const float rs = (j0 + lane < nr) ? p.row_scale[row0 + j0 + lane] : 0.f;
          // v[j] = out[row j0 + j][col]: the hi plane's and the lo plane's sums
          float v[32];
          tmem_ld32_sum2(tb + h * 2 * kQRows + j0, kQRows, v);
          if (SWIGLU) {
            float u[32];
            tmem_ld32_sum2(tb + 2 * kQRows + j0, kQRows, u);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float r = __shfl_sync(0xffffffffu, rs, j);
              const float gt = v[j] * (sc1 * r), up = u[j] * (sc3 * r);
              v[j] = silu_times(gt, up);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= sc1 * __shfl_sync(0xffffffffu, rs, j);
          }
          // transpose through shared memory: stage[row j][column lane]
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[j * S::kStageRowWords + lane] = v[j];
          __syncwarp();
          if (SWIGLU) {  // bf16 rows: 8 lanes x 8 bytes per 64-byte row segment, 4 rows per step
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = i * 4 + (lane >> 3), q = lane & 7;
              const int grow = row0 + j0 + j, gcol = col0 + q * 4;
              const float4 f =
                  *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
              if (j0 + j < nr && gcol < p.N) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(f.x, f.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(f.z, f.w);
                uint2 w;
                w.x = *reinterpret_cast<uint32_t *>(&lo);
                w.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                           (size_t)grow * p.N + gcol) = w;
              }
            }
          } else {  // fp32 rows: 8 lanes x 16 bytes, 4 rows per step
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = i * 4 + (lane >> 3), q = lane & 7;
              const int grow = row0 + j0 + j, gcol = col0 + q * 4;
              float4 o = *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
              if (j0 + j < nr && gcol < p.N) {
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

// ---------------------------------------------------------------------------
// Activation planes
// ---------------------------------------------------------------------------
// Row r (r < the row count) of `src` -- or, with row_src, token row
// row_src[r] / k_max of it (the dispatch gather) -- split into two e4m3
// planes with a power-of-two scale (see the top of this file): planes[q *
// rows_cap + r][:] = q-th plane, row_scale[r] = s.  One CTA of 128 threads
// per row: the row's largest magnitude, then the planes, 8 elements (one
// 16-byte load) per thread step.
constexpr int kSplitThreads = 128;

__device__ __forceinline__ float e4m3_value(uint8_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
  return __half2float(__half(h));
}

__global__ void __launch_bounds__(kSplitThreads)
    k_split_planes(const __nv_bfloat16 *__restrict__ src, const int32_t *__restrict__ n_rows,
                   int fixed_rows, const int32_t *__restrict__ row_src, int k_max, int src_rows,
                   int rows_cap, int K, uint8_t *__restrict__ planes,
                   float *__restrict__ row_scale, uint32_t *err) {
  grid_dependency();  // the previous grid is complete; the next may launch
  __shared__ float s_red[kSplitThreads / 32];
  int R = n_rows ? *n_rows : fixed_rows;
  if (R < 0 || R > rows_cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrIndex);
    R = R < 0 ? 0 : rows_cap;
  }
  const int vecs = K / 8;  // K % 16 == 0
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    int t = r;
    if (row_src) {
      const int a = row_src[r];
      t = a / k_max;
      if (a < 0 || t >= src_rows) {
        if (threadIdx.x == 0) raise_error(err, kErrIndex);
        continue;
      }
    }
    const uint4 *row = reinterpret_cast<const uint4 *>(src + (size_t)t * K);
    float m = 0.0f;
    for (int v = threadIdx.x; v < vecs; v += kSplitThreads) {
      const uint4 u = row[v];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)),
                           fabsf(__uint_as_float(w[i] & 0xffff0000u))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (threadIdx.x % 32 == 0) s_red[threadIdx.x / 32] = m;
    __syncthreads();
    m = s_red[0];
#pragma unroll
    for (int i = 1; i < kSplitThreads / 32; ++i) m = fmaxf(m, s_red[i]);
    __syncthreads();  // s_red is reused by the next row
    // m = M * 2^E with M in [1, 2): the smallest k with m / 2^k <= 448 = 1.75 * 2^8
    // is E - 8, or E - 7 when M > 1.75.  Zero and non-finite rows take k = 0;
    // k is clamped so that 2^k and 2^-k are normal fp32 values.
    int k = 0;
    if (m > 0.0f && m <= 3.4028234e38f) {
      int e2;
      const float M2 = 2.0f * frexpf(m, &e2);  // frexp: m = (M2 / 2) * 2^e2
      k = (e2 - 1) - 8 + (M2 > 1.75f ? 1 : 0);
      k = max(-120, min(120, k));
    }
    const float inv = ldexpf(1.0f, -k);
    uint8_t *p0 = planes + (size_t)r * K;
    uint8_t *p1 = planes + ((size_t)rows_cap + r) * K;
    for (int v = threadIdx.x; v < vecs; v += kSplitThreads) {
      const uint4 u = row[v];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t q0w[2] = {0, 0}, q1w[2] = {0, 0};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(w[i] << 16) * inv;
        const float b = __uint_as_float(w[i] & 0xffff0000u) * inv;
        const __nv_fp8x2_storage_t c0 =
            __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
        const float ra = a - e4m3_value((uint8_t)(c0 & 0xff));
        const float rb = b - e4m3_value((uint8_t)(c0 >> 8));
        const __nv_fp8x2_storage_t c1 =
            __nv_cvt_float2_to_fp8x2(make_float2(ra, rb), __NV_SATFINITE, __NV_E4M3);
        q0w[i / 2] |= (uint32_t)c0 << (16 * (i % 2));
        q1w[i / 2] |= (uint32_t)c1 << (16 * (i % 2));
      }
      *reinterpret_cast<uint2 *>(p0 + 8 * (size_t)v) = make_uint2(q0w[0], q0w[1]);
      *reinterpret_cast<uint2 *>(p1 + 8 * (size_t)v) = make_uint2(q1w[0], q1w[1]);
    }
    if (threadIdx.x == 0) row_scale[r] = ldexpf(1.0f, k);
  }
}

// 2-D map over the planes [2 * rows_cap, K] (one byte each), box 128 (K) x 16
// rows, 128-byte swizzle.
bool make_map_planes(CUtensorMap *m, const void *planes, int rows_cap, int K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)kPlanes * (rows_cap > 0 ? rows_cap : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {(cuuint32_t)kQK, (cuuint32_t)kRowBoxQ};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(planes), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over e4m3 codes Q [G, N, K] (K contiguous), box 128 (K) x 128 (N) x 1,
// 128-byte swizzle: the K-major A tile of the MMA.
bool make_map_codes_k128(CUtensorMap *m, const void *Q, int G, int N, int K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)N, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)N * K};
  cuuint32_t box[3] = {(cuuint32_t)kQK, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(Q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SWIGLU>
cudaError_t launch_f8(int rows_cap, int K, int N, int G, const int32_t *offsets,
                      const uint8_t *planes, const float *row_scale, const void *B1,
                      const void *B3, const float *s1, const float *s3, void *out,
                      const float *row_w, const int32_t *w_row_src, uint32_t *err,
                      cudaStream_t s) {
  using S = ShapeF8<SWIGLU>;
  CUtensorMap mp, mw1, mw3;
  if (!make_map_planes(&mp, planes, rows_cap, K) || !make_map_codes_k128(&mw1, B1, G, N, K) ||
      !make_map_codes_k128(&mw3, SWIGLU ? B3 : B1, G, N, K))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_f8<SWIGLU>,
                                    S::kSmemFixed + sizeof(int32_t) * (kMaxGroups + 1)))
    return e;
  const char *pf = getenv("MOE_F8_PREFETCH");
  const char *ks = getenv("MOE_F8_KSTAGGER");
  ParamsF8 p{offsets, G, rows_cap, K, N, out, s1, SWIGLU ? s3 : nullptr, row_scale,
             row_w, w_row_src, err, pipeline_wait_limit_ns(), pf ? atoi(pf) : 0,
             (ks && ks[0] == '1') ? 1 : 0};
  const long long max_tiles = (long long)((rows_cap + kQRows - 1) / kQRows + G) *
                              ((N + S::kTileCols - 1) / S::kTileCols);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  launch_k(k_grouped_gemm_f8<SWIGLU>, grid, kThreads, smem, s, mp, mw1, mw3, p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

size_t fp8_planes_bytes(int rows_cap, int K) { return (size_t)2 * rows_cap * K; }

cudaError_t launch_split_planes(const void *src, const int32_t *n_rows, int fixed_rows,
                                const int32_t *row_src, int k_max, int src_rows, int rows_cap,
                                int K, uint8_t *planes, float *row_scale, uint32_t *err,
                                cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  if (K % 16) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = rows_cap < 8 * sms ? rows_cap : 8 * sms;
  launch_k(tc::k_split_planes, grid, tc::kSplitThreads, 0, s, 
      static_cast<const __nv_bfloat16 *>(src), n_rows, fixed_rows, row_src, k_max, src_rows,
      rows_cap, K, planes, row_scale, err);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm_f8(bool swiglu, int rows_cap, int K, int N, int G,
                                   const int32_t *offsets, const uint8_t *planes,
                                   const float *row_scale, const void *B1, const void *B3,
                                   const float *s1, const float *s3, void *out, uint32_t *err,
                                   cudaStream_t s, const float *row_w,
                                   const int32_t *w_row_src) {
  if (rows_cap <= 0) return cudaSuccess;
  if (!offsets || G <= 0 || G > tc::kMaxGroups || N % 16 || K % 16) return cudaErrorInvalidValue;
  if (row_w && swiglu) return cudaErrorInvalidValue;  // gate weights: the down projection only
  return swiglu ? tc::launch_f8<true>(rows_cap, K, N, G, offsets, planes, row_scale, B1, B3, s1,
                                      s3, out, nullptr, nullptr, err, s)
                : tc::launch_f8<false>(rows_cap, K, N, G, offsets, planes, row_scale, B1, B1, s1,
                                       nullptr, out, row_w, w_row_src, err, s);
}

}  // namespace moe
