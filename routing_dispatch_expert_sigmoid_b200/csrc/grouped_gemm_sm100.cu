// K5/K6 -- grouped GEMM for the expert FFN on the 5th-generation tensor cores.
//
// "LLM MoE Expert Parallel 生产实战", section "为什么 MoE 推理会慢在'最热专家'",
// step 3 (each expert computes on the rows routed to it) and "Paralelismo
// experto para el servicio MoE", "Información técnica" (the expert GEMMs see
// data-dependent row counts).  Rows of group g are offsets[g]..offsets[g+1]-1
// of A; the counts stay on the device and each CTA derives its tile list from
// them, so no host synchronisation is needed between routing and the FFN.
//
//   SWIGLU: out[r, n] = silu(A[r].B1[g][:, n]) * (A[r].B3[g][:, n])   (K5, x_perm -> h, bf16)
//   PLAIN:  out[r, n] = A[r].B1[g][:, n]                              (K6, h -> y_perm, fp32)
//
// A [rows_cap, K] bf16 row-major (K-major); B [G, K, N] bf16 row-major, i.e.
// N-major for the MMA ("MN-major" operand); fp32 accumulation in tensor
// memory.  h is stored bf16 (it is the next GEMM's operand); y_perm is kept
// fp32 so that the layer output sees a single bf16 rounding after the
// weighted sum.
//
// Design (one CTA per SM, persistent, warp-specialised, 192 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tiles 64 x 64 (one 128-byte
//               swizzle span of N each) into a STAGES-deep shared-memory ring;
//   warp 1      allocates tensor memory and issues tcgen05.mma (M=128, N=256,
//               K=16) from one thread; tcgen05.commit releases ring slots and
//               hands finished accumulators to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld of the 128 x 256 fp32 accumulator (warp w
//               reads TMEM lanes 32*(w%4)...), SiLU-gate multiply for K5,
//               bf16 conversion; each 32 x 32 chunk is staged in shared
//               memory and written back row-wise (whole 64/128-byte row
//               segments per warp store), masked to the group's rows.
// The accumulator is double-buffered in tensor memory (2 x 256 columns) so
// the epilogue of one tile overlaps the main loop of the next.
// For SWIGLU the W1 and W3 tiles of the same 128 output columns sit next to
// each other in shared memory, so one N=256 MMA produces gate (columns
// 0..127) and up (columns 128..255) of the same rows.
//
// Tiles are enumerated (group, n-tile, m-tile) with m fastest and dealt
// round-robin to the CTAs: CTAs running at the same time share the weight
// tile of one expert and its rows of A, so weights are read from HBM about
// once and A stays in L2.  All tiles of a launch have the same K, so the
// deal is balanced to within one tile.
//
// FP8 weights (single engine, FP8W): B holds e4m3 codes and one fp32 scale
// per output column of each group.  TMA brings the codes (64 x 64 bytes per
// span) into a staging area of the stage; warps 6-9 widen them to bf16 --
// exact, every e4m3 value is a bf16 value; integer bit moves and one packed
// multiply, see e4m3x2_to_bf16x2 -- into the swizzled B layout the
// MMA reads, fence the generic-proxy stores for the tensor cores and arrive
// on the stage's "converted" barrier, which the MMA thread waits on instead
// of "full".  The epilogue multiplies each column by its scale before SiLU.
//
// Every wait on an mbarrier is bounded (by %globaltimer): on expiry the CTA
// records kErrWait in the device error word, tells its other roles to stop,
// waits (again bounded) for its own copies and MMAs in flight, frees its
// tensor memory and returns.  No TMA multicast is used.
#include <cuda.h>
#include <stdlib.h>

#include <atomic>

#include "tcgen05_common.cuh"

namespace moe {
namespace tc {

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
struct Params {
  const int32_t *offsets;  // [G+1] or nullptr
  int G;
  int fixed_rows;  // rows of the single group when offsets == nullptr
  int rows_cap;    // rows of A and out
  int K, N;
  void *out;  // [rows_cap, N]: bf16 for SWIGLU (h), fp32 for PLAIN (y, logits)
  const float *bias;  // PLAIN only: [N] added to every row (router logit bias), or nullptr
  // Gathered A rows: when row_src is set, row r of A is row row_src[r] / k_max
  // of the tensor map (the token rows x), fetched with TMA gather4; this fuses
  // the dispatch copy into the GEMM.
  const int32_t *row_src;
  int k_max;
  uint32_t *err;
  // Split K (single engine, PLAIN, offsets == nullptr): group g multiplies
  // the same fixed_rows rows of A by K columns g*k_split .. g*k_split+k_split-1
  // (B is one [K, N] matrix) and writes its partial product to output rows
  // g*fixed_rows .. ; columns past K read the TMA zero fill.
  int k_split = 0;
  // Word set to zero by the first thread of block 0 (a ticket the next
  // launch on the stream counts with), or nullptr.
  int32_t *clear = nullptr;
  // FP8 weights: per-column scales of B1 and B3, [G, N] fp32
  const float *scale1 = nullptr, *scale3 = nullptr;
  // PLAIN: output row r is multiplied by row_w[w_row_src[r]] (the gate weight
  // of the slot the row serves), or nothing when row_w is nullptr
  const float *row_w = nullptr;
  const int32_t *w_row_src = nullptr;
  // Limit of one pipeline wait (the single-CTA and swap-AB engines)
  uint64_t wait_limit_ns = kWaitLimitNs;
  // PLAIN, single-CTA and pair engines: when set, out receives the compact
  // y16 form of the rows, with nblk = ceil(N / 32) block exponents per row
  int8_t *yexp = nullptr;
  int nblk = 0;
  // L2 eviction hints on the TMA loads (bf16 single-CTA and pair engines)
  int l2_hints = 0;
  // pair engine swap-AB tiles: 0 none; 1 groups under 256 rows (a light
  // list dealt evenly among the others); 2 those and every group's last,
  // partial 256-row chunk
  int pair_swap = 0;
  int swap_rows = 0;  // the light list: groups of 1 .. swap_rows rows (< 256)
};

// Gate weights to apply in the down projection's epilogue (both nullptr: none).
struct RowWeights {
  const float *w = nullptr;
  const int32_t *row_src = nullptr;
};

template <bool SWIGLU, int SPANS, bool FP8W = false>
struct Shape {
  static constexpr int kSpans = SPANS;                // 64-column spans per B operand
  static constexpr int BN = 64 * SPANS;               // output columns per tile
  static constexpr int kBOps = SWIGLU ? 2 : 1;
  static constexpr uint32_t kABytes = BM * BK * 2;    // 16 KB
  static constexpr uint32_t kSpanBytes = BK * 128;    // 8 KB: 64 K-rows x 128 B
  static constexpr uint32_t kBBytes = kBOps * kSpans * kSpanBytes;
  // compute ring: A and (widened) B of one k-block per stage
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  // bf16: as many stages as fit in ~192 KB, at most 8.  FP8W: two compute
  // stages; the rest of the 192 KB is a deeper ring of e4m3 codes (64 K-rows
  // x 64 bytes per span), the HBM stream, at most 8 deep.
  static constexpr int kStages =
      FP8W ? 2 : ((196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes));
  // FP8W codes are K-contiguous ([G, N, K]): per operand one box of BN
  // columns x 64 K-codes, 64-byte rows with the 64-byte swizzle
  static constexpr uint32_t kQOpBytes = FP8W ? BN * BK : 0;
  static constexpr uint32_t kQBytes = kBOps * kQOpBytes;
  static constexpr int kQStages =
      !FP8W ? 0
            : ((196608 - kStages * kStageBytes) / kQBytes > 8
                   ? 8
                   : (196608 - kStages * kStageBytes) / kQBytes);
  static constexpr uint32_t kRingBytes = kStages * kStageBytes + kQStages * kQBytes;
  static constexpr uint32_t kTxBytes = FP8W ? kABytes : kStageBytes;  // TMA bytes per stage
  // FP8W: + 4 converter warps (6-9) and an A-loading warp (10)
  static constexpr int kCtaThreads = FP8W ? 352 : 192;
  static constexpr int kConvThreads = 128;
  static constexpr int kMmaN = kBOps * BN;            // 256
  static constexpr uint32_t kAccCols = kMmaN;         // fp32 columns per accumulator
  static constexpr uint32_t kTmemCols = 2 * kAccCols; // 512
  // bf16 weights are an MN-major B tile; widened fp8 weights a K-major one
  static constexpr uint32_t kIdesc = FP8W ? instr_desc_kk(BM, kMmaN) : instr_desc(BM, kMmaN);
  // epilogue staging: per epilogue warp a 32-row x 32-column fp32 chunk, rows
  // padded to 36 words so both the row-wise writes and the column-wise reads
  // are free of bank conflicts
  static constexpr uint32_t kStageRowWords = 36;
  static constexpr uint32_t kEpiBytes = 4 * 32 * kStageRowWords * 4;  // 18 KB
  static constexpr size_t kSmemFixed =
      1024 /*align slack*/ + kRingBytes + 256 + kEpiBytes;
  // barriers: full, empty per stage, 2 + 2 accumulator, drain; FP8W also
  // converted per stage and code-full, code-empty per code stage
  static constexpr int kBars = FP8W ? 3 * kStages + 2 * kQStages + 5 : 2 * kStages + 5;
  static_assert(kBars * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");
  static_assert(!FP8W || kQStages >= 2, "code ring");
  static_assert(!FP8W || (kMmaN % kConvThreads == 0 && BN <= 256), "whole B rows per converter");
  static_assert(kMmaN % 16 == 0 && kMmaN <= 256, "UMMA N");
  static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                "TMEM allocation: a power of two in [32, 512] columns");
};

__device__ __forceinline__ void tile_of(int tile, const int32_t *s_tstart, const int32_t *s_off,
                                        int G, int &g, int &m, int &n) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with s_tstart[g] <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  g = lo;
  const int rows = s_off[g + 1] - s_off[g];
  const int mt = (rows + BM - 1) / BM;
  const int local = tile - s_tstart[g];
  n = local / mt;
  m = local - n * mt;
}

// Two e4m3 codes (bytes 0 and 1 of `two`) to two bf16 values (the low half
// from byte 0), on the integer and FMA pipes (the conversion instructions'
// pipe is the narrow one).  Each byte goes to the top of a 16-bit half, so
// its sign sits on the bf16 sign bit and its 4 exponent and 3 fraction bits,
// shifted right by 4, on the low end of the bf16 exponent and the top of the
// fraction.  Read as bf16 that is value * 2^-120 (exponent bias 127 instead
// of 7) -- for e4m3 subnormals a bf16 subnormal of the same significand -- so
// one exact multiply by 2^120 gives the value.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  const uint32_t y = __byte_perm(two, 0u, 0x1404);  // bytes: 0, b0, 0, b1
  const uint32_t bits = ((y >> 4) & 0x07F007F0u) | (y & 0x80008000u);
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&bits);
  const __nv_bfloat162 k = __floats2bfloat162_rn(0x1p120f, 0x1p120f);  // exact in bf16
  v = __hmul2(v, k);
  return *reinterpret_cast<const uint32_t *>(&v);
}
// Four e4m3 codes (one 32-bit word, byte i = K element i) to four bf16 values
// (two bf16 pairs, low halves first), with fewer integer-pipe operations: the
// magnitudes' exponent and fraction bits reach their bf16 positions by a byte
// permute and a multiply by 16 (the FMA pipe), the exact multiply by 2^120
// rebiases them, and the signs are or-ed back in by a second byte permute.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t &p01, uint32_t &p23) {
  const uint32_t mag = w & 0x7F7F7F7Fu;
  const uint32_t m01 = __byte_perm(mag, 0u, 0x4140) * 16u;  // |b0| -> bits 4-10, |b1| -> 20-26
  const uint32_t m23 = __byte_perm(mag, 0u, 0x4342) * 16u;
  const __nv_bfloat162 k = __floats2bfloat162_rn(0x1p120f, 0x1p120f);
  __nv_bfloat162 v01 = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&m01), k);
  __nv_bfloat162 v23 = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&m23), k);
  p01 = *reinterpret_cast<const uint32_t *>(&v01) | (__byte_perm(w, 0u, 0x1404) & 0x80008000u);
  p23 = *reinterpret_cast<const uint32_t *>(&v23) | (__byte_perm(w, 0u, 0x3424) & 0x80008000u);
}
__device__ __forceinline__ void e4m3x16_to_bf16(uint4 c, uint4 &lo, uint4 &hi) {
  lo = make_uint4(e4m3x2_to_bf16x2(c.x & 0xffffu), e4m3x2_to_bf16x2(c.x >> 16),
                  e4m3x2_to_bf16x2(c.y & 0xffffu), e4m3x2_to_bf16x2(c.y >> 16));
  hi = make_uint4(e4m3x2_to_bf16x2(c.z & 0xffffu), e4m3x2_to_bf16x2(c.z >> 16),
                  e4m3x2_to_bf16x2(c.w & 0xffffu), e4m3x2_to_bf16x2(c.w >> 16));
}
// Shared-memory stores of this thread become visible to the tensor cores'
// (async proxy) reads that are ordered after it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// The 64 codes of one column of a code box (64-byte rows, 64-byte TMA
// swizzle: 16-byte chunk j of row r sits in slot j ^ ((r >> 1) & 3)), widened
// to 32 bf16 pairs, K ascending (pair i = K elements 2i, 2i+1).  Eight
// threads on consecutive rows read 8 distinct bank groups.
// NC of the 4 16-code chunks of row r, from chunk j0 (K = 16*j0 ..).
template <int NC>
__device__ __forceinline__ void widen_chunks(const uint8_t *__restrict__ box, int r, int j0,
                                             uint32_t (&out)[8 * NC]) {
  const uint8_t *row = box + r * 64;
  uint4 c[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j)
    c[j] = *reinterpret_cast<const uint4 *>(row + (((j0 + j) ^ ((r >> 1) & 3)) << 4));
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    const uint32_t w[4] = {c[j].x, c[j].y, c[j].z, c[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) e4m3x4_to_bf16x4(w[i], out[8 * j + 2 * i], out[8 * j + 2 * i + 1]);
  }
}
__device__ __forceinline__ void widen_column(const uint8_t *__restrict__ box, int r,
                                             uint32_t (&out)[32]) {
  widen_chunks<4>(box, r, 0, out);
}

// Single engine: widen the stage's codes (per operand a box of BN columns x
// 64 K) into the K-major B tile the MMA reads: row r (operand r / BN, column
// r % BN) holds 64 bf16 = 128 bytes, 16-byte chunk c in slot c ^ (r & 7)
// (the 128-byte swizzle).  Thread ct widens rows ct, ct + 128, ...
template <int kRowsPerThread>
__device__ __forceinline__ void widen_rows(const uint8_t *__restrict__ q, uint8_t *__restrict__ b,
                                           int ct, int BN) {
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) {
    const int r = ct + 128 * i, op = r / BN, rn = r - op * BN;
    uint32_t v[32];
    widen_column(q + op * BN * 64, rn, v);
    uint8_t *row = b + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) =
          make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}

// v[i] *= scale[col + i] for the columns below N (N a multiple of 16, col a
// multiple of 32, scale 16-byte aligned: a float4 is whole or absent).
__device__ __forceinline__ void scale_cols(float (&v)[32], const float *scale, int col, int N) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (col + 4 * q < N) {
      const float4 sc = __ldg(reinterpret_cast<const float4 *>(scale + col + 4 * q));
      v[4 * q] *= sc.x;
      v[4 * q + 1] *= sc.y;
      v[4 * q + 2] *= sc.z;
      v[4 * q + 3] *= sc.w;
    }
  }
}

template <bool SWIGLU, int SPANS, bool FP8W = false>
__global__ void __launch_bounds__(Shape<SWIGLU, SPANS, FP8W>::kCtaThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmB3, const Params p) {
  grid_dependency();  // the previous grid is complete; the next may launch
  using S = Shape<SWIGLU, SPANS, FP8W>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;                                  // compute stages
  uint8_t *qring = ring + S::kStages * S::kStageBytes;   // FP8W: code stages
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + S::kRingBytes);
  // bars: full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain[1];
  // FP8W: converted[kStages], code_full[kQStages], code_empty[kQStages]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + S::kBars);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  float *s_epi = reinterpret_cast<float *>(ring + S::kRingBytes + 256);
  int32_t *s_off = reinterpret_cast<int32_t *>(ring + S::kRingBytes + 256 + S::kEpiBytes);
  int32_t *s_tstart = s_off + (p.G + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S::kStages);
  const uint32_t accf0 = smem_addr(bars + 2 * S::kStages);
  const uint32_t acce0 = smem_addr(bars + 2 * S::kStages + 2);
  const uint32_t drain = smem_addr(bars + 2 * S::kStages + 4);
  const uint32_t conv0 = smem_addr(bars + 2 * S::kStages + 5);
  const uint32_t qfull0 = smem_addr(bars + 3 * S::kStages + 5);
  const uint32_t qempty0 = smem_addr(bars + 3 * S::kStages + 5 + S::kQStages);
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
    if (FP8W) {
      for (int s = 0; s < S::kStages; ++s) mbar_init(conv0 + 8 * s, S::kConvThreads / 32);
      for (int s = 0; s < S::kQStages; ++s) {
        mbar_init(qfull0 + 8 * s, 1);
        mbar_init(qempty0 + 8 * s, S::kConvThreads / 32);
      }
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB1);
    if (SWIGLU) prefetch_tmap(&tmB3);
  }
  // Group table: row offsets, then tile starts (exclusive scan of the
  // per-group tile counts), checked against the buffer size.
  bool bad = false;
  if (p.clear && blockIdx.x == 0 && threadIdx.x == 0) *p.clear = 0;
  for (int g = threadIdx.x; g <= p.G; g += S::kCtaThreads) {
    const int v = p.offsets ? p.offsets[g]
                            : (p.k_split ? g * p.fixed_rows : (g == 0 ? 0 : p.fixed_rows));
    s_off[g] = v;
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  const int n_tiles = (p.N + S::BN - 1) / S::BN;
  for (int g = threadIdx.x; g < p.G; g += S::kCtaThreads) {
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
  const int num_kb = p.k_split ? p.k_split / BK : (p.K + BK - 1) / BK;

  if (warp == 0 || (FP8W && warp == 10)) {
    // ------------------------------------------------------------ producers
    // Lane 0 waits and issues the tiled loads; when the A rows are gathered,
    // every lane issues one gather4 (4 of the tile's 128 rows).  With fp8
    // weights warp 0 streams the e4m3 codes through the code ring and warp
    // 10 loads the A tiles into the compute ring, so the code stream runs
    // ahead of the compute stages.
    const bool codes = FP8W && warp == 0;
    const bool load_a = !FP8W || warp == 10;
    const bool gather = p.row_src != nullptr;
    const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
    const int nst = codes ? S::kQStages : S::kStages;
    const uint32_t fullb = codes ? qfull0 : full0, emptyb = codes ? qempty0 : empty0;
    int s = 0;
    uint32_t ph = 0, issued_parity = 0, issued_mask = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      int g, m, n;
      tile_of(tile, s_tstart, s_off, p.G, g, m, n);
      // split K: every group reads the same A rows, at its own K offset
      const int row = p.k_split ? m * BM : s_off[g] + m * BM;
      const int k0 = p.k_split ? g * p.k_split : 0;
      const int gb = p.k_split ? 0 : g;  // B's group coordinate
      int tok[4] = {0, 0, 0, 0};  // rows past the group read token 0 (masked later)
      if (gather) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = row + 4 * lane + q;
          if (r < s_off[g + 1]) tok[q] = p.row_src[r] / p.k_max;
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        int okw = 1;
        if (lane == 0) okw = wait(emptyb + 8 * s, ph ^ 1, ctl) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) {
          ok = false;
          break;
        }
        const uint32_t fb = fullb + 8 * s;
        if (codes) {
          const uint32_t qt = smem_addr(qring + s * S::kQBytes);
          if (lane == 0) {  // codes [G, N, K]: coordinates (k, n, group)
            mbar_expect_tx(fb, S::kQBytes);
            tma_load_3d(qt, &tmB1, fb, k0 + kb * BK, n * S::BN, gb);
            if (SWIGLU) tma_load_3d(qt + S::kQOpBytes, &tmB3, fb, k0 + kb * BK, n * S::BN, gb);
          }
        } else {
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          if (lane == 0) mbar_expect_tx(fb, S::kTxBytes);
          if (gather)
            tma_gather4(st + lane * 4 * 128, &tmA, fb, kb * BK, tok[0], tok[1], tok[2], tok[3]);
          if (lane == 0) {
            if (!gather && load_a) {
              if (p.l2_hints)
                tma_load_2d_hint(st, &tmA, fb, k0 + kb * BK, row, pol_keep);
              else
                tma_load_2d(st, &tmA, fb, k0 + kb * BK, row);
            }
            if (!FP8W) {
#pragma unroll
              for (int j = 0; j < S::kSpans * S::kBOps; ++j) {
                const CUtensorMap *mb = (SWIGLU && j >= S::kSpans) ? &tmB3 : &tmB1;
                const int col = n * S::BN + (j % S::kSpans) * 64;
                if (p.l2_hints)
                  tma_load_3d_hint(st + S::kABytes + j * S::kSpanBytes, mb, fb, col,
                                   k0 + kb * BK, gb, pol_stream);
                else
                  tma_load_3d(st + S::kABytes + j * S::kSpanBytes, mb, fb, col, k0 + kb * BK, gb);
              }
            }
          }
        }
        issued_mask |= 1u << s;
        issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
        if (++s == nst) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {  // stopped early: let the copies already issued land first
      for (int q = 0; q < nst; ++q)
        if ((issued_mask >> q) & 1u) wait_drain(fullb + 8 * q, (issued_parity >> q) & 1u, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, buf = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true, any = false;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!wait(acce0 + 8 * buf, acc_ph ^ 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * S::kAccCols;
        for (int kb = 0; kb < num_kb; ++kb) {
          // FP8W: the A tile has landed and the converters have filled B
          if (!wait(full0 + 8 * s, ph, ctl) || (FP8W && !wait(conv0 + 8 * s, ph, ctl))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // A: K-major, 128-byte rows, 8-row groups 1024 B apart; step K by 32 B.
            const uint64_t ad = smem_desc(st + kk * 32, 16, 1024);
            // B: MN-major, 64-column spans kSpanBytes apart (LBO), 8-row K
            // groups 1024 B apart (SBO); step K by 16 rows = 2048 B.  Widened
            // fp8 weights: K-major like A.
            const uint64_t bd = FP8W ? smem_desc(st + S::kABytes + kk * 32, 16, 1024)
                                     : smem_desc(st + S::kABytes + kk * 2048, S::kSpanBytes, 1024);
            umma(d_tmem, ad, bd, S::kIdesc, (kb | kk) != 0);
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
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int buf = 0;
    uint32_t acc_ph = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, m, n;
      tile_of(tile, s_tstart, s_off, p.G, g, m, n);
      // One lane waits, the warp follows: tcgen05.ld needs a converged warp.
      int ready = 0;
      if (lane == 0) ready = wait(accf0 + 8 * buf, acc_ph, ctl) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      // This warp owns rows row0 .. row0+31 of the tile (TMEM lanes 32*quarter ..).
      const int row0 = s_off[g] + m * BM + quarter * 32;
      const int row_end = s_off[g + 1];
      const uint32_t tb = tmem_base + buf * S::kAccCols + ((uint32_t)(quarter * 32) << 16);
      float *stg = s_epi + (warp - 2) * 32 * S::kStageRowWords;
#pragma unroll 1
      for (int c = 0; c < S::BN; c += 32) {
        // lane = row: 32 consecutive columns of its row from tensor memory
        float v[32], u[32];
        if (SWIGLU)
          tmem_ld32x2(tb + c, tb + S::BN + c, v, u);
        else
          tmem_ld32(tb + c, v);
        const int col = n * S::BN + c;
        // split K: every split is the same weight group 0
        if (FP8W) scale_cols(v, p.scale1 + (size_t)(p.k_split ? 0 : g) * p.N, col, p.N);
        if (SWIGLU) {
          if (FP8W) scale_cols(u, p.scale3 + (size_t)(p.k_split ? 0 : g) * p.N, col, p.N);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu_times(v[i], u[i]);
        }
        // Stage the 32 x 32 chunk in shared memory, then write it back row by
        // row so that each warp store covers whole 64/128-byte row segments.
        if (SWIGLU) {  // h: bf16, a row is 16 words
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
            const uint4 val = *reinterpret_cast<const uint4 *>(st + r * S::kStageRowWords + 4 * q);
            if (grow < row_end && gcol < p.N)
              *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                         (size_t)grow * p.N + gcol) = val;
          }
        } else if (p.yexp) {  // y16: fp16 rows, one exponent per 32-column block
          if (p.row_w && row0 + lane < row_end) {
            const float wr = p.row_w[p.w_row_src[row0 + lane]];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= wr;
          }
          store_y16_lane_rows(v, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords, lane, row0,
                              row_end, col, p.N, p.out, p.yexp, p.nblk);
        } else {  // fp32 (+ bias), a row is 32 words
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
            if (grow < row_end && gcol < p.N) {
              if (p.bias) {  // the bias is only 4-byte aligned: scalar loads
                const float *b = p.bias + gcol;
                o.x += b[0];
                o.y += b[1];
                o.z += b[2];
                o.w += b[3];
              }
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
      buf ^= 1;
      if (buf == 0) acc_ph ^= 1;
    }
  } else if (FP8W && warp >= 6 && warp < 10) {
    // ------------------------------------------------------------ fp8 converters
    // Per k-block: wait for its codes (code stage qs) and for a free compute
    // stage s, widen them into the stage's B tile, release the code stage and
    // mark the compute stage converted.
    const int ct = threadIdx.x - 192;
    int s = 0, qs = 0;
    uint32_t ph = 0, qph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb) {
        int okw = 1;
        if (lane == 0)
          okw = (wait(qfull0 + 8 * qs, qph, ctl) && wait(empty0 + 8 * s, ph ^ 1, ctl)) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) {
          ok = false;
          break;
        }
        widen_rows<S::kMmaN / S::kConvThreads>(qring + qs * S::kQBytes,
                                                ring + s * S::kStageBytes + S::kABytes, ct,
                                                S::BN);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(qempty0 + 8 * qs);
          mbar_arrive(conv0 + 8 * s);
        }
        if (++qs == S::kQStages) {
          qs = 0;
          qph ^= 1;
        }
        if (++s == S::kStages) {
          s = 0;
          ph ^= 1;
        }
      }
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
// The same grouped GEMM on CTA pairs (tcgen05 cta_group::2)
//
// A cluster of two CTAs (two SMs of one TPC) computes a 256-row tile: CTA r
// loads rows r*128.. of the tile's A and half of the B columns (SWIGLU: CTA 0
// the W1 span pair, CTA 1 the W3 span pair; PLAIN: columns r*128..r*128+127
// of the 256), so each SM streams 32 KB per k-block instead of 48 KB and the
// same shared-memory ring covers 1.5 times the tensor-core time.  CTA 0 (the
// leader) issues one M=256, N=256, K=16 MMA per step for both SMs; each
// CTA's tensor memory receives its own 128 rows of the accumulator.
// Barriers: both CTAs' TMA loads complete on the leader's "full" barrier
// (cta_group::2 form), the leader's commits arrive on "empty" and
// "accumulator full" in both CTAs (cluster multicast of the commit, not of
// any load), and both CTAs' epilogue warps arrive on the leader's
// "accumulator empty" barrier.
// ---------------------------------------------------------------------------
constexpr int BM2 = 256;  // rows per pair tile
// Groups of at most this many rows run as swap-AB pair tiles (the light
// list); larger ones as 256-row pair tiles, padded.  Alternated call by call,
// swap tiles paid off for groups of a few dozen rows (GPT-OSS-shaped
// sub-experts) and lost for groups of about 128 (DeepSeek-V3-shaped prefill),
// whose plain-output swap epilogue is slower than a padded tile's.
constexpr int kPairSwapRows = 32;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t leader_bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t leader_bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap *map,
                                                      uint32_t leader_bar, int c0, int c1,
                                                      uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(leader_bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair_hint(uint32_t dst, const CUtensorMap *map,
                                                      uint32_t leader_bar, int c0, int c1, int c2,
                                                      uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(leader_bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` (same shared-memory offset) in both CTAs of the pair when
// every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}\n" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair_self(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// kind::f16 descriptor of a swap-AB pair tile: M = 256 weight columns (128
// per CTA, MN-major), N = the chunk's rows rounded up to 16 (K-major, N/2 of
// them in each CTA's shared memory).
__device__ __forceinline__ uint32_t instr_desc_pair_swap(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(BM2 >> 4) << 24);
}
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <bool SWIGLU, int KPS>
struct Shape2 {
  static_assert(KPS == 1 || KPS == 2, "k-blocks per ring stage");
  static constexpr int BN = SWIGLU ? 128 : 256;       // output columns per tile
  static constexpr int kSpansPerCta = 2;              // 64-column B spans each CTA loads
  static constexpr uint32_t kABytes = 128 * BK * 2;   // 16 KB: this CTA's 128 rows
  static constexpr uint32_t kSpanBytes = BK * 128;    // 8 KB
  static constexpr uint32_t kBBytes = kSpansPerCta * kSpanBytes;  // 16 KB
  static constexpr uint32_t kKbBytes = kABytes + kBBytes;         // one k-block: 32 KB per CTA
  // k-blocks per ring stage: the loads of a stage complete on one barrier
  // and the MMAs of a stage release it with one commit, so two k-blocks a
  // stage halve the barrier round trips per byte (same bytes in flight)
  static constexpr int kKbPerStage = KPS;
  static constexpr uint32_t kStageBytes = kKbPerStage * kKbBytes;
  static constexpr int kStages = 6 / kKbPerStage;
  static constexpr int kMmaN = 256;                   // N of the pair instruction
  static constexpr uint32_t kAccCols = 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdesc = instr_desc(BM2, kMmaN);
  static constexpr uint32_t kStageRowWords = 36;
  static constexpr uint32_t kEpiBytes = 4 * 32 * kStageRowWords * 4;
  static constexpr size_t kSmemFixed =
      1024 + kStages * kStageBytes + 256 + kEpiBytes;
};

template <bool SWIGLU, int KPS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ CUtensorMap tmB3,
                        const __grid_constant__ CUtensorMap tmX32,
                        const __grid_constant__ CUtensorMap tmX8, const Params p) {
  grid_dependency();  // the previous grid is complete; the next may launch
  using S = Shape2<SWIGLU, KPS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + S::kStages * S::kStageBytes);
  // bars: full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain[1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S::kStages + 5);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  // per tile parity and epilogue warp: whether its accumulator became ready
  volatile int *s_ready = reinterpret_cast<volatile int *>(abort_flag + 1);
  float *s_epi = reinterpret_cast<float *>(ring + S::kStages * S::kStageBytes + 256);
  int32_t *s_off = reinterpret_cast<int32_t *>(ring + S::kStages * S::kStageBytes + 256 +
                                               S::kEpiBytes);
  int32_t *s_tstart = s_off + (p.G + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x / 2, npairs = gridDim.x / 2;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S::kStages);
  const uint32_t accf0 = smem_addr(bars + 2 * S::kStages);
  const uint32_t acce0 = smem_addr(bars + 2 * S::kStages + 2);
  const uint32_t drain = smem_addr(bars + 2 * S::kStages + 4);
  // A pair stops only on the long limit: its CTAs complete copies on each
  // other's barriers, so one CTA stopping early must not outrun its peer.
  const Ctl ctl{abort_flag, p.err, kWaitLimitNs};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);   // the leader's arrive.expect_tx (both CTAs' bytes)
      mbar_init(empty0 + 8 * s, 1);  // the leader's multicast commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);   // the leader's multicast commit
      mbar_init(acce0 + 8 * b, 8);   // 4 epilogue warps x 2 CTAs (leader's copy is used)
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB1);
    if (SWIGLU) prefetch_tmap(&tmB3);
    if (p.pair_swap) {
      prefetch_tmap(&tmX32);
      prefetch_tmap(&tmX8);
    }
  }
  bool bad = false;
  for (int g = threadIdx.x; g <= p.G; g += kThreads) {
    const int v = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.fixed_rows);
    s_off[g] = v;
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc_pair(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  // Two tile lists, each an exclusive scan of per-group tile counts: heavy
  // (groups of at least 256 rows: their chunks, the partial last one
  // included, chunks fastest within a column tile) and -- when partial chunks
  // run swap-AB -- light (smaller groups: one swap-AB tile per column tile).
  // The deal merges them evenly (tile t is light when the count of light
  // tiles among the first t+1, round-down of (t+1) L / total, steps up), so
  // every wave mixes compute-bound heavy tiles with light tiles that mostly
  // stream their group's weights.
  int32_t *s_lstart = s_tstart + (p.G + 1);
  const int n_tiles = (p.N + S::BN - 1) / S::BN;
  for (int g = threadIdx.x; g < p.G; g += kThreads) {
    const int rows = s_off[g + 1] - s_off[g];
    if (rows < 0) bad = true;
    const bool light = p.pair_swap && rows > 0 && rows <= p.swap_rows;
    s_tstart[g] = (rows > 0 && !light) ? ((rows + BM2 - 1) / BM2) * n_tiles : 0;
    s_lstart[g] = light ? n_tiles : 0;
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
  if (warp == 1) tmem_relinquish_pair();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Both CTAs see the same offsets, so they agree on the tile list; a CTA
  // that found bad offsets stops, and its peer's waits time out.
  const int n_heavy = s_tstart[p.G], n_light = s_lstart[p.G];
  const int total = *abort_flag ? 0 : n_heavy + n_light;
  const int num_kb = (p.K + BK - 1) / BK;
  const uint32_t leader_full0 = mapa_shared(full0, 0);
  const uint32_t leader_acce0 = mapa_shared(acce0, 0);

  // tile -> group g, column tile n, 256-row chunk from row0 with nr rows;
  // chunks fastest.  A light tile (and, with p.pair_swap == 2, a group's last,
  // partial chunk) runs swap-AB: the weights are the MMA's M (256 columns,
  // 128 per CTA), the rows its N, rounded up to 16, so a group of a few rows
  // costs a 16-row MMA, not a 256-row one, while each CTA still streams only
  // half of the weights.
  struct PairTile {
    int g, n, row0, nr;
    bool swap;
  };
  // Every role walks the same tiles, pair, pair + npairs, ..., in order, so
  // the deal's counts and the group lookups advance from one tile to the
  // next: no 64-bit division and no binary search per tile.  (The MMA
  // thread's time between two tiles is a bubble for the tensor pipe; with
  // both, it was about a microsecond, a fifth of a 12-k-block tile.)
  //   light tile t:  floor((t+1) L / N) > floor(t L / N), L = n_light, N = total
  //   light index:   floor(t L / N); heavy index: t - floor(t L / N)
  struct Walk {
    long long r0, r1;  // t L mod N, (t + 1) L mod N
    int l0, l1;        // floor(t L / N), floor((t + 1) L / N)
    int gh, gl;        // group cursors in the heavy and light lists
  };
  const long long w_n = total > 0 ? total : 1, w_l = n_light;
  const int w_q = (int)((long long)npairs * w_l / w_n);
  const long long w_r = (long long)npairs * w_l - (long long)w_q * w_n;
  auto walk_start = [&]() {
    Walk w;
    const long long a0 = (long long)pair * w_l, a1 = a0 + w_l;
    w.l0 = (int)(a0 / w_n);
    w.r0 = a0 - (long long)w.l0 * w_n;
    w.l1 = (int)(a1 / w_n);
    w.r1 = a1 - (long long)w.l1 * w_n;
    w.gh = 0;
    w.gl = 0;
    return w;
  };
  auto walk_next = [&](Walk &w) {  // to tile + npairs
    w.l0 += w_q;
    w.r0 += w_r;
    if (w.r0 >= w_n) {
      w.r0 -= w_n;
      ++w.l0;
    }
    w.l1 += w_q;
    w.r1 += w_r;
    if (w.r1 >= w_n) {
      w.r1 -= w_n;
      ++w.l1;
    }
  };
  // the group of list index idx: the largest g with start[g] <= idx (a group
  // with tiles: an empty one shares its start with the next), from the
  // previous tile's group on
  auto advance = [&](const int32_t *start, int &g, int idx) {
    while (g + 1 < p.G && start[g + 1] <= idx) ++g;
    return g;
  };
  auto pair_tile = [&](int tile, Walk &w) {
    PairTile t;
    const bool light = w.l1 > w.l0;
    if (light) {  // light: the whole group, column tile n
      const int li = w.l0;
      t.g = advance(s_lstart, w.gl, li);
      t.n = li - s_lstart[t.g];
      t.row0 = s_off[t.g];
      t.nr = s_off[t.g + 1] - s_off[t.g];
    } else {  // heavy: chunk m of column tile n
      const int hi = tile - w.l0;
      t.g = advance(s_tstart, w.gh, hi);
      const int rows = s_off[t.g + 1] - s_off[t.g];
      const int mt = (rows + BM2 - 1) / BM2;
      const int local = hi - s_tstart[t.g];
      t.n = local / mt;
      const int m = local - t.n * mt;
      t.row0 = s_off[t.g] + m * BM2;
      t.nr = min(BM2, rows - m * BM2);
    }
    t.swap = light || (p.pair_swap == 2 && t.nr < BM2);
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      Walk w = walk_start();
      for (int tile = pair; tile < total && ok; tile += npairs, walk_next(w)) {
        const PairTile t = pair_tile(tile, w);
        const int h = t.swap ? ((t.nr + 15) & ~15) / 2 : 0;  // swap: rows of B per CTA
        // bytes this CTA loads per k-block
        const uint32_t cta_bytes = t.swap ? (uint32_t)h * 128u + S::kBBytes : S::kKbBytes;
        const int row = t.row0 + (int)rank * 128;  // full tile: this CTA's 128 rows of A
        for (int kb0 = 0; kb0 < num_kb; kb0 += S::kKbPerStage) {
          if (!wait(empty0 + 8 * s, ph ^ 1, ctl)) {
            ok = false;
            break;
          }
          const int nk = min(S::kKbPerStage, num_kb - kb0);
          const uint32_t lfb = leader_full0 + 8 * s;
          if (rank == 0) mbar_expect_tx(full0 + 8 * s, 2 * cta_bytes * (uint32_t)nk);
          for (int hk = 0; hk < nk; ++hk) {
            const int kb = kb0 + hk;
            const uint32_t st = smem_addr(ring + s * S::kStageBytes + hk * S::kKbBytes);
            if (t.swap) {
              // B: this CTA's h rows (32-row, then 8-row boxes); A: its 128
              // weight columns, two 64-column spans (the up projection: gate
              // and up of the same 64 columns, so each CTA's accumulator holds
              // both halves of its columns' SwiGLU)
              const int xrow = t.row0 + (int)rank * h;
              int q = 0;
              for (; q + 32 <= h; q += 32)
                tma_load_2d_pair(st + q * 128, &tmX32, lfb, kb * BK, xrow + q);
              for (; q < h; q += 8) tma_load_2d_pair(st + q * 128, &tmX8, lfb, kb * BK, xrow + q);
              if (SWIGLU) {
                const int col = t.n * S::BN + (int)rank * 64;
                tma_load_3d_pair(st + S::kABytes, &tmB1, lfb, col, kb * BK, t.g);
                tma_load_3d_pair(st + S::kABytes + S::kSpanBytes, &tmB3, lfb, col, kb * BK, t.g);
              } else {
                const int col = t.n * S::BN + (int)rank * 128;
#pragma unroll
                for (int j = 0; j < 2; ++j)
                  tma_load_3d_pair(st + S::kABytes + j * S::kSpanBytes, &tmB1, lfb, col + j * 64,
                                   kb * BK, t.g);
              }
            } else {
              const CUtensorMap *mb = (SWIGLU && rank == 1) ? &tmB3 : &tmB1;
              const int bcol = SWIGLU ? t.n * S::BN : t.n * S::BN + (int)rank * 128;
              if (p.l2_hints) {
                // 1: rows evict-last, weights evict-first; 2: rows evict-last,
                // weights unhinted; 3: rows unhinted, weights evict-last
                if (p.l2_hints == 3)
                  tma_load_2d_pair(st, &tmA, lfb, kb * BK, row);
                else
                  tma_load_2d_pair_hint(st, &tmA, lfb, kb * BK, row, pol_keep);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  if (p.l2_hints == 2)
                    tma_load_3d_pair(st + S::kABytes + j * S::kSpanBytes, mb, lfb, bcol + j * 64,
                                     kb * BK, t.g);
                  else
                    tma_load_3d_pair_hint(st + S::kABytes + j * S::kSpanBytes, mb, lfb,
                                          bcol + j * 64, kb * BK, t.g,
                                          p.l2_hints == 3 ? pol_keep : pol_stream);
                }
              } else {
                tma_load_2d_pair(st, &tmA, lfb, kb * BK, row);
#pragma unroll
                for (int j = 0; j < 2; ++j)
                  tma_load_3d_pair(st + S::kABytes + j * S::kSpanBytes, mb, lfb, bcol + j * 64,
                                   kb * BK, t.g);
              }
            }
          }
          ++issued;
          if (++s == S::kStages) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok && issued > 0) {
        // Stopped early.  The leader waits for the stages it armed; both CTAs'
        // copies complete there.  The peer gives its copies a moment to land.
        if (rank == 0) {
          for (int q = 0; q < S::kStages && q < issued; ++q) {
            int st_i = s - 1 - q;
            uint32_t par = ph;
            if (st_i < 0) {
              st_i += S::kStages;
              par ^= 1;
            }
            wait_drain(full0 + 8 * st_i, par, p.err);
          }
        } else {
          const uint64_t t0 = global_timer();
          while (global_timer() - t0 < 2000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (rank == 0 && lane == 0) {
      int s = 0, buf = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true, any = false;
      // descriptors of stage 0 (rows: K-major; weights: MN-major 64-column
      // spans, LBO = span stride); stage s and K step kk are additions to the
      // 16-byte address field (every stage lies below 256 KB)
      const uint64_t rows_d0 = smem_desc(smem_addr(ring), 16, 1024);
      const uint64_t w_d0 = smem_desc(smem_addr(ring) + S::kABytes, S::kSpanBytes, 1024);
      constexpr uint32_t kStageStep = S::kStageBytes >> 4, kKbStep = S::kKbBytes >> 4;
      constexpr uint32_t kRowK = 32 >> 4, kWK = 2048 >> 4;
      Walk w = walk_start();
      for (int tile = pair; tile < total && ok; tile += npairs, walk_next(w)) {
        const PairTile t = pair_tile(tile, w);
        const uint32_t idesc_swap = instr_desc_pair_swap((t.nr + 15) & ~15);
        if (!wait(acce0 + 8 * buf, acc_ph ^ 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * S::kAccCols;
        for (int kb0 = 0; kb0 < num_kb; kb0 += S::kKbPerStage) {
          if (!wait(full0 + 8 * s, ph, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(S::kKbPerStage, num_kb - kb0);
          for (int hk = 0; hk < nk; ++hk) {
            const uint64_t rd = rows_d0 + s * kStageStep + hk * kKbStep;
            const uint64_t wd = w_d0 + s * kStageStep + hk * kKbStep;
            const uint32_t acc0 = (kb0 + hk) != 0;
            if (t.swap) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_pair(d_tmem, wd + kk * kWK, rd + kk * kRowK, idesc_swap, kk ? 1u : acc0);
            } else {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_pair(d_tmem, rd + kk * kRowK, wd + kk * kWK, S::kIdesc, kk ? 1u : acc0);
            }
          }
          any = true;
          umma_commit_pair_both(empty0 + 8 * s);
          if (++s == S::kStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_both(accf0 + 8 * buf);
        buf ^= 1;
        if (buf == 0) acc_ph ^= 1;
      }
      if (!ok && any) {
        umma_commit_pair_self(drain);
        wait_drain(drain, 0, p.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Warp w reads TMEM lanes 32*quarter ..  The warps of quarters q and
    // q ^ 2 form a pair: on an up-projection swap tile one holds the gate and
    // the other the up values of the same 32 columns, and they meet through
    // shared memory (named barrier 1 + (q & 1)).  So that neither ever waits
    // there for a partner that has stopped, the pair decides together, tile
    // by tile, whether to go on.
    const int quarter = warp & 3;
    const int partner = ((quarter ^ 2) < 2 ? (quarter ^ 2) + 4 : (quarter ^ 2));  // its warp
    const int bar_id = 1 + (quarter & 1);
    int buf = 0, it = 0;
    uint32_t acc_ph = 0;
    float *stg = s_epi + (warp - 2) * 32 * S::kStageRowWords;
    const float *pstg = s_epi + (partner - 2) * 32 * S::kStageRowWords;
    Walk w = walk_start();
    for (int tile = pair; tile < total; tile += npairs, ++it, walk_next(w)) {
      const PairTile t = pair_tile(tile, w);
      const int g = t.g, n = t.n;
      int ready = 0;
      if (lane == 0) ready = wait(accf0 + 8 * buf, acc_ph, ctl) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (lane == 0) s_ready[(it & 1) * 4 + (warp - 2)] = ready;
      named_bar_sync(bar_id, 64);
      ready = ready && s_ready[(it & 1) * 4 + (partner - 2)];
      if (!ready) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + buf * S::kAccCols + ((uint32_t)(quarter * 32) << 16);
      if (t.swap) {
        // lane = weight column of this CTA's half, TMEM column = row of the chunk
        if (SWIGLU) {
          // lanes 0-63: gate of columns n*128 + rank*64 .. +63; lanes 64-127: up
          const bool gate = quarter < 2;
          const float *g_stg = gate ? stg : pstg;
          const float *u_stg = gate ? pstg : stg;
          const int col0 = n * S::BN + (int)rank * 64 + (quarter & 1) * 32;
          const int jb = gate ? 0 : 16;  // the 16 rows of each chunk this warp writes
#pragma unroll 1
          for (int j0 = 0; j0 < t.nr; j0 += 32) {
            float v[32];
            tmem_ld32(tb + j0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[j * S::kStageRowWords + lane] = v[j];
            named_bar_sync(bar_id, 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = jb + i * 4 + (lane >> 3), q = lane & 7;
              const int grow = t.row0 + j0 + j, gcol = col0 + q * 4;
              const float4 gv =
                  *reinterpret_cast<const float4 *>(g_stg + j * S::kStageRowWords + 4 * q);
              const float4 uv =
                  *reinterpret_cast<const float4 *>(u_stg + j * S::kStageRowWords + 4 * q);
              if (j0 + j < t.nr && gcol < p.N) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(silu_times(gv.x, uv.x),
                                                          silu_times(gv.y, uv.y));
                __nv_bfloat162 hi = __floats2bfloat162_rn(silu_times(gv.z, uv.z),
                                                          silu_times(gv.w, uv.w));
                uint2 w;
                w.x = *reinterpret_cast<uint32_t *>(&lo);
                w.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                           (size_t)grow * p.N + gcol) = w;
              }
            }
            named_bar_sync(bar_id, 64);  // both read before the next chunk is staged
          }
        } else {
          const int col0 = n * S::BN + (int)rank * 128 + quarter * 32;
#pragma unroll 1
          for (int j0 = 0; j0 < t.nr; j0 += 32) {
            float v[32];
            tmem_ld32(tb + j0, v);  // v[j] = y[row j0 + j][col0 + lane]
            if (p.yexp) {
              store_y16_lane_cols(v, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords, lane,
                                  t.row0 + j0, t.nr - j0, col0, p.N, p.out, p.yexp, p.nblk,
                                  p.row_w, p.w_row_src);
              continue;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) stg[j * S::kStageRowWords + lane] = v[j];
            __syncwarp();
            {
#pragma unroll
              for (int i = 0; i < 8; ++i) {  // fp32 rows: 8 lanes x 16 bytes, 4 rows per step
                const int j = i * 4 + (lane >> 3), q = lane & 7;
                const int grow = t.row0 + j0 + j, gcol = col0 + q * 4;
                float4 o = *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
                if (j0 + j < t.nr && gcol < p.N) {
                  if (p.row_w) {
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
            __syncwarp();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(acce0 + 8 * buf);
          else
            mbar_arrive_cluster(leader_acce0 + 8 * buf);
        }
        buf ^= 1;
        if (buf == 0) acc_ph ^= 1;
        continue;
      }
      const int row0 = t.row0 + (int)rank * 128 + quarter * 32;
      const int row_end = s_off[g + 1];
      // one 32-column chunk of this warp's 32 rows, from registers to memory
      auto store_chunk = [&](float(&v)[32], int c) {
        const int col = n * S::BN + c;
        if (SWIGLU) {
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
          for (int i = 0; i < 4; ++i) {
            const int r = i * 8 + (lane >> 2), q = lane & 3;
            const int grow = row0 + r, gcol = col + q * 8;
            const uint4 val = *reinterpret_cast<const uint4 *>(st + r * S::kStageRowWords + 4 * q);
            if (grow < row_end && gcol < p.N)
              *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) +
                                         (size_t)grow * p.N + gcol) = val;
          }
        } else if (p.yexp) {  // y16: fp16 rows, one exponent per 32-column block
          if (p.row_w && row0 + lane < row_end) {
            const float wr = p.row_w[p.w_row_src[row0 + lane]];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= wr;
          }
          store_y16_lane_rows(v, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords, lane, row0,
                              row_end, col, p.N, p.out, p.yexp, p.nblk);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(stg + lane * S::kStageRowWords + 4 * q) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = i * 4 + (lane >> 3), q = lane & 7;
            const int grow = row0 + r, gcol = col + q * 4;
            float4 o = *reinterpret_cast<const float4 *>(stg + r * S::kStageRowWords + 4 * q);
            if (grow < row_end && gcol < p.N) {
              if (p.bias) {
                const float *b = p.bias + gcol;
                o.x += b[0];
                o.y += b[1];
                o.z += b[2];
                o.w += b[3];
              }
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
        __syncwarp();
      };
      // two chunks per wait for tensor memory: gate and up of the same
      // columns, or two neighbouring column chunks of the plain product;
      // y16: the row's eight block exponents of the tile gathered in exps
      uint64_t exps = 0;
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
            if (p.row_w && row0 + lane < row_end) {
              const float wr = p.row_w[p.w_row_src[row0 + lane]];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                v[i] *= wr;
                u[i] *= wr;
              }
            }
            uint32_t e2;
            store_y16_lane_rows2(v, u, reinterpret_cast<uint32_t *>(stg), S::kStageRowWords, lane,
                                 row0, row_end, n * S::BN + c, p.N, p.out, nullptr, p.nblk, &e2);
            exps |= (uint64_t)e2 << (2 * c / 8);  // blocks c/32 and c/32 + 1 of the tile
          } else {
            store_chunk(v, c);
            store_chunk(u, c + 32);
          }
        }
      }
      if (!SWIGLU && p.yexp && row0 + lane < row_end) {
        // one 8-byte store per row when the tile's 8 blocks are whole and
        // aligned, else the valid ones a byte each
        const int b0 = n * (S::BN / 32), nb = min(S::BN / 32, p.nblk - b0);
        int8_t *ye = p.yexp + (size_t)(row0 + lane) * p.nblk + b0;
        const uintptr_t al = reinterpret_cast<uintptr_t>(ye);
        if (nb == 8 && (al & 7) == 0) {
          *reinterpret_cast<uint64_t *>(ye) = exps;
        } else if (nb == 8 && (al & 1) == 0) {  // e.g. 90 blocks a row: 2-byte aligned
#pragma unroll
          for (int b = 0; b < 8; b += 2)
            *reinterpret_cast<uint16_t *>(ye + b) = (uint16_t)(exps >> (8 * b));
        } else {
          for (int b = 0; b < nb; ++b) ye[b] = (int8_t)(exps >> (8 * b));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(acce0 + 8 * buf);
        else
          mbar_arrive_cluster(leader_acce0 + 8 * buf);
      }
      buf ^= 1;
      if (buf == 0) acc_ph ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair's MMAs may still use its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Small groups: the same products with the operands swapped ("swap-AB")
//
// When most groups hold a few rows (decode, or thousands of fine-grained
// experts), a 128-row tile is mostly padding.  Here a tile is 128 output
// columns x at most 128 rows of one group: the weights are the MMA's M
// operand (MN-major, the same 64 x 64 TMA boxes as above), the group's rows
// are its N operand (K-major, loaded in 32-row boxes, only as many as the tile
// has rows), and N is the row count rounded up to 16, set per tile in the
// instruction descriptor.  Tensor memory then holds the transposed tile
// (lane = output column, column = row); the epilogue transposes it back
// through its shared-memory stage.
//   SWIGLU: two MMAs per step, gate = W1^T.x^T and up = W3^T.x^T, into TMEM
//           columns [0,128) and [128,256) of the accumulator buffer;
//   PLAIN:  one MMA per step, y^T = W^T.h^T.
// ---------------------------------------------------------------------------
constexpr int kRowBox = 32;  // rows per TMA box of the N operand

template <bool SWIGLU, bool FP8W = false>
struct ShapeSwap {
  static constexpr int kCols = 128;                      // output columns per tile (MMA M)
  // rows per tile (MMA N): fp8 weights keep decode-sized row tiles so that
  // a stage stays small and the code stream can run deep
  static constexpr int kMaxRows = FP8W ? 32 : 128;
  // fp8 down projection: 256-column tiles as two 128-column halves (the MMA's
  // M is 128), so that decode-sized layers fill the GPU in one wave
  static constexpr bool kWide = FP8W && !SWIGLU;
  static constexpr int kTileCols = kWide ? 256 : 128;
  static constexpr int kWOps = (SWIGLU || kWide) ? 2 : 1;  // operands or column halves
  static constexpr uint32_t kSpanBytes = BK * 128;       // 8 KB: 64 K-rows x 64 columns
  static constexpr uint32_t kWBytes = kWOps * 2 * kSpanBytes;   // 16 or 32 KB (bf16)
  static constexpr uint32_t kRowBoxBytes = kRowBox * BK * 2;    // 4 KB
  static constexpr uint32_t kXBytes = kMaxRows * BK * 2;        // 16 KB (fp8: 4 KB)
  // FP8W codes are K-contiguous ([G, N, K]): per operand one box of 128
  // columns x 64 K-codes (64-byte rows, 64-byte TMA swizzle)
  static constexpr uint32_t kQOpBytes = FP8W ? kCols * BK : 0;
  static constexpr uint32_t kQBytes = kWOps * kQOpBytes;
  // a stage: the weights (bf16, or e4m3 codes) and the rows of one k-block
  static constexpr uint32_t kStageBytes = (FP8W ? kQBytes : kWBytes) + kXBytes;
  static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
  static constexpr uint32_t kRingBytes = kStages * kStageBytes;
  // FP8W: + 8 converter warps (6-13), two per tensor-memory lane quarter
  static constexpr int kCtaThreads = FP8W ? 448 : 192;
  static constexpr int kConvThreads = 256;
  // Tensor memory: two accumulators (W1 [and W3] x rows), and with fp8
  // weights kASlots k-blocks of widened weights, the MMA's A operand
  // (lane = output column, 32 columns = 64 bf16 K-values per operand).
  static constexpr uint32_t kW3Off = FP8W ? kMaxRows : 128;     // W3 accumulator columns
  static constexpr uint32_t kAccCols = kWOps * kW3Off;
  static constexpr int kASlots = FP8W ? 6 : 0;
  static constexpr uint32_t kACol0 = 2 * kAccCols;
  static constexpr uint32_t kASlotCols = kWOps * 32;
  static constexpr uint32_t kTmemCols = FP8W ? 512 : 2 * kAccCols;
  static constexpr uint32_t kStageRowWords = 36;
  static constexpr uint32_t kEpiBytes = 4 * 32 * kStageRowWords * 4;
  static constexpr uint32_t kBarBytes = FP8W ? 512 : 256;
  static constexpr size_t kSmemFixed = 1024 + kRingBytes + kBarBytes + kEpiBytes;
  // barriers: full, empty per stage, 2 + 2 accumulator, drain; FP8W also
  // converted and free per A slot
  static constexpr int kBars = 2 * kStages + 2 * kASlots + 5;
  static_assert(kBars * 8 + 8 <= kBarBytes, "barriers, TMEM slot and abort flag fit");
  static_assert(kACol0 + kASlots * kASlotCols <= kTmemCols, "tensor memory");
  static_assert(kStageBytes % 1024 == 0 && (FP8W ? kQBytes : kWBytes) % 1024 == 0,
                "swizzled tiles start on 1024-byte boundaries");
};

// kind::f16 descriptor: fp32 accumulator, bf16 A and B, A MN-major, B K-major.
__device__ __forceinline__ uint32_t instr_desc_swap(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

template <bool SWIGLU, bool FP8W = false>
__global__ void __launch_bounds__(ShapeSwap<SWIGLU, FP8W>::kCtaThreads, 1)
    k_grouped_gemm_swap(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW1,
                        const __grid_constant__ CUtensorMap tmW3, const Params p) {
  grid_dependency();  // the previous grid is complete; the next may launch
  using S = ShapeSwap<SWIGLU, FP8W>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + S::kRingBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + S::kBars);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  float *s_epi = reinterpret_cast<float *>(ring + S::kRingBytes + S::kBarBytes);
  int32_t *s_off =
      reinterpret_cast<int32_t *>(ring + S::kRingBytes + S::kBarBytes + S::kEpiBytes);
  int32_t *s_tstart = s_off + (p.G + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + S::kStages);
  const uint32_t accf0 = smem_addr(bars + 2 * S::kStages);
  const uint32_t acce0 = smem_addr(bars + 2 * S::kStages + 2);
  const uint32_t drain = smem_addr(bars + 2 * S::kStages + 4);
  // FP8W: A slot converted[kASlots], A slot free[kASlots]
  const uint32_t conv0 = smem_addr(bars + 2 * S::kStages + 5);
  const uint32_t cempty0 = smem_addr(bars + 2 * S::kStages + 5 + S::kASlots);
  const Ctl ctl{abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf0 + 8 * b, 1);
      mbar_init(acce0 + 8 * b, 4);
    }
    mbar_init(drain, 1);
    for (int c = 0; c < S::kASlots; ++c) {
      mbar_init(conv0 + 8 * c, 4);  // the 4 warps of the group converting that k-block
      mbar_init(cempty0 + 8 * c, 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW1);
    if (SWIGLU) prefetch_tmap(&tmW3);
  }
  bool bad = false;
  for (int g = threadIdx.x; g <= p.G; g += S::kCtaThreads) {
    const int v = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.fixed_rows);
    s_off[g] = v;
    if (v < 0 || v > p.rows_cap) bad = true;
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), S::kTmemCols);
  __syncthreads();
  const int col_tiles = (p.N + S::kTileCols - 1) / S::kTileCols;
  for (int g = threadIdx.x; g < p.G; g += S::kCtaThreads) {
    const int rows = s_off[g + 1] - s_off[g];
    if (rows < 0) bad = true;
    s_tstart[g] = rows > 0 ? ((rows + S::kMaxRows - 1) / S::kMaxRows) * col_tiles : 0;
  }
  if (bad) {
    *abort_flag = 1;
    raise_error(p.err, kErrIndex);
  }
  __syncthreads();
  if (warp == 0) {
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

  // tile -> (group g, column tile c, row tile r); rows fastest, so CTAs
  // running together share a weight tile
  auto tile_coords = [&](int tile, int &g, int &c, int &r, int &row0, int &nr) {
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int rows = s_off[g + 1] - s_off[g];
    const int rt = (rows + S::kMaxRows - 1) / S::kMaxRows;
    const int local = tile - s_tstart[g];
    c = local / rt;
    r = local - c * rt;
    row0 = s_off[g] + r * S::kMaxRows;
    nr = min(S::kMaxRows, rows - r * S::kMaxRows);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool gather = p.row_src != nullptr;
    int s = 0;
    uint32_t ph = 0, issued_parity = 0, issued_mask = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      int g, c, r, row0, nr;
      tile_coords(tile, g, c, r, row0, nr);
      // rows loaded: 32-row boxes, or (gathering) gather4s up to the MMA's N
      const int nq = gather ? ((nr + 15) & ~15) / 4 : (nr + kRowBox - 1) / kRowBox;
      const uint32_t wbytes = FP8W ? S::kQBytes : S::kWBytes;  // where the rows start
      const uint32_t bytes = wbytes + (gather ? nq * 512 : nq * S::kRowBoxBytes);
      int tok[4] = {0, 0, 0, 0};
      if (gather && lane < nq) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int rr = 4 * lane + q;
          if (rr < nr) tok[q] = p.row_src[row0 + rr] / p.k_max;
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
        const uint32_t fb = full0 + 8 * s;
        if (lane == 0) mbar_expect_tx(fb, bytes);
        if (gather && lane < nq)
          tma_gather4(st + wbytes + lane * 4 * 128, &tmX, fb, kb * BK, tok[0], tok[1], tok[2],
                      tok[3]);
        if (lane == 0) {
          if (FP8W) {  // codes [G, N, K]: one box (64 K x 128 columns) per operand / half
            tma_load_3d(st, &tmW1, fb, kb * BK, c * S::kTileCols, g);
            if (SWIGLU) tma_load_3d(st + S::kQOpBytes, &tmW3, fb, kb * BK, c * S::kTileCols, g);
            if (S::kWide)
              tma_load_3d(st + S::kQOpBytes, &tmW1, fb, kb * BK, c * S::kTileCols + 128, g);
          } else {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_3d(st + j * S::kSpanBytes, &tmW1, fb, c * S::kCols + j * 64, kb * BK, g);
            if (SWIGLU) {
#pragma unroll
              for (int j = 0; j < 2; ++j)
                tma_load_3d(st + (2 + j) * S::kSpanBytes, &tmW3, fb, c * S::kCols + j * 64,
                            kb * BK, g);
            }
          }
          if (!gather)
            for (int q = 0; q < nq; ++q)
              tma_load_2d(st + wbytes + q * S::kRowBoxBytes, &tmX, fb, kb * BK,
                          row0 + q * kRowBox);
        }
        issued_mask |= 1u << s;
        issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
        if (++s == S::kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (!ok && lane == 0) {
      for (int q = 0; q < S::kStages; ++q)
        if ((issued_mask >> q) & 1u) wait_drain(full0 + 8 * q, (issued_parity >> q) & 1u, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, buf = 0, cs = 0;
      uint32_t ph = 0, acc_ph = 0, cph = 0;
      bool ok = true, any = false;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int g, c, r, row0, nr;
        tile_coords(tile, g, c, r, row0, nr);
        // bf16: weights an MN-major smem A; fp8: the widened weights in
        // tensor memory (K-major); the rows K-major in both
        const uint32_t idesc = FP8W ? instr_desc_kk(S::kCols, (nr + 15) & ~15)
                                    : instr_desc_swap(S::kCols, (nr + 15) & ~15);
        if (!wait(acce0 + 8 * buf, acc_ph ^ 1, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * S::kAccCols;
        for (int kb = 0; kb < num_kb; ++kb) {
          // FP8W: the rows have landed and the converters have filled the weights
          if (!wait(full0 + 8 * s, ph, ctl) || (FP8W && !wait(conv0 + 8 * cs, cph, ctl))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_addr(ring + s * S::kStageBytes);
          const uint32_t xt = st + (FP8W ? S::kQBytes : S::kWBytes);
          const uint32_t at = tmem_base + S::kACol0 + cs * S::kASlotCols;  // FP8W
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // rows: K-major 128-byte rows; bf16 weights: MN-major spans (LBO
            // = span stride); fp8: 8 tensor-memory columns per 16 K-values
            const uint64_t xd = smem_desc(xt + kk * 32, 16, 1024);
            const uint32_t acc = (kb | kk) != 0;
            if (FP8W) {
              umma_ts(d_tmem, at + kk * 8, xd, idesc, acc);
              if (S::kWOps == 2) umma_ts(d_tmem + S::kW3Off, at + 32 + kk * 8, xd, idesc, acc);
            } else {
              const uint64_t w1d = smem_desc(st + kk * 2048, S::kSpanBytes, 1024);
              umma(d_tmem, w1d, xd, idesc, acc);
              if (SWIGLU) {
                const uint64_t w3d =
                    smem_desc(st + 2 * S::kSpanBytes + kk * 2048, S::kSpanBytes, 1024);
                umma(d_tmem + S::kW3Off, w3d, xd, idesc, acc);
              }
            }
          }
          any = true;
          umma_commit(empty0 + 8 * s);
          if (FP8W) umma_commit(cempty0 + 8 * cs);
          if (++s == S::kStages) {
            s = 0;
            ph ^= 1;
          }
          if (FP8W && ++cs == S::kASlots) {
            cs = 0;
            cph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * buf);
        buf ^= 1;
        if (buf == 0) acc_ph ^= 1;
      }
      if (!ok && any) {
        umma_commit(drain);
        wait_drain(drain, 0, p.err);
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    // TMEM lane = output column (this warp: columns 32*quarter ..), TMEM
    // column = row of the tile.
    const int quarter = warp & 3;
    int buf = 0;
    uint32_t acc_ph = 0;
    float *stg = s_epi + (warp - 2) * 32 * S::kStageRowWords;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, c, r, row0, nr;
      tile_coords(tile, g, c, r, row0, nr);
      int ready = 0;
      if (lane == 0) ready = wait(accf0 + 8 * buf, acc_ph, ctl) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      // wide fp8 tiles: two 128-column halves, each its own accumulator
      for (int h = 0; h < (S::kWide ? 2 : 1); ++h) {
      const uint32_t tb = tmem_base + buf * S::kAccCols + h * S::kW3Off +
                          ((uint32_t)(quarter * 32) << 16);
      const int col0 = c * S::kTileCols + h * 128 + quarter * 32;  // this warp's 32 columns
      // FP8W: this lane's column scales (lane = column)
      float sc1 = 1.f, sc3 = 1.f;
      if (FP8W && col0 + lane < p.N) {
        sc1 = p.scale1[(size_t)g * p.N + col0 + lane];
        if (SWIGLU) sc3 = p.scale3[(size_t)g * p.N + col0 + lane];
      }
#pragma unroll 1
      for (int j0 = 0; j0 < nr; j0 += 32) {
        float v[32], u[32];  // v[j] = out[row j0 + j][col0 + lane]
        if (SWIGLU)
          tmem_ld32x2(tb + j0, tb + S::kW3Off + j0, v, u);
        else
          tmem_ld32(tb + j0, v);
        if (FP8W) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= sc1;
        }
        if (SWIGLU) {
          if (FP8W) {
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] *= sc3;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = silu_times(v[i], u[i]);
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
            const float4 f = *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
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
        } else {  // fp32 (+ bias) rows: 8 lanes x 16 bytes, 4 rows per step
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int j = i * 4 + (lane >> 3), q = lane & 7;
            const int grow = row0 + j0 + j, gcol = col0 + q * 4;
            float4 o = *reinterpret_cast<const float4 *>(stg + j * S::kStageRowWords + 4 * q);
            if (j0 + j < nr && gcol < p.N) {
              if (p.bias) {
                const float *b = p.bias + gcol;
                o.x += b[0];
                o.y += b[1];
                o.z += b[2];
                o.w += b[3];
              }
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
        __syncwarp();
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * buf);
      buf ^= 1;
      if (buf == 0) acc_ph ^= 1;
    }
  } else if (FP8W) {
    // ------------------------------------------------------------ fp8 converters
    // Per k-block: wait for its codes (stage s) and a free A slot cs; each
    // thread widens the 64 codes of its weight column (= its tensor-memory
    // lane, warp w holding lanes 32*(w%4)..) per operand and stores them as
    // 32 tensor-memory columns, then the slot is marked converted.  Warps 6-9
    // take the even k-blocks and warps 10-13 the odd ones, so that two
    // k-blocks are in flight at a time.
    const int quarter = warp & 3, half = (warp - 6) >> 2;
    const int m = quarter * 32 + lane;  // weight column within the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int s = 0, cs = 0, it = 0;
    uint32_t ph = 0, cph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        if ((it & 1) == half) {
          int okw = 1;
          if (lane == 0)
            okw = (wait(full0 + 8 * s, ph, ctl) && wait(cempty0 + 8 * cs, cph ^ 1, ctl)) ? 1 : 0;
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t *q = ring + s * S::kStageBytes;
          const uint32_t at = tmem_base + lane_base + S::kACol0 + cs * S::kASlotCols;
#pragma unroll
          for (int op = 0; op < S::kWOps; ++op) {
            uint32_t v[32];
            widen_column(q + op * S::kQOpBytes, m, v);
            tmem_st32(at + op * 32, v);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(conv0 + 8 * cs);
        }
        if (++s == S::kStages) {
          s = 0;
          ph ^= 1;
        }
        if (++cs == S::kASlots) {
          cs = 0;
          cph ^= 1;
        }
      }
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
// Host side
// ---------------------------------------------------------------------------
// 2-D map over A [rows, K] (K contiguous), box 64 x 128, 128-byte swizzle.
bool make_map_a(CUtensorMap *m, const void *A, int rows, int K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)BM};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(A), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over rows [rows, K] with a box of `box_rows` rows.
bool make_map_rows(CUtensorMap *m, const void *A, int rows, int K, int box_rows) {
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

// 3-D map over B [G, K, N] (N contiguous), box 64 (N) x 64 (K) x 1, 128-byte swizzle.
bool make_map_b(CUtensorMap *m, const void *B, int G, int K, int N) {
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

// 3-D map over e4m3 codes Q [G, N, K] (one byte each, K contiguous: the
// transposed weights), box 64 (K) x box_n (N) x 1, 64-byte swizzle (the
// converters read one column's 64 codes per thread without bank conflicts).
bool make_map_codes(CUtensorMap *m, const void *Q, int G, int N, int K, int box_n) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)N, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)K, (cuuint64_t)N * K};
  cuuint32_t box[3] = {(cuuint32_t)BK, (cuuint32_t)box_n, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(Q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The single engine on e4m3 weights with per-column scales.
template <bool SWIGLU, int SPANS>
cudaError_t launch_q8(int rows_cap, int K, int N, int G, const int32_t *offsets, int fixed_rows,
                      const void *A, const void *B1, const void *B3, const float *s1,
                      const float *s3, void *out, uint32_t *err, cudaStream_t s,
                      RowWeights rw = RowWeights()) {
  using S = Shape<SWIGLU, SPANS, true>;
  CUtensorMap ma, mb1, mb3;
  if (!make_map_a(&ma, A, rows_cap, K) || !make_map_codes(&mb1, B1, G, N, K, S::BN) ||
      !make_map_codes(&mb3, SWIGLU ? B3 : B1, G, N, K, S::BN))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm<SWIGLU, SPANS, true>,
                                    S::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  Params p{offsets, G, fixed_rows, rows_cap, K, N, out, nullptr, nullptr, 1, err};
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.row_w = rw.w;
  p.w_row_src = rw.row_src;
  p.scale1 = s1;
  p.scale3 = SWIGLU ? s3 : nullptr;
  const long long max_tiles = (long long)((rows_cap + BM - 1) / BM + (offsets ? G : 0)) *
                              ((N + S::BN - 1) / S::BN);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  launch_k(k_grouped_gemm<SWIGLU, SPANS, true>, grid, S::kCtaThreads, smem, s, ma, mb1, mb3, p);
  return cudaGetLastError();
}

template <bool SWIGLU, int SPANS>
cudaError_t launch(int rows_cap, int K, int N, int G, const int32_t *offsets, int fixed_rows,
                   const void *A, const void *B1, const void *B3, void *out, const float *bias,
                   uint32_t *err, cudaStream_t s, const int32_t *row_src = nullptr,
                   int k_max = 1, int a_rows = 0, RowWeights rw = RowWeights(),
                   int8_t *yexp = nullptr) {
  using S = Shape<SWIGLU, SPANS>;
  CUtensorMap ma, mb1, mb3;
  const bool map_ok = row_src ? make_map_rows(&ma, A, a_rows, K, 1) : make_map_a(&ma, A, rows_cap, K);
  if (!map_ok || !make_map_b(&mb1, B1, G, K, N) ||
      !make_map_b(&mb3, SWIGLU ? B3 : B1, G, K, N))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm<SWIGLU, SPANS>,
                                    S::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  Params p{offsets, G, fixed_rows, rows_cap, K, N, out, bias, row_src, k_max, err};
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.row_w = rw.w;
  p.w_row_src = rw.row_src;
  p.yexp = yexp;
  p.nblk = (N + 31) / 32;
  p.l2_hints = l2_hints_enabled();
  // never more CTAs than tiles can exist (a group holds at most rows_cap rows)
  const long long max_tiles = (long long)((rows_cap + BM - 1) / BM + (offsets ? G : 0)) *
                              ((N + S::BN - 1) / S::BN);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  launch_k(k_grouped_gemm<SWIGLU, SPANS>, grid, kThreads, smem, s, ma, mb1, mb3, p);
  return cudaGetLastError();
}

template <bool SWIGLU, int KPS>
cudaError_t launch_pair_kps(int rows_cap, int K, int N, int G, const int32_t *offsets,
                            int fixed_rows, const void *A, const void *B1, const void *B3,
                            void *out, uint32_t *err, cudaStream_t s, RowWeights rw,
                            int8_t *yexp, const float *bias) {
  using S = Shape2<SWIGLU, KPS>;
  CUtensorMap ma, mb1, mb3;
  if (!make_map_a(&ma, A, rows_cap, K) || !make_map_b(&mb1, B1, G, K, N) ||
      !make_map_b(&mb3, SWIGLU ? B3 : B1, G, K, N))
    return cudaErrorInvalidValue;
  // group tables: row offsets, heavy and light tile starts
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 3 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_pair<SWIGLU, KPS>,
                                    S::kSmemFixed + sizeof(int32_t) * 3 * (kMaxGroups + 1)))
    return e;
  Params p{offsets, G, fixed_rows, rows_cap, K, N, out, bias, nullptr, 1, err};
  p.row_w = rw.w;
  p.w_row_src = rw.row_src;
  p.yexp = yexp;
  p.nblk = (N + 31) / 32;
  p.l2_hints = l2_hints_enabled();
  // Swap-AB pair tiles for groups under 256 rows by default (MOE_PAIR_SWAP=0:
  // none; =2: every group's partial last chunk too).  Alternated call by
  // call, the light list made the GPT-OSS- and DeepSeek-V3-shaped layers
  // faster, while swapping the large remainders of big groups made the
  // Qwen3- and Mixtral-shaped ones slower (their plain-output swap epilogue
  // takes twice as long as a row-major one).
  const char *ps = getenv("MOE_PAIR_SWAP");
  p.pair_swap = (ps && ps[0] == '0') ? 0 : ((ps && ps[0] == '2') ? 2 : 1);
  // the light list's largest group (MOE_PAIR_SWAP_ROWS, 1..255)
  const char *sr = getenv("MOE_PAIR_SWAP_ROWS");
  const int swap_rows = sr ? atoi(sr) : kPairSwapRows;
  p.swap_rows = swap_rows < 1 ? 1 : (swap_rows > BM2 - 1 ? BM2 - 1 : swap_rows);
  CUtensorMap mx32, mx8;
  if (!make_map_rows(&mx32, A, rows_cap, K, 32) || !make_map_rows(&mx8, A, rows_cap, K, 8))
    return cudaErrorInvalidValue;
  const long long max_tiles = (long long)((rows_cap + BM2 - 1) / BM2 + (offsets ? G : 0)) *
                              ((N + S::BN - 1) / S::BN);
  long long pairs = sms / 2;
  if (max_tiles < pairs) pairs = max_tiles < 1 ? 1 : max_tiles;
  launch_k(k_grouped_gemm_pair<SWIGLU, KPS>, (int)(2 * pairs), kThreads, smem, s, ma, mb1, mb3,
           mx32, mx8, p);
  return cudaGetLastError();
}

// Two k-blocks per ring stage for long K (at least 32 k-blocks), one for
// short K.  Alternated call by call on one B200, two per stage made the
// Mixtral-shaped layer 3% faster (up and down), the DeepSeek-V3-shaped
// prefill 3-5% and the Qwen3-shaped up projection (K = 2048) 2.6%, while the
// short-K down projections (K = 720-768, 12 k-blocks) lost 3.6% with half
// as many stages.  MOE_PAIR_KPS=1|2 forces the choice.
template <bool SWIGLU>
cudaError_t launch_pair(int rows_cap, int K, int N, int G, const int32_t *offsets,
                        int fixed_rows, const void *A, const void *B1, const void *B3, void *out,
                        uint32_t *err, cudaStream_t s, RowWeights rw = RowWeights(),
                        int8_t *yexp = nullptr, const float *bias = nullptr) {
  const char *ks = getenv("MOE_PAIR_KPS");
  const int num_kb = (K + BK - 1) / BK;
  const int kps = ks && (ks[0] == '1' || ks[0] == '2') ? ks[0] - '0' : (num_kb >= 32 ? 2 : 1);
  if (kps == 2)
    return launch_pair_kps<SWIGLU, 2>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3, out, err,
                                      s, rw, yexp, bias);
  return launch_pair_kps<SWIGLU, 1>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3, out, err, s,
                                    rw, yexp, bias);
}

template <bool SWIGLU>
cudaError_t launch_swap(int rows_cap, int K, int N, int G, const int32_t *offsets,
                        int fixed_rows, const void *A, const void *B1, const void *B3, void *out,
                        uint32_t *err, cudaStream_t s, const int32_t *row_src = nullptr,
                        int k_max = 1, int a_rows = 0, RowWeights rw = RowWeights()) {
  using S = ShapeSwap<SWIGLU>;
  CUtensorMap mx, mw1, mw3;
  const bool map_ok = row_src ? make_map_rows(&mx, A, a_rows, K, 1)
                              : make_map_rows(&mx, A, rows_cap, K, kRowBox);
  if (!map_ok || !make_map_b(&mw1, B1, G, K, N) ||
      !make_map_b(&mw3, SWIGLU ? B3 : B1, G, K, N))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_swap<SWIGLU>,
                                    S::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  Params p{offsets, G, fixed_rows, rows_cap, K, N, out, nullptr, row_src, k_max, err};
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.row_w = rw.w;
  p.w_row_src = rw.row_src;
  const long long max_tiles = (long long)((rows_cap + S::kMaxRows - 1) / S::kMaxRows +
                                          (offsets ? G : 0)) *
                              ((N + S::kCols - 1) / S::kCols);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  launch_k(k_grouped_gemm_swap<SWIGLU>, grid, kThreads, smem, s, mx, mw1, mw3, p);
  return cudaGetLastError();
}

// The swap-AB engine on e4m3 weights with per-column scales.
template <bool SWIGLU>
cudaError_t launch_swap_q8(int rows_cap, int K, int N, int G, const int32_t *offsets,
                           int fixed_rows, const void *A, const void *B1, const void *B3,
                           const float *s1, const float *s3, void *out, uint32_t *err,
                           cudaStream_t s, RowWeights rw = RowWeights()) {
  using S = ShapeSwap<SWIGLU, true>;
  CUtensorMap mx, mw1, mw3;
  if (!make_map_rows(&mx, A, rows_cap, K, kRowBox) ||
      !make_map_codes(&mw1, B1, G, N, K, S::kCols) ||
      !make_map_codes(&mw3, SWIGLU ? B3 : B1, G, N, K, S::kCols))
    return cudaErrorInvalidValue;
  const size_t smem = S::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(G + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm_swap<SWIGLU, true>,
                                    S::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  Params p{offsets, G, fixed_rows, rows_cap, K, N, out, nullptr, nullptr, 1, err};
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.row_w = rw.w;
  p.w_row_src = rw.row_src;
  p.scale1 = s1;
  p.scale3 = SWIGLU ? s3 : nullptr;
  const long long max_tiles = (long long)((rows_cap + S::kMaxRows - 1) / S::kMaxRows +
                                          (offsets ? G : 0)) *
                              ((N + S::kTileCols - 1) / S::kTileCols);
  const int grid = (int)(max_tiles < sms ? (max_tiles < 1 ? 1 : max_tiles) : sms);
  launch_k(k_grouped_gemm_swap<SWIGLU, true>, grid, S::kCtaThreads, smem, s, mx, mw1, mw3, p);
  return cudaGetLastError();
}

}  // namespace tc

// Engines, all correct for every shape (the tests run each):
//   single  one CTA per 128-row tile; up projection 128 columns of gate and of
//           up (N=256 MMA), down projection 256 columns;
//   narrow  the same with 64-column up-projection tiles (twice the tiles);
//   pair    CTA pairs on 256-row tiles (tcgen05 cta_group::2);
//   swap    weights as the M operand, rows in steps of 16 (swap-AB);
//   mixed   routed groups only: each group's full 128-row chunks as single
//           tiles and its remainder as a swap-AB tile, in one launch
//           (grouped_gemm_mixed.cu).
// Defaults, from B200 measurements with the engines alternated call by call
// in one process (whole layers, the same box):
//   - decode-sized groups (at most 32 rows per group on average): swap-AB for
//     the up projection, which loads only the valid rows (Mixtral-shaped
//     decode: 0.298 vs 0.320 ms single-CTA), single-CTA for the down
//     projection (CTA pairs: 0.171 vs 0.146 ms);
//   - routed groups of at most 256 rows on average (ragged layers: many
//     small experts next to a few large ones), both projections: mixed tiles
//     (each group's full 128-row chunks single-CTA, its remainder swap-AB,
//     heavy and light tiles interleaved in the deal).  Alternated call by
//     call on two boxes: GPT-OSS-shaped sub-experts 2.41 vs 2.73 ms (pairs),
//     DeepSeek-V3-shaped prefill 7.34 vs 8.06 ms; a light tile mostly streams
//     its group's weights, and a single CTA keeps 128 KB of them in flight
//     where a CTA of a pair keeps 96 KB;
//   - every other shape, both projections: CTA pairs.  Sharing each weight
//     tile between two SMs halves the weight bytes each SM streams and cuts
//     the shared-memory and L2 traffic per FLOP by a third, which under the
//     1 kW power cap keeps the clock up: Mixtral-shaped prefill 4.36 vs 7.47
//     ms (single CTA), Qwen3-shaped 1.35 vs 1.64 ms (mixed 1.72; its 2048-wide
//     down projection 0.39 vs 0.46 ms single).  A pair's partial last
//     256-row chunk can run swap-AB (MOE_PAIR_SWAP=1: weights as M, the
//     chunk's rows as N): the tensor pipe then does far less padding work
//     (ncu, GPT-OSS-shaped up projection: 74% → 28% tensor-active), but no
//     layer measured faster (Qwen3-shaped: 1.52 vs 1.46 ms), so it is off.
// MOE_GEMM_ENGINE=single|narrow|pair|swap|mixed selects one engine for every
// GEMM (mixed: for routed groups; a single group of rows runs single-CTA).
enum class Engine { kSingle, kNarrow, kPair, kSwap, kMixed };

static Engine pick_engine(bool swiglu, int rows_cap, int G, const int32_t *offsets,
                          int fixed_rows, int N) {
  const char *env = getenv("MOE_GEMM_ENGINE");
  if (env && env[0] == 's' && env[1] == 'i') return Engine::kSingle;
  if (env && env[0] == 'n') return Engine::kNarrow;
  if (env && env[0] == 'p') return Engine::kPair;
  if (env && env[0] == 's' && env[1] == 'w') return Engine::kSwap;
  if (env && env[0] == 'm') return offsets ? Engine::kMixed : Engine::kSingle;
  const long long mean_rows = offsets ? (long long)rows_cap / G : fixed_rows;
  if (mean_rows <= 32) return swiglu ? Engine::kSwap : Engine::kSingle;
  return Engine::kPair;
}

bool grouped_gemm_can_gather(bool swiglu, int rows_cap, int G, const int32_t *offsets,
                             int fixed_rows) {
  if (!swiglu) return false;
  const Engine e = pick_engine(swiglu, rows_cap, G, offsets, fixed_rows, 0);
  return e == Engine::kSingle || e == Engine::kNarrow || e == Engine::kSwap ||
         e == Engine::kMixed;
}

bool grouped_gemm_y16_out(int rows_cap, int G, const int32_t *offsets, int fixed_rows, int N) {
  return pick_engine(false, rows_cap, G, offsets, fixed_rows, N) != Engine::kSwap;
}

cudaError_t launch_grouped_gemm_bf16(bool swiglu, int rows_cap, int K, int N, int G,
                                     const int32_t *offsets, int fixed_rows, const void *A,
                                     const void *B1, const void *B3, void *out, uint32_t *err,
                                     cudaStream_t s, const int32_t *row_src, int k_max,
                                     int a_rows, const float *row_w,
                                     const int32_t *w_row_src, int8_t *yexp) {
  if (G <= 0 || G > tc::kMaxGroups) return cudaErrorInvalidValue;
  if (rows_cap == 0) return cudaSuccess;
  const Engine e = pick_engine(swiglu, rows_cap, G, offsets, fixed_rows, N);
  if (row_src && (!swiglu || e == Engine::kPair)) return cudaErrorInvalidValue;
  if (yexp && (swiglu || e == Engine::kSwap)) return cudaErrorInvalidValue;
  if (row_w && swiglu) return cudaErrorInvalidValue;  // gate weights: the down projection only
  tc::RowWeights rw;
  rw.w = row_w;
  rw.row_src = w_row_src;
  switch (e) {
    case Engine::kMixed:
      return launch_grouped_gemm_mixed(swiglu, rows_cap, K, N, G, offsets, A, B1, B3, out, err,
                                       s, row_w, w_row_src, yexp, row_src, k_max, a_rows);
    case Engine::kPair:
      return swiglu ? tc::launch_pair<true>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                            out, err, s)
                    : tc::launch_pair<false>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                             out, err, s, rw, yexp);
    case Engine::kSwap:
      return swiglu ? tc::launch_swap<true>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                            out, err, s, row_src, k_max, a_rows)
                    : tc::launch_swap<false>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                             out, err, s, nullptr, 1, 0, rw);
    case Engine::kNarrow:
      if (swiglu)
        return tc::launch<true, 1>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3, out,
                                   nullptr, err, s, row_src, k_max, a_rows);
      [[fallthrough]];
    default:
      return swiglu ? tc::launch<true, 2>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                          out, nullptr, err, s, row_src, k_max, a_rows)
                    : tc::launch<false, 4>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                           out, nullptr, err, s, nullptr, 1, 0, rw, yexp);
  }
}

cudaError_t launch_grouped_gemm_fp8(bool swiglu, int rows_cap, int K, int N, int G,
                                    const int32_t *offsets, int fixed_rows, const void *A,
                                    const void *B1, const void *B3, const float *s1,
                                    const float *s3, void *out, uint32_t *err, cudaStream_t s,
                                    const float *row_w, const int32_t *w_row_src) {
  if (rows_cap <= 0) return cudaSuccess;
  if (G <= 0 || G > tc::kMaxGroups || N % 16 != 0) return cudaErrorInvalidValue;
  if (row_w && swiglu) return cudaErrorInvalidValue;  // gate weights: the down projection only
  tc::RowWeights rw;
  rw.w = row_w;
  rw.row_src = w_row_src;
  // fp8 weights: swap-AB for decode-sized groups (at most 32 rows per group
  // on average, as for bf16), the single engine otherwise;
  // MOE_GEMM_ENGINE=single|narrow|swap forces one (narrow: 64-column up
  // projection tiles on the single engine)
  const char *env = getenv("MOE_GEMM_ENGINE");
  const long long mean_rows = offsets ? (long long)rows_cap / G : fixed_rows;
  const bool swap = env ? (env[0] == 's' && env[1] == 'w') : mean_rows <= 32;
  if (swap)
    return swiglu ? tc::launch_swap_q8<true>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3,
                                             s1, s3, out, err, s)
                  : tc::launch_swap_q8<false>(rows_cap, K, N, G, offsets, fixed_rows, A, B1,
                                              B1, s1, nullptr, out, err, s, rw);
  if (swiglu && env && env[0] == 'n')
    return tc::launch_q8<true, 1>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3, s1, s3,
                                  out, err, s);
  return swiglu ? tc::launch_q8<true, 2>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B3, s1,
                                         s3, out, err, s)
                : tc::launch_q8<false, 4>(rows_cap, K, N, G, offsets, fixed_rows, A, B1, B1, s1,
                                          nullptr, out, err, s, rw);
}

namespace tc {

// Split-K launch of the single engine without SwiGLU (fp32 output): S groups
// of the same T rows, group s at K offset s*k_split (its tiles read past K as
// zeros).  The A map holds exactly T rows, so a tile's rows past T read as
// zeros too.
template <int SPANS, bool FP8W>
cudaError_t launch_split(int T, int K, int N, int S, int k_split, const void *A, const void *B,
                         const float *scale, float *out, int32_t *clear, uint32_t *err,
                         cudaStream_t s) {
  using Sh = Shape<false, SPANS, FP8W>;
  if (T <= 0 || S < 1 || S > kMaxGroups || k_split <= 0 || k_split % BK)
    return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!make_map_a(&ma, A, T, K)) return cudaErrorInvalidValue;
  if (FP8W ? !make_map_codes(&mb, B, 1, N, K, Sh::BN) : !make_map_b(&mb, B, 1, K, N))
    return cudaErrorInvalidValue;
  const size_t smem = Sh::kSmemFixed + sizeof(int32_t) * 2 * (size_t)(S + 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = set_smem_once(attr_set, k_grouped_gemm<false, SPANS, FP8W>,
                                    Sh::kSmemFixed + sizeof(int32_t) * 2 * (kMaxGroups + 1)))
    return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  Params p{nullptr, S, T, S * T, K, N, out, nullptr, nullptr, 1, err, k_split, clear};
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.scale1 = scale;
  const long long tiles = (long long)S * ((T + BM - 1) / BM) * ((N + Sh::BN - 1) / Sh::BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  launch_k(k_grouped_gemm<false, SPANS, FP8W>, grid, Sh::kCtaThreads, smem, s, ma, mb, mb, p);
  return cudaGetLastError();
}

}  // namespace tc

cudaError_t launch_router_split(int T, int d, int E, int S, int k_split, const void *x,
                                const void *Wr, float *partials, int32_t *clear, uint32_t *err,
                                cudaStream_t s) {
  return tc::launch_split<1, false>(T, d, E, S, k_split, x, Wr, nullptr, partials, clear, err, s);
}

// 256-column output tiles (the down projection's single-engine shapes).
cudaError_t launch_gemm_split(bool fp8, int T, int K, int N, int S, const void *A, const void *B,
                              const float *scale, float *out, uint32_t *err, cudaStream_t s) {
  if (S < 1 || K % (S * tc::BK)) return cudaErrorInvalidValue;
  if (fp8) {
    if (N % 16) return cudaErrorInvalidValue;
    return tc::launch_split<4, true>(T, K, N, S, K / S, A, B, scale, out, nullptr, err, s);
  }
  return tc::launch_split<4, false>(T, K, N, S, K / S, A, B, nullptr, out, nullptr, err, s);
}

cudaError_t launch_router_tc(int T, int d, int E, const void *x, const void *Wr,
                             const float *bias, float *logits, uint32_t *err, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  // One group of T rows; B = Wr viewed as [1, d, E].  A tile is 128 rows by
  // 64 x spans columns.  Wide tiles read a block of x once for all experts,
  // narrow ones give more CTAs when T is short: take the width with the
  // fewest waves x spans (the time of the busiest CTA), ties to the widest.
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Many experts and a long batch: CTA pairs (256 x 256 tiles, half the
  // operand bytes per SM of a single-CTA tile), as for the expert GEMMs.
  // MOE_ROUTER_PAIR=0/1 forces the choice.
  const char *rp = getenv("MOE_ROUTER_PAIR");
  const bool pair = rp ? rp[0] == '1' : (E >= 512 && T >= 2048);
  if (pair)
    return tc::launch_pair<false>(T, d, E, 1, nullptr, T, x, Wr, Wr, logits, err, s,
                                  tc::RowWeights(), nullptr, bias);
  const long long row_tiles = (T + tc::BM - 1) / tc::BM;
  int spans = 1;
  long long best = -1;
  for (int sp = 4; sp >= 1; sp /= 2) {
    if (sp > 1 && E <= 64 * sp / 2) continue;  // wider than E needs
    const long long tiles = row_tiles * ((E + 64 * sp - 1) / (64 * sp));
    const long long cost = (tiles + sms - 1) / sms * sp;
    if (best < 0 || cost < best) {
      best = cost;
      spans = sp;
    }
  }
  if (spans == 1)
    return tc::launch<false, 1>(T, d, E, 1, nullptr, T, x, Wr, Wr, logits, bias, err, s);
  if (spans == 2)
    return tc::launch<false, 2>(T, d, E, 1, nullptr, T, x, Wr, Wr, logits, bias, err, s);
  return tc::launch<false, 4>(T, d, E, 1, nullptr, T, x, Wr, Wr, logits, bias, err, s);
}

}  // namespace moe
