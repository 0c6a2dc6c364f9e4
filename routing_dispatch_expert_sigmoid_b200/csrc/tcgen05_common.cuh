// Shared pieces of the tcgen05 GEMM kernels of libmoe.so: tile constants,
// inline PTX wrappers (mbarriers, bounded waits, TMA loads, tensor-memory
// allocation and loads, tcgen05.mma and its descriptors) and the host-side
// helpers every launcher uses (the tensor-map encoder, the wait limit, the
// per-device shared-memory attribute).  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdlib.h>

#include <atomic>

#include "moe_internal.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;          // rows per tile (UMMA M, one TMEM lane per row)
constexpr int BK = 64;           // K per stage: one 128-byte swizzle span of bf16
constexpr int kThreads = 192;    // 6 warps
constexpr int kMaxGroups = 1024;
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

struct Ctl {
  volatile int *abort;
  uint32_t *err;
  uint64_t limit_ns;  // how long one pipeline wait may take before the CTA stops
};

// Wait until the phase of parity `parity` of barrier `bar` has completed.
// Returns false (and stops the CTA) on time-out or when another role stopped.
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, const Ctl &c) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort) return false;
    if (global_timer() - t0 > c.limit_ns) {
      *c.abort = 1;
      raise_error(c.err, kErrWait);
      return false;
    }
  }
}

// Wait without honouring the stop flag (used to drain work in flight); always
// the long limit, so that every copy and MMA already issued lands before the
// CTA frees its tensor memory and exits.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, uint32_t *err) {
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kWaitLimitNs) {
      raise_error(err, kErrWait);
      return;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
// L2 eviction policies for TMA loads: operands that later tiles read again
// (the rows of A, reused by every column tile of a group) are kept, operands
// that stream through once (expert weights, shared only by the CTAs that run
// a group's row tiles at the same time) go first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar, int c0, int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap *map,
                                                 uint32_t bar, int c0, int c1, int c2,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(pol)
      : "memory");
}
// Whether the GEMMs give their TMA loads L2 eviction hints: MOE_L2_HINTS=1
// turns them on (read at every launch).  Off by default: on B200, alternated
// call by call, the hints made the Mixtral-shaped prefill layer 6% slower
// (4.63 vs 4.36 ms) and the Qwen3- and GPT-OSS-shaped layers 2-3% slower;
// streamed weights marked evict-first leave L2 before the other CTAs of the
// same row tiles read them.
// MOE_L2_HINTS: 0 none (default); 1 rows evict-last and weights
// evict-first; the CTA-pair engine also takes 2 (rows evict-last only) and 3
// (weights evict-last only).
inline int l2_hints_enabled() {
  const char *env = getenv("MOE_L2_HINTS");
  return (env && env[0] >= '1' && env[0] <= '3') ? env[0] - '0' : 0;
}

// Four rows (r0..r3) of 64 columns starting at column c0 into 4 consecutive
// 128-byte rows of shared memory (the map's box is one row high).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3),
      "r"(bar)
      : "memory");
}
// Bring a box of a 3-D tensor into L2 ahead of its TMA load: no shared
// memory, no completion to wait for.  A stream of weights that each SM reads
// once is paced by the bytes it keeps in flight; prefetches add to them.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap *map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                     uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
// The same MMA with A read from tensor memory (a_tmem: lane = row of A,
// 32-bit column c = K elements 2c, 2c+1).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive 32-bit columns of this warp's 32 lanes; completion is
// waited for with tmem_wait_st.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Load 32 consecutive fp32 columns of this thread's TMEM lane (and wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Two 32-column loads of this thread's lane (at ta into v, at tb into u) with
// a single wait for both.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, float *v, float *u) {
  uint32_t a[32], b[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __uint_as_float(a[i]);
    u[i] = __uint_as_float(b[i]);
  }
}
// Sum of two 32-column loads `off` columns apart (partial sums of one output
// kept in two accumulators).
__device__ __forceinline__ void tmem_ld32_sum2(uint32_t taddr, uint32_t off, float *v) {
  float w[32];
  tmem_ld32x2(taddr, taddr + off, v, w);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] += w[i];
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // version
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A
// K-major, B MN-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t instr_desc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// The same with B K-major too (the widened fp8 weight tiles).
__host__ __device__ constexpr uint32_t instr_desc_kk(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Compact expert outputs ("y16"): the down projection's fp32 rows stored as
// fp16 values with one power-of-two scale per 32-column block of a row,
// value = y16 * 2^e.  For a block whose largest magnitude is M * 2^E (M in
// [1, 2)), e = E - 14, so the scaled block lies within 2^15 and fp16 keeps a
// relative error of at most 2^-11 on every value down to 2^-29 of the
// block's largest (below that, an absolute error under 2^-40 of it).  Half
// the bytes of fp32 rows; the combine undoes the scale.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int y16_exponent(float m) {
  if (!(m > 0.0f) || !(m <= 3.4028234e38f)) return 0;  // zero or non-finite block
  // E from the exponent field: exact for normal m; a subnormal m reads as
  // E = -127 and, like its true exponent, ends at the clamp below
  const int e = (((__float_as_int(m) >> 23) & 0xFF) - 127) - 14;
  return e < -120 ? -120 : (e > 120 ? 120 : e);
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// Largest magnitude of 32 values as a tree of maxima (depth 5 instead of a
// chain of 32 dependent steps).  A NaN is skipped, like fmaxf does.
__device__ __forceinline__ float absmax32(const float (&v)[32]) {
  float m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = fmaxf(fabsf(v[i]), fabsf(v[i + 16]));
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

// One warp, lane = row: its row's 32 values v (columns col .. col+31 of rows
// row0 + lane) into y16 rows of N columns and their block exponents
// (nblk = ceil(N / 32) per row), through the warp's staging buffer st (32
// rows of row_words words); rows from row_end on are not written.
__device__ __forceinline__ void store_y16_lane_rows(const float (&v)[32], uint32_t *st,
                                                    int row_words, int lane, int row0,
                                                    int row_end, int col, int N, void *out,
                                                    int8_t *yexp, int nblk) {
  const int e = y16_exponent(absmax32(v));
  const float inv = pow2f(-e);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h2 = __floats2half2_rn(v[q * 8 + 2 * i] * inv, v[q * 8 + 2 * i + 1] * inv);
      w[i] = *reinterpret_cast<uint32_t *>(&h2);
    }
    *reinterpret_cast<uint4 *>(st + lane * row_words + 4 * q) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (row0 + lane < row_end && col < N) yexp[(size_t)(row0 + lane) * nblk + col / 32] = (int8_t)e;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // 8 rows x 64 bytes per instruction
    const int r = i * 8 + (lane >> 2), q = lane & 3;
    const int grow = row0 + r, gcol = col + q * 8;
    const uint4 val = *reinterpret_cast<const uint4 *>(st + r * row_words + 4 * q);
    if (grow < row_end && gcol < N)
      *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + (size_t)grow * N + gcol) = val;
  }
}

// The same for two neighbouring 32-column blocks (v: columns col .., u:
// col + 32 ..; col a multiple of 64): both blocks of a row are staged as one
// 128-byte fp16 row, written by 8 lanes with 16-byte stores, 4 rows per
// instruction.  With yexp == nullptr the two exponents are returned in
// *e2 (block col/32 in the low byte) for the caller to store with others.
__device__ __forceinline__ void store_y16_lane_rows2(const float (&v)[32], const float (&u)[32],
                                                     uint32_t *st, int row_words, int lane,
                                                     int row0, int row_end, int col, int N,
                                                     void *out, int8_t *yexp, int nblk,
                                                     uint32_t *e2 = nullptr) {
  const int ev = y16_exponent(absmax32(v)), eu = y16_exponent(absmax32(u));
  const float iv = pow2f(-ev), iu = pow2f(-eu);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // packed scaling by the powers of two (exact)
      __half2 h = __float22half2_rn(
          __fmul2_rn(make_float2(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]), make_float2(iv, iv)));
      a[i] = *reinterpret_cast<uint32_t *>(&h);
      h = __float22half2_rn(
          __fmul2_rn(make_float2(u[q * 8 + 2 * i], u[q * 8 + 2 * i + 1]), make_float2(iu, iu)));
      b[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(st + lane * row_words + 4 * q) = make_uint4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<uint4 *>(st + lane * row_words + 16 + 4 * q) =
        make_uint4(b[0], b[1], b[2], b[3]);
  }
  if (!yexp) {
    *e2 = (uint32_t)(uint8_t)ev | ((uint32_t)(uint8_t)eu << 8);
  } else if (row0 + lane < row_end) {
    int8_t *ye = yexp + (size_t)(row0 + lane) * nblk + col / 32;
    if (col < N) ye[0] = (int8_t)ev;
    if (col + 32 < N) ye[1] = (int8_t)eu;
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // 4 rows x 128 bytes per instruction
    const int r = i * 4 + (lane >> 3), q = lane & 7;
    const int grow = row0 + r, gcol = col + q * 8;
    const uint4 val = *reinterpret_cast<const uint4 *>(st + r * row_words + 4 * q);
    if (grow < row_end && gcol < N)
      *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + (size_t)grow * N + gcol) = val;
  }
  __syncwarp();
}

// One warp, lane = column: v[j] is row row0 + j, column col0 + lane (col0 a
// multiple of 32, so the warp holds exactly one exponent block of each row).
// Rows j < nr into y16 rows and their block exponents: each row's largest
// magnitude is one warp reduction on the magnitudes' bit patterns (their
// order as unsigned integers is the order of the values; a NaN counts as 0,
// as fmaxf skips it); the fp16 values go through the staging buffer st (32
// rows of row_words words) and leave as whole 64-byte row segments.  wr:
// per-row factor source (row_w[w_row_src[row]]) or nullptr.
__device__ __forceinline__ void store_y16_lane_cols(float (&v)[32], uint32_t *st, int row_words,
                                                    int lane, int row0, int nr, int col0, int N,
                                                    void *out, int8_t *yexp, int nblk,
                                                    const float *row_w,
                                                    const int32_t *w_row_src) {
  if (row_w) {
    const float wl = lane < nr ? row_w[w_row_src[row0 + lane]] : 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= __shfl_sync(0xffffffffu, wl, j);
  }
  __half *sh = reinterpret_cast<__half *>(st);
  const int rh = 2 * row_words;  // halves per staged row
  int my_e = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float a = fabsf(v[j]);
    const uint32_t key = a != a ? 0u : __float_as_uint(a);
    const int e = y16_exponent(__uint_as_float(__reduce_max_sync(0xffffffffu, key)));
    if (lane == j) my_e = e;
    sh[j * rh + lane] = __float2half_rn(v[j] * pow2f(-e));
  }
  if (lane < nr && col0 < N) yexp[(size_t)(row0 + lane) * nblk + col0 / 32] = (int8_t)my_e;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // 8 rows x 64 bytes per instruction
    const int r = i * 8 + (lane >> 2), q = lane & 3;
    const int gcol = col0 + q * 8;
    const uint4 val = *reinterpret_cast<const uint4 *>(sh + r * rh + q * 8);
    if (r < nr && gcol < N)
      *reinterpret_cast<uint4 *>(static_cast<__half *>(out) + (size_t)(row0 + r) * N + gcol) = val;
  }
  __syncwarp();
}

// One warp, rows staged transposed (stg[j * row_words + c] = value of row j,
// column col0 + c): rows j < nr of rows row0 .. into y16 rows and their block
// exponents; 8 lanes per row, 4 columns each.  wr: per-row factor source
// (row_w[w_row_src[row]]) or nullptr.
__device__ __forceinline__ void store_y16_staged(const float *stg, int row_words, int lane,
                                                 int row0, int nr, int col0, int N, void *out,
                                                 int8_t *yexp, int nblk, const float *row_w,
                                                 const int32_t *w_row_src) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // 4 rows per step
    const int j = i * 4 + (lane >> 3), q = lane & 7;
    const int grow = row0 + j, gcol = col0 + q * 4;
    const bool live = j < nr;
    float4 f = *reinterpret_cast<const float4 *>(stg + j * row_words + 4 * q);
    if (live && row_w) {
      const float wr = row_w[w_row_src[grow]];
      f.x *= wr;
      f.y *= wr;
      f.z *= wr;
      f.w *= wr;
    }
    float m = fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w)));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    const int e = y16_exponent(m);
    const float inv = pow2f(-e);
    if (live && gcol < N) {
      __half2 lo = __floats2half2_rn(f.x * inv, f.y * inv);
      __half2 hi = __floats2half2_rn(f.z * inv, f.w * inv);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t *>(&lo);
      w.y = *reinterpret_cast<uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(static_cast<__half *>(out) + (size_t)grow * N + gcol) = w;
      if (q == 0) yexp[(size_t)grow * nblk + col0 / 32] = (int8_t)e;
    }
  }
}

// ---------------------------------------------------------------------------
// Host helpers
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

// Limit of one pipeline wait of the single-CTA and swap-AB engines, read at
// every launch: MOE_WAIT_LIMIT_NS when it holds a number of nanoseconds up to
// the default (a diagnostic knob: a tiny limit makes the waits run out, so
// the stop path can be exercised), else the default 4 s.
inline uint64_t pipeline_wait_limit_ns() {
  const char *env = getenv("MOE_WAIT_LIMIT_NS");
  if (!env || !*env) return kWaitLimitNs;
  char *end = nullptr;
  const unsigned long long v = strtoull(env, &end, 10);
  return (end && *end == '\0' && v <= kWaitLimitNs) ? (uint64_t)v : kWaitLimitNs;
}

// Raise a kernel's dynamic shared-memory limit once per device.  The flags are
// atomics: host threads that launch on the same device for the first time at
// once may both set the (same) attribute, without a data race.
template <typename Kernel>
cudaError_t set_smem_once(std::atomic<bool> (&done)[64], Kernel kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_release);
  return e;
}

}  // namespace tc
}  // namespace moe
