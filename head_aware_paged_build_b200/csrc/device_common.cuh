// Device-side helpers of libsegpaged.so: pool page layouts, mbarriers, bulk
// copies, warp-level MMA and the status word.  All inline PTX here is written
// from the PTX ISA (sm_90 / sm_100a instructions).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sp_internal.h"

namespace sp {

// --------------------------------------------------------------------------
// Pool page layouts.
//
// bf16 (page size 64): a K page is the tcgen05 "K-major, 128-byte swizzle"
// operand layout of a [P tokens x D dims] tile: D/64 column blocks of
// [P rows x 128 B]; within a row the 16-byte chunk c is stored at c ^ (row & 7).
// A V page is stored transposed, [D rows x P tokens] with the same swizzle, so
// that it is the K-major operand of O += P V.  Both are exactly what the
// tensor cores and ldmatrix read, so a page moves with one plain bulk copy.
// fp32: K page row-major [P][D], V page transposed [D][P], no swizzle.
// --------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t kpage_chunk_offset_bf16(int t, int c16, int P) {
  // c16: 16-byte chunk index inside the token's D*2-byte row
  return int64_t(c16 >> 3) * (P * 128) + t * 128 + (((c16 & 7) ^ (t & 7)) << 4);
}
__host__ __device__ __forceinline__ int64_t vpage_chunk_offset_bf16(int i, int c16) {
  // row i (dimension), chunk c16 holds tokens 8*c16 .. 8*c16+7 (P = 64)
  return int64_t(i) * 128 + ((c16 ^ (i & 7)) << 4);
}
// E4M3 pages (P = 64): K page [64 tokens][D] codes, V page [D][64 positions]
// codes.  A byte lives at its linear address with the 16-byte chunks of each
// 128-byte line XOR-swizzled by the line index, in the pattern that keeps the
// decode's shared-memory reads free of bank conflicts:
//  K: each half-warp reads 32 contiguous bytes of 4 consecutive token rows
//     (64-bit loads): chunks XOR 2 * (line mod 4) give the 4 rows distinct
//     32-byte bank groups for D = 64 and 128;
//  V: a warp reads 16 bytes of 8 consecutive dimension rows (32-bit loads):
//     chunks XOR (line mod 8) give the 8 rows distinct 16-byte bank groups.
__host__ __device__ __forceinline__ int fp8_kpage_offset(int t, int col, int D) {
  const int a = t * D + col;
  const int line = a >> 7;
  return (line << 7) | ((((a >> 4) & 7) ^ ((line & 3) << 1)) << 4) | (a & 15);
}
__host__ __device__ __forceinline__ int fp8_vpage_offset(int i, int pos) {
  const int a = i * 64 + pos;
  const int line = a >> 7;
  return (line << 7) | ((((a >> 4) & 7) ^ (line & 7)) << 4) | (a & 15);
}
// Position of token u (0 .. 63) inside a V row of an E4M3 page.  Within each
// group of 16 tokens, tokens 2i, 2i+1, 8+2i, 9+2i sit at positions 4i .. 4i+3:
// exactly the four values one lane's mma.sync B fragment (two f16x2
// registers) needs, so one 32-bit load feeds both registers.
__host__ __device__ __forceinline__ int fp8_vtok_pos(int u) {
  const int w = u & 15;
  return (u & ~15) + ((w & 7) >> 1) * 4 + ((w >> 3) << 1) + (w & 1);
}
__host__ __device__ __forceinline__ int fp8_vpos_tok(int p) {  // inverse of fp8_vtok_pos
  const int w = p & 15;
  return (p & ~15) + ((w >> 1) & 1) * 8 + (w >> 2) * 2 + (w & 1);
}

// --------------------------------------------------------------------------
// Status word (workspace word 0).  The first error sticks.
// --------------------------------------------------------------------------
__device__ __forceinline__ void record_error(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// --------------------------------------------------------------------------
// mbarrier
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: ~2 s of wall time, then give up (returns false).  The fast
// path is one try_wait; the slow path re-checks the clock every 256 tries.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0) {
      if (global_timer_ns() - t0 > kWaitLimitNs) return false;
      __nanosleep(64);
    }
  }
}

// Order this thread's earlier generic-proxy global writes before later
// async-proxy accesses (bulk copies) of the same memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// --------------------------------------------------------------------------
// Bulk (non-tensor) asynchronous copy global -> shared, completing on an mbarrier.
// Both addresses 16-byte aligned, size a multiple of 16.
// --------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// --------------------------------------------------------------------------
// Warp-level MMA (decode).  m16n8k16, bf16 inputs, fp32 accumulate.
// --------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values to two FP8 E4M3 codes (round to nearest even, saturating);
// `lo` lands in the low byte.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two E4M3 codes (low byte first) to two fp16 values (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(codes));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__uint_as_float(x & 0xffff0000u)), "f"(__uint_as_float(x << 16)));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Named barrier `id` over `count` threads (whole warps) that also ANDs a
// predicate across them: every participant gets the same answer.
__device__ __forceinline__ bool bar_red_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// 2^x on the SFU (ex2.approx, flush-to-zero); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) and 3-input max ----------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair, on the FMA and integer pipes instead of the SFU.
// x = n + f with n = round(x) (adding 1.5 * 2^23 rounds to an integer held in
// the low mantissa bits) and f in [-1/2, 1/2]; 2^f is a cubic fitted by
// relative-error least squares on 64 Chebyshev nodes of [-1/2, 1/2]
// (csrc/exp2_cubic_fit.py; maximum relative error 7.74e-5, 7.8e-5 with the
// fp32 evaluation, below bf16's 2^-8 rounding of P); n is added to the
// exponent field.  x is clamped at -126 so the exponent never wraps: lanes
// below that (masked, -inf) give ~1e-38, which vanishes next to the row's
// largest weight (>= 1) in every fp32 sum.
__device__ __forceinline__ void exp2_poly_pair(uint64_t x2, float& e0, float& e1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x0 = fmaxf(x0, -126.f), x1 = fmaxf(x1, -126.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t t = f2_add(xc, f2_pack(kRound, kRound));
  const uint64_t j = f2_add(t, f2_pack(-kRound, -kRound));
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), xc);
  uint64_t p = f2_fma(f2_pack(0.05508868396282196f, 0.05508868396282196f), f,
                      f2_pack(0.24260404706001282f, 0.24260404706001282f));
  p = f2_fma(p, f, f2_pack(0.6932762265205383f, 0.6932762265205383f));
  p = f2_fma(p, f, f2_pack(0.9999289512634277f, 0.9999289512634277f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  e0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  e1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// Visibility of key position `a` for query position `p` of a head:
// causal, and for a local head inside the sink or the recent window.
__device__ __forceinline__ bool sees(int local, int sink, int window, int p, int a) {
  return a <= p && (!local || a < sink || a > p - window);
}

}  // namespace sp
