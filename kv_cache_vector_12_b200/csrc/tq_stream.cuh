// Device helpers shared by the kernels that stream the packed cache (decode
// and prefill attention): PTX wrappers for mbarriers, bulk copies and the
// mma.sync shapes they use, and the expansion of packed codes into tensor-core
// fragments by byte-permute lookups.  Internal to the library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier waits: 2 s

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One suspending test of phase `parity`: a thread whose phase is not complete
// sleeps until it completes or kSuspendNs pass, instead of spinning (a spinning
// producer would take issue slots from the consumer warps of its SM).
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier; false once 2 s have passed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) return false;
  }
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <bool ASigned, bool BSigned>
__device__ __forceinline__ void mma_i8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  if constexpr (ASigned && BSigned)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else if constexpr (ASigned && !BSigned)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else if constexpr (!ASigned && BSigned)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// x0, x1 as bf16 pairs hi + lo (x0 in the low halves): hi = bf16(x), lo =
// bf16(x - hi), so x - hi - lo is below 2^-16 |x|.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSqrtHalfPi = 1.2533141373155003f;  // sqrt(pi / 2), the QJL constant's numerator

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// 2^x with the hardware approximation (relative error ~2^-22; flushes
// subnormal results to zero, which only affects weights below 2^-126).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// ------------------------------------------------------- code expansion
// A selector holds four codes in the low three (or four) bits of the nibbles
// of its low 16 bits.  lookup() returns the low bytes and the high bytes of
// the four table entries (one byte per code).
template <int B>
__device__ __forceinline__ void lookup(const Lut &t, uint32_t sel, uint32_t &lo, uint32_t &hi) {
  if constexpr (B <= 3) {
    lo = prmt(t.lo[0], t.lo[1], sel);
    hi = prmt(t.hi[0], t.hi[1], sel);
  } else {
    const uint32_t s7 = sel & 0x7777u;
    // byte n of m is 0xFF when nibble n of sel has its top bit set
    const uint32_t m = prmt(sel << 4, sel, 0xD9C8u);
    const uint32_t l0 = prmt(t.lo[0], t.lo[1], s7), l1 = prmt(t.lo[2], t.lo[3], s7);
    const uint32_t h0 = prmt(t.hi[0], t.hi[1], s7), h1 = prmt(t.hi[2], t.hi[3], s7);
    lo = (l1 & m) | (l0 & ~m);
    hi = (h1 & m) | (h0 & ~m);
  }
}

// Spare-column codes of the 3-bit layout: bit k of each code is the top bit
// of the same nibble of word k.
__device__ __forceinline__ uint32_t spare3(uint32_t w0, uint32_t w1, uint32_t w2) {
  return ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
}

// Selector sigma (0..7) of the 32 K codes a thread owns for one token
// (the words of its 32-coordinate group).  Code order: see kperm on the host.
template <int B>
__device__ __forceinline__ uint32_t k_selector(const uint32_t (&w)[B], int sigma) {
  if constexpr (B == 3) {
    const int k = sigma >> 1;
    const uint32_t x = k < 3 ? (w[k < 3 ? k : 0] & 0x77777777u) : spare3(w[0], w[1], w[2]);
    return (sigma & 1) ? x >> 16 : x;
  } else if constexpr (B == 2) {
    const int wd = sigma >> 2, par = (sigma >> 1) & 1;
    const uint32_t x = (w[wd] >> (2 * par)) & 0x33333333u;
    return (sigma & 1) ? x >> 16 : x;
  } else {
    const uint32_t x = w[sigma >> 1];
    return (sigma & 1) ? x >> 16 : x;
  }
}

// fp16 pairs (token A, token B) for two coordinates from one V selector whose
// nibbles are [A.x, A.y, B.x, B.y].
template <int B>
__device__ __forceinline__ void v_pairs(const Lut &t, uint32_t sel, uint32_t &px, uint32_t &py) {
  uint32_t lo, hi;
  lookup<B>(t, sel, lo, hi);
  px = prmt(lo, hi, 0x6240u);
  py = prmt(lo, hi, 0x7351u);
}

// -------------------------------------------------------- shared layout
// One stage of TOK tokens of every plane of DH-dimensional vectors, packed
// back to back (every plane offset a multiple of 16 bytes for TOK a multiple
// of 8).
template <int BK, int BV, bool QJL, int TOK, int DH = D>
struct Stage {
  static constexpr int kc = 0;                           // K codes
  static constexpr int vc = kc + TOK * DH * BK / 8;      // V codes
  static constexpr int jb = vc + TOK * DH * BV / 8;      // QJL sign bits
  static constexpr int kn = jb + (QJL ? TOK * DH / 8 : 0);
  static constexpr int vn = kn + TOK * 2;
  static constexpr int jg = vn + TOK * 2;
  static constexpr int bytes = jg + (QJL ? TOK * 2 : 0);
};

}  // namespace
}  // namespace tq
