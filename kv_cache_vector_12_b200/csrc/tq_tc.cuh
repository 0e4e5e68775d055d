// Shared pieces of the tensor-core quantize kernels (sm_100a): PTX wrappers
// for mbarriers, TMA tile loads and tcgen05 (MMA, commit, tensor-memory
// loads), the exact code computation from the rotated coordinates against
// thresholds scaled by ||x|| ("ステップ1: PolarQuant", ai-accelerate.xyz
// TurboQuant explainer), its bit-packing into the cache layout, and the host
// construction of the 128-byte-swizzled tensor maps.  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_f32x2.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kTileRows = 128;
constexpr int kTileBytes = kTileRows * kHeadDim * 2;  // 32 KB: two 128x64 16-bit boxes
constexpr int kBoxBytes = kTileBytes / 2;
constexpr uint32_t kSuspendNs = 1000000;                 // longest sleep of one barrier test: 1 ms
constexpr unsigned long long kWaitNs = 2000000000ull;   // bounded barrier waits: 2 s

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void bar_init(uint32_t b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(n));
}
__device__ __forceinline__ void bar_expect_tx(uint32_t b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
}
// A suspending test: the thread sleeps until the phase completes or
// kSuspendNs pass, so waiting warps leave the issue slots to working ones.
__device__ __forceinline__ bool bar_try(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(ok)
               : "r"(b), "r"(parity), "r"(kSuspendNs)
               : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase `parity`; false once kWaitNs have passed.
__device__ __forceinline__ bool bar_wait(uint32_t b, uint32_t parity) {
  if (bar_try(b, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (bar_try(b, parity)) return true;
    if (global_ns() - t0 > kWaitNs) return false;
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (start address and offsets in 16-byte units).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 128, M = 128.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "l"(a), "l"(b), "r"(kInstrDesc), "r"(accumulate)
               : "memory");
}
// The same with the instruction descriptor as an argument (other N).
__device__ __forceinline__ void tc_mma_n(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
               : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 1 when a b + c > 0 (exact product and sum, one rounding), else 0 when the
// result rounds to at most 0; values in (0, 1) only for exact results below 1.
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float mul_sat(float a, float b) {
  float d;
  asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Per-row constants of the code computation.  A row whose stored fp16 norm is
// zero (||x|| <= 2^-25) is the zero vector (y = 0): sc = zc = 0.  Otherwise
// sc = 2^64 / ||x|| (at most 2^89), zc = 2^127, and nt_j = -t_j 2^64 for the
// positive unit thresholds t_j.  [|z| / ||x|| > t_j] is fma_sat(|z|, sc, nt_j):
// the exact value |z| sc - t_j 2^64 is either <= 0 or at least t_j 2^16 > 1 (a
// product of two floats differs from a float by at least 2^-48 of it unless
// equal), so the saturated result is exactly 0 or 1; the comparison differs
// from |z| > t_j ||x|| only by the rounding of 2^64 / ||x||.
//
// m = #{j : t_j < |z| / ||x||} is found by binary search over the sorted nt_j,
// one saturating test per level, the next level's threshold selected with
// fused multiply-adds by the bits found so far (sel = b D + base).  The
// differences D (below) are exact in fp32 for the codebooks in use, so every
// selection yields one of the nt_j exactly; the host checks this for each
// codebook before a context is created (threshold_search_exact).
//   3 bits (t0 < t1 < t2): b1 = [> t1]; b0 = [> (b1 ? t2 : t0)]; m = 2 b1 + b0.
//   4 bits (t0 .. t6):     b2 = [> t3]; b1 = [> (b2 ? t5 : t1)];
//                          b0 = [> t(4 b2 + 2 b1)]; m = 4 b2 + 2 b1 + b0.
template <int B>
struct CodeConsts {
  float sc, zc, nt[(1 << (B - 1)) - 1];
  float d20;                  // 3 bits: nt2 - nt0
  float d51, d40, d20b, ddd;  // 4 bits: nt5 - nt1, nt4 - nt0, nt2 - nt0, (nt6 - nt4) - (nt2 - nt0)
};

template <int B>
__device__ __forceinline__ void search_consts(CodeConsts<B> &k) {
  if constexpr (B == 3) {
    k.d20 = k.nt[2] - k.nt[0];
  } else if constexpr (B == 4) {
    k.d51 = k.nt[5] - k.nt[1];
    k.d40 = k.nt[4] - k.nt[0];
    k.d20b = k.nt[2] - k.nt[0];
    k.ddd = (k.nt[6] - k.nt[4]) - k.d20b;
  }
}

// m for two coordinates (|z| in a0, a1).
template <int B>
__device__ __forceinline__ float2 threshold_count2(float a0, float a1, const CodeConsts<B> &k) {
  if constexpr (B == 2) {
    return make_float2(fma_sat(a0, k.sc, k.nt[0]), fma_sat(a1, k.sc, k.nt[0]));
  } else if constexpr (B == 3) {
    const float2 b1 = make_float2(fma_sat(a0, k.sc, k.nt[1]), fma_sat(a1, k.sc, k.nt[1]));
    const float2 sel = fma2(b1, make_float2(k.d20, k.d20), make_float2(k.nt[0], k.nt[0]));
    const float2 b0 = make_float2(fma_sat(a0, k.sc, sel.x), fma_sat(a1, k.sc, sel.y));
    return fma2(b1, make_float2(2.f, 2.f), b0);
  } else {
    const float2 b2 = make_float2(fma_sat(a0, k.sc, k.nt[3]), fma_sat(a1, k.sc, k.nt[3]));
    const float2 sel1 = fma2(b2, make_float2(k.d51, k.d51), make_float2(k.nt[1], k.nt[1]));
    const float2 b1 = make_float2(fma_sat(a0, k.sc, sel1.x), fma_sat(a1, k.sc, sel1.y));
    const float2 base = fma2(b2, make_float2(k.d40, k.d40), make_float2(k.nt[0], k.nt[0]));
    const float2 step = fma2(b2, make_float2(k.ddd, k.ddd), make_float2(k.d20b, k.d20b));
    const float2 sel0 = fma2(b1, step, base);
    const float2 b0 = make_float2(fma_sat(a0, k.sc, sel0.x), fma_sat(a1, k.sc, sel0.y));
    return fma2(b2, make_float2(4.f, 4.f), fma2(b1, make_float2(2.f, 2.f), b0));
  }
}

// Offsets from half - 1 of the codes #{j : T_j < z} of two rotated
// coordinates, exactly, as floats on the FMA pipe: m = #{j : t_j < |z| / ||x||}
// (threshold_count2; the saturating tests run per lane, as the paired form
// has no saturation), p = [z > 0] (z zc 2^127 saturates to 1 for every
// positive float when zc = 2^127, and to 0 otherwise), and the offset
// m (2 p - 1) + p, i.e. m + 1 for z > 0, -m otherwise; the sums and products
// after the tests run on both lanes at once.
template <int B>
__device__ __forceinline__ float2 code_offset_f2(float z0, float z1, const CodeConsts<B> &k) {
  const float2 m = threshold_count2<B>(fabsf(z0), fabsf(z1), k);
  const float2 s = mul2(make_float2(z0, z1), make_float2(k.zc, k.zc));
  const float2 p = make_float2(mul_sat(s.x, 0x1p127f), mul_sat(s.y, 0x1p127f));
  const float2 q = fma2(p, make_float2(2.f, 2.f), make_float2(-1.f, -1.f));
  return fma2(m, q, p);
}

// 16 bits of codes (n codes of `bits` bits, LSB first): their offsets summed
// at their positions (even and odd codes in the two lanes, the even lane
// starting from 2^23 + (half - 1) in every field), the lanes added, and the
// integer read out of the mantissa.  Every partial sum is an integer below
// 2^24, so all of it is exact.
template <int B, int n, int bits>
__device__ __forceinline__ uint32_t pack16(const float *z, const CodeConsts<B> &k) {
  constexpr int half_m1 = (1 << (B - 1)) - 1;
  int ones = 0;
#pragma unroll
  for (int j = 0; j < n; ++j) ones += 1 << (bits * j);
  float2 acc = make_float2(8388608.f + (float)(half_m1 * ones), 0.f);
#pragma unroll
  for (int j = 0; j < n; j += 2)
    acc = fma2(code_offset_f2<B>(z[j], z[j + 1], k),
               make_float2((float)(1 << (bits * j)), (float)(1 << (bits * (j + 1)))), acc);
  return __float_as_uint(acc.x + acc.y) & 0xFFFFu;
}

__device__ __forceinline__ uint32_t join16(uint32_t lo, uint32_t hi) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(d) : "r"(lo), "r"(hi));
  return d;
}

// Codes of coordinates 16 c .. 16 c + 15 packed into the words of the cache
// layout: LSB-first for 2 and 4 bits; for 3 bits, in each 32-coordinate group
// nibble l % 8 of word l / 8 (l < 24), and the eight spare-column codes
// gathered into the nibbles of one word whose bit k of every nibble then
// moves to bit 3 of word k.
template <int B, int N>
__device__ __forceinline__ void code_chunk(int c, const float (&z)[16], const CodeConsts<B> &k, uint32_t (&w)[N]) {
  if constexpr (B == 3) {
    const int g = c >> 1;
    const uint32_t x0 = join16(pack16<3, 4, 4>(z, k), pack16<3, 4, 4>(z + 4, k));
    const uint32_t x1 = join16(pack16<3, 4, 4>(z + 8, k), pack16<3, 4, 4>(z + 12, k));
    if ((c & 1) == 0) {
      w[3 * g] = x0;
      w[3 * g + 1] = x1;
    } else {
      w[3 * g] |= (x1 << 3) & 0x88888888u;
      w[3 * g + 1] |= (x1 << 2) & 0x88888888u;
      w[3 * g + 2] = x0 | ((x1 << 1) & 0x88888888u);
    }
  } else if constexpr (B == 2) {
    w[c] = join16(pack16<2, 8, 2>(z, k), pack16<2, 8, 2>(z + 8, k));
  } else {
    w[2 * c] = join16(pack16<4, 4, 4>(z, k), pack16<4, 4, 4>(z + 4, k));
    w[2 * c + 1] = join16(pack16<4, 4, 4>(z + 8, k), pack16<4, 4, 4>(z + 12, k));
  }
}

// One row of C chunks of 16 columns (C = d / 16): its C / 2 * B code words.
template <int B, int C = 8>
__device__ __forceinline__ void epilogue_row(const float (&thr)[kMaxLevels], float n, uint32_t tmem_row,
                                             uint32_t (&words)[C / 2 * B]) {
  constexpr int half = 1 << (B - 1);
  CodeConsts<B> k;
  const bool live = n > 0x1p-25f;  // stored fp16 norm nonzero
  k.sc = live ? 0x1p64f / n : 0.f;
  k.zc = live ? 0x1p127f : 0.f;
#pragma unroll
  for (int j = 0; j < half - 1; ++j) k.nt[j] = -thr[half + j] * 0x1p64f;  // positive thresholds x -2^64
  search_consts<B>(k);
#pragma unroll
  for (int c = 0; c < C; ++c) {
    float z[16];
    tmem_ld16(tmem_row + 16 * c, z);
    code_chunk<B>(c, z, k, words);
  }
}

// ------------------------------------------------------------------ host
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a row-major [rows][width] matrix of 16-bit elements (bf16
// unless `type` says otherwise), boxes of box_rows rows x 64 columns (128
// bytes) with the 128-byte swizzle the MMA descriptors expect.
bool make_row_map(CUtensorMap *m, const void *base, long rows,
                  CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int width = kHeadDim,
                  int box_rows = kTileRows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)width * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(m, type, 2, const_cast<void *>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace tq
