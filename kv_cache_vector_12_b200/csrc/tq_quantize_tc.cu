// Quantize-on-append on the 5th-generation tensor cores (sm_100a).
//
// "ステップ1: PolarQuant" (ai-accelerate.xyz TurboQuant explainer): every
// head vector x is rotated by the random orthogonal matrix Pi and each rotated
// coordinate is quantized with the Lloyd-Max codebook.  Here the rotation of
// a tile of 128 head vectors is one 128x128x128 bf16 GEMM, z = X Pi^T:
//
//   producer warp   TMA (cp.async.bulk.tensor, 128-byte swizzle) loads each
//                   128-row tile of K or V into a 4-deep shared-memory ring;
//                   Pi stays resident in shared memory for the CTA's lifetime.
//   MMA warp        one thread issues 8 tcgen05.mma (kind::f16, bf16 inputs,
//                   fp32 accumulation in tensor memory) per tile and commits
//                   to mbarriers.
//   4 epilogue      warpgroups, one TMEM accumulator each; every thread owns
//   warpgroups      one row (vector): ||x|| from the shared-memory tile,
//                   z from TMEM (tcgen05.ld 32x32b), codes against the
//                   thresholds scaled by ||x||, bit-packing into the cache
//                   layout, 16-byte stores, fp16 norm.
//
// The kernel is persistent (one CTA per SM, tiles strided by the grid).  Every
// mbarrier wait is bounded; on expiry the kernel flags the error, stops, waits
// for its copies and MMAs in flight (bounded) and releases its tensor memory.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
constexpr int kTileRows = 128;
constexpr int kRingStages = 4;
constexpr int kEpiGroups = 4;
constexpr int kQThreads = 32 * (2 + 4 * kEpiGroups);
constexpr int kTileBytes = kTileRows * D * 2;     // 32 KB: two 128x64 bf16 boxes
constexpr int kBoxBytes = kTileBytes / 2;
constexpr unsigned kTmemCols = 512;               // 4 accumulators of 128 columns
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

struct QuantTcArgs {
  DeviceParams p;
  tq_cache c;
  const int32_t *seq_idx;
  const int32_t *pos;
  int n_rows;       // n_tok * n_kv_heads rows per matrix
  int tiles_k;      // tiles of K handled here (0 when K goes elsewhere)
  int tiles_v;
};

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

// Two fp32 lanes in one 64-bit register pair: multiply and fused multiply-add
// of both lanes in one instruction (f32x2, sm_100), round to nearest like
// their scalar forms.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
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
template <int B>
__device__ __forceinline__ void code_chunk(int c, const float (&z)[16], const CodeConsts<B> &k,
                                           uint32_t (&w)[4 * B]) {
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

template <int B>
__device__ __forceinline__ void epilogue_row(const float (&thr)[kMaxLevels], float n, uint32_t tmem_row,
                                             uint32_t (&words)[4 * B]) {
  constexpr int half = 1 << (B - 1);
  CodeConsts<B> k;
  const bool live = n > 0x1p-25f;  // stored fp16 norm nonzero
  k.sc = live ? 0x1p64f / n : 0.f;
  k.zc = live ? 0x1p127f : 0.f;
#pragma unroll
  for (int j = 0; j < half - 1; ++j) k.nt[j] = -thr[half + j] * 0x1p64f;  // positive thresholds x -2^64
  search_consts<B>(k);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float z[16];
    tmem_ld16(tmem_row + 16 * c, z);
    code_chunk<B>(c, z, k, words);
  }
}

template <int BK, int BV>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                       const __grid_constant__ CUtensorMap map_pi, const QuantTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned region: Pi (32 KB) then the ring
  unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char *pi_tile = smem;
  unsigned char *ring = smem + kTileBytes;
  __shared__ __align__(8) uint64_t full_bar[kRingStages], empty_bar[kRingStages];
  __shared__ __align__(8) uint64_t tfull_bar[kEpiGroups], tempty_bar[kEpiGroups], pi_bar;
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.tiles_k + a.tiles_v;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingStages; ++i) {
      bar_init(smem_addr(&full_bar[i]), 1);
      bar_init(smem_addr(&empty_bar[i]), 1 + 4);  // MMA commit + the 4 norm-reading warps
    }
    for (int g = 0; g < kEpiGroups; ++g) {
      bar_init(smem_addr(&tfull_bar[g]), 1);
      bar_init(smem_addr(&tempty_bar[g]), 4);
    }
    bar_init(smem_addr(&pi_bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the MMA warp owns the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_base_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  if (warp == 0 && lane == 0) {  // Pi belongs to the context: no earlier kernel writes it
    const uint32_t pb = smem_addr(&pi_bar);
    bar_expect_tx(pb, kTileBytes);
    tma_load_2d(smem_addr(pi_tile), &map_pi, 0, 0, pb);
    tma_load_2d(smem_addr(pi_tile + kBoxBytes), &map_pi, 64, 0, pb);
  }
  // launched as a programmatic dependent: inputs and the cache are touched
  // only once the previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------ producer (TMA)
    if (lane == 0) {
      const uint32_t pb = smem_addr(&pi_bar);
      int i = 0, issued = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
        const int slot = i % kRingStages;
        if (i >= kRingStages && !bar_wait(smem_addr(&empty_bar[slot]), ((i / kRingStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        const bool is_k = t < a.tiles_k;
        const CUtensorMap *map = is_k ? &map_k : &map_v;
        const int row0 = (is_k ? t : t - a.tiles_k) * kTileRows;
        const uint32_t fb = smem_addr(&full_bar[slot]);
        unsigned char *st = ring + slot * kTileBytes;
        bar_expect_tx(fb, kTileBytes);
        tma_load_2d(smem_addr(st), map, 0, row0, fb);
        tma_load_2d(smem_addr(st + kBoxBytes), map, 64, row0, fb);
        issued = i + 1;
      }
      bar_wait(pb, 0);
      if (*(volatile int *)&abort_flag)  // drain: never leave copies in flight
        for (int k = (issued > kRingStages ? issued - kRingStages : 0); k < issued; ++k)
          bar_wait(smem_addr(&full_bar[k % kRingStages]), (k / kRingStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = bar_wait(smem_addr(&pi_bar), 0);
      int i = 0;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
        const int slot = i % kRingStages, acc = i % kEpiGroups;
        ok = bar_wait(smem_addr(&full_bar[slot]), (i / kRingStages) & 1);
        if (ok && i >= kEpiGroups) ok = bar_wait(smem_addr(&tempty_bar[acc]), ((i / kEpiGroups) - 1) & 1);
        if (!ok || *(volatile int *)&abort_flag) break;
        tc_fence_after();
        const uint32_t a0 = smem_addr(ring + slot * kTileBytes), b0 = smem_addr(pi_tile);
        const uint32_t d = tmem_base + acc * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;  // 16 bf16 along K per MMA
          tc_mma(d, sw128_desc(a0 + off), sw128_desc(b0 + off), kk > 0);
        }
        tc_commit(smem_addr(&tfull_bar[acc]));
        tc_commit(smem_addr(&empty_bar[slot]));
      }
      if (!ok) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------ epilogue warpgroups
    const int g = (warp - 2) / 4;
    const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
    const int r = 32 * quarter + lane;             // the row this thread owns
    // thresholds of both codebooks, once
    float tk[kMaxLevels], tv[kMaxLevels];
#pragma unroll
    for (int e = 0; e < kMaxLevels; ++e) {
      tk[e] = a.p.cb[1 * kMaxLevels + e];
      tv[e] = a.p.cb[3 * kMaxLevels + e];
    }
    for (int j = 0, t = blockIdx.x + g * gridDim.x; t < n_tiles; ++j, t += kEpiGroups * gridDim.x) {
      const int i = g + j * kEpiGroups;            // tile sequence number within this CTA
      const int slot = i % kRingStages;
      const bool is_k = t < a.tiles_k;
      const int row = (is_k ? t : t - a.tiles_k) * kTileRows + r;
      // destination of this row: loaded now, checked after the codes, so the
      // loads' latency overlaps the barrier waits and the epilogue
      const bool live = row < a.n_rows;
      const int tok = live ? row / a.c.n_kv_heads : 0;
      const int tok_h = live ? row - tok * a.c.n_kv_heads : 0;
      // (no index arrays: token t goes to position t of sequence 0, the
      // weight-row layout of tq_weight_quantize)
      const int s_dst = a.seq_idx ? a.seq_idx[tok] : 0, p_dst = a.pos ? a.pos[tok] : tok;
      if (!bar_wait(smem_addr(&full_bar[slot]), (i / kRingStages) & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      // ||x|| from the swizzled tile.  Row r's 128-byte segment holds its 16-byte
      // chunks permuted by r % 8; reading chunk c ^ (r % 8) keeps a warp's loads
      // conflict-free, and the order does not matter to a sum of squares.  bf16
      // squares are exact in fp32.
      const unsigned char *st = ring + slot * kTileBytes;
      float2 ss = make_float2(0.f, 0.f);  // sums of the squares of the low and the high halves
#pragma unroll
      for (int box = 0; box < 2; ++box)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u =
              *reinterpret_cast<const uint4 *>(st + box * kBoxBytes + r * 128 + ((ch ^ (r & 7)) * 16));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = make_float2(__uint_as_float(w4[e] << 16), __uint_as_float(w4[e] & 0xffff0000u));
            ss = fma2(x, x, ss);
          }
        }
      const float nrm = sqrtf(ss.x + ss.y);
      __syncwarp();
      if (lane == 0) bar_arrive(smem_addr(&empty_bar[slot]));

      if (!bar_wait(smem_addr(&tfull_bar[g]), j & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t trow = tmem_base + g * 128 + ((uint32_t)(32 * quarter) << 16);
      uint32_t words[16];
      if constexpr (BK == BV) {  // one copy of the epilogue code for K and V tiles
        float thr[kMaxLevels];
#pragma unroll
        for (int e = 0; e < kMaxLevels; ++e) thr[e] = is_k ? tk[e] : tv[e];
        uint32_t w[4 * BK];
        epilogue_row<BK>(thr, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < 4 * BK; ++e) words[e] = w[e];
      } else if (is_k) {
        uint32_t w[4 * BK];
        epilogue_row<BK>(tk, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < 4 * BK; ++e) words[e] = w[e];
      } else {
        uint32_t w[4 * BV];
        epilogue_row<BV>(tv, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < 4 * BV; ++e) words[e] = w[e];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(smem_addr(&tempty_bar[g]));

      long slot_i = -1;
      if (live) {
        slot_i = cache_slot(a.c, s_dst, tok_h, p_dst);
        if (slot_i < 0 && tok_h == 0 && is_k) atomicOr(a.p.err, kErrTokenRange);
      }
      if (slot_i >= 0) {
        const int bits = is_k ? BK : BV;
        uint4 *dst = reinterpret_cast<uint4 *>((is_k ? a.c.codes_k : a.c.codes_v) + slot_i * (long)(16 * bits));
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < bits) dst[q] = make_uint4(words[4 * q], words[4 * q + 1], words[4 * q + 2], words[4 * q + 3]);
        (is_k ? a.c.norm_k : a.c.norm_v)[slot_i] = __half_as_ushort(__float2half_rn(fminf(nrm, 65504.f)));
      }
      if (*(volatile int *)&abort_flag) break;
    }
  }

  // release tensor memory once every MMA and every tcgen05.ld is finished
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
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

// 2-D map over a row-major [rows][128] bf16 matrix, boxes of 128 rows x 64
// columns (128 bytes) with the 128-byte swizzle the MMA descriptors expect.
bool make_row_map(CUtensorMap *m, const void *base, long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTileRows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kQuantTcSmem = 1024 + kTileBytes * (1 + kRingStages);

using QuantTcFn = void (*)(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                           const __grid_constant__ CUtensorMap, const QuantTcArgs);

template <int BK>
QuantTcFn pick_bv(int bv) {
  return bv == 2 ? quantize_tc_kernel<BK, 2> : bv == 3 ? quantize_tc_kernel<BK, 3> : quantize_tc_kernel<BK, 4>;
}

QuantTcFn pick(int bk, int bv) { return bk == 2 ? pick_bv<2>(bv) : bk == 3 ? pick_bv<3>(bv) : pick_bv<4>(bv); }

}  // namespace

int launch_quantize_tc(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                       const int32_t *seq_idx, const int32_t *pos, int n_tok, bool include_k, bool include_v,
                       void *stream) {
  // cached per device (the attribute applies to the current device), and
  // atomically, as calls may come from several threads
  static std::atomic<int> cached_sm[kMaxDevices];
  static std::atomic<bool> configured[kMaxDevices][3][3];
  const int dev = current_device();
  int n_sm = cached_sm[dev].load(std::memory_order_relaxed);
  if (n_sm == 0) {
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
    cached_sm[dev].store(n_sm, std::memory_order_relaxed);
  }
  const QuantTcFn fn = pick(p.bits_k, p.bits_v);
  std::atomic<bool> &done = configured[dev][p.bits_k - 2][p.bits_v - 2];
  if (!done.load(std::memory_order_acquire)) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantTcSmem);
    done.store(true, std::memory_order_release);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  CUtensorMap mk, mv, mp;
  std::memset(&mk, 0, sizeof mk);
  std::memset(&mv, 0, sizeof mv);
  if ((include_v && !make_row_map(&mv, v, rows)) || !make_row_map(&mp, p.pi, D) ||
      (include_k && !make_row_map(&mk, k, rows)))
    return (int)cudaErrorInvalidValue;
  if (!include_k) mk = mv;
  if (!include_v) mv = mk;
  QuantTcArgs args{p, c, seq_idx, pos, (int)rows, 0, 0};
  const int tiles = (int)((rows + kTileRows - 1) / kTileRows);
  args.tiles_k = include_k ? tiles : 0;
  args.tiles_v = include_v ? tiles : 0;
  const int total = args.tiles_k + args.tiles_v;
  const int grid = total < n_sm ? total : n_sm;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = kQuantTcSmem;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, mk, mv, mp, args);
}

}  // namespace tq
