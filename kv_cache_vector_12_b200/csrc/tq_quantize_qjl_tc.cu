// Quantize-on-append with the 1-bit QJL residual stage on K, on the
// 5th-generation tensor cores (sm_100a); V rows of the same batch (MSE codes
// only) run in the same launch.
//
// The method ("ステップ2: QJL", ai-accelerate.xyz TurboQuant explainer; the
// residual 1-bit QJL transform of "Tether QVACのTurboQuant実装", qxai.app):
// after the rotation and the Lloyd-Max codes, the residual r = y - c[code] of
// each K vector (y = Pi x / ||x||) is projected by a Gaussian matrix S, and
// only the signs of S r are kept, with ||r||.
//
// Head dimension d = 128 or 64 (a template parameter W).  Per tile of 128
// rows, on tcgen05 with fp32 accumulators in tensor memory:
//   MMA 1   Z = X Pi^T: X by TMA (128-byte swizzle) from a 3-deep ring, Pi
//           resident in shared memory (bf16, exact products).
//   epilogue A (two threads per row, d / 2 coordinates each): ||x|| from the
//           shared-memory tile, z from tensor memory, the codes against the
//           thresholds scaled by ||x|| (the exact saturating-FMA search of
//           the MSE kernel); for K also the residual r 2^14 = y 2^14 -
//           c[code] 2^14 (the centroid selected by fused multiply-adds from
//           the search's bits, exact), ||r||^2, and r 2^14 split into two
//           fp16 parts hi + lo written back over the row's Z columns in
//           tensor memory (hi and lo of each 16 coordinates side by side: the
//           A operand of MMA 2).
//   MMA 2   (K) S r = R_hi S_hi^T + R_hi S_lo^T + R_lo S_hi^T with A from
//           tensor memory and S 2^sigma = S_hi + S_lo (fp16, resident in
//           shared memory): 22 significant bits on each side, so the signs
//           agree with an exact dot product wherever |S r| is above about
//           2^-21 |S| |r|.
//   epilogue B (K): the signs (bit n of the row = [(S r)_n >= 0]) from
//           tensor memory; then the stores: packed codes, fp16 ||x||, and for
//           K the sign bits and fp16 ||r||.
// The K tiles come first in the tile order and the cheaper V tiles fill the
// tail.  Two tile groups (each two warpgroups, one per half row) take
// alternate tiles with 2 d columns of tensor memory each (Z / R, then S r),
// so one group's MMAs run while the other computes.  One thread issues both
// GEMMs, polling the barriers of both stages.  Every wait is bounded; on
// expiry the kernel flags the error and stops, after waiting (bounded) for
// its copies and MMAs in flight, and releases its tensor memory.
#include <atomic>
#include <cstring>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"
#include "tq_tc.cuh"

namespace tq {
namespace {

constexpr int kJStages = 3;                          // X ring depth
constexpr int kJGroups = 2;                          // tile groups (two warpgroups each)
constexpr int kJThreads = 32 * (2 + 8 * kJGroups);   // producer, MMA issuer, epilogue
constexpr float kRScale = 0x1p14f;  // |r| < 1.3: r 2^14 stays below fp16's largest finite value

// The shapes that depend on the head dimension W: an X tile is W / 64 boxes
// of 128 rows x 64 coordinates; Pi, S hi and S lo are W / 64 boxes of W rows.
template <int W>
struct JShape {
  static constexpr int boxes = W / 64;
  static constexpr int tile_bytes = kTileRows * W * 2;
  static constexpr int mat_bytes = W * W * 2;
  static constexpr int mat_box = W * 128;
  static constexpr unsigned tmem_cols = kJGroups * 2 * W;  // per group: Z / R (W columns), S r (W)
  static constexpr int smem = 1024 + 3 * mat_bytes + kJStages * tile_bytes;  // Pi, S hi, S lo, the ring
  // instruction descriptors, kind::f16, fp32 accumulator, K-major, M = 128,
  // N = W: bf16 A and B (MMA 1), fp16 A and B (MMA 2)
  static constexpr uint32_t idesc_bf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(W >> 3) << 17) | ((128u >> 4) << 24);
  static constexpr uint32_t idesc_f16 = (1u << 4) | ((uint32_t)(W >> 3) << 17) | ((128u >> 4) << 24);
};

// D (tensor memory) += A (tensor memory) B (shared-memory descriptor).
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
               : "memory");
}

// 8 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// Non-blocking test of phase `parity`.
__device__ __forceinline__ bool bar_test(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(ok)
               : "r"(b), "r"(parity)
               : "memory");
  return ok != 0;
}

struct QjlTcArgs {
  DeviceParams p;
  tq_cache c;
  const int32_t *seq_idx;
  const int32_t *pos;
  int n_rows;   // n_tok * n_kv_heads rows per matrix
  int tiles_k;  // K tiles (with QJL), then as many V tiles (MSE only)
};

// Centroid magnitudes of the positive half, times 2^14, and the differences
// that select one of them by fused multiply-adds from the search's bits.  The
// centroids are fp16 values within a few binades of each other, so every
// difference (and difference of differences) below is exact in fp32 and
// every selection yields a centroid exactly.
template <int B>
struct ResConsts {
  float c0;
  float d1;        // B = 2: c1 - c0
  float d2, e3;    // B = 3: c2 - c0; (c3 - c2) - (c1 - c0)
  float d4, e6;    // B = 4: c4 - c0; (c6 - c4) - (c2 - c0)
  float f0, f40, f2, f62;  // B = 4: d0 = c1 - c0, d4 - d0, d2 = c3 - c2, d6 - d2 (d_m = c_{m+1} - c_m)
};

template <int B>
__device__ __forceinline__ void res_consts(const float *cent, ResConsts<B> &rc) {
  constexpr int half = 1 << (B - 1);
  float cm[half];
#pragma unroll
  for (int j = 0; j < half; ++j) cm[j] = cent[half + j] * kRScale;
  rc.c0 = cm[0];
  if constexpr (B == 2) {
    rc.d1 = cm[1] - cm[0];
  } else if constexpr (B == 3) {
    rc.d1 = cm[1] - cm[0];
    rc.d2 = cm[2] - cm[0];
    rc.e3 = (cm[3] - cm[2]) - (cm[1] - cm[0]);
  } else {
    rc.d2 = cm[2] - cm[0];
    rc.d4 = cm[4] - cm[0];
    rc.e6 = (cm[6] - cm[4]) - (cm[2] - cm[0]);
    rc.f0 = cm[1] - cm[0];
    rc.f40 = (cm[5] - cm[4]) - (cm[1] - cm[0]);
    rc.f2 = cm[3] - cm[2];
    rc.f62 = (cm[7] - cm[6]) - (cm[3] - cm[2]);
  }
}

// Bits of m = #{j : t_j < |z| / ||x||} for two coordinates (|z| in a0, a1),
// by the same saturating tests and threshold selections as threshold_count2,
// and the centroid magnitude c_m 2^14 they select.
template <int B>
__device__ __forceinline__ void search_select2(float a0, float a1, const CodeConsts<B> &k, const ResConsts<B> &rc,
                                               float2 &m, float2 &cmag) {
  if constexpr (B == 2) {
    const float2 b0 = make_float2(fma_sat(a0, k.sc, k.nt[0]), fma_sat(a1, k.sc, k.nt[0]));
    m = b0;
    cmag = fma2(b0, make_float2(rc.d1, rc.d1), make_float2(rc.c0, rc.c0));
  } else if constexpr (B == 3) {
    const float2 b1 = make_float2(fma_sat(a0, k.sc, k.nt[1]), fma_sat(a1, k.sc, k.nt[1]));
    const float2 sel = fma2(b1, make_float2(k.d20, k.d20), make_float2(k.nt[0], k.nt[0]));
    const float2 b0 = make_float2(fma_sat(a0, k.sc, sel.x), fma_sat(a1, k.sc, sel.y));
    m = fma2(b1, make_float2(2.f, 2.f), b0);
    const float2 t = fma2(b1, make_float2(rc.d2, rc.d2), make_float2(rc.c0, rc.c0));      // c0 or c2
    const float2 dd = fma2(b1, make_float2(rc.e3, rc.e3), make_float2(rc.d1, rc.d1));     // c1 - c0 or c3 - c2
    cmag = fma2(b0, dd, t);
  } else {
    const float2 b2 = make_float2(fma_sat(a0, k.sc, k.nt[3]), fma_sat(a1, k.sc, k.nt[3]));
    const float2 sel1 = fma2(b2, make_float2(k.d51, k.d51), make_float2(k.nt[1], k.nt[1]));
    const float2 b1 = make_float2(fma_sat(a0, k.sc, sel1.x), fma_sat(a1, k.sc, sel1.y));
    const float2 base = fma2(b2, make_float2(k.d40, k.d40), make_float2(k.nt[0], k.nt[0]));
    const float2 step = fma2(b2, make_float2(k.ddd, k.ddd), make_float2(k.d20b, k.d20b));
    const float2 sel0 = fma2(b1, step, base);
    const float2 b0 = make_float2(fma_sat(a0, k.sc, sel0.x), fma_sat(a1, k.sc, sel0.y));
    m = fma2(b2, make_float2(4.f, 4.f), fma2(b1, make_float2(2.f, 2.f), b0));
    const float2 u = fma2(b2, make_float2(rc.d4, rc.d4), make_float2(rc.c0, rc.c0));        // c0 or c4
    const float2 e = fma2(b2, make_float2(rc.e6, rc.e6), make_float2(rc.d2, rc.d2));        // c2 - c0 or c6 - c4
    const float2 v = fma2(b1, e, u);                                                        // c_{4 b2 + 2 b1}
    const float2 x = fma2(b2, make_float2(rc.f40, rc.f40), make_float2(rc.f0, rc.f0));      // d0 or d4
    const float2 y = fma2(b2, make_float2(rc.f62, rc.f62), make_float2(rc.f2, rc.f2));      // d2 or d6
    const float2 dd = fma2(b1, make_float2(y.x - x.x, y.y - x.y), x);
    cmag = fma2(b0, dd, v);
  }
}

// For two rotated coordinates z0, z1: the code offsets from half - 1 (as
// code_offset_f2: m + 1 for z > 0, -m otherwise) and the residuals
// r 2^14 = z rinv - (2 p - 1) c_m 2^14 with rinv = 2^14 / ||x|| (0 for the
// zero vector).
template <int B>
__device__ __forceinline__ void code_res2(float z0, float z1, const CodeConsts<B> &k, const ResConsts<B> &rc,
                                          float rinv, float2 &off, float2 &res) {
  float2 m, cmag;
  search_select2<B>(fabsf(z0), fabsf(z1), k, rc, m, cmag);
  const float2 s = mul2(make_float2(z0, z1), make_float2(k.zc, k.zc));
  const float2 p = make_float2(mul_sat(s.x, 0x1p127f), mul_sat(s.y, 0x1p127f));
  const float2 q = fma2(p, make_float2(2.f, 2.f), make_float2(-1.f, -1.f));   // 2 p - 1
  const float2 nq = fma2(p, make_float2(-2.f, -2.f), make_float2(1.f, 1.f));  // 1 - 2 p
  off = fma2(m, q, p);
  res = fma2(nq, cmag, mul2(make_float2(z0, z1), make_float2(rinv, rinv)));
}

// 16 bits of codes (n codes of `bits` bits, LSB first) from their offsets, as
// pack16 does from z.
template <int B, int n, int bits>
__device__ __forceinline__ uint32_t pack16_off(const float *off) {
  constexpr int half_m1 = (1 << (B - 1)) - 1;
  int ones = 0;
#pragma unroll
  for (int j = 0; j < n; ++j) ones += 1 << (bits * j);
  float2 acc = make_float2(8388608.f + (float)(half_m1 * ones), 0.f);
#pragma unroll
  for (int j = 0; j < n; j += 2)
    acc = fma2(make_float2(off[j], off[j + 1]), make_float2((float)(1 << (bits * j)), (float)(1 << (bits * (j + 1)))),
               acc);
  return __float_as_uint(acc.x + acc.y) & 0xFFFFu;
}

// Codes of coordinates 16 c .. 16 c + 15 (c counted from the first of the
// words in w) into the cache words (code_chunk's layout).
template <int B>
__device__ __forceinline__ void code_chunk_off(int c, const float (&off)[16], uint32_t (&w)[4 * B]) {
  if constexpr (B == 3) {
    const int g = c >> 1;
    const uint32_t x0 = join16(pack16_off<3, 4, 4>(off), pack16_off<3, 4, 4>(off + 4));
    const uint32_t x1 = join16(pack16_off<3, 4, 4>(off + 8), pack16_off<3, 4, 4>(off + 12));
    if ((c & 1) == 0) {
      w[3 * g] = x0;
      w[3 * g + 1] = x1;
    } else {
      w[3 * g] |= (x1 << 3) & 0x88888888u;
      w[3 * g + 1] |= (x1 << 2) & 0x88888888u;
      w[3 * g + 2] = x0 | ((x1 << 1) & 0x88888888u);
    }
  } else if constexpr (B == 2) {
    w[c] = join16(pack16_off<2, 8, 2>(off), pack16_off<2, 8, 2>(off + 8));
  } else {
    w[2 * c] = join16(pack16_off<4, 4, 4>(off), pack16_off<4, 4, 4>(off + 4));
    w[2 * c + 1] = join16(pack16_off<4, 4, 4>(off + 8), pack16_off<4, 4, 4>(off + 12));
  }
}

// The code words of a half row (W/2 coordinates: W/64 groups of 32, B words
// each) at dst: 16-byte stores for W = 128 where B is even, else 8- or
// 4-byte stores (the half row starts on a multiple of 4 B bytes).
template <int W, int B>
__device__ __forceinline__ void store_half_codes(unsigned char *dst, const uint32_t (&words)[4 * B]) {
  if constexpr (W == 128 && B != 3) {
#pragma unroll
    for (int q = 0; q < B / 2; ++q)
      reinterpret_cast<uint4 *>(dst)[q] = make_uint4(words[4 * q], words[4 * q + 1], words[4 * q + 2], words[4 * q + 3]);
  } else if constexpr (W == 128) {
#pragma unroll
    for (int q = 0; q < 3; ++q) reinterpret_cast<uint2 *>(dst)[q] = make_uint2(words[2 * q], words[2 * q + 1]);
  } else if constexpr (B != 3) {
#pragma unroll
    for (int q = 0; q < B / 2; ++q) reinterpret_cast<uint2 *>(dst)[q] = make_uint2(words[2 * q], words[2 * q + 1]);
  } else {
#pragma unroll
    for (int q = 0; q < 3; ++q) reinterpret_cast<uint32_t *>(dst)[q] = words[q];
  }
}

// 18 warps: one of the four schedulers holds five, whose registers (at most
// 16384 per scheduler) cap a thread at 96
template <int W, int BK, int BV>
__global__ void __launch_bounds__(kJThreads, 1)
    quantize_qjl_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                           const __grid_constant__ CUtensorMap map_pi, const __grid_constant__ CUtensorMap map_s,
                           const QjlTcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  using Sh = JShape<W>;
  unsigned char *pi_tile = smem;                     // Pi, bf16
  unsigned char *s_hi = smem + Sh::mat_bytes;        // S 2^sigma, fp16 high parts
  unsigned char *s_lo = smem + 2 * Sh::mat_bytes;    // and low parts
  unsigned char *ring = smem + 3 * Sh::mat_bytes;
  __shared__ __align__(8) uint64_t full_bar[kJStages], empty_bar[kJStages];
  __shared__ __align__(8) uint64_t zfull[kJGroups], rfull[kJGroups], sfull[kJGroups], tfree[kJGroups];
  __shared__ __align__(8) uint64_t rr_bar[kJGroups];  // both halves' ||r||^2 written
  __shared__ __align__(8) uint64_t const_bar, s_bar, mma_done;  // Pi; S hi and lo
  __shared__ float s_rr[kJGroups][2][2][kTileRows];  // ||r||^2 of each half row, by tile parity
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's tiles: first the K tiles bx + i gridDim.x, then the V tiles
  // (gridDim.x - 1 - bx) + j gridDim.x, so that the CTAs with one K tile more
  // than the others get one V tile less (the K tiles cost about twice as much)
  const int bx = (int)blockIdx.x, grid = (int)gridDim.x, bv = grid - 1 - bx;
  const int my_k = bx < a.tiles_k ? (a.tiles_k - 1 - bx) / grid + 1 : 0;
  const int my_v = bv < a.tiles_k ? (a.tiles_k - 1 - bv) / grid + 1 : 0;
  const int my_tiles = my_k + my_v;
  // first row (of K or V) of the CTA's i-th tile
  auto tile_row0 = [&](int i) { return (i < my_k ? bx + i * grid : bv + (i - my_k) * grid) * kTileRows; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kJStages; ++i) {
      bar_init(smem_addr(&full_bar[i]), 1);
      bar_init(smem_addr(&empty_bar[i]), 1 + 8);  // MMA 1 commit + the 8 norm-reading warps
    }
    for (int g = 0; g < kJGroups; ++g) {
      bar_init(smem_addr(&zfull[g]), 1);
      bar_init(smem_addr(&rfull[g]), 8);
      bar_init(smem_addr(&sfull[g]), 1);
      bar_init(smem_addr(&tfree[g]), 8);
      bar_init(smem_addr(&rr_bar[g]), 8);
    }
    bar_init(smem_addr(&const_bar), 1);
    bar_init(smem_addr(&s_bar), 1);
    bar_init(smem_addr(&mma_done), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the MMA warp owns the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_base_slot)),
                 "r"(Sh::tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  if (warp == 0 && lane == 0) {  // Pi and S belong to the context: no earlier kernel writes them
    const uint32_t cb = smem_addr(&const_bar);
    bar_expect_tx(cb, Sh::mat_bytes);
#pragma unroll
    for (int b = 0; b < Sh::boxes; ++b) tma_load_2d(smem_addr(pi_tile + b * Sh::mat_box), &map_pi, 64 * b, 0, cb);
  }
  // launched as a programmatic dependent: inputs and the cache are touched
  // only once the previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------ producer (TMA)
    if (lane == 0) {
      bool s_issued = false;
      auto load_s = [&]() {  // S belongs to the context: no earlier kernel writes it
        s_issued = true;
        const uint32_t sb = smem_addr(&s_bar);
        bar_expect_tx(sb, 2 * Sh::mat_bytes);
#pragma unroll
        for (int b = 0; b < Sh::boxes; ++b) {
          tma_load_2d(smem_addr(s_hi + b * Sh::mat_box), &map_s, 64 * b, 0, sb);  // S rows 0 .. W - 1: hi
          tma_load_2d(smem_addr(s_lo + b * Sh::mat_box), &map_s, 64 * b, W, sb);  // rows W .. 2 W - 1: lo
        }
      };
      int issued = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int slot = i % kJStages;
        if (i >= kJStages && !bar_wait(smem_addr(&empty_bar[slot]), ((i / kJStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        const bool is_k = i < my_k;
        const int row0 = tile_row0(i);
        const CUtensorMap *map = is_k ? &map_k : &map_v;
        const uint32_t fb = smem_addr(&full_bar[slot]);
        unsigned char *st = ring + slot * Sh::tile_bytes;
        bar_expect_tx(fb, Sh::tile_bytes);
#pragma unroll
        for (int b = 0; b < Sh::boxes; ++b) tma_load_2d(smem_addr(st + b * kBoxBytes), map, 64 * b, row0, fb);
        issued = i + 1;
        // S (hi, lo) is needed only by the second GEMM of the first K tile:
        // its copies queue behind the ring's first tiles
        if (i == min(kJStages, my_tiles) - 1) load_s();
      }
      if (!s_issued) load_s();  // (stopped early: S is still copied, and waited for below)
      bar_wait(smem_addr(&const_bar), 0);
      bar_wait(smem_addr(&s_bar), 0);
      if (*(volatile int *)&abort_flag)  // drain: never leave copies in flight
        for (int k = (issued > kJStages ? issued - kJStages : 0); k < issued; ++k)
          bar_wait(smem_addr(&full_bar[k % kJStages]), (k / kJStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer: MMA 1 of the
    // next tile whenever its X has landed and its group's tensor memory is
    // free, MMA 2 of the oldest K tile whose residuals are written
    if (lane == 0) {
      bool ok = bar_wait(smem_addr(&const_bar), 0);
      int n1 = 0, n2 = 0;
      bool s_ready = false;  // S hi and lo have landed (the second GEMM)
      unsigned long long t_last = global_ns();
      while (ok && n2 < my_k) {
        if (*(volatile int *)&abort_flag) break;
        bool progress = false;
        if (n1 < my_tiles) {
          const int slot = n1 % kJStages, g = n1 % kJGroups;
          if (bar_test(smem_addr(&full_bar[slot]), (n1 / kJStages) & 1) &&
              (n1 < kJGroups || bar_test(smem_addr(&tfree[g]), ((n1 / kJGroups) - 1) & 1))) {
            tc_fence_after();
            const uint32_t a0 = smem_addr(ring + slot * Sh::tile_bytes), b0 = smem_addr(pi_tile);
            const uint32_t d = tmem_base + g * 2 * W;
#pragma unroll
            for (int kk = 0; kk < W / 16; ++kk) {  // 16 elements along K per MMA
              const uint32_t ao = (kk >> 2) * kBoxBytes + (kk & 3) * 32, bo = (kk >> 2) * Sh::mat_box + (kk & 3) * 32;
              tc_mma_n(d, sw128_desc(a0 + ao), sw128_desc(b0 + bo), Sh::idesc_bf16, kk > 0);
            }
            tc_commit(smem_addr(&zfull[g]));
            tc_commit(smem_addr(&empty_bar[slot]));
            ++n1;
            progress = true;
          }
        }
        if (n2 < n1) {
          const int g = n2 % kJGroups;
          if (!s_ready) s_ready = bar_test(smem_addr(&s_bar), 0);
          if (s_ready && bar_test(smem_addr(&rfull[g]), (n2 / kJGroups) & 1)) {
            tc_fence_after();
            const uint32_t ra = tmem_base + g * 2 * W, d = ra + W;
            const uint32_t bh = smem_addr(s_hi), bl = smem_addr(s_lo);
#pragma unroll
            for (int kk = 0; kk < W / 16; ++kk) {
              const uint32_t off = (kk >> 2) * Sh::mat_box + (kk & 3) * 32;
              tc_mma_ts(d, ra + 16 * kk, sw128_desc(bh + off), Sh::idesc_f16, kk > 0);  // R_hi S_hi^T
              tc_mma_ts(d, ra + 16 * kk, sw128_desc(bl + off), Sh::idesc_f16, 1);       // R_hi S_lo^T
              tc_mma_ts(d, ra + 16 * kk + 8, sw128_desc(bh + off), Sh::idesc_f16, 1);   // R_lo S_hi^T
            }
            tc_commit(smem_addr(&sfull[g]));
            ++n2;
            progress = true;
          }
        }
        if (progress) {
          t_last = global_ns();
        } else {
          if (global_ns() - t_last > kWaitNs) ok = false;
          __nanosleep(32);
        }
      }
      // the V tiles need MMA 1 only
      for (int i = n1; ok && i < my_tiles; ++i) {
        const int slot = i % kJStages, g = i % kJGroups;
        ok = bar_wait(smem_addr(&full_bar[slot]), (i / kJStages) & 1);
        if (ok && i >= kJGroups) ok = bar_wait(smem_addr(&tfree[g]), ((i / kJGroups) - 1) & 1);
        if (!ok || *(volatile int *)&abort_flag) break;
        tc_fence_after();
        const uint32_t a0 = smem_addr(ring + slot * Sh::tile_bytes), b0 = smem_addr(pi_tile);
        const uint32_t d = tmem_base + g * 2 * W;
#pragma unroll
        for (int kk = 0; kk < W / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * kBoxBytes + (kk & 3) * 32, bo = (kk >> 2) * Sh::mat_box + (kk & 3) * 32;
          tc_mma_n(d, sw128_desc(a0 + ao), sw128_desc(b0 + bo), Sh::idesc_bf16, kk > 0);
        }
        tc_commit(smem_addr(&zfull[g]));
        tc_commit(smem_addr(&empty_bar[slot]));
      }
      if (!ok) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
      }
      // every MMA issued here has completed before the tensor memory is released
      tc_commit(smem_addr(&mma_done));
      bar_wait(smem_addr(&mma_done), 0);
    }
  } else {
    // ------------------------------------------------ epilogue: tile group g,
    // half h of every row (coordinates and projections W/2 h .. W/2 h + W/2 - 1)
    const int g = (warp - 2) / 8, h = ((warp - 2) / 4) & 1;
    const int quarter = warp & 3;       // TMEM lanes 32 quarter .. + 31
    const int r = 32 * quarter + lane;  // the row this thread shares
    constexpr int hk = 1 << (BK - 1), hv = 1 << (BV - 1);
    ResConsts<BK> rc;
    res_consts<BK>(a.p.cb, rc);
    CodeConsts<BK> kk;
    CodeConsts<BV> kv;
#pragma unroll
    for (int j = 0; j < hk - 1; ++j) kk.nt[j] = -a.p.cb[1 * kMaxLevels + hk + j] * 0x1p64f;  // positive thresholds x -2^64
#pragma unroll
    for (int j = 0; j < hv - 1; ++j) kv.nt[j] = -a.p.cb[3 * kMaxLevels + hv + j] * 0x1p64f;
    search_consts<BK>(kk);
    search_consts<BV>(kv);
    const uint32_t tz = tmem_base + g * 2 * W + (W / 2) * h + ((uint32_t)(32 * quarter) << 16);
    constexpr int kHalfChunks = W / 32;  // chunks of 16 coordinates per half row

    for (int j = 0, i = g; i < my_tiles; ++j, i += kJGroups) {
      const int slot = i % kJStages;
      const bool is_k = i < my_k;
      const int row = tile_row0(i) + r;
      // destination, loaded now and checked after the codes
      const bool in_range = row < a.n_rows;
      const int tok = in_range ? row / a.c.n_kv_heads : 0;
      const int tok_h = in_range ? row - tok * a.c.n_kv_heads : 0;
      const int s_dst = a.seq_idx ? a.seq_idx[tok] : 0, p_dst = a.pos ? a.pos[tok] : tok;
      if (!bar_wait(smem_addr(&full_bar[slot]), (i / kJStages) & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      // ||x|| from the swizzled tile (chunk c of row r sits at c ^ (r % 8));
      // bf16 squares are exact in fp32.  Both halves read the whole row.
      const unsigned char *st = ring + slot * Sh::tile_bytes;
      float2 ss = make_float2(0.f, 0.f);
#pragma unroll
      for (int box = 0; box < Sh::boxes; ++box)
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

      if (!bar_wait(smem_addr(&zfull[g]), j & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const bool live = nrm > 0x1p-25f;  // stored fp16 norm nonzero
      long slot_i = -1;
      if (in_range) {
        slot_i = cache_slot(a.c, s_dst, tok_h, p_dst);
        if (slot_i < 0 && tok_h == 0 && h == 0 && is_k) atomicOr(a.p.err, kErrTokenRange);
      }
      if (is_k) {
        // ---- epilogue A: codes, residuals, R into tensor memory
        kk.sc = live ? 0x1p64f / nrm : 0.f;
        kk.zc = live ? 0x1p127f : 0.f;
        const float rinv = live ? kRScale / nrm : 0.f;
        uint32_t words[4 * BK];
        float2 rr = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kHalfChunks; ++c) {
          float z[16];
          tmem_ld16(tz + 16 * c, z);
          float off[16];
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float2 o2, r2;
            code_res2<BK>(z[2 * e], z[2 * e + 1], kk, rc, rinv, o2, r2);
            off[2 * e] = o2.x;
            off[2 * e + 1] = o2.y;
            rr = fma2(r2, r2, rr);
            split_f16x2(r2.x, r2.y, hi[e], lo[e]);
          }
          code_chunk_off<BK>(c, off, words);
          tmem_st8(tz + 16 * c, hi);
          tmem_st8(tz + 16 * c + 8, lo);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(smem_addr(&rfull[g]));
        // ||r||^2 of the row from both halves (the group's eight warps meet on
        // rr_bar; double-buffered by tile parity, so a half never overwrites a
        // value its partner has yet to read)
        s_rr[g][j & 1][h][r] = rr.x + rr.y;
        __syncwarp();
        if (lane == 0) bar_arrive(smem_addr(&rr_bar[g]));
        if (!bar_wait(smem_addr(&rr_bar[g]), j & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        const float rr_row = s_rr[g][j & 1][0][r] + s_rr[g][j & 1][1][r];

        // ---- epilogue B: the signs of S r
        if (!bar_wait(smem_addr(&sfull[g]), j & 1)) {  // K tiles are a prefix: j K tiles before
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        uint32_t sb[2] = {0u, 0u};  // bit n of the row = [(S r)_n >= 0], LSB first, n = W/2 h ..
#pragma unroll
        for (int c = 0; c < kHalfChunks; ++c) {
          float v[16];
          tmem_ld16(tz + W + 16 * c, v);
          uint32_t b = 0;
#pragma unroll
          for (int e = 0; e < 16; ++e) b |= (v[e] >= 0.f ? 1u : 0u) << e;
          sb[c >> 1] |= b << (16 * (c & 1));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(smem_addr(&tfree[g]));

        if (slot_i >= 0) {
          // the half row's code groups: W/16 BK bytes from byte W/16 BK h of the row
          store_half_codes<W, BK>(a.c.codes_k + slot_i * (long)(W / 8 * BK) + W / 16 * BK * h, words);
          if constexpr (W == 128) reinterpret_cast<uint2 *>(a.c.qjl_bits + slot_i * 16)[h] = make_uint2(sb[0], sb[1]);
          else reinterpret_cast<uint32_t *>(a.c.qjl_bits + slot_i * (W / 8))[h] = sb[0];
          if (h == 0) {
            a.c.norm_k[slot_i] = __half_as_ushort(__float2half_rn(fminf(nrm, 65504.f)));
            const float gamma = sqrtf(rr_row) * (1.f / kRScale);
            a.c.qjl_norm[slot_i] = __half_as_ushort(__float2half_rn(fminf(gamma, 65504.f)));
          }
        }
      } else {
        // ---- V: codes only
        kv.sc = live ? 0x1p64f / nrm : 0.f;
        kv.zc = live ? 0x1p127f : 0.f;
        uint32_t words[4 * BV];
#pragma unroll
        for (int c = 0; c < kHalfChunks; ++c) {
          float z[16];
          tmem_ld16(tz + 16 * c, z);
          code_chunk<BV>(c, z, kv, words);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(smem_addr(&tfree[g]));
        if (slot_i >= 0) {
          store_half_codes<W, BV>(a.c.codes_v + slot_i * (long)(W / 8 * BV) + W / 16 * BV * h, words);
          if (h == 0) a.c.norm_v[slot_i] = __half_as_ushort(__float2half_rn(fminf(nrm, 65504.f)));
        }
      }
      if (*(volatile int *)&abort_flag) break;
    }
  }

  // release tensor memory once every MMA and every tensor-memory access is finished
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Sh::tmem_cols)
                 : "memory");
  }
}

using QjlTcFn = void (*)(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                         const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, const QjlTcArgs);

template <int W, int BK>
QjlTcFn pick_bv(int bv) {
  return bv == 2 ? quantize_qjl_tc_kernel<W, BK, 2> : bv == 3 ? quantize_qjl_tc_kernel<W, BK, 3>
                                                               : quantize_qjl_tc_kernel<W, BK, 4>;
}

template <int W>
QjlTcFn pick(int bk, int bv) {
  return bk == 2 ? pick_bv<W, 2>(bv) : bk == 3 ? pick_bv<W, 3>(bv) : pick_bv<W, 4>(bv);
}

}  // namespace

int launch_quantize_qjl_tc(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                           const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream) {
  // cached per device (the attribute applies to the current device), and
  // atomically, as calls may come from several threads
  static std::atomic<int> cached_sm[kMaxDevices];
  if (p.d != 64 && p.d != kHeadDim) return (int)cudaErrorInvalidValue;
  const int W = p.d;
  static std::atomic<bool> configured[kMaxDevices][2][3][3];
  const int dev = current_device();
  int n_sm = cached_sm[dev].load(std::memory_order_relaxed);
  if (n_sm == 0) {
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
    cached_sm[dev].store(n_sm, std::memory_order_relaxed);
  }
  const QjlTcFn fn = W == 64 ? pick<64>(p.bits_k, p.bits_v) : pick<kHeadDim>(p.bits_k, p.bits_v);
  const int smem = W == 64 ? JShape<64>::smem : JShape<kHeadDim>::smem;
  std::atomic<bool> &done = configured[dev][W == 64 ? 0 : 1][p.bits_k - 2][p.bits_v - 2];
  if (!done.load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    done.store(true, std::memory_order_release);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  CUtensorMap mk, mv, mp, ms;
  const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_row_map(&mk, k, rows, bf16, W) || !make_row_map(&mv, v, rows, bf16, W) ||
      !make_row_map(&mp, p.pi, W, bf16, W, W) ||
      !make_row_map(&ms, p.ssplit, 2 * W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, W, W))
    return (int)cudaErrorInvalidValue;
  QjlTcArgs args{p, c, seq_idx, pos, (int)rows, (int)((rows + kTileRows - 1) / kTileRows)};
  const int n_tiles = 2 * args.tiles_k;
  const int grid = n_tiles < n_sm ? n_tiles : n_sm;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kJThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, mk, mv, mp, ms, args);
}

}  // namespace tq
