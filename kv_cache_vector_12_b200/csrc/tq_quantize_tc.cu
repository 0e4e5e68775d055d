// Quantize-on-append on the 5th-generation tensor cores (sm_100a).
//
// "ステップ1: PolarQuant" (ai-accelerate.xyz TurboQuant explainer): every
// head vector x is rotated by the random orthogonal matrix Pi and each rotated
// coordinate is quantized with the Lloyd-Max codebook.  Here the rotation of
// a tile of 128 head vectors is one 128 x d x d bf16 GEMM, z = X Pi^T, for
// head dimension d = 128 or 64 (d = 256 has its own kernel):
//
//   producer warp   TMA (cp.async.bulk.tensor, 128-byte swizzle) loads each
//                   128-row tile of K or V into a 4-deep shared-memory ring;
//                   Pi stays resident in shared memory for the CTA's lifetime.
//   MMA warp        one thread issues d / 16 tcgen05.mma (kind::f16, bf16
//                   inputs, fp32 accumulation in tensor memory) per tile and
//                   commits to mbarriers.
//   4 epilogue      warpgroups, one TMEM accumulator each; every thread owns
//   warpgroups      one row (vector): ||x|| from the shared-memory tile,
//                   z from TMEM (tcgen05.ld 32x32b), codes against the
//                   thresholds scaled by ||x||, bit-packing into the cache
//                   layout, 16-byte stores, fp16 norm.
//
// The kernel is persistent (one CTA per SM, tiles strided by the grid).  Every
// mbarrier wait is bounded; on expiry the kernel flags the error, stops, waits
// for its copies and MMAs in flight (bounded) and releases its tensor memory.

#include <atomic>
#include <cmath>
#include <cstring>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"
#include "tq_tc.cuh"

namespace tq {
namespace {

constexpr int kRingStages = 4;
constexpr int kEpiGroups = 4;
constexpr int kQThreads = 32 * (2 + 4 * kEpiGroups);

// The shapes that depend on the head dimension W: a tile is W / 64 boxes of
// 128 rows x 64 coordinates, Pi W / 64 boxes of W rows.
template <int W>
struct TcShape {
  static constexpr int boxes = W / 64;
  static constexpr int tile_bytes = kTileRows * W * 2;
  static constexpr int pi_bytes = W * W * 2;
  static constexpr int pi_box = W * 128;
  static constexpr unsigned tmem_cols = kEpiGroups * W;  // one accumulator of W columns per group
  // instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both K-major, N = W, M = 128
  static constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(W >> 3) << 17) | ((128u >> 4) << 24);
  static constexpr int smem = 1024 + pi_bytes + kRingStages * tile_bytes;
};


struct QuantTcArgs {
  DeviceParams p;
  tq_cache c;
  const int32_t *seq_idx;
  const int32_t *pos;
  int n_rows;       // n_tok * n_kv_heads rows per matrix
  int tiles_k;      // tiles of K handled here (0 when K goes elsewhere)
  int tiles_v;
};



template <int W, int BK, int BV>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                       const __grid_constant__ CUtensorMap map_pi, const QuantTcArgs a) {
  using Sh = TcShape<W>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned region: Pi then the ring
  unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char *pi_tile = smem;
  unsigned char *ring = smem + Sh::pi_bytes;
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
                 "r"(Sh::tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  if (warp == 0 && lane == 0) {  // Pi belongs to the context: no earlier kernel writes it
    const uint32_t pb = smem_addr(&pi_bar);
    bar_expect_tx(pb, Sh::pi_bytes);
#pragma unroll
    for (int b = 0; b < Sh::boxes; ++b) tma_load_2d(smem_addr(pi_tile + b * Sh::pi_box), &map_pi, 64 * b, 0, pb);
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
        unsigned char *st = ring + slot * Sh::tile_bytes;
        bar_expect_tx(fb, Sh::tile_bytes);
#pragma unroll
        for (int b = 0; b < Sh::boxes; ++b) tma_load_2d(smem_addr(st + b * kBoxBytes), map, 64 * b, row0, fb);
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
        const uint32_t a0 = smem_addr(ring + slot * Sh::tile_bytes), b0 = smem_addr(pi_tile);
        const uint32_t d = tmem_base + acc * W;
#pragma unroll
        for (int kk = 0; kk < W / 16; ++kk) {  // 16 bf16 along K per MMA
          const uint32_t ao = (kk >> 2) * kBoxBytes + (kk & 3) * 32, bo = (kk >> 2) * Sh::pi_box + (kk & 3) * 32;
          tc_mma_n(d, sw128_desc(a0 + ao), sw128_desc(b0 + bo), Sh::idesc, kk > 0);
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
      const unsigned char *st = ring + slot * Sh::tile_bytes;
      float2 ss = make_float2(0.f, 0.f);  // sums of the squares of the low and the high halves
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

      if (!bar_wait(smem_addr(&tfull_bar[g]), j & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t trow = tmem_base + g * W + ((uint32_t)(32 * quarter) << 16);
      constexpr int C = W / 16;  // chunks of 16 columns; C / 2 * bits words per row
      uint32_t words[C / 2 * 4];
      if constexpr (BK == BV) {  // one copy of the epilogue code for K and V tiles
        float thr[kMaxLevels];
#pragma unroll
        for (int e = 0; e < kMaxLevels; ++e) thr[e] = is_k ? tk[e] : tv[e];
        uint32_t w[C / 2 * BK];
        epilogue_row<BK, C>(thr, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < C / 2 * BK; ++e) words[e] = w[e];
      } else if (is_k) {
        uint32_t w[C / 2 * BK];
        epilogue_row<BK, C>(tk, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < C / 2 * BK; ++e) words[e] = w[e];
      } else {
        uint32_t w[C / 2 * BV];
        epilogue_row<BV, C>(tv, nrm, trow, w);
#pragma unroll
        for (int e = 0; e < C / 2 * BV; ++e) words[e] = w[e];
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
        const int bits = is_k ? BK : BV;  // W / 8 * bits bytes per row
        unsigned char *row_dst = (is_k ? a.c.codes_k : a.c.codes_v) + slot_i * (long)(W / 8 * bits);
        if constexpr (W == 128) {
          uint4 *dst = reinterpret_cast<uint4 *>(row_dst);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < bits) dst[q] = make_uint4(words[4 * q], words[4 * q + 1], words[4 * q + 2], words[4 * q + 3]);
        } else {
          uint2 *dst = reinterpret_cast<uint2 *>(row_dst);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < bits) dst[q] = make_uint2(words[2 * q], words[2 * q + 1]);
        }
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(Sh::tmem_cols)
                 : "memory");
  }
}


using QuantTcFn = void (*)(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                           const __grid_constant__ CUtensorMap, const QuantTcArgs);

template <int W, int BK>
QuantTcFn pick_bv(int bv) {
  return bv == 2 ? quantize_tc_kernel<W, BK, 2> : bv == 3 ? quantize_tc_kernel<W, BK, 3> : quantize_tc_kernel<W, BK, 4>;
}

template <int W>
QuantTcFn pick(int bk, int bv) {
  return bk == 2 ? pick_bv<W, 2>(bv) : bk == 3 ? pick_bv<W, 3>(bv) : pick_bv<W, 4>(bv);
}

}  // namespace

int launch_quantize_tc(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                       const int32_t *seq_idx, const int32_t *pos, int n_tok, bool include_k, bool include_v,
                       void *stream) {
  if (p.d != 64 && p.d != kHeadDim) return (int)cudaErrorInvalidValue;
  const int W = p.d;
  // cached per device (the attribute applies to the current device), and
  // atomically, as calls may come from several threads
  static std::atomic<int> cached_sm[kMaxDevices];
  static std::atomic<bool> configured[kMaxDevices][2][3][3];
  const int dev = current_device();
  int n_sm = cached_sm[dev].load(std::memory_order_relaxed);
  if (n_sm == 0) {
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
    cached_sm[dev].store(n_sm, std::memory_order_relaxed);
  }
  const QuantTcFn fn = W == 64 ? pick<64>(p.bits_k, p.bits_v) : pick<kHeadDim>(p.bits_k, p.bits_v);
  const int smem = W == 64 ? TcShape<64>::smem : TcShape<kHeadDim>::smem;
  std::atomic<bool> &done = configured[dev][W == 64 ? 0 : 1][p.bits_k - 2][p.bits_v - 2];
  if (!done.load(std::memory_order_acquire)) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    done.store(true, std::memory_order_release);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  const CUtensorMapDataType bf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mk, mv, mp;
  std::memset(&mk, 0, sizeof mk);
  std::memset(&mv, 0, sizeof mv);
  if ((include_v && !make_row_map(&mv, v, rows, bf16, W)) || !make_row_map(&mp, p.pi, W, bf16, W, W) ||
      (include_k && !make_row_map(&mk, k, rows, bf16, W)))
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
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, mk, mv, mp, args);
}

}  // namespace tq
