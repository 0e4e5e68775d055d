// Quantize-on-append for head dimension 256 on the 5th-generation tensor
// cores (sm_100a): the method's norm, rotation by Pi and Lloyd-Max codes
// ("ステップ1: PolarQuant", ai-accelerate.xyz TurboQuant explainer) for every
// V row and the K rows without QJL.
//
// Per tile of 128 vectors, z = X Pi^T is one tcgen05 GEMM with M = 128 and
// N = 256 over 16 steps of K = 16 (bf16 operands, fp32 accumulator of 256
// columns in tensor memory):
//   producer warp   TMA (128-byte swizzle) loads each tile as two K halves
//                   (128 rows x 128 coordinates, 32 KB) into a 3-deep ring;
//                   Pi (256 x 256 bf16, 128 KB) stays resident in shared
//                   memory as four 256-row boxes of 64 coordinates.
//   MMA warp        one thread issues the 16 MMAs of a tile into the
//                   accumulator of its tile group and commits.
//   epilogue        two tile groups (alternate tiles, one accumulator each)
//                   of two warpgroups; thread (row, half) reads ||x|| over the
//                   whole row from the shared-memory tile, the row's 128
//                   accumulator columns of its half from tensor memory, and
//                   packs their codes (the exact saturating-FMA search of the
//                   d = 128 kernel) into the cache layout.
// The kernel is persistent (one CTA per SM, tiles strided by the grid).  Every
// mbarrier wait is bounded; on expiry the kernel flags the error, stops, waits
// for its copies and MMAs in flight (bounded) and releases its tensor memory.
#include <atomic>
#include <cstring>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"
#include "tq_tc.cuh"

namespace tq {
namespace {

constexpr int kW = 256;                             // the head dimension of this kernel
constexpr int kHalfStages = 3;                      // ring of K halves
constexpr int kHalfBytes = kTileRows * 128 * 2;     // 32 KB: two 128 x 64 boxes
constexpr int kHalfBox = kHalfBytes / 2;
constexpr int kPiBox = kW * 64 * 2;                 // 32 KB: Pi rows 0..255, 64 input coordinates
constexpr int kPiBytes = 4 * kPiBox;                // 128 KB
constexpr int kThreads256 = 32 * (2 + 16);          // producer, MMA issuer, 2 tile groups x 2 halves x 4 warps
constexpr unsigned kTmemCols256 = 512;              // two accumulators of 256 columns
constexpr int kSmem256 = 1024 + kPiBytes + kHalfStages * kHalfBytes;

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc256 = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma256(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "l"(a), "l"(b), "r"(kIdesc256), "r"(accumulate)
               : "memory");
}

struct Quant256Args {
  DeviceParams p;
  tq_cache c;
  const int32_t *seq_idx;
  const int32_t *pos;
  int n_rows;   // n_tok * n_kv_heads rows per matrix
  int tiles_k;  // tiles of K handled here (0 when K goes elsewhere)
  int tiles_v;
};

template <int BK, int BV>
__global__ void __launch_bounds__(kThreads256, 1)
    quantize_tc256_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                          const __grid_constant__ CUtensorMap map_pi, const Quant256Args a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char *pi = smem;               // four 256-row boxes
  unsigned char *ring = smem + kPiBytes;  // K halves
  __shared__ __align__(8) uint64_t full_bar[kHalfStages], empty_bar[kHalfStages];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], pi_bar, mma_done;
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.tiles_k + a.tiles_v;
  const int bx = (int)blockIdx.x, grid = (int)gridDim.x;
  const int my_tiles = bx < n_tiles ? (n_tiles - 1 - bx) / grid + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kHalfStages; ++i) {
      bar_init(smem_addr(&full_bar[i]), 1);
      bar_init(smem_addr(&empty_bar[i]), 1 + 8);  // MMA commit + the tile group's 8 norm-reading warps
    }
    for (int g = 0; g < 2; ++g) {
      bar_init(smem_addr(&tfull_bar[g]), 1);
      bar_init(smem_addr(&tempty_bar[g]), 8);
    }
    bar_init(smem_addr(&pi_bar), 1);
    bar_init(smem_addr(&mma_done), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the MMA warp owns the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_base_slot)),
                 "r"(kTmemCols256)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_slot;
  if (warp == 0 && lane == 0) {  // Pi belongs to the context: no earlier kernel writes it
    const uint32_t pb = smem_addr(&pi_bar);
    bar_expect_tx(pb, kPiBytes);
    for (int kb = 0; kb < 4; ++kb) tma_load_2d(smem_addr(pi + kb * kPiBox), &map_pi, 64 * kb, 0, pb);
  }
  // launched as a programmatic dependent: inputs and the cache are touched
  // only once the previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------ producer (TMA): half
    // hh of tile i is ring entry 2 i + hh
    if (lane == 0) {
      int issued = 0;
      for (int e = 0; e < 2 * my_tiles; ++e) {
        const int slot = e % kHalfStages;
        if (e >= kHalfStages && !bar_wait(smem_addr(&empty_bar[slot]), ((e / kHalfStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        const int t = bx + (e >> 1) * grid, hh = e & 1;
        const bool is_k = t < a.tiles_k;
        const CUtensorMap *map = is_k ? &map_k : &map_v;
        const int row0 = (is_k ? t : t - a.tiles_k) * kTileRows;
        const uint32_t fb = smem_addr(&full_bar[slot]);
        unsigned char *st = ring + slot * kHalfBytes;
        bar_expect_tx(fb, kHalfBytes);
        tma_load_2d(smem_addr(st), map, 128 * hh, row0, fb);
        tma_load_2d(smem_addr(st + kHalfBox), map, 128 * hh + 64, row0, fb);
        issued = e + 1;
      }
      bar_wait(smem_addr(&pi_bar), 0);
      if (*(volatile int *)&abort_flag)  // drain: never leave copies in flight
        for (int k = (issued > kHalfStages ? issued - kHalfStages : 0); k < issued; ++k)
          bar_wait(smem_addr(&full_bar[k % kHalfStages]), (k / kHalfStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = bar_wait(smem_addr(&pi_bar), 0);
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int g = i & 1;
        if (i >= 2) ok = bar_wait(smem_addr(&tempty_bar[g]), ((i >> 1) - 1) & 1);
        if (!ok || *(volatile int *)&abort_flag) break;
        const uint32_t d = tmem_base + 256 * g;
        for (int hh = 0; ok && hh < 2; ++hh) {
          const int e = 2 * i + hh, slot = e % kHalfStages;
          ok = bar_wait(smem_addr(&full_bar[slot]), (e / kHalfStages) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = smem_addr(ring + slot * kHalfBytes), b0 = smem_addr(pi);
#pragma unroll
          for (int kl = 0; kl < 8; ++kl) {
            const int kk = 8 * hh + kl;  // 16 input coordinates per MMA
            const uint32_t aoff = (kl >> 2) * kHalfBox + (kl & 3) * 32;
            const uint32_t boff = (kk >> 2) * kPiBox + (kk & 3) * 32;
            tc_mma256(d, sw128_desc(a0 + aoff), sw128_desc(b0 + boff), kk > 0);
          }
          tc_commit(smem_addr(&empty_bar[slot]));
        }
        if (ok) tc_commit(smem_addr(&tfull_bar[g]));
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
    // half h of every row's coordinates (128 h .. 128 h + 127)
    const int ew = warp - 2;
    const int g = ew >> 3, h = (ew >> 2) & 1;
    const int quarter = warp & 3;       // TMEM lanes 32 quarter .. + 31
    const int r = 32 * quarter + lane;  // the row this thread shares
    float tk[kMaxLevels], tv[kMaxLevels];
#pragma unroll
    for (int e = 0; e < kMaxLevels; ++e) {
      tk[e] = a.p.cb[1 * kMaxLevels + e];
      tv[e] = a.p.cb[3 * kMaxLevels + e];
    }
    const uint32_t trow = tmem_base + 256 * g + 128 * h + ((uint32_t)(32 * quarter) << 16);
    for (int j = 0, i = g; i < my_tiles; ++j, i += 2) {
      const int t = bx + i * grid;
      const bool is_k = t < a.tiles_k;
      const int row = (is_k ? t : t - a.tiles_k) * kTileRows + r;
      // destination of this row: loaded now, checked after the codes
      const bool live_row = row < a.n_rows;
      const int tok = live_row ? row / a.c.n_kv_heads : 0;
      const int tok_h = live_row ? row - tok * a.c.n_kv_heads : 0;
      const int s_dst = a.seq_idx ? a.seq_idx[tok] : 0, p_dst = a.pos ? a.pos[tok] : tok;
      // ||x|| over both K halves of the row (chunk c of row r sits at
      // c ^ (r % 8)); bf16 squares are exact in fp32
      float2 ss = make_float2(0.f, 0.f);
      bool ok = true;
      for (int hh = 0; ok && hh < 2; ++hh) {
        const int e = 2 * i + hh, slot = e % kHalfStages;
        ok = bar_wait(smem_addr(&full_bar[slot]), (e / kHalfStages) & 1);
        if (!ok) break;
        const unsigned char *st = ring + slot * kHalfBytes;
#pragma unroll
        for (int box = 0; box < 2; ++box)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 u = *reinterpret_cast<const uint4 *>(st + box * kHalfBox + r * 128 + ((ch ^ (r & 7)) * 16));
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 x = make_float2(__uint_as_float(w4[q] << 16), __uint_as_float(w4[q] & 0xffff0000u));
              ss = fma2(x, x, ss);
            }
          }
        __syncwarp();
        if (lane == 0) bar_arrive(smem_addr(&empty_bar[slot]));
      }
      if (ok) ok = bar_wait(smem_addr(&tfull_bar[g]), j & 1);
      if (!ok) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const float nrm = sqrtf(ss.x + ss.y);
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
      if (live_row) {
        slot_i = cache_slot(a.c, s_dst, tok_h, p_dst);
        if (slot_i < 0 && tok_h == 0 && is_k && h == 0) atomicOr(a.p.err, kErrTokenRange);
      }
      if (slot_i >= 0) {
        const int bits = is_k ? BK : BV;
        // groups 4 h .. 4 h + 3 of the row: 16 bits bytes from byte 16 bits h
        uint4 *dst = reinterpret_cast<uint4 *>((is_k ? a.c.codes_k : a.c.codes_v) + slot_i * (long)(32 * bits) +
                                               16 * bits * h);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < bits) dst[q] = make_uint4(words[4 * q], words[4 * q + 1], words[4 * q + 2], words[4 * q + 3]);
        if (h == 0)
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols256)
                 : "memory");
  }
}

// 2-D map over a row-major [rows][256] bf16 matrix, boxes of `box_rows` rows
// x 64 columns (128 bytes) with the 128-byte swizzle.
bool make_map256(CUtensorMap *m, const void *base, long rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kW, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kW * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using Quant256Fn = void (*)(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                            const __grid_constant__ CUtensorMap, const Quant256Args);

template <int BK>
Quant256Fn pick256_bv(int bv) {
  return bv == 2 ? quantize_tc256_kernel<BK, 2> : bv == 3 ? quantize_tc256_kernel<BK, 3> : quantize_tc256_kernel<BK, 4>;
}

}  // namespace

int launch_quantize_tc256(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
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
  const Quant256Fn fn = p.bits_k == 2 ? pick256_bv<2>(p.bits_v) : p.bits_k == 3 ? pick256_bv<3>(p.bits_v)
                                                                               : pick256_bv<4>(p.bits_v);
  std::atomic<bool> &done = configured[dev][p.bits_k - 2][p.bits_v - 2];
  if (!done.load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem256);
    if (e != cudaSuccess) return (int)e;
    done.store(true, std::memory_order_release);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  CUtensorMap mk, mv, mp;
  std::memset(&mk, 0, sizeof mk);
  std::memset(&mv, 0, sizeof mv);
  if ((include_v && !make_map256(&mv, v, rows, kTileRows)) || !make_map256(&mp, p.pi, kW, kW) ||
      (include_k && !make_map256(&mk, k, rows, kTileRows)))
    return (int)cudaErrorInvalidValue;
  if (!include_k) mk = mv;
  if (!include_v) mv = mk;
  Quant256Args args{p, c, seq_idx, pos, (int)rows, 0, 0};
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
  cfg.blockDim = dim3(kThreads256);
  cfg.dynamicSmemBytes = kSmem256;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, mk, mv, mp, args);
}

}  // namespace tq
