// Quantize-on-append in tiles for head dimension 64 (sm_100a): the method's
// norm, rotation by Pi and Lloyd-Max codes ("ステップ1: PolarQuant",
// ai-accelerate.xyz TurboQuant explainer) for the K rows without QJL and for
// every V row, 64 vectors per CTA tile.
//
// Each of the four warps takes 16 rows (one m16 tile):
//   z = X Pi^T     mma m16n8k16 bf16 (X and Pi are bf16: exact products,
//                  fp32 sums), ||x|| from the same X fragments;
//   codes          #{j : t_j < z / ||x||} against the positive thresholds
//                  scaled by ||x|| (the symmetric codebook), into shared
//                  memory;
//   store          the packed 32-code groups of every row (thread q of a
//                  quad packs groups q, q + 4, ...), the fp16 norm.
// Pi's B-fragment table (8 KB) is copied once per CTA into shared memory.
// The kernel is persistent: tiles are strided over the grid.  d = 128 and
// d = 256 use the tcgen05 kernels instead.
#include <atomic>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

// warps per CTA (16 rows each)
template <int DH>
__host__ __device__ constexpr int tile_warps() { return 4; }

__device__ __forceinline__ void mma_bf16_t(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int B>
__device__ __forceinline__ int tile_code(float z, const float (&tp)[(1 << (B - 1)) - 1]) {
  constexpr int half = 1 << (B - 1);
  const float a = fabsf(z);
  int m = 0;
#pragma unroll
  for (int j = 0; j < half - 1; ++j) m += a > tp[j] ? 1 : 0;
  return z > 0.f ? half + m : half - 1 - m;
}

// Word k of the packed 32-code group `cd` (the cache layout: LSB-first for 2
// and 4 bits; nibbles plus the spare column for 3 bits).
template <int B>
__device__ __forceinline__ uint32_t tile_pack_word(const uint8_t *cd, int k) {
  uint32_t x = 0;
  if constexpr (B == 3) {
#pragma unroll
    for (int j = 0; j < 8; ++j) x |= (uint32_t)cd[8 * k + j] << (4 * j);
#pragma unroll
    for (int j = 0; j < 8; ++j) x |= (((uint32_t)cd[24 + j] >> k) & 1u) << (4 * j + 3);
  } else {
#pragma unroll
    for (int j = 0; j < 32 / B; ++j) x |= (uint32_t)cd[(32 / B) * k + j] << (B * j);
  }
  return x;
}

template <int B, int DH>
__global__ void __launch_bounds__(32 * tile_warps<DH>()) quantize_tile_kernel(DeviceParams p, tq_cache c,
                                                                     const uint16_t *__restrict__ x_in,
                                                                     const int32_t *__restrict__ seq_idx,
                                                                     const int32_t *__restrict__ pos, int n_rows,
                                                                     int is_v) {
  constexpr int half = 1 << (B - 1);
  constexpr int NT = DH / 8;      // n-tiles of z
  constexpr int KS = DH / 16;     // k-steps
  constexpr int CH = DH / 32;     // 16-byte chunks per lane per n-tile in the fragment table
  constexpr int kTWarps = tile_warps<DH>();
  constexpr int kTRows = 16 * kTWarps;  // rows per tile
  extern __shared__ __align__(16) uint4 s_pif[];  // Pi fragments
  __shared__ __align__(16) uint8_t s_code[kTRows][DH + 4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = lane >> 2, q = lane & 3;
  const float *thr = p.cb + (is_v ? 3 : 1) * kMaxLevels;
  float tpos[half - 1];
#pragma unroll
  for (int j = 0; j < half - 1; ++j) tpos[j] = thr[half + j];
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(p.pif);
    for (int i = tid; i < NT * CH * 32; i += 32 * kTWarps) s_pif[i] = src[i];
  }
  const uint4 *pif = s_pif;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncthreads();
  uint8_t *codes = is_v ? c.codes_v : c.codes_k;
  uint16_t *norms = is_v ? c.norm_v : c.norm_k;

  const int n_tiles = (n_rows + kTRows - 1) / kTRows;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const long row0 = (long)tile * kTRows + 16 * warp;
    const long rows[2] = {row0 + r, row0 + r + 8};
    uint32_t a[KS][4];
    float ss[2] = {0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long row = rows[e & 1];
        const int col = 16 * ks + 8 * (e >> 1) + 2 * q;
        const uint32_t w = row < n_rows ? *reinterpret_cast<const uint32_t *>(x_in + row * DH + col) : 0u;
        a[ks][e] = w;
        const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
        ss[e & 1] = fmaf(lo, lo, fmaf(hi, hi, ss[e & 1]));  // bf16 squares are exact in fp32
      }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      ss[e] += __shfl_xor_sync(0xffffffffu, ss[e], 1);
      ss[e] += __shfl_xor_sync(0xffffffffu, ss[e], 2);
    }
    const float nrm[2] = {sqrtf(ss[0]), sqrtf(ss[1])};
    // a vector whose stored fp16 norm is zero (||x|| <= 2^-25) is the zero vector
    const bool live[2] = {nrm[0] > 0x1p-25f, nrm[1] > 0x1p-25f};
    float tp[2][half - 1];
#pragma unroll
    for (int j = 0; j < half - 1; ++j) {
      tp[0][j] = tpos[j] * nrm[0];
      tp[1][j] = tpos[j] * nrm[1];
    }
    // z = X Pi^T, eight n-tiles at a time (independent accumulators between
    // consecutive MMAs), codes straight into shared memory
#pragma unroll
    for (int g = 0; g < NT / 8; ++g) {
      float z[8][4];
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) z[t][e] = 0.f;
#pragma unroll
      for (int j = 0; j < CH; ++j)
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint4 v = pif[((8 * g + t) * CH + j) * 32 + lane];
          mma_bf16_t(z[t], a[2 * j], v.x, v.y);
          mma_bf16_t(z[t], a[2 * j + 1], v.z, v.w);
        }
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {  // 0: row r, 1: row r + 8; columns 8 nt + 2 q and + 1
          const int c0 = tile_code<B>(live[hr] ? z[t][2 * hr] : 0.f, tp[hr]);
          const int c1 = tile_code<B>(live[hr] ? z[t][2 * hr + 1] : 0.f, tp[hr]);
          *reinterpret_cast<uint16_t *>(&s_code[16 * warp + r + 8 * hr][8 * (8 * g + t) + 2 * q]) =
              (uint16_t)(c0 | (c1 << 8));
        }
    }
    __syncwarp();  // this warp's code rows are complete
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const long row = rows[e];
      if (row >= n_rows) continue;
      const int tok = (int)(row / c.n_kv_heads), h = (int)(row - (long)tok * c.n_kv_heads);
      const long slot = cache_slot(c, seq_idx ? seq_idx[tok] : 0, h, pos ? pos[tok] : tok);
      if (slot < 0) {
        if (q == 0 && h == 0 && !is_v) atomicOr(p.err, kErrTokenRange);
        continue;
      }
      uint32_t *dst = reinterpret_cast<uint32_t *>(codes + slot * (DH * B / 8));
      for (int gr = q; gr < DH / 32; gr += 4) {
        const uint8_t *cd = &s_code[16 * warp + r + 8 * e][32 * gr];
#pragma unroll
        for (int k = 0; k < B; ++k) dst[B * gr + k] = tile_pack_word<B>(cd, k);
      }
      if (q == 0) norms[slot] = __half_as_ushort(__float2half_rn(fminf(nrm[e], 65504.f)));
    }
    __syncwarp();  // this warp's code rows are read before the next tile writes them
  }
}

using TileFn = void (*)(DeviceParams, tq_cache, const uint16_t *, const int32_t *, const int32_t *, int, int);

template <int DH>
TileFn pick_tile(int bits) {
  return bits == 2 ? quantize_tile_kernel<2, DH> : bits == 3 ? quantize_tile_kernel<3, DH> : quantize_tile_kernel<4, DH>;
}

}  // namespace

int launch_quantize_tile(const DeviceParams &p, const tq_cache &c, const void *x, const int32_t *seq_idx,
                         const int32_t *pos, int n_tok, bool is_v, void *stream) {
  const int bits = is_v ? p.bits_v : p.bits_k;
  if (p.d != 64) return (int)cudaErrorInvalidValue;  // d = 64 only
  const TileFn fn = pick_tile<64>(bits);
  const int warps = tile_warps<64>();
  const int smem = (p.d / 8) * (p.d / 32) * 32 * 16;  // the fragment table
  // resident CTAs on the device, cached per device and width
  static std::atomic<int> slots[kMaxDevices][3];
  const int dev = current_device();
  std::atomic<int> &slot = slots[dev][bits - 2];
  int n_slots = slot.load(std::memory_order_relaxed);
  if (n_slots == 0) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    int n_sm = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 32 * warps, smem) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    n_slots = n_sm * per_sm;
    slot.store(n_slots, std::memory_order_relaxed);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  const long tiles = (rows + 16 * warps - 1) / (16 * warps);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles < n_slots ? tiles : n_slots));
  cfg.blockDim = dim3(32 * warps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, p, c, static_cast<const uint16_t *>(x), seq_idx, pos, (int)rows,
                                 is_v ? 1 : 0);
}

}  // namespace tq
