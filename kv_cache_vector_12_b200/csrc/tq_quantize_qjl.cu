// Quantize-on-append of K with the 1-bit QJL residual stage, in tiles on the
// tensor cores (sm_100a).
//
// The method ("ステップ2: QJL", ai-accelerate.xyz TurboQuant explainer; the
// residual 1-bit QJL transform of "Tether QVACのTurboQuant実装", qxai.app):
// after the rotation and the Lloyd-Max codes, the residual r = y - c[code] of
// each K vector is projected by a Gaussian matrix S and only the signs of
// S r are kept, with ||r||, so that the score's residual term can be
// estimated without bias.
//
// One CTA of four warps takes 64 K rows (16 per warp, one m16 tile):
//   z = X Pi^T     mma m16n8k16 bf16 (X and Pi are bf16: exact products,
//                  fp32 sums), ||x|| from the same X fragments;
//   codes, y = z / ||x||, r = y - c[code], ||r||;
//   S r            the residual goes from the accumulator fragments straight
//                  into the A fragments of the second product (the k-steps
//                  are the accumulators' column pairs); r 2^14 and S 2^sigma
//                  are each split into two fp16 parts (22 significant bits;
//                  the power-of-two scales keep the low parts out of fp16's
//                  subnormal range and do not change a sign), and the three
//                  products hi hi, hi lo, lo hi give S r to within about
//                  2^-21 of |S| |r|, so its signs agree with an fp32 dot
//                  product wherever |S r| is above that level;
//   store          packed codes, fp16 ||x||, sign bits (LSB first), fp16 ||r||.
// Pi and S are read as coalesced B-fragment tables (built on the host),
// 128 KB per 64 rows from L2, instead of 96 KB per row.
#include <atomic>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_cache_slot.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
constexpr int kWarps = 4;
constexpr int kRows = 16 * kWarps;           // K rows per CTA
constexpr int kFragWords = 16 * 4 * 32 * 4;  // 32-bit words of one B-fragment table (128 x 128 bf16)

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t half2_bits(__half2 v) { return *reinterpret_cast<const uint32_t *>(&v); }

// Residuals r0, r1 (r0 in the low halves), scaled by 2^14, as two fp16 pairs
// hi + lo.  |r| is below 1.3 (a coordinate of a unit direction minus a
// centroid), so r 2^14 stays below fp16's largest finite value; hi + lo
// differs from r 2^14 by at most 2^-22 |r| 2^14 + 2^-24 (lo's rounding, in
// the normal or the subnormal range).
constexpr float kResidualScale = 0x1p14f;
__device__ __forceinline__ void split2(float r0, float r1, uint32_t &hi, uint32_t &lo) {
  const float x0 = r0 * kResidualScale, x1 = r1 * kResidualScale;
  const __half2 h = __floats2half2_rn(x0, x1);
  const __half2 l = __floats2half2_rn(x0 - __low2float(h), x1 - __high2float(h));
  hi = half2_bits(h);
  lo = half2_bits(l);
}

// Code #{j : T_j < z} of one coordinate against the positive thresholds tp
// (already scaled by ||x||) of the symmetric codebook.
template <int B>
__device__ __forceinline__ int code_of(float z, const float (&tp)[(1 << (B - 1)) - 1]) {
  constexpr int half = 1 << (B - 1);
  const float a = fabsf(z);
  int m = 0;
#pragma unroll
  for (int j = 0; j < half - 1; ++j) m += a > tp[j] ? 1 : 0;
  return z > 0.f ? half + m : half - 1 - m;
}

// Word k of the packed 32-code group `cd` (layout of the cache planes: LSB-first
// for 2 and 4 bits; nibbles plus the spare column for 3 bits).
template <int B>
__device__ __forceinline__ uint32_t pack_word(const uint8_t *cd, int k) {
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

// Persistent: each CTA stages the Pi and S fragment tables (96 KB) in shared
// memory once, then takes 64-row tiles strided over the grid; two CTAs per SM.
constexpr int kTabVec = kFragWords / 4;           // 16-byte vectors of one fragment table
constexpr int kTabBytes = 3 * kTabVec * 16;       // Pi, S hi, S lo
template <int BK>
__global__ void __launch_bounds__(32 * kWarps, 2) quantize_qjl_kernel(DeviceParams p, tq_cache c,
                                                                    const uint16_t *__restrict__ k_in,
                                                                    const int32_t *__restrict__ seq_idx,
                                                                    const int32_t *__restrict__ pos, int n_rows) {
  constexpr int half = 1 << (BK - 1);
  __shared__ __align__(16) uint8_t s_code[kRows][D + 4];  // rows padded by one bank
  __shared__ float s_cent[1 << BK];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = lane >> 2, q = lane & 3;
  extern __shared__ __align__(16) uint4 s_tab[];             // [Pi | S hi | S lo] fragment tables
  // parameters (written long before) first, then wait for the previous kernel
  if (tid < (1 << BK)) s_cent[tid] = p.cb[tid];
  float thr[half - 1];
#pragma unroll
  for (int j = 0; j < half - 1; ++j) thr[j] = p.cb[kMaxLevels + half + j];
  {
    const uint4 *gp = reinterpret_cast<const uint4 *>(p.pif), *gs = reinterpret_cast<const uint4 *>(p.sf);
    for (int i = tid; i < kTabVec; i += 32 * kWarps) s_tab[i] = gp[i];
    for (int i = tid; i < 2 * kTabVec; i += 32 * kWarps) s_tab[kTabVec + i] = gs[i];
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncthreads();

  const int n_tiles = (n_rows + kRows - 1) / kRows;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const long row0 = (long)tile * kRows + 16 * warp;
    const long rows[2] = {row0 + r, row0 + r + 8};
    // ---- X fragments (a0: row r, a1: row r + 8, a2 / a3: the same rows, columns + 8) and ||x||^2
    uint32_t a[8][4];
    float ss[2] = {0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long row = rows[e & 1];
        const int col = 16 * ks + 8 * (e >> 1) + 2 * q;
        const uint32_t w = row < n_rows ? *reinterpret_cast<const uint32_t *>(k_in + row * D + col) : 0u;
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
    const float inv[2] = {live[0] ? 1.f / nrm[0] : 0.f, live[1] ? 1.f / nrm[1] : 0.f};

    // ---- z = X Pi^T: z[nt][0..1] = row r, columns 8 nt + 2 q (+1); [2..3] = row r + 8.
    // The n-tiles are the inner loop, so consecutive MMAs feed 16 independent
    // accumulators.
    float z[16][4];
    const uint4 *pif = s_tab;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) z[nt][e] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const uint4 v = pif[(nt * 4 + j) * 32 + lane];
        mma_bf16(z[nt], a[2 * j], v.x, v.y);
        mma_bf16(z[nt], a[2 * j + 1], v.z, v.w);
      }

    // ---- codes (to shared memory), residuals r = y - c[code], ||r||^2
    float tp[2][half - 1];
#pragma unroll
    for (int j = 0; j < half - 1; ++j) {
      tp[0][j] = thr[j] * nrm[0];
      tp[1][j] = thr[j] * nrm[1];
    }
    float gg[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {  // 0: row r, 1: row r + 8; columns 8 nt + 2 q and + 1
        int code[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float zz = live[hr] ? z[nt][2 * hr + u] : 0.f;
          code[u] = code_of<BK>(zz, tp[hr]);
          const float y = zz * inv[hr];  // within an ulp of z / ||x||; only r and ||r|| use it
          const float res = y - s_cent[code[u]];
          z[nt][2 * hr + u] = res;
          gg[hr] = fmaf(res, res, gg[hr]);
        }
        *reinterpret_cast<uint16_t *>(&s_code[16 * warp + r + 8 * hr][8 * nt + 2 * q]) =
            (uint16_t)(code[0] | (code[1] << 8));
      }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      gg[e] += __shfl_xor_sync(0xffffffffu, gg[e], 1);
      gg[e] += __shfl_xor_sync(0xffffffffu, gg[e], 2);
    }

    // ---- S r: A fragments of k-step j are the residual accumulators of
    // n-tiles 2 j (columns 16 j + 2 q ..) and 2 j + 1 (columns 16 j + 8 + 2 q ..)
    uint32_t ah[8][4], al[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      split2(z[2 * j][0], z[2 * j][1], ah[j][0], al[j][0]);
      split2(z[2 * j][2], z[2 * j][3], ah[j][1], al[j][1]);
      split2(z[2 * j + 1][0], z[2 * j + 1][1], ah[j][2], al[j][2]);
      split2(z[2 * j + 1][2], z[2 * j + 1][3], ah[j][3], al[j][3]);
    }
    const uint4 *sfh = s_tab + kTabVec;
    const uint4 *sfl = sfh + kTabVec;
    // projection m = 8 nt + 2 q (+1) is bit m of the row; a projection of exactly
    // 0 stores 1.  Two halves of 8 n-tiles: 8 independent accumulators between
    // consecutive MMAs.
    uint32_t sb[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};  // sign bits of rows r, r + 8 (LSB first)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float acc[8][4];
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int f = ((8 * hf + t) * 4 + j) * 32 + lane;
          const uint4 h = sfh[f], l = sfl[f];
#pragma unroll
          for (int u = 0; u < 2; ++u) {  // k-steps 2 j and 2 j + 1
            const int ks = 2 * j + u;
            const uint32_t hb0 = u ? h.z : h.x, hb1 = u ? h.w : h.y;
            const uint32_t lb0 = u ? l.z : l.x, lb1 = u ? l.w : l.y;
            mma_f16(acc[t], ah[ks], hb0, hb1);
            mma_f16(acc[t], ah[ks], lb0, lb1);
            mma_f16(acc[t], al[ks], hb0, hb1);
          }
        }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int nt = 8 * hf + t, sh = 8 * (nt & 3) + 2 * q;
        sb[0][nt >> 2] |= ((acc[t][0] >= 0.f ? 1u : 0u) | (acc[t][1] >= 0.f ? 2u : 0u)) << sh;
        sb[1][nt >> 2] |= ((acc[t][2] >= 0.f ? 1u : 0u) | (acc[t][3] >= 0.f ? 2u : 0u)) << sh;
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        sb[e][w] |= __shfl_xor_sync(0xffffffffu, sb[e][w], 1);
        sb[e][w] |= __shfl_xor_sync(0xffffffffu, sb[e][w], 2);
      }
    __syncwarp();  // this warp's code rows are complete

    // ---- stores: thread q of a quad packs code group q of its two rows
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const long row = rows[e];
      if (row >= n_rows) continue;
      const int tok = (int)(row / c.n_kv_heads), h = (int)(row - (long)tok * c.n_kv_heads);
      const long slot = cache_slot(c, seq_idx[tok], h, pos[tok]);
      if (slot < 0) {
        if (q == 0 && h == 0) atomicOr(p.err, kErrTokenRange);
        continue;
      }
      const uint8_t *cd = &s_code[16 * warp + r + 8 * e][32 * q];
      uint32_t *dst = reinterpret_cast<uint32_t *>(c.codes_k + slot * (D * BK / 8)) + BK * q;
#pragma unroll
      for (int k = 0; k < BK; ++k) dst[k] = pack_word<BK>(cd, k);
      if (q == 0) {
        reinterpret_cast<uint4 *>(c.qjl_bits + slot * (D / 8))[0] = make_uint4(sb[e][0], sb[e][1], sb[e][2], sb[e][3]);
        c.norm_k[slot] = __half_as_ushort(__float2half_rn(fminf(nrm[e], 65504.f)));
        c.qjl_norm[slot] = __half_as_ushort(__float2half_rn(fminf(sqrtf(gg[e]), 65504.f)));
      }
    }
    __syncwarp();  // this warp's code rows are read before the next tile writes them
  }
}

}  // namespace

int launch_quantize_qjl(const DeviceParams &p, const tq_cache &c, const void *k, const int32_t *seq_idx,
                        const int32_t *pos, int n_tok, void *stream) {
  using Fn = void (*)(DeviceParams, tq_cache, const uint16_t *, const int32_t *, const int32_t *, int);
  const Fn fn = p.bits_k == 2 ? quantize_qjl_kernel<2> : p.bits_k == 3 ? quantize_qjl_kernel<3> : quantize_qjl_kernel<4>;
  // resident CTAs on the device, per bit width; cached per device (the
  // attribute and the occupancy query apply to the current device) and
  // atomically, as calls may come from several threads
  static std::atomic<int> slots[kMaxDevices][3];
  const int dev = current_device();
  int n_slots = slots[dev][p.bits_k - 2].load(std::memory_order_relaxed);
  if (n_slots == 0) {
    int n_sm = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kTabBytes);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 32 * kWarps, kTabBytes) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    n_slots = n_sm * per_sm;
    slots[dev][p.bits_k - 2].store(n_slots, std::memory_order_relaxed);
  }
  const long rows = (long)n_tok * c.n_kv_heads;
  const long tiles = (rows + kRows - 1) / kRows;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles < n_slots ? tiles : n_slots));
  cfg.blockDim = dim3(32 * kWarps);
  cfg.dynamicSmemBytes = kTabBytes;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, fn, p, c, static_cast<const uint16_t *>(k), seq_idx, pos, (int)rows);
}

}  // namespace tq
