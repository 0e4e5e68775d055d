// TurboQuant quantize-on-append for sm_100a, small batches and QJL rows:
// norm, rotation by Pi, Lloyd-Max codes, bit-pack, optional QJL residual
// signs (one CTA per vector; batches of K rows with QJL at head dimension 256
// on mma.sync tensor cores, 32 vectors per CTA); and the dispatch between
// these kernels and the tcgen05 kernels.
//
// The method: ai-accelerate.xyz TurboQuant explainer, "TurboQuantの仕組み"
// (rotation + per-coordinate Lloyd-Max, then the 1-bit QJL residual
// correction); decode reads the packed cache without reconstructing K or V.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>

#include "tq_cache_slot.cuh"
#include "tq_f32x2.cuh"
#include "tq_internal.h"
#include "tq_stream.cuh"

namespace tq {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float((uint32_t)h << 16);
}

__device__ __forceinline__ uint16_t f32_to_f16_bits_sat(float x) {
  return __half_as_ushort(__float2half_rn(fminf(x, 65504.f)));
}

// Bit position of bit k of coordinate i's code inside a packed vector (the
// layout documented in tq.h).
__device__ __forceinline__ int code_bit_pos(int bits, int i, int k) {
  if (bits != 3) return i * bits + k;
  const int g = i >> 5, l = i & 31;
  if (l < 24) return 96 * g + 32 * (l >> 3) + 4 * (l & 7) + k;
  return 96 * g + 32 * k + 4 * (l - 24) + 3;
}

// ---------------------------------------------------------------------------
// quantize, one CTA per head vector (small batches, K rows with QJL, and every
// batch of a head dimension other than 128): thread i owns coordinate i of a
// DH-dimensional vector.  z_i = (Pi x)_i from row i of Pi (16-byte loads,
// L2-resident), ||x|| by a block reduction (fp32 over exact bf16 squares), the
// code against the thresholds scaled by ||x||, packing by warp OR-reductions
// (one warp = one 32-coordinate group of the layout).  With QJL:
// r = z/||x|| - c[code], ||r||, (S r)_m from row m of S, one sign ballot per
// warp.  grid = (rows, 2): y = 0 for K, 1 for V.
// ---------------------------------------------------------------------------
// Row of Pi held in registers (up to 128 coordinates: loaded before the
// dependency wait) or read on the fly (256).
template <int DH>
struct PiRow {
  static constexpr int kHeld = DH <= 128 ? DH / 8 : 1;
  uint4 w[kHeld];
  const uint16_t *row;
  __device__ __forceinline__ void load(const uint16_t *r) {
    row = r;
    if constexpr (DH <= 128) {
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) w[c] = reinterpret_cast<const uint4 *>(r)[c];
    }
  }
  __device__ __forceinline__ uint4 get(int c) const {
    if constexpr (DH <= 128) return w[c];
    else return reinterpret_cast<const uint4 *>(row)[c];
  }
};

template <int DH>
__device__ __forceinline__ float row_dot_bf16(const PiRow<DH> &pr, const float *x) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < DH / 8; ++c) {
    const uint4 w = pr.get(c);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[e] = fmaf(__uint_as_float(u[e] << 16), x[8 * c + 2 * e], acc[e]);
      acc[e] = fmaf(__uint_as_float(u[e] & 0xffff0000u), x[8 * c + 2 * e + 1], acc[e]);
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <int DH>
__device__ __forceinline__ float row_dot_f32(const float *row, const float *x) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int c = 0; c < DH / 4; ++c) {
    const float4 w = reinterpret_cast<const float4 *>(row)[c];
    acc[0] = fmaf(w.x, x[4 * c], acc[0]);
    acc[1] = fmaf(w.y, x[4 * c + 1], acc[1]);
    acc[2] = fmaf(w.z, x[4 * c + 2], acc[2]);
    acc[3] = fmaf(w.w, x[4 * c + 3], acc[3]);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <int DH>
__device__ __forceinline__ float block_sum(float v, float *red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < DH / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

template <int DH>
__global__ void __launch_bounds__(DH) quantize_row_kernel(DeviceParams p, tq_cache c,
                                                          const uint16_t *__restrict__ k_in,
                                                          const uint16_t *__restrict__ v_in,
                                                          const int32_t *__restrict__ seq_idx,
                                                          const int32_t *__restrict__ pos) {
  __shared__ float s_x[DH], s_r[DH];
  __shared__ float red[DH / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // row tid of Pi is a parameter, written long before: load it while the
  // previous kernel finishes
  PiRow<DH> pw;
  pw.load(p.pi + tid * DH);
  // warm L2 with this row's inputs (a prefetch only moves lines into L2, the
  // point of coherence, so it may run before the previous kernel is done)
  if (tid == 0) {
    const long row = blockIdx.x;
    for (int ch = 0; ch < DH * 2; ch += 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"((blockIdx.y == 1 ? v_in : k_in) + row * DH + ch / 2));
    if (seq_idx) asm volatile("prefetch.global.L2 [%0];" ::"l"(seq_idx + row / c.n_kv_heads));
    if (pos) asm volatile("prefetch.global.L2 [%0];" ::"l"(pos + row / c.n_kv_heads));
  }
  // launched as a programmatic dependent: no input is read before the
  // previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool is_v = blockIdx.y == 1;
  const int bits = is_v ? p.bits_v : p.bits_k;
  const bool qjl = !is_v && p.qjl;
  const long row = blockIdx.x;
  const int t = (int)(row / c.n_kv_heads), h = (int)(row % c.n_kv_heads);
  // the input is loaded beside the indices, not after the destination check
  const float x = bf16_bits_to_f32((is_v ? v_in : k_in)[row * DH + tid]);
  // (no index arrays: token t goes to position t of sequence 0)
  const long slot = cache_slot(c, seq_idx ? seq_idx[t] : 0, h, pos ? pos[t] : t);
  if (slot < 0) {
    if (tid == 0 && !is_v) atomicOr(p.err, kErrTokenRange);
    return;
  }
  s_x[tid] = x;
  const float n = sqrtf(block_sum<DH>(x * x, red));  // also orders s_x
  // a vector whose stored fp16 norm is zero (n <= 2^-25) is the zero vector
  const bool live = n > 0x1p-25f;
  const float z = live ? row_dot_bf16<DH>(pw, s_x) : 0.f;
  const float *thr = p.cb + (is_v ? 3 : 1) * kMaxLevels;
  const int half = 1 << (bits - 1);
  const float a = fabsf(z);
  int m = 0;
  for (int j = 0; j < half - 1; ++j) m += a > thr[half + j] * n ? 1 : 0;
  const int code = z > 0.f ? half + m : half - 1 - m;

  uint32_t *dst = reinterpret_cast<uint32_t *>((is_v ? c.codes_v : c.codes_k) + slot * (DH * bits / 8));
  for (int wd = 0; wd < bits; ++wd) {  // warp w owns words w*bits .. w*bits+bits-1
    uint32_t contrib = 0;
    for (int kb = 0; kb < bits; ++kb) {
      const int pbit = code_bit_pos(bits, tid, kb) - 32 * bits * warp;
      if ((pbit >> 5) == wd) contrib |= (uint32_t)((code >> kb) & 1) << (pbit & 31);
    }
    const uint32_t word = __reduce_or_sync(0xffffffffu, contrib);
    if (lane == 0) dst[warp * bits + wd] = word;
  }
  if (tid == 0) (is_v ? c.norm_v : c.norm_k)[slot] = f32_to_f16_bits_sat(n);

  if (qjl) {
    const float *cent = p.cb;  // K centroids
    const float y = live ? z / n : 0.f;
    const float r = y - cent[code];
    s_r[tid] = r;
    const float gamma = sqrtf(block_sum<DH>(r * r, red));
    const float proj = row_dot_f32<DH>(p.s + tid * DH, s_r);  // (S r)_tid
    const uint32_t sb = __ballot_sync(0xffffffffu, proj >= 0.f);
    if (lane == 0) reinterpret_cast<uint32_t *>(c.qjl_bits + slot * (DH / 8))[warp] = sb;
    if (tid == 0) c.qjl_norm[slot] = f32_to_f16_bits_sat(gamma);
  }
}

// ---------------------------------------------------------------------------
// K rows with QJL in batches at head dimension 256 on the mma.sync tensor
// cores (Pi, S hi and S lo at d = 256 do not fit in shared memory beside a
// tcgen05 tile ring).  A CTA takes 32 vectors (two m-tiles of 16); warp w
// owns output coordinates 64 w .. 64 w + 63 in two chunks of 32, each one
// coordinate block of the cache layout (BK words of codes, one word of signs).
//   z = X Pi^T on m16n8k16 bf16 (exact products, fp32 sums): A = the bf16
//   rows from shared memory (ldmatrix), B = Pi's bf16 fragment table;
//   the codes, the packed words and r = z / ||x|| - c[code] come straight
//   from the accumulator fragments (the four lanes of a quad hold a row's 32
//   coordinates of the chunk, and OR-reduce its words);
//   S r with r 2^14 and S 2^sigma as two-part fp16 splits, three m16n8k16
//   f16 products (hi hi, hi lo, lo hi: about 22 significant bits, of which
//   only the sign is kept; both scales are positive): A = the split
//   residuals of all four warps from shared memory, B = S's fragment tables.
// grid = ceil(rows / 32), 128 threads, four CTAs per SM (51 KB of shared
// memory and at most 128 registers each): sixteen warps per SM hide more of
// the MMA and L2 latency than eight warps with 64 vectors per CTA did, although
// every fragment of Pi and S is then read once per 32 vectors instead of 64.
// ---------------------------------------------------------------------------
constexpr int kQmMT = 2;        // m-tiles of 16 vectors per CTA
constexpr int kQmM = 16 * kQmMT;  // vectors per CTA
constexpr int kQmLd = 256 + 8;  // row stride in 16-bit elements: 528 B puts ldmatrix rows on distinct banks
constexpr int kQmSmem = kQmM * kQmLd * 2 * 3 + kQmM * (4 + 16 + 8) + 16 * 4;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}

// OR the code of in-block coordinate 8 jn + pe (jn < 4, pe < 8) into the BK
// words of its 32-coordinate block (the cache layout: LSB-first for 2 and 4
// bits; nibbles for the first 24 coordinates and the spare column of the
// nibbles' top bits for the last 8 at 3 bits)
template <int BK>
__device__ __forceinline__ void or_code(uint32_t (&w)[BK], int jn, int pe, uint32_t code) {
  if constexpr (BK == 2) {
    w[jn >> 1] |= code << (16 * (jn & 1) + 2 * pe);
  } else if constexpr (BK == 4) {
    w[jn] |= code << (4 * pe);
  } else {
    if (jn < 3) {
      w[jn < 3 ? jn : 0] |= code << (4 * pe);
    } else {
#pragma unroll
      for (int k = 0; k < 3; ++k) w[k] |= ((code >> k) & 1u) << (4 * pe + 3);
    }
  }
}

template <int BK>
__global__ void __launch_bounds__(128, 4) quantize_qjl_mma256_kernel(DeviceParams p, tq_cache c,
                                                                      const uint16_t *__restrict__ k_in,
                                                                      const int32_t *__restrict__ seq_idx,
                                                                      const int32_t *__restrict__ pos, long n_rows) {
  constexpr int DH = 256, M = kQmM, LD = kQmLd;
  extern __shared__ __align__(16) unsigned char qm_smem[];
  uint16_t *s_x = reinterpret_cast<uint16_t *>(qm_smem);   // [M][LD] bf16 rows
  uint16_t *s_rh = s_x + M * LD;                             // [M][LD] fp16 hi of r 2^14
  uint16_t *s_rl = s_rh + M * LD;                            // [M][LD] fp16 lo
  float *s_n = reinterpret_cast<float *>(s_rl + M * LD);     // [M] ||x||
  float *s_gp = s_n + M;                                     // [4][M] the warps' parts of ||r||^2
  long *s_slot = reinterpret_cast<long *>(s_gp + 4 * M);     // [M]
  float *s_cent = reinterpret_cast<float *>(s_slot + M);     // [16] K centroids
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
  const long row0 = (long)blockIdx.x * M;
  if (tid < 16) s_cent[tid] = p.cb[tid];
  // launched as a programmatic dependent: no input is read before the
  // previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  {  // the M rows in 16-byte pieces (32 per row), every load issued first; rows past the end are zero
    uint4 v[M / 4];
#pragma unroll
    for (int k = 0; k < M / 4; ++k) {
      const int idx = tid + 128 * k;
      const long row = row0 + (idx >> 5);
      v[k] = row < n_rows ? reinterpret_cast<const uint4 *>(k_in + row * DH)[idx & 31] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < M / 4; ++k) {
      const int idx = tid + 128 * k;
      *reinterpret_cast<uint4 *>(s_x + (idx >> 5) * LD + 8 * (idx & 31)) = v[k];
    }
  }
  if (tid < M) {
    const long row = row0 + tid;
    long slot = -1;
    if (row < n_rows) {
      const int tk = (int)(row / c.n_kv_heads), hd = (int)(row % c.n_kv_heads);
      // (no index arrays: token t goes to position t of sequence 0)
      slot = cache_slot(c, seq_idx ? seq_idx[tk] : 0, hd, pos ? pos[tk] : tk);
      if (slot < 0 && hd == 0) atomicOr(p.err, kErrTokenRange);
    }
    s_slot[tid] = slot;
  }
  __syncthreads();
  // ||x||, fp32 over exact bf16 squares: warp w takes rows M w / 4 .. M (w + 1) / 4 - 1
  for (int rr = 0; rr < M / 4; ++rr) {
    const int r = (M / 4) * warp + rr;
    const uint4 u = *reinterpret_cast<const uint4 *>(s_x + r * LD + 8 * lane);
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    float v = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xffff0000u);
      v = fmaf(lo, lo, v);
      v = fmaf(hi, hi, v);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_n[r] = sqrtf(v);
  }
  __syncthreads();

  constexpr int half = 1 << (BK - 1);
  float thr[half - 1];  // the positive thresholds
#pragma unroll
  for (int j = 0; j < half - 1; ++j) thr[j] = p.cb[1 * kMaxLevels + half + j];
  // this lane's ldmatrix address: row lane % 16 of an m-tile, columns 8 (lane / 16) of a k-step
  const uint32_t a_off = (uint32_t)(((lane & 15) * LD + ((lane >> 4) << 3)) * 2);
  const uint32_t xs = smem_u32(s_x) + a_off, rhs = smem_u32(s_rh) + a_off, rls = smem_u32(s_rl) + a_off;
  const uint4 *pif4 = reinterpret_cast<const uint4 *>(p.pif);
  float gs[kQmMT][2];  // this thread's part of ||r||^2 for rows 16 mt + g + 8 hf
#pragma unroll
  for (int mt = 0; mt < kQmMT; ++mt) gs[mt][0] = gs[mt][1] = 0.f;

#pragma unroll 1
  for (int cc = 0; cc < 2; ++cc) {
    const int nt0 = 8 * warp + 4 * cc;  // first n-tile (8 coordinates each) of the chunk
    float acc[kQmMT][4][4];
#pragma unroll
    for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll 2
    for (int j = 0; j < DH / 32; ++j) {  // k-steps 2 j and 2 j + 1: one 16-byte fragment load per n-tile
      uint4 b[4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) b[nt] = pif4[((nt0 + nt) * (DH / 32) + j) * 32 + lane];
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        uint32_t a[kQmMT][4];
#pragma unroll
        for (int mt = 0; mt < kQmMT; ++mt) ldsm_x4(xs + (uint32_t)((mt * 16 * LD + (2 * j + s2) * 16) * 2), a[mt]);
#pragma unroll
        for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
            mma_bf16(acc[mt][nt], a[mt][0], a[mt][1], a[mt][2], a[mt][3], s2 ? b[nt].z : b[nt].x,
                     s2 ? b[nt].w : b[nt].y);
      }
    }
    // codes, packed words and residuals of the chunk; fragment element e of
    // n-tile nt0 + nt is row 16 mt + g + 8 (e / 2), coordinate 8 (nt0 + nt) + 2 t + e % 2
#pragma unroll
    for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * mt + g + 8 * hf;
        const float n = s_n[r];
        // a vector whose stored fp16 norm is zero (n <= 2^-25) is the zero vector
        const bool live = n > 0x1p-25f;
        const float inv = live ? 1.f / n : 0.f;
        float tn[half - 1];
#pragma unroll
        for (int j = 0; j < half - 1; ++j) tn[j] = thr[j] * n;
        uint32_t wds[BK];
#pragma unroll
        for (int k = 0; k < BK; ++k) wds[k] = 0u;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          float rv[2];
#pragma unroll
          for (int e1 = 0; e1 < 2; ++e1) {
            const float z = live ? acc[mt][nt][2 * hf + e1] : 0.f;
            const float a = fabsf(z);
            int m = 0;
#pragma unroll
            for (int j = 0; j < half - 1; ++j) m += a > tn[j] ? 1 : 0;
            const int code = z > 0.f ? half + m : half - 1 - m;
            or_code<BK>(wds, nt, 2 * t + e1, (uint32_t)code);
            rv[e1] = z * inv - s_cent[code];
            gs[mt][hf] = fmaf(rv[e1], rv[e1], gs[mt][hf]);
          }
          uint32_t hi, lo;
          split_f16x2(rv[0] * 16384.f, rv[1] * 16384.f, hi, lo);
          const int col = 8 * (nt0 + nt) + 2 * t;
          *reinterpret_cast<uint32_t *>(s_rh + r * LD + col) = hi;
          *reinterpret_cast<uint32_t *>(s_rl + r * LD + col) = lo;
        }
#pragma unroll
        for (int k = 0; k < BK; ++k) {
          wds[k] |= __shfl_xor_sync(0xffffffffu, wds[k], 1);
          wds[k] |= __shfl_xor_sync(0xffffffffu, wds[k], 2);
        }
        const long slot = s_slot[r];
        if (t == 0 && slot >= 0) {
          uint32_t *dst = reinterpret_cast<uint32_t *>(c.codes_k + slot * (DH * BK / 8)) + (2 * warp + cc) * BK;
#pragma unroll
          for (int k = 0; k < BK; ++k) dst[k] = wds[k];
        }
      }
  }
#pragma unroll
  for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v = gs[mt][hf];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (t == 0) s_gp[warp * M + 16 * mt + g + 8 * hf] = v;
    }
  __syncthreads();  // every warp's residuals and ||r||^2 parts are in shared memory
  if (tid < M) {
    const long slot = s_slot[tid];
    if (slot >= 0) {
      c.norm_k[slot] = f32_to_f16_bits_sat(s_n[tid]);
      const float g2 = (s_gp[tid] + s_gp[M + tid]) + (s_gp[2 * M + tid] + s_gp[3 * M + tid]);
      c.qjl_norm[slot] = f32_to_f16_bits_sat(sqrtf(g2));
    }
  }
  const uint4 *sf4 = reinterpret_cast<const uint4 *>(p.sf);
  constexpr int kLoPart = DH * DH / 8;  // the lo table, in 16-byte units
#pragma unroll 1
  for (int cc = 0; cc < 2; ++cc) {
    const int nt0 = 8 * warp + 4 * cc;
    float acc[kQmMT][4][4];
#pragma unroll
    for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll 1
    for (int j = 0; j < DH / 32; ++j) {
      uint4 bh[4], bl[4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        bh[nt] = sf4[((nt0 + nt) * (DH / 32) + j) * 32 + lane];
        bl[nt] = sf4[kLoPart + ((nt0 + nt) * (DH / 32) + j) * 32 + lane];
      }
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        uint32_t ah[kQmMT][4], al[kQmMT][4];
#pragma unroll
        for (int mt = 0; mt < kQmMT; ++mt) {
          ldsm_x4(rhs + (uint32_t)((mt * 16 * LD + (2 * j + s2) * 16) * 2), ah[mt]);
          ldsm_x4(rls + (uint32_t)((mt * 16 * LD + (2 * j + s2) * 16) * 2), al[mt]);
        }
#pragma unroll
        for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const uint32_t h0 = s2 ? bh[nt].z : bh[nt].x, h1 = s2 ? bh[nt].w : bh[nt].y;
            const uint32_t l0 = s2 ? bl[nt].z : bl[nt].x, l1 = s2 ? bl[nt].w : bl[nt].y;
            mma_f16(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], h0, h1);
            mma_f16(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], l0, l1);
            mma_f16(acc[mt][nt], al[mt][0], al[mt][1], al[mt][2], al[mt][3], h0, h1);
          }
      }
    }
    // sign of (S r)_i, i = 8 (nt0 + nt) + 2 t + e % 2: bit i % 32 of word i / 32 = 2 w + cc
#pragma unroll
    for (int mt = 0; mt < kQmMT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sb = 0u;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e1 = 0; e1 < 2; ++e1)
            sb |= (acc[mt][nt][2 * hf + e1] >= 0.f ? 1u : 0u) << (8 * nt + 2 * t + e1);
        sb |= __shfl_xor_sync(0xffffffffu, sb, 1);
        sb |= __shfl_xor_sync(0xffffffffu, sb, 2);
        const long slot = s_slot[16 * mt + g + 8 * hf];
        if (t == 0 && slot >= 0) reinterpret_cast<uint32_t *>(c.qjl_bits + slot * (DH / 8))[2 * warp + cc] = sb;
      }
  }
}
}  // namespace

// Batches of up to kRowKernelMaxRows rows per matrix (decode-time appends) use
// the one-CTA-per-row kernel; larger batches one tcgen05 kernel for K and V:
// the MSE kernel (tq_quantize_tc.cu) without QJL, the QJL kernel
// (tq_quantize_qjl_tc.cu) with it.
constexpr long kRowKernelMaxRows = 1024;

int launch_quantize(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                    const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream) {
  const long rows = (long)n_tok * c.n_kv_heads;
  cudaStream_t st = (cudaStream_t)stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const uint16_t *kk = (const uint16_t *)k, *vv = (const uint16_t *)v;
  if (p.d != kHeadDim) {
    // other head dimensions: the per-row kernel for small batches, else the
    // tcgen05 kernels: at d = 64 the MSE kernel (tq_quantize_tc.cu) or, with
    // QJL, the QJL kernel (tq_quantize_qjl_tc.cu), both templated on d; at
    // d = 256 the MSE kernel of tq_quantize_tc256.cu for V and for K without
    // QJL, and the mma.sync QJL kernel above for K with QJL (Pi, S hi and
    // S lo at d = 256 do not fit in shared memory beside a tile ring)
    if (rows <= kRowKernelMaxRows) {
      cfg.gridDim = dim3((unsigned)rows, 2);
      cfg.blockDim = dim3(p.d);
      if (p.d == 64) return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<64>, p, c, kk, vv, seq_idx, pos);
      return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<256>, p, c, kk, vv, seq_idx, pos);
    }
    if (p.d == 256) {  // tcgen05: K and V in one launch, or V alone next to the QJL rows of K
      const int e = launch_quantize_tc256(p, c, k, v, seq_idx, pos, n_tok, !p.qjl, true, stream);
      if (e != 0 || !p.qjl) return e;
      return launch_quantize_rows_k(p, c, k, seq_idx, pos, n_tok, stream);
    }
    if (p.qjl) return launch_quantize_qjl_tc(p, c, k, v, seq_idx, pos, n_tok, stream);
    return launch_quantize_tc(p, c, k, v, seq_idx, pos, n_tok, true, true, stream);
  }
  if (rows <= kRowKernelMaxRows) {
    cfg.gridDim = dim3((unsigned)rows, 2);
    return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<kHeadDim>, p, c, kk, vv, seq_idx, pos);
  }
  if (p.qjl) return launch_quantize_qjl_tc(p, c, k, v, seq_idx, pos, n_tok, stream);
  return launch_quantize_tc(p, c, k, v, seq_idx, pos, n_tok, true, true, stream);
}

int launch_quantize_rows_k(const DeviceParams &p, const tq_cache &c, const void *k, const int32_t *seq_idx,
                           const int32_t *pos, int n_tok, void *stream) {
  const long rows = (long)n_tok * c.n_kv_heads;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(p.d);
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const uint16_t *kk = (const uint16_t *)k;
  if (p.d == 256 && p.qjl) {  // 32 vectors per CTA on the mma.sync tensor cores
    cfg.gridDim = dim3((unsigned)((rows + kQmM - 1) / kQmM));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = kQmSmem;
    using QjlMmaFn = void (*)(DeviceParams, tq_cache, const uint16_t *, const int32_t *, const int32_t *, long);
    const QjlMmaFn fn = p.bits_k == 2   ? quantize_qjl_mma256_kernel<2>
                        : p.bits_k == 3 ? quantize_qjl_mma256_kernel<3>
                                        : quantize_qjl_mma256_kernel<4>;
    // cached per device (the attribute applies to the current device), and
    // atomically, as calls may come from several threads
    static std::atomic<bool> configured[kMaxDevices][3];
    std::atomic<bool> &done = configured[current_device()][p.bits_k - 2];
    if (!done.load(std::memory_order_acquire)) {
      const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kQmSmem);
      if (e != cudaSuccess) return (int)e;
      done.store(true, std::memory_order_release);
    }
    return (int)cudaLaunchKernelEx(&cfg, fn, p, c, kk, seq_idx, pos, rows);
  }
  cfg.gridDim = dim3((unsigned)rows, 1);  // y = 0: K only
  if (p.d == 64) return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<64>, p, c, kk, kk, seq_idx, pos);
  if (p.d == 256) return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<256>, p, c, kk, kk, seq_idx, pos);
  return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<kHeadDim>, p, c, kk, kk, seq_idx, pos);
}

}  // namespace tq
