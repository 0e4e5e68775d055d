// TurboQuant quantize-on-append for sm_100a, small batches and QJL rows:
// norm, rotation by Pi, Lloyd-Max codes, bit-pack, optional QJL residual
// signs (one CTA per vector, or 32 vectors per CTA for batches of K rows with
// QJL at head dimension 256); and the dispatch between these kernels and the
// tensor-core kernels.
//
// The method: ai-accelerate.xyz TurboQuant explainer, "TurboQuantの仕組み"
// (rotation + per-coordinate Lloyd-Max, then the 1-bit QJL residual
// correction); decode reads the packed cache without reconstructing K or V.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq_cache_slot.cuh"
#include "tq_f32x2.cuh"
#include "tq_internal.h"

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
// K rows with QJL in batches at head dimension 256 (d = 64 and 128 batches run
// on the tcgen05 QJL kernel): the per-row kernel's arithmetic for R vectors per
// CTA.  Thread t owns coordinates t + h d / C (h < C) of all R vectors, so each
// row of Pi and of S is read once per R vectors (the per-row kernel reads all
// of S, d x d fp32, for every vector), and every broadcast shared-memory load
// of a vector's coordinates feeds C rows of Pi or S.  The R vectors sit in
// shared memory as fp32 (x, then z, then the residuals r in the same buffer),
// interleaved by pairs (vectors 2 j and 2 j + 1 alternate coordinate by
// coordinate), so that one packed f32x2 FMA advances a row of Pi or S against
// both vectors of a pair, each lane rounding as the scalar FMA would; the
// norms and ||r|| are warp reductions, one vector per warp in turn.  A
// coordinate block of 32 (one word of the cache layout per bit, one word of
// sign bits) belongs to warp w = block % (d / 32 C).  grid = ceil(rows / R).
// ---------------------------------------------------------------------------
template <int DH, int R, int BK, int C>
__global__ void __launch_bounds__(DH / C) quantize_qjl_rows_kernel(DeviceParams p, tq_cache c,
                                                                   const uint16_t *__restrict__ k_in,
                                                                   const int32_t *__restrict__ seq_idx,
                                                                   const int32_t *__restrict__ pos, long n_rows) {
  constexpr int kThreads = DH / C, kWarps = kThreads / 32;
  static_assert(R % 2 == 0, "vectors are held in pairs");
  __shared__ __align__(16) float s_v[R / 2][DH][2];  // x, then z, then r; vector r at [r / 2][.][r % 2]
  auto V = [&](int r, int i) -> float & { return s_v[r >> 1][i][r & 1]; };
  __shared__ float s_n[R], s_g[R];
  __shared__ long s_slot[R];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long row0 = (long)blockIdx.x * R;
  PiRow<DH> pw[C];
#pragma unroll
  for (int h = 0; h < C; ++h) pw[h].load(p.pi + (tid + h * kThreads) * DH);
  // launched as a programmatic dependent: no input is read before the
  // previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#pragma unroll 4
  for (int r = 0; r < R; ++r) {  // rows past the end are zero vectors that are never stored
    const long row = row0 + r;
#pragma unroll
    for (int h = 0; h < C; ++h)
      V(r, tid + h * kThreads) = row < n_rows ? bf16_bits_to_f32(k_in[row * DH + tid + h * kThreads]) : 0.f;
  }
  if (tid < R) {
    const long row = row0 + tid;
    long slot = -1;
    if (row < n_rows) {
      const int t = (int)(row / c.n_kv_heads), hd = (int)(row % c.n_kv_heads);
      // (no index arrays: token t goes to position t of sequence 0)
      slot = cache_slot(c, seq_idx ? seq_idx[t] : 0, hd, pos ? pos[t] : t);
      if (slot < 0 && hd == 0) atomicOr(p.err, kErrTokenRange);
    }
    s_slot[tid] = slot;
  }
  __syncthreads();
  for (int r = warp; r < R; r += kWarps) {  // ||x||, fp32 over exact bf16 squares
    float v = 0.f;
#pragma unroll
    for (int j = lane; j < DH; j += 32) v = fmaf(V(r, j), V(r, j), v);
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_n[r] = sqrtf(v);
  }
  // z_i = (Pi x)_i of the R vectors: rows i of Pi against each pair of vectors
  float2 acc[C][R / 2];
#pragma unroll
  for (int h = 0; h < C; ++h)
#pragma unroll
    for (int j = 0; j < R / 2; ++j) acc[h][j] = make_float2(0.f, 0.f);
#pragma unroll(DH <= 128 ? DH / 8 : 1)
  for (int c8 = 0; c8 < DH / 8; ++c8) {
    float pf[C][8];
#pragma unroll
    for (int h = 0; h < C; ++h) {
      const uint4 w = pw[h].get(c8);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pf[h][2 * e] = __uint_as_float(u[e] << 16);
        pf[h][2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int j = 0; j < R / 2; ++j) {
      // coordinates 8 c8 .. 8 c8 + 7 of vectors 2 j and 2 j + 1
      const float4 *xp = reinterpret_cast<const float4 *>(&s_v[j][8 * c8][0]);
      const float4 x[4] = {xp[0], xp[1], xp[2], xp[3]};
#pragma unroll
      for (int h = 0; h < C; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[h][j] = fma2(make_float2(pf[h][2 * e], pf[h][2 * e]), make_float2(x[e].x, x[e].y), acc[h][j]);
          acc[h][j] = fma2(make_float2(pf[h][2 * e + 1], pf[h][2 * e + 1]), make_float2(x[e].z, x[e].w), acc[h][j]);
        }
    }
  }
  __syncthreads();  // every thread is done with x: the buffer takes z, then r
#pragma unroll
  for (int h = 0; h < C; ++h)
#pragma unroll
    for (int j = 0; j < R / 2; ++j) {
      V(2 * j, tid + h * kThreads) = acc[h][j].x;
      V(2 * j + 1, tid + h * kThreads) = acc[h][j].y;
    }
  constexpr int half = 1 << (BK - 1);
  const float *cent = p.cb;
  float thr[half - 1];  // the positive thresholds
#pragma unroll
  for (int j = 0; j < half - 1; ++j) thr[j] = p.cb[1 * kMaxLevels + half + j];
  // this thread's bit positions inside the BK words of its coordinate blocks
  // (the cache layout: LSB-first for 2 and 4 bits, nibbles plus the spare
  // column for 3 bits)
  int wd_of[C][BK], sh_of[C][BK];
#pragma unroll
  for (int h = 0; h < C; ++h)
#pragma unroll
    for (int kb = 0; kb < BK; ++kb) {
      const int i = tid + h * kThreads;
      const int pbit = code_bit_pos(BK, i, kb) - 32 * BK * (i >> 5);
      wd_of[h][kb] = pbit >> 5;
      sh_of[h][kb] = pbit & 31;
    }
#pragma unroll 1
  for (int r = 0; r < R; ++r) {
    const float n = s_n[r];
    // a vector whose stored fp16 norm is zero (n <= 2^-25) is the zero vector
    const bool live = n > 0x1p-25f;
    const long slot = s_slot[r];
    uint32_t *dst = reinterpret_cast<uint32_t *>(c.codes_k + (slot < 0 ? 0 : slot) * (DH * BK / 8));
#pragma unroll
    for (int h = 0; h < C; ++h) {
      const int i = tid + h * kThreads;
      const float z = live ? V(r, i) : 0.f;
      const float a = fabsf(z);
      int m = 0;
#pragma unroll
      for (int j = 0; j < half - 1; ++j) m += a > thr[j] * n ? 1 : 0;
      const int code = z > 0.f ? half + m : half - 1 - m;
#pragma unroll
      for (int wd = 0; wd < BK; ++wd) {  // block i / 32 owns words BK (i / 32) ..
        uint32_t contrib = 0;
#pragma unroll
        for (int kb = 0; kb < BK; ++kb)
          if (wd_of[h][kb] == wd) contrib |= (uint32_t)((code >> kb) & 1) << sh_of[h][kb];
        const uint32_t word = __reduce_or_sync(0xffffffffu, contrib);
        if (lane == 0 && slot >= 0) dst[(i >> 5) * BK + wd] = word;
      }
      const float y = live ? z / n : 0.f;
      V(r, i) = y - cent[code];
    }
    if (tid == 0 && slot >= 0) c.norm_k[slot] = f32_to_f16_bits_sat(n);
  }
  __syncthreads();
  for (int r = warp; r < R; r += kWarps) {  // ||r||
    float v = 0.f;
#pragma unroll
    for (int j = lane; j < DH; j += 32) v = fmaf(V(r, j), V(r, j), v);
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_g[r] = sqrtf(v);
  }
  // (S r)_i of the R residuals: rows i of S (fp32) against each pair of residuals
#pragma unroll
  for (int h = 0; h < C; ++h)
#pragma unroll
    for (int j = 0; j < R / 2; ++j) acc[h][j] = make_float2(0.f, 0.f);
#pragma unroll 2
  for (int c4 = 0; c4 < DH / 4; ++c4) {
    float4 w[C];
#pragma unroll
    for (int h = 0; h < C; ++h) w[h] = reinterpret_cast<const float4 *>(p.s + (size_t)(tid + h * kThreads) * DH)[c4];
#pragma unroll
    for (int j = 0; j < R / 2; ++j) {
      const float4 *xp = reinterpret_cast<const float4 *>(&s_v[j][4 * c4][0]);
      const float4 x0 = xp[0], x1 = xp[1];
#pragma unroll
      for (int h = 0; h < C; ++h) {
        acc[h][j] = fma2(make_float2(w[h].x, w[h].x), make_float2(x0.x, x0.y), acc[h][j]);
        acc[h][j] = fma2(make_float2(w[h].y, w[h].y), make_float2(x0.z, x0.w), acc[h][j]);
        acc[h][j] = fma2(make_float2(w[h].z, w[h].z), make_float2(x1.x, x1.y), acc[h][j]);
        acc[h][j] = fma2(make_float2(w[h].w, w[h].w), make_float2(x1.z, x1.w), acc[h][j]);
      }
    }
  }
  __syncthreads();  // s_g
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const long slot = s_slot[r];
#pragma unroll
    for (int h = 0; h < C; ++h) {
      const uint32_t sb = __ballot_sync(0xffffffffu, ((r & 1) ? acc[h][r >> 1].y : acc[h][r >> 1].x) >= 0.f);
      if (slot >= 0 && lane == 0) reinterpret_cast<uint32_t *>(c.qjl_bits + slot * (DH / 8))[warp + h * kWarps] = sb;
    }
    if (slot >= 0 && tid == 0) c.qjl_norm[slot] = f32_to_f16_bits_sat(s_g[r]);
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
    // QJL, and the batched QJL kernel above for K with QJL (Pi, S hi and S lo
    // at d = 256 do not fit in shared memory beside a tile ring)
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
  if (p.d == 256 && p.qjl) {  // R = 32 vectors per CTA, two coordinates per thread
    constexpr int R = 32;
    cfg.gridDim = dim3((unsigned)((rows + R - 1) / R));
    cfg.blockDim = dim3(128);
    using QjlRowsFn = void (*)(DeviceParams, tq_cache, const uint16_t *, const int32_t *, const int32_t *, long);
    const QjlRowsFn fn = p.bits_k == 2   ? quantize_qjl_rows_kernel<256, R, 2, 2>
                         : p.bits_k == 3 ? quantize_qjl_rows_kernel<256, R, 3, 2>
                                         : quantize_qjl_rows_kernel<256, R, 4, 2>;
    // the largest shared-memory carveout: the CTAs per SM are then bounded by registers only
    cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return (int)cudaLaunchKernelEx(&cfg, fn, p, c, kk, seq_idx, pos, rows);
  }
  cfg.gridDim = dim3((unsigned)rows, 1);  // y = 0: K only
  if (p.d == 64) return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<64>, p, c, kk, kk, seq_idx, pos);
  if (p.d == 256) return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<256>, p, c, kk, kk, seq_idx, pos);
  return (int)cudaLaunchKernelEx(&cfg, quantize_row_kernel<kHeadDim>, p, c, kk, kk, seq_idx, pos);
}

}  // namespace tq
