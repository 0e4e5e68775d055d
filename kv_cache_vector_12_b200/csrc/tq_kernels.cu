// TurboQuant quantize-on-append kernel for sm_100a: norm, rotation by Pi,
// Lloyd-Max codes, bit-pack, optional QJL residual signs.
//
// The method: ai-accelerate.xyz TurboQuant explainer, "TurboQuantの仕組み"
// (rotation + per-coordinate Lloyd-Max, then the 1-bit QJL residual
// correction); decode reads the packed cache without reconstructing K or V.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;

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
// quantize: one CTA (128 threads = one thread per coordinate) per chunk of
// rows; Pi^T staged in shared memory once per CTA.
// ---------------------------------------------------------------------------
constexpr int kQuantRowsPerCta = 64;

__global__ void __launch_bounds__(128) quantize_kernel(DeviceParams p, tq_cache c,
                                                       const uint16_t *__restrict__ k_in,
                                                       const uint16_t *__restrict__ v_in,
                                                       const int32_t *__restrict__ seq_idx,
                                                       const int32_t *__restrict__ pos, int n_tok) {
  __shared__ uint16_t s_pit[D * D];
  __shared__ float s_x[D];
  __shared__ float s_r[D];
  __shared__ double s_red[4];
  __shared__ float s_redf[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool is_v = blockIdx.y == 1;
  const int bits = is_v ? p.bits_v : p.bits_k;
  const bool qjl = !is_v && p.qjl;
  const float *cent = p.cb + (is_v ? 2 : 0) * kMaxLevels;
  const float *thr = p.cb + (is_v ? 3 : 1) * kMaxLevels;
  const int levels = 1 << bits;
  const uint16_t *x_in = is_v ? v_in : k_in;
  uint8_t *codes_plane = is_v ? c.codes_v : c.codes_k;
  uint16_t *norm_plane = is_v ? c.norm_v : c.norm_k;
  const int cbytes = D * bits / 8;

  for (int e = tid; e < D * D; e += 128) s_pit[e] = p.pit[e];
  __syncthreads();

  const long n_rows = (long)n_tok * c.n_kv_heads;
  const long row0 = (long)blockIdx.x * kQuantRowsPerCta;
  for (long row = row0; row < row0 + kQuantRowsPerCta && row < n_rows; ++row) {
    const int t = (int)(row / c.n_kv_heads), h = (int)(row % c.n_kv_heads);
    const int s = seq_idx[t], ps = pos[t];
    const bool ok = s >= 0 && s < c.n_seqs && ps >= 0 && ps < c.capacity;
    if (!ok) {
      if (tid == 0 && !is_v) atomicOr(p.err, kErrTokenRange);
      continue;
    }
    const float x = bf16_bits_to_f32(x_in[row * D + tid]);
    s_x[tid] = x;
    // ||x||^2 in fp64: every square of a bf16 value is exact.
    double sq = (double)x * (double)x;
    for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) s_red[warp] = sq;
    __syncthreads();
    const double n64 = sqrt(s_red[0] + s_red[1] + s_red[2] + s_red[3]);
    float z = 0.f;
#pragma unroll 8
    for (int j = 0; j < D; ++j) z = fmaf(bf16_bits_to_f32(s_pit[j * D + tid]), s_x[j], z);
    const float n = (float)n64;
    const float y = n > 0.f ? z / n : 0.f;
    int code = 0;
    for (int j = 0; j < levels - 1; ++j) code += thr[j] < y ? 1 : 0;

    const long slot = ((long)s * c.n_kv_heads + h) * c.capacity + ps;
    // pack: warp w owns coordinates 32w..32w+31 (one group for 3 bits)
    uint8_t *dst = codes_plane + slot * cbytes;
    const int words = bits;  // 32 coordinates * bits / 32 bits per word
    for (int wd = 0; wd < words; ++wd) {
      uint32_t contrib = 0;
      for (int kb = 0; kb < bits; ++kb) {
        const int pbit = code_bit_pos(bits, tid, kb) - 32 * bits * warp;  // within this warp's words
        if ((pbit >> 5) == wd) contrib |= (uint32_t)((code >> kb) & 1) << (pbit & 31);
      }
      const uint32_t word = __reduce_or_sync(0xffffffffu, contrib);
      if (lane == 0) reinterpret_cast<uint32_t *>(dst)[warp * words + wd] = word;
    }
    if (tid == 0) norm_plane[slot] = __half_as_ushort(__double2half(fmin(n64, 65504.0)));

    if (qjl) {
      const float r = y - cent[code];
      s_r[tid] = r;
      float r2 = r * r;
      for (int o = 16; o; o >>= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, o);
      if (lane == 0) s_redf[warp] = r2;
      __syncthreads();
      const float gamma = sqrtf(s_redf[0] + s_redf[1] + s_redf[2] + s_redf[3]);
      float proj = 0.f;  // (S r)_tid
      for (int i = 0; i < D; ++i) proj = fmaf(p.st[i * D + tid], s_r[i], proj);
      const uint32_t sb = __ballot_sync(0xffffffffu, proj >= 0.f);
      if (lane == 0) reinterpret_cast<uint32_t *>(c.qjl_bits + slot * (D / 8))[warp] = sb;
      if (tid == 0) c.qjl_norm[slot] = f32_to_f16_bits_sat(gamma);
    }
    __syncthreads();
  }
}

}  // namespace

// MSE-only rows (all of V; K without QJL) go through the tensor-core kernel;
// K rows with the QJL stage use quantize_kernel (grid.y = 1 selects K only).
int launch_quantize(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                    const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream) {
  const bool k_on_tc = !p.qjl;
  const int e = launch_quantize_tc(p, c, k, v, seq_idx, pos, n_tok, k_on_tc, stream);
  if (e != 0 || k_on_tc) return e;
  const long rows = (long)n_tok * c.n_kv_heads;
  dim3 grid((unsigned)((rows + kQuantRowsPerCta - 1) / kQuantRowsPerCta), 1);
  quantize_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(p, c, (const uint16_t *)k, (const uint16_t *)v,
                                                          seq_idx, pos, n_tok);
  return (int)cudaGetLastError();
}

}  // namespace tq
