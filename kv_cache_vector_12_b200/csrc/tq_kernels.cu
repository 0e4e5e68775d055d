// TurboQuant kernels for sm_100a.
//
// quantize_kernel      norm, rotation by Pi, Lloyd-Max codes, bit-pack, QJL
// rotate_q_kernel      q_hat = Pi q (and q_tilde = S q_hat)
// decode_attn_kernel   split-K attention over the packed cache, partials (m, l, o~)
// merge_kernel         log-sum-exp merge of the splits, o = Pi^T o~
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

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Bit position of bit k of coordinate i's code inside a packed vector (the
// layout documented in tq.h).
__device__ __forceinline__ int code_bit_pos(int bits, int i, int k) {
  if (bits != 3) return i * bits + k;
  const int g = i >> 5, l = i & 31;
  if (l < 24) return 96 * g + 32 * (l >> 3) + 4 * (l & 7) + k;
  return 96 * g + 32 * k + 4 * (l - 24) + 3;
}

__device__ __forceinline__ int read_code(const uint8_t *vec, int bits, int i) {
  int c = 0;
  for (int k = 0; k < bits; ++k) {
    const int p = code_bit_pos(bits, i, k);
    c |= ((vec[p >> 3] >> (p & 7)) & 1) << k;
  }
  return c;
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

// ---------------------------------------------------------------------------
// rotate_q: q_hat = Pi q, q_tilde = S q_hat; one CTA per (sequence, q head).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) rotate_q_kernel(DeviceParams p, const void *q, int q_dtype,
                                                       float *q_hat, float *q_tilde) {
  __shared__ float s_q[D];
  __shared__ float s_qh[D];
  const int row = blockIdx.x, tid = threadIdx.x;
  s_q[tid] = q_dtype == TQ_F32 ? static_cast<const float *>(q)[(long)row * D + tid]
                               : bf16_bits_to_f32(static_cast<const uint16_t *>(q)[(long)row * D + tid]);
  __syncthreads();
  float acc = 0.f;
  for (int j = 0; j < D; ++j) acc = fmaf(bf16_bits_to_f32(p.pit[j * D + tid]), s_q[j], acc);
  q_hat[(long)row * D + tid] = acc;
  if (p.qjl) {
    s_qh[tid] = acc;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < D; ++i) t = fmaf(p.st[i * D + tid], s_qh[i], t);
    q_tilde[(long)row * D + tid] = t;
  }
}

// ---------------------------------------------------------------------------
// decode attention, one CTA per (split, KV head, sequence); 4 warps, each
// warp walks every 4th token of the split; lane l owns coordinates 4l..4l+3.
// ---------------------------------------------------------------------------
constexpr int kMaxGroup = 16;

__global__ void __launch_bounds__(128) decode_attn_kernel(DeviceParams p, tq_cache c, int n_q_heads,
                                                          const int32_t *__restrict__ seq_lens,
                                                          int max_seq_len, float scale, int chunk,
                                                          int n_splits, const float *__restrict__ q_hat,
                                                          const float *__restrict__ q_tilde,
                                                          float *__restrict__ partials) {
  __shared__ float s_m[4][kMaxGroup], s_l[4][kMaxGroup];
  __shared__ float s_o[4][kMaxGroup][D];
  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = n_q_heads / c.n_kv_heads;
  int len = seq_lens[s];
  if (len < 0 || len > max_seq_len) {
    if (tid == 0 && split == 0 && h == 0) atomicOr(p.err, kErrSeqLen);
    len = len < 0 ? 0 : max_seq_len;
  }
  const int t0 = split * chunk, t1 = min(len, t0 + chunk);
  const float *ck = p.cb, *cv = p.cb + 2 * kMaxLevels;
  const int bk = p.bits_k, bv = p.bits_v;
  const int kbytes = D * bk / 8, vbytes = D * bv / 8;
  const long base = ((long)s * c.n_kv_heads + h) * c.capacity;

  float qh[kMaxGroup][4], qt[kMaxGroup][4];
  for (int g = 0; g < G; ++g)
    for (int e = 0; e < 4; ++e) {
      const long r = ((long)s * n_q_heads + h * G + g) * D + 4 * lane + e;
      qh[g][e] = q_hat[r];
      qt[g][e] = p.qjl ? q_tilde[r] : 0.f;
    }
  float m[kMaxGroup], l[kMaxGroup], o[kMaxGroup][4];
  for (int g = 0; g < kMaxGroup; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
    for (int e = 0; e < 4; ++e) o[g][e] = 0.f;
  }
  const float qjl_c = sqrtf(0.5f * (float)M_PI) / (float)D;
  for (int t = t0 + warp; t < t1; t += 4) {
    const uint8_t *kv = c.codes_k + (base + t) * kbytes;
    const uint8_t *vv = c.codes_v + (base + t) * vbytes;
    float kc[4], vc[4], sg[4];
    for (int e = 0; e < 4; ++e) {
      kc[e] = ck[read_code(kv, bk, 4 * lane + e)];
      vc[e] = cv[read_code(vv, bv, 4 * lane + e)];
      if (p.qjl) {
        const int mm = 4 * lane + e;
        sg[e] = ((c.qjl_bits[(base + t) * (D / 8) + (mm >> 3)] >> (mm & 7)) & 1) ? 1.f : -1.f;
      }
    }
    const float nk = f16_bits_to_f32(c.norm_k[base + t]);
    const float nv = f16_bits_to_f32(c.norm_v[base + t]);
    const float gam = p.qjl ? f16_bits_to_f32(c.qjl_norm[base + t]) : 0.f;
    for (int g = 0; g < G; ++g) {
      float dot = 0.f, cor = 0.f;
      for (int e = 0; e < 4; ++e) {
        dot = fmaf(qh[g][e], kc[e], dot);
        if (p.qjl) cor = fmaf(qt[g][e], sg[e], cor);
      }
      for (int off = 16; off; off >>= 1) {
        dot += __shfl_xor_sync(0xffffffffu, dot, off);
        cor += __shfl_xor_sync(0xffffffffu, cor, off);
      }
      const float sc = scale * nk * (dot + (p.qjl ? qjl_c * gam * cor : 0.f));
      const float mn = fmaxf(m[g], sc);
      const float alpha = __expf(m[g] - mn);
      const float pw = __expf(sc - mn);
      l[g] = l[g] * alpha + pw;
      for (int e = 0; e < 4; ++e) o[g][e] = o[g][e] * alpha + pw * nv * vc[e];
      m[g] = mn;
    }
  }
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      s_m[warp][g] = m[g];
      s_l[warp][g] = l[g];
    }
    for (int e = 0; e < 4; ++e) s_o[warp][g][4 * lane + e] = o[g][e];
  }
  __syncthreads();
  // thread tid combines the 4 warps for coordinate tid of every head
  for (int g = 0; g < G; ++g) {
    float mm = -INFINITY;
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, s_m[w][g]);
    float ll = 0.f, oo = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = s_m[w][g] == -INFINITY ? 0.f : __expf(s_m[w][g] - mm);
      ll += f * s_l[w][g];
      oo += f * s_o[w][g][tid];
    }
    float *dst = partials + (((long)s * n_q_heads + h * G + g) * n_splits + split) * (D + 2);
    dst[2 + tid] = oo;
    if (tid == 0) {
      dst[0] = mm;
      dst[1] = ll;
    }
  }
}

// ---------------------------------------------------------------------------
// merge: one CTA per (sequence, q head): combine splits, o = Pi^T o~ / L.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) merge_kernel(DeviceParams p, int n_q_heads,
                                                    const int32_t *__restrict__ seq_lens, int max_seq_len,
                                                    int chunk, int n_splits,
                                                    const float *__restrict__ partials, float *out,
                                                    float *lse) {
  __shared__ float s_ot[D];
  const int row = blockIdx.x, tid = threadIdx.x;
  const int s = row / n_q_heads;
  int len = seq_lens[s];
  len = len < 0 ? 0 : (len > max_seq_len ? max_seq_len : len);
  const int used = (len + chunk - 1) / chunk;
  const float *src = partials + (long)row * n_splits * (D + 2);
  float mm = -INFINITY;
  for (int sp = 0; sp < used; ++sp) mm = fmaxf(mm, src[sp * (D + 2)]);
  float ll = 0.f, oo = 0.f;
  for (int sp = 0; sp < used; ++sp) {
    const float ms = src[sp * (D + 2)];
    if (ms == -INFINITY) continue;
    const float f = __expf(ms - mm);
    ll += f * src[sp * (D + 2) + 1];
    oo += f * src[sp * (D + 2) + 2 + tid];
  }
  s_ot[tid] = ll > 0.f ? oo / ll : 0.f;
  __syncthreads();
  float acc = 0.f;  // (Pi^T o~)_tid = sum_k Pi[k][tid] o~_k
  for (int kk = 0; kk < D; ++kk) acc = fmaf(bf16_bits_to_f32(p.pi[kk * D + tid]), s_ot[kk], acc);
  out[(long)row * D + tid] = acc;
  if (lse && tid == 0) lse[row] = ll > 0.f ? mm + logf(ll) : -INFINITY;
}

}  // namespace

int launch_quantize(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                    const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream) {
  const long rows = (long)n_tok * c.n_kv_heads;
  dim3 grid((unsigned)((rows + kQuantRowsPerCta - 1) / kQuantRowsPerCta), 2);
  quantize_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(p, c, (const uint16_t *)k, (const uint16_t *)v,
                                                          seq_idx, pos, n_tok);
  return (int)cudaGetLastError();
}

int launch_decode(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype, int n_q_heads,
                  const int32_t *seq_lens, int max_seq_len, float scale, float *out, float *lse,
                  char *workspace, const DecodeSplit &split, const DecodeWorkspace &ws, void *stream) {
  cudaStream_t st = (cudaStream_t)stream;
  float *q_hat = (float *)(workspace + ws.q_hat);
  float *q_tilde = (float *)(workspace + ws.q_tilde);
  float *partials = (float *)(workspace + ws.partials);
  const int rows = c.n_seqs * n_q_heads;
  rotate_q_kernel<<<rows, 128, 0, st>>>(p, q, q_dtype, q_hat, q_tilde);
  dim3 grid(split.n_splits, c.n_kv_heads, c.n_seqs);
  decode_attn_kernel<<<grid, 128, 0, st>>>(p, c, n_q_heads, seq_lens, max_seq_len, scale, split.chunk,
                                           split.n_splits, q_hat, q_tilde, partials);
  merge_kernel<<<rows, 128, 0, st>>>(p, n_q_heads, seq_lens, max_seq_len, split.chunk, split.n_splits,
                                     partials, out, lse);
  return (int)cudaGetLastError();
}

}  // namespace tq
