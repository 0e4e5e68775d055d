// Weight quantization with the method, and the matrix product over the
// packed weights, sm_100a.
//
// The same algorithm serves the weights of a linear layer (ai-accelerate.xyz
// TurboQuant explainer, "重みの量子化にも応用できる"): every row of W
// [n_out][n_in] is cut into n_in / d blocks of d coordinates and every block
// is one vector of the method (its norm, the rotation by Pi, the K codebook).
// The packed rows live in a tq_cache of one sequence whose KV heads are the
// blocks and whose positions are the rows, written by the quantize kernels.
//
// y = W~ x is never expanded back to bf16: in rotated space
//   y[t][i] = sum_b n_ib (Pi x_tb) . c[code_ib].
//   rotate  x_hat[b][t] = Pi x_tb per (block, token), as 16-bit fixed point
//           (hi, lo bytes) in the decode kernel's K fragment order, with its
//           scale factor; one CTA of d threads per (block, token), which also
//           zeroes a share of y.
//   gemm    per CTA 128 weight rows x 8 or 16 tokens, over a range of blocks: the
//           rows' codes, norms and the blocks' x_hat stream in by TMA bulk
//           copies (one producer warp, mbarrier ring, bounded waits); four
//           consumer warps of 32 rows compute each block's dot products on
//           the int8 tensor cores exactly as the decode scores (codes
//           expanded by byte permutes into exact fixed-point centroids, four
//           hi/lo products), scale them by n_ib and the token's factor and
//           sum over the blocks in fp32; partial sums over block ranges meet
//           in y by atomic adds.  It is a programmatic dependent of the
//           rotation: its first weight rows stream in while that still runs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "tq_internal.h"
#include "tq_stream.cuh"

namespace tq {
namespace {

constexpr int kWWarps = 4;
constexpr int kWThreads = 32 * (kWWarps + 1);
constexpr int kWRows = 32 * kWWarps;  // weight rows per CTA
constexpr int kWTok = 16;             // token padding of the workspace (up to two n-tiles of 8 per CTA)
constexpr int kWStages = 4;

// ------------------------------------------------------------------ rotate
// x_hat = Pi x for one (block b, token t < n_tok): thread kappa computes
// fragment position kappa (row kperm[kappa] of Pi), then the block's scale.
// The padding tokens up to a multiple of 16 are never written: the product
// reads them but never stores their results.
// It also zeroes its share of y (token t, outputs b y_chunk ..), which the
// product then accumulates into.
__global__ void __launch_bounds__(kHeadDim) weight_rotate_kernel(DeviceParams p, const void *x, int x_dtype,
                                                                 int n_tok, int n_in, int t_pad, uint8_t *xq,
                                                                 float *xf, float *y, int n_out, int y_chunk) {
  __shared__ float s_x[kHeadDim];
  __shared__ float red[kHeadDim / 32];
  const int b = blockIdx.x, t = blockIdx.y, k = threadIdx.x;
  const uint16_t *prow = p.pi + (size_t)p.kperm[k] * kHeadDim;
  // launched as a programmatic dependent: x and y are touched only once the
  // previous kernel in the stream has completed; the product may launch
  // from then on (it reads the packed weights, final by now, before it
  // waits for this grid)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (t < n_tok) {
    const int i1 = min(n_out, (b + 1) * y_chunk);
    for (int i = b * y_chunk + k; i < i1; i += kHeadDim) y[(size_t)t * n_out + i] = 0.f;
  }
  float xv = 0.f;
  if (t < n_tok) {
    const size_t idx = (size_t)t * n_in + (size_t)b * kHeadDim + k;
    xv = x_dtype == TQ_F32 ? static_cast<const float *>(x)[idx]
                           : __uint_as_float((uint32_t) static_cast<const uint16_t *>(x)[idx] << 16);
  }
  s_x[k] = xv;
  __syncthreads();
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < kHeadDim / 8; ++c) {
    const uint4 w = reinterpret_cast<const uint4 *>(prow)[c];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[e] = fmaf(__uint_as_float(u[e] << 16), s_x[8 * c + 2 * e], acc[e]);
      acc[e] = fmaf(__uint_as_float(u[e] & 0xffff0000u), s_x[8 * c + 2 * e + 1], acc[e]);
    }
  }
  const float v = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  float m = fabsf(v);
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((k & 31) == 0) red[k >> 5] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float mu = m > 0.f ? 32767.f / m : 1.f;
  const int vi = (int)rintf(v * mu);
  uint8_t *dst = xq + ((size_t)b * t_pad + t) * 2 * kHeadDim;
  dst[k] = (uint8_t)((vi >> 8) & 0xFF);
  dst[kHeadDim + k] = (uint8_t)(vi & 0xFF);
  if (k == 0) xf[(size_t)b * t_pad + t] = 1.f / (mu * ldexpf(1.f, p.k_shift));
}

// -------------------------------------------------------------------- gemm
template <int BK, int NT>
struct WStage {
  static constexpr int tok = 8 * NT;                               // tokens per CTA
  static constexpr int codes = 0;                                  // [128 rows][16 BK]
  static constexpr int norms = codes + kWRows * 16 * BK;           // [128 rows] fp16
  static constexpr int xq = norms + kWRows * 2;                    // [tok][2][128] bytes
  static constexpr int xf = xq + tok * 2 * kHeadDim;               // [tok] fp32
  static constexpr int bytes = xf + tok * 4;
};

struct WeightArgs {
  DeviceParams p;
  tq_cache w;        // one sequence; KV heads = blocks, positions = rows
  int n_out, n_blocks, n_tok, t_pad, blocks_per_split;
  const uint8_t *xq;
  const float *xf;
  float *y;          // [n_tok][n_out], accumulated with atomic adds
};

template <int BK, int NT>
__global__ void __launch_bounds__(kWThreads) weight_gemm_kernel(const WeightArgs a) {
  using St = WStage<BK, NT>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kWStages], empty_bar[kWStages];
  __shared__ int abort_flag;
  const int tile = blockIdx.x, split = blockIdx.y, tg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = lane >> 2, q = lane & 3;
  const int row0 = tile * kWRows;
  const int b0 = split * a.blocks_per_split, b1 = min(a.n_blocks, b0 + a.blocks_per_split);
  const int n_stage = b1 - b0;
  if (n_stage <= 0) return;
  if (tid == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), kWWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kWWarps) {
    // ---------------- producer: one stage per block, the tile's rows (the
    // capacity is a multiple of 64, so a ragged last tile copies 64 rows).
    // The first stages' weight rows are requested before the wait for the
    // rotation kernel (they were final before it started); their x_hat after.
    if (lane == 0) {
      const uint32_t n_rows = (uint32_t)min(kWRows, a.w.capacity - row0);
      const int pre = min(kWStages, n_stage);
      auto weights = [&](int it) {
        unsigned char *st = smem + (it % kWStages) * St::bytes;
        const uint32_t bar = smem_u32(&full_bar[it % kWStages]);
        const long tok = (long)(b0 + it) * a.w.capacity + row0;  // sequence 0, KV head b, position row0
        mbar_arrive_expect_tx(bar, n_rows * (16 * BK + 2) + St::tok * (2 * kHeadDim + 4));
        bulk_g2s(smem_u32(st + St::codes), a.w.codes_k + tok * (16 * BK), n_rows * (16 * BK), bar);
        bulk_g2s(smem_u32(st + St::norms), a.w.norm_k + tok, n_rows * 2, bar);
      };
      auto activations = [&](int it) {
        unsigned char *st = smem + (it % kWStages) * St::bytes;
        const uint32_t bar = smem_u32(&full_bar[it % kWStages]);
        const int b = b0 + it;
        bulk_g2s(smem_u32(st + St::xq), a.xq + ((size_t)b * a.t_pad + (size_t)tg * St::tok) * 2 * kHeadDim,
                 St::tok * 2 * kHeadDim, bar);
        bulk_g2s(smem_u32(st + St::xf), a.xf + (size_t)b * a.t_pad + (size_t)tg * St::tok, St::tok * 4, bar);
      };
      for (int it = 0; it < pre; ++it) weights(it);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int it = 0; it < pre; ++it) activations(it);
      int issued = pre;
      for (int it = pre; it < n_stage; ++it) {
        const int slot = it % kWStages;
        if (!mbar_wait(smem_u32(&empty_bar[slot]), ((it / kWStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        weights(it);
        activations(it);
        issued = it + 1;
      }
      if (*(volatile int *)&abort_flag) {
        for (int it = max(0, issued - kWStages); it < issued; ++it)
          mbar_wait(smem_u32(&full_bar[it % kWStages]), (it / kWStages) & 1);
      }
    }
    return;
  }

  // ---------------- consumers: rows 32 warp + 16 rb + r (+ 8), tokens 8 nt + 2 q (+ 1)
  // (y, zeroed by the rotation kernel, is accumulated into only after it completed)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const Lut lk = a.p.lut_k;
  float yacc[2][NT][4];
#pragma unroll
  for (int rb = 0; rb < 2; ++rb)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) yacc[rb][nt][e] = 0.f;
  for (int it = 0; it < n_stage; ++it) {
    const int slot = it % kWStages;
    if (!mbar_wait(smem_u32(&full_bar[slot]), (it / kWStages) & 1)) {
      atomicOr(a.p.err, kErrWaitExpired);
      abort_flag = 1;
      break;
    }
    const unsigned char *st = smem + slot * St::bytes;
    // B fragments of x_hat (tokens 8 nt + r), the tokens' factors and the rows' norms
    uint32_t xh[NT][4][2], xl[NT][4][2];
    float xfac[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t *xb = st + St::xq + (8 * nt + r) * 2 * kHeadDim;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int off = 32 * ks + 16 * sl + 4 * q;
          xh[nt][ks][sl] = *reinterpret_cast<const uint32_t *>(xb + off);
          xl[nt][ks][sl] = *reinterpret_cast<const uint32_t *>(xb + kHeadDim + off);
        }
      const float *xfs = reinterpret_cast<const float *>(st + St::xf);
      xfac[nt][0] = xfs[8 * nt + 2 * q];
      xfac[nt][1] = xfs[8 * nt + 2 * q + 1];
    }
    const __half *nrm = reinterpret_cast<const __half *>(st + St::norms);
#pragma unroll
    for (int rb = 0; rb < 2; ++rb) {
      const int lr = 32 * warp + 16 * rb + r;  // local rows lr, lr + 8
      uint32_t wk0[BK], wk1[BK];
      const unsigned char *kr0 = st + St::codes + lr * (16 * BK) + q * 4 * BK;
      const unsigned char *kr1 = kr0 + 8 * (16 * BK);
#pragma unroll
      for (int i = 0; i < BK; ++i) {
        wk0[i] = reinterpret_cast<const uint32_t *>(kr0)[i];
        wk1[i] = reinterpret_cast<const uint32_t *>(kr1)[i];
      }
      int chh[NT][4], cmid[NT][4], cll[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) chh[nt][e] = cmid[nt][e] = cll[nt][e] = 0;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t alo[4], ahi[4];
        lookup<BK>(lk, k_selector<BK>(wk0, 2 * ks), alo[0], ahi[0]);
        lookup<BK>(lk, k_selector<BK>(wk1, 2 * ks), alo[1], ahi[1]);
        lookup<BK>(lk, k_selector<BK>(wk0, 2 * ks + 1), alo[2], ahi[2]);
        lookup<BK>(lk, k_selector<BK>(wk1, 2 * ks + 1), alo[3], ahi[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_i8<true, true>(chh[nt], ahi[0], ahi[1], ahi[2], ahi[3], xh[nt][ks][0], xh[nt][ks][1]);
          mma_i8<true, false>(cmid[nt], ahi[0], ahi[1], ahi[2], ahi[3], xl[nt][ks][0], xl[nt][ks][1]);
          mma_i8<false, true>(cmid[nt], alo[0], alo[1], alo[2], alo[3], xh[nt][ks][0], xh[nt][ks][1]);
          mma_i8<false, false>(cll[nt], alo[0], alo[1], alo[2], alo[3], xl[nt][ks][0], xl[nt][ks][1]);
        }
      }
      const float n0 = __half2float(nrm[lr]), n1 = __half2float(nrm[lr + 8]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hm = (chh[nt][e] << 8) + cmid[nt][e];
          const float dot = fmaf(256.f, (float)hm, (float)cll[nt][e]);
          yacc[rb][nt][e] = fmaf(dot * xfac[nt][e & 1], e < 2 ? n0 : n1, yacc[rb][nt][e]);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[slot]));
    if (*(volatile int *)&abort_flag) break;
  }
  if (*(volatile int *)&abort_flag) return;
#pragma unroll
  for (int rb = 0; rb < 2; ++rb)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = row0 + 32 * warp + 16 * rb + r + 8 * (e >> 1);
        const int t = tg * St::tok + 8 * nt + 2 * q + (e & 1);
        if (row < a.n_out && t < a.n_tok) atomicAdd(a.y + (size_t)t * a.n_out + row, yacc[rb][nt][e]);
      }
}

using WeightFn = void (*)(const WeightArgs);

int sm_count_here() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace

size_t weight_workspace_bytes(int n_tok, int n_in) {
  const size_t t_pad = (size_t)(n_tok + kWTok - 1) / kWTok * kWTok, nb = (size_t)n_in / kHeadDim;
  const size_t xq = (nb * t_pad * 2 * kHeadDim + 255) / 256 * 256;
  return xq + (nb * t_pad * 4 + 255) / 256 * 256;
}

int launch_weight_gemm(const DeviceParams &p, const tq_cache &w, int n_out, int n_in, const void *x, int x_dtype,
                       int n_tok, float *y, char *workspace, void *stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int nb = n_in / kHeadDim;
  const int t_pad = (n_tok + kWTok - 1) / kWTok * kWTok;
  uint8_t *xq = reinterpret_cast<uint8_t *>(workspace);
  float *xf = reinterpret_cast<float *>(workspace + ((size_t)nb * t_pad * 2 * kHeadDim + 255) / 256 * 256);
  // two launches, the second a programmatic dependent of the first: the
  // rotation (which also zeroes y) and the product
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t rcfg = {};
  rcfg.gridDim = dim3(nb, n_tok);
  rcfg.blockDim = dim3(kHeadDim);
  rcfg.stream = st;
  rcfg.attrs = pdl;
  rcfg.numAttrs = 1;
  const int y_chunk = (n_out + nb - 1) / nb;
  cudaError_t e = cudaLaunchKernelEx(&rcfg, weight_rotate_kernel, p, x, x_dtype, n_tok, n_in, t_pad, xq, xf, y, n_out,
                                     y_chunk);
  if (e != cudaSuccess) return (int)e;
  // split the blocks so that the grid fills about four CTAs per SM
  // one n-tile of 8 tokens per CTA for up to 8 tokens, else two
  const int nt = n_tok <= 8 ? 1 : 2;
  const int tiles = (n_out + kWRows - 1) / kWRows, groups = (n_tok + 8 * nt - 1) / (8 * nt);
  const long units = (long)tiles * groups;
  const long want = 2L * sm_count_here() * 2;
  int splits = (int)std::max(1L, std::min<long>(nb, (want + units - 1) / units));
  const int per = (nb + splits - 1) / splits;
  splits = (nb + per - 1) / per;
  const WeightFn fn = nt == 1 ? (p.bits_k == 2 ? weight_gemm_kernel<2, 1> : p.bits_k == 3 ? weight_gemm_kernel<3, 1>
                                                                                         : weight_gemm_kernel<4, 1>)
                              : (p.bits_k == 2 ? weight_gemm_kernel<2, 2> : p.bits_k == 3 ? weight_gemm_kernel<3, 2>
                                                                                         : weight_gemm_kernel<4, 2>);
  const int smem = kWStages * (nt == 1 ? (p.bits_k == 2 ? WStage<2, 1>::bytes : p.bits_k == 3 ? WStage<3, 1>::bytes
                                                                                             : WStage<4, 1>::bytes)
                                       : (p.bits_k == 2 ? WStage<2, 2>::bytes : p.bits_k == 3 ? WStage<3, 2>::bytes
                                                                                             : WStage<4, 2>::bytes));
  static std::atomic<bool> configured[kMaxDevices][3][2];
  std::atomic<bool> &done = configured[current_device()][p.bits_k - 2][nt - 1];
  if (!done.load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    done.store(true, std::memory_order_release);
  }
  WeightArgs args{p, w, n_out, nb, n_tok, t_pad, per, xq, xf, y};
  cudaLaunchConfig_t gcfg = {};
  gcfg.gridDim = dim3(tiles, splits, groups);
  gcfg.blockDim = dim3(kWThreads);
  gcfg.dynamicSmemBytes = smem;
  gcfg.stream = st;
  gcfg.attrs = pdl;
  gcfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&gcfg, fn, args);
}

}  // namespace tq
