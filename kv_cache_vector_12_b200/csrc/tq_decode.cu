// Decode attention over the packed TurboQuant cache, sm_100a.
//
// The method reads K and V straight from their codes ("TurboQuantの仕組み",
// ai-accelerate.xyz explainer: rotate once, per-coordinate Lloyd-Max codes,
// optional 1-bit QJL residual signs).  Per (sequence, KV head, split of the
// sequence) one CTA streams the split's packed codes and norms into a shared
// memory ring with TMA bulk copies (one producer warp, mbarrier pipeline with
// bounded waits) while four consumer warps each take 32 tokens of every
// 128-token stage.  Before the first stage arrives the consumers rotate the
// KV head's queries themselves:
//
//   q_hat   Pi q for the G query heads on the tensor cores (mma m16n8k16
//           bf16, fp32 q as an exact hi + lo pair), then 16-bit fixed point;
//           with QJL also q_tilde = S q_hat (fp32).
//   scores  S[tok][head] = q_hat . c_K[code]   int8 tensor cores (mma m16n8k32):
//           K centroids are exact 16-bit fixed-point integers (c * 2^17), split
//           into hi/lo bytes by two byte-permute lookups per 4 codes; q_hat is
//           16-bit fixed point (hi/lo bytes), so the dot product is exact up to
//           q_hat's rounding.  QJL signs become 0/-1 bytes (sign-replicating
//           byte permute) against q_tilde in the same int8 MMA.
//   softmax online per warp and query head (exp2), masked past seq_len.
//   values  O^T[coord][head] += V~^T[coord][tok] P[tok][head]   fp16 tensor
//           cores (mma m16n8k16): fp16 centroids looked up by byte permutes,
//           P transposed into the B fragment with movmatrix.
//
// The coordinate order inside the MMA fragments is a fixed permutation of the
// head dimension chosen so that every code is expanded where it is loaded; the
// host computes the permutations (tq_fragments.cpp) and stores Pi's rows in
// the K order (so q_hat comes out of its MMA already in that order) and S in
// the QJL and K orders; merge applies Pi^T with rows in the V order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>

#include "tq_internal.h"
#include "tq_stream.cuh"

namespace tq {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kWarpTokens = 32;                            // tokens per consumer warp per stage
constexpr int kStageTokens = kWarpTokens * kConsumerWarps;  // 128
constexpr int kStages = 4;
constexpr int kPrefetchTokens = kStages * kStageTokens;  // L2 prefetch before the dependency wait

// Barrier of the four consumer warps only (the producer warp never joins).
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(32 * kConsumerWarps) : "memory");
}

struct DecodeArgs {
  DeviceParams p;
  tq_cache c;
  int n_q_heads, max_seq_len, chunk, n_splits;
  const int32_t *seq_lens;
  const void *q;          // [n_seqs][n_q_heads][d], fp32 or bf16 (q_dtype)
  int q_dtype;
  float scale;
  float *partials;        // [rows][n_splits][d + 4]
};

// Two register budgets of the same kernel, chosen per call from the split
// length (tq_api.cu): CTAS = 2 (168 registers) for short splits, where fewer
// CTAs amortise the per-CTA prologue and each warp has room for more
// independent work; CTAS = 3 (128 registers) for long splits, where twelve
// consumer warps per SM hide more latency in the steady state.
//
// PAGED selects the paged cache layout (the stage copies follow the block
// table); it is its own instantiation so that the contiguous kernels keep
// their code and register allocation.
template <int BK, int BV, bool QJL, int NT, int CTAS, bool PAGED>
__global__ void __maxnreg__(CTAS == 3 ? 128 : 168) decode_mma_kernel(const DecodeArgs a) {
  static_assert(kStageTokens % 64 == 0 && kWarpTokens == 32, "stages start on 64-token boundaries");
  using St = Stage<BK, BV, QJL, kStageTokens>;
  constexpr int kRows = 8 * NT;  // query-head rows of the score MMAs
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ int abort_flag;
  __shared__ float sm_m[kConsumerWarps][kRows], sm_l[kConsumerWarps][kRows];
  __shared__ __align__(16) uint8_t s_q8[kRows][QJL ? 4 : 2][D];  // q_hat hi, lo; q_tilde hi, lo (fragment orders)
  __shared__ __align__(16) float s_qf[QJL ? kRows : 1][D];       // q_hat, fp32, K order (QJL input)
  __shared__ float s_qs[kRows][4];                                // score factor, QJL factor, sum of q_tilde ints
  __shared__ float s_red[kConsumerWarps][kRows];

  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, q = lane & 3;
  const int G = a.n_q_heads / a.c.n_kv_heads;
  // B fragments of Pi (rows in the K fragment order) for this consumer warp's
  // 32 output positions: parameters, loaded before waiting for the previous
  // kernel in the stream
  uint32_t bfr[4][8][2];
  if (warp < kConsumerWarps) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = reinterpret_cast<const uint4 *>(a.p.pikf)[((warp * 4 + nt) * 4 + j) * 32 + lane];
        bfr[nt][2 * j][0] = v.x;
        bfr[nt][2 * j][1] = v.y;
        bfr[nt][2 * j + 1][0] = v.z;
        bfr[nt][2 * j + 1][1] = v.w;
      }
  }
  // While the previous kernel (typically the append) still runs, warm L2 with
  // the first stages this CTA will stream.  A prefetch only moves lines into
  // L2, the point of coherence, so whatever the previous kernel writes there
  // is what the copies read after the wait; lengths are not known yet, so the
  // split's whole range (below the length bound and the capacity) is fetched.
  if (warp == kConsumerWarps && lane == 0) {
    // this KV head's query rows and the sequence length (read right after the wait)
    const size_t qbytes = (size_t)G * D * (a.q_dtype == TQ_F32 ? 4 : 2);
    prefetch_l2(static_cast<const char *>(a.q) + ((size_t)s * a.n_q_heads + (size_t)h * G) * D *
                                                     (a.q_dtype == TQ_F32 ? 4 : 2),
                (uint32_t)qbytes);
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.seq_lens + s));
    const int first = split * a.chunk;
    const int last = min(min(first + a.chunk, a.max_seq_len), min(first + kPrefetchTokens, a.c.capacity));
    // (contiguous layout only: a paged cache's block table is not read before the wait)
    if (!PAGED && first < last) {
      const long tok = ((long)s * a.c.n_kv_heads + h) * a.c.capacity + first;
      const uint32_t n = (uint32_t)(last - first);
      prefetch_l2(a.c.codes_k + tok * (D * BK / 8), n * (D * BK / 8));
      prefetch_l2(a.c.codes_v + tok * (D * BV / 8), n * (D * BV / 8));
      prefetch_l2(a.c.norm_k + tok, (n * 2 + 15) & ~15u);
      prefetch_l2(a.c.norm_v + tok, (n * 2 + 15) & ~15u);
      if constexpr (QJL) {
        prefetch_l2(a.c.qjl_bits + tok * (D / 8), n * (D / 8));
        prefetch_l2(a.c.qjl_norm + tok, (n * 2 + 15) & ~15u);
      }
    }
  }
  // launched as a programmatic dependent: the cache, q and seq_lens are final
  // once the previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int len = a.seq_lens[s];
  if (len < 0 || len > a.max_seq_len) {
    if (tid == 0 && split == 0 && h == 0) atomicOr(a.p.err, kErrSeqLen);
    len = len < 0 ? 0 : a.max_seq_len;
  }
  const int t0 = split * a.chunk;
  if (t0 >= len) return;  // this split holds no tokens; merge skips it
  const int t1 = min(len, t0 + a.chunk);
  const int n_stage = (t1 - t0 + kStageTokens - 1) / kStageTokens;
  const long base = ((long)s * a.c.n_kv_heads + h) * a.c.capacity;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), kConsumerWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one elected lane issues the bulk copies
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_stage; ++it) {
        const int slot = it % kStages;
        if (it >= kStages && !mbar_wait(smem_u32(&empty_bar[slot]), ((it / kStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        unsigned char *st = smem + slot * St::bytes;
        const uint32_t bar = smem_u32(&full_bar[slot]);
        const int first = t0 + it * kStageTokens;  // multiple of 64, below the split's end t1
        // a stage copies its tokens below t1 rounded up to a multiple of 64:
        // never past the capacity (a multiple of 64 at or above t1), and in a
        // paged cache never from a block that holds no position below t1, so
        // the table entries of blocks past the length are not read
        const uint32_t n = (uint32_t)min(kStageTokens, (t1 - first + 63) & ~63);
        const uint32_t bytes = n * (D * BK / 8 + D * BV / 8 + 4 + (QJL ? D / 8 + 2 : 0));
        mbar_arrive_expect_tx(bar, bytes);
        if constexpr (!PAGED) {
          const long tok = base + first;
          bulk_g2s(smem_u32(st + St::kc), a.c.codes_k + tok * (D * BK / 8), n * (D * BK / 8), bar);
          bulk_g2s(smem_u32(st + St::vc), a.c.codes_v + tok * (D * BV / 8), n * (D * BV / 8), bar);
          bulk_g2s(smem_u32(st + St::kn), a.c.norm_k + tok, n * 2, bar);
          bulk_g2s(smem_u32(st + St::vn), a.c.norm_v + tok, n * 2, bar);
          if constexpr (QJL) {
            bulk_g2s(smem_u32(st + St::jb), a.c.qjl_bits + tok * (D / 8), n * (D / 8), bar);
            bulk_g2s(smem_u32(st + St::jg), a.c.qjl_norm + tok, n * 2, bar);
          }
        } else {
          // the stage in runs of consecutive slots, one per block it touches
          // (block sizes are multiples of 64, so every run is too and every
          // copy stays 16-byte aligned at both ends)
          for (uint32_t done = 0; done < n;) {
            const int p = first + (int)done, j = p / a.c.block_size, off = p - j * a.c.block_size;
            const uint32_t run = min(n - done, (uint32_t)(a.c.block_size - off));
            int blk = a.c.block_table[(long)s * (a.c.capacity / a.c.block_size) + j];
            if (blk < 0 || blk >= a.c.n_blocks) {  // flagged; a valid block is read in its place
              atomicOr(a.p.err, kErrTokenRange);
              blk = 0;
            }
            const long tok = ((long)blk * a.c.n_kv_heads + h) * a.c.block_size + off;
            bulk_g2s(smem_u32(st + St::kc + done * (D * BK / 8)), a.c.codes_k + tok * (D * BK / 8),
                     run * (D * BK / 8), bar);
            bulk_g2s(smem_u32(st + St::vc + done * (D * BV / 8)), a.c.codes_v + tok * (D * BV / 8),
                     run * (D * BV / 8), bar);
            bulk_g2s(smem_u32(st + St::kn + done * 2), a.c.norm_k + tok, run * 2, bar);
            bulk_g2s(smem_u32(st + St::vn + done * 2), a.c.norm_v + tok, run * 2, bar);
            if constexpr (QJL) {
              bulk_g2s(smem_u32(st + St::jb + done * (D / 8)), a.c.qjl_bits + tok * (D / 8), run * (D / 8), bar);
              bulk_g2s(smem_u32(st + St::jg + done * 2), a.c.qjl_norm + tok, run * 2, bar);
            }
            done += run;
          }
        }
        issued = it + 1;
      }
      // never leave the CTA with copies in flight: wait (bounded) for the
      // last stages issued if the consumers stopped early
      if (*(volatile int *)&abort_flag) {
        for (int it = max(0, issued - kStages); it < issued; ++it)
          mbar_wait(smem_u32(&full_bar[it % kStages]), (it / kStages) & 1);
      }
    }
  } else {
    // ---------------- consumers
    // q_hat = Pi q for this KV head's query heads on the tensor cores: mma
    // m16n8k16 bf16 with the heads as rows and the K fragment positions as
    // columns (Pi's rows are stored in that order), fp32 q split into a bf16
    // hi + lo pair so every product is exact and the sums are fp32.  Warp w
    // computes positions 32 w .. 32 w + 31.
    {
      const long qrow0 = (long)s * a.n_q_heads + (long)h * G;
      const bool f32 = a.q_dtype == TQ_F32;
      float c[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // a0: row r; a1: row r + 8; a2, a3: the same rows, columns + 8
          const int row = r + 8 * (e & 1), col = 16 * ks + 8 * (e >> 1) + 2 * q;
          float x0 = 0.f, x1 = 0.f;
          if (row < G) {
            if (f32) {
              const float2 v = *reinterpret_cast<const float2 *>(static_cast<const float *>(a.q) + (qrow0 + row) * D + col);
              x0 = v.x;
              x1 = v.y;
            } else {
              const uint32_t v = *reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(a.q) + (qrow0 + row) * D + col);
              x0 = __uint_as_float(v << 16);
              x1 = __uint_as_float(v & 0xffff0000u);
            }
          }
          split_bf16x2(x0, x1, ahi[e], alo[e]);
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          mma_bf16(c[nt], ahi[0], ahi[1], ahi[2], ahi[3], bfr[nt][ks][0], bfr[nt][ks][1]);
          if (f32) mma_bf16(c[nt], alo[0], alo[1], alo[2], alo[3], bfr[nt][ks][0], bfr[nt][ks][1]);
        }
      }
      // per head: mu = 32767 / max |q_hat|, q_hat as 16-bit fixed point (hi, lo bytes)
      float mx0 = 0.f, mx1 = 0.f;  // rows r, r + 8
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(fabsf(c[nt][0]), fabsf(c[nt][1])));
        mx1 = fmaxf(mx1, fmaxf(fabsf(c[nt][2]), fabsf(c[nt][3])));
      }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (q == 0) {
        s_red[warp][r] = mx0;
        if constexpr (kRows > 8) s_red[warp][r + 8] = mx1;
      }
      consumer_sync();
      float mu[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (kRows <= 8 && e == 1) break;
        const int row = r + 8 * e;
        const float m = fmaxf(fmaxf(s_red[0][row], s_red[1][row]), fmaxf(s_red[2][row], s_red[3][row]));
        mu[e] = m > 0.f ? 32767.f / m : 1.f;
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int kap = 32 * warp + 8 * nt + 2 * q;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (kRows <= 8 && e == 1) break;
          const int row = r + 8 * e;
          const int v0 = (int)rintf(c[nt][2 * e] * mu[e]), v1 = (int)rintf(c[nt][2 * e + 1] * mu[e]);
          *reinterpret_cast<uint16_t *>(&s_q8[row][0][kap]) = (uint16_t)(((v0 >> 8) & 0xFF) | (((v1 >> 8) & 0xFF) << 8));
          *reinterpret_cast<uint16_t *>(&s_q8[row][1][kap]) = (uint16_t)((v0 & 0xFF) | ((v1 & 0xFF) << 8));
          if constexpr (QJL) *reinterpret_cast<float2 *>(&s_qf[row][kap]) = make_float2(c[nt][2 * e], c[nt][2 * e + 1]);
        }
      }
      if (warp == 0 && q == 0) {
        s_qs[r][0] = a.scale * kLog2e / (mu[0] * (float)(1 << kKFixedShift));
        if constexpr (kRows > 8) s_qs[r + 8][0] = a.scale * kLog2e / (mu[1] * (float)(1 << kKFixedShift));
      }
      if constexpr (QJL) {
        // q_tilde = S q_hat: position tid (QJL fragment order) of every head,
        // from row tid of S permuted into the QJL (rows) and K (columns) orders
        consumer_sync();
        float qt[kRows];
#pragma unroll
        for (int g = 0; g < kRows; ++g) qt[g] = 0.f;
        const float4 *srow = reinterpret_cast<const float4 *>(a.p.sjk + tid * D);
#pragma unroll 4
        for (int c4 = 0; c4 < D / 4; ++c4) {
          const float4 w4 = srow[c4];
#pragma unroll
          for (int g = 0; g < kRows; ++g) {
            const float4 x = *reinterpret_cast<const float4 *>(&s_qf[g][4 * c4]);
            qt[g] = fmaf(w4.x, x.x, fmaf(w4.y, x.y, fmaf(w4.z, x.z, fmaf(w4.w, x.w, qt[g]))));
          }
        }
        // nu = 32767 / max |q_tilde| per head, then the ints and their sum
#pragma unroll
        for (int g = 0; g < kRows; ++g) {
          float m = fabsf(qt[g]);
#pragma unroll
          for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) s_red[warp][g] = m;
        }
        consumer_sync();
        float nu[kRows];
#pragma unroll
        for (int g = 0; g < kRows; ++g) {
          const float m = fmaxf(fmaxf(s_red[0][g], s_red[1][g]), fmaxf(s_red[2][g], s_red[3][g]));
          nu[g] = m > 0.f ? 32767.f / m : 1.f;
          if (tid == g) s_qs[g][1] = a.scale * kLog2e * kSqrtHalfPi / ((float)D * nu[g]);
        }
        consumer_sync();  // s_red is reused for the sums
#pragma unroll
        for (int g = 0; g < kRows; ++g) {
          const int vi = (int)rintf(qt[g] * nu[g]);
          s_q8[g][2][tid] = (uint8_t)(vi >> 8);
          s_q8[g][3][tid] = (uint8_t)(vi & 0xFF);
          int sum = vi;
#pragma unroll
          for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) s_red[warp][g] = (float)sum;  // |sum| < 2^22: exact
        }
        consumer_sync();
        if (tid < kRows) s_qs[tid][2] = (s_red[0][tid] + s_red[1][tid]) + (s_red[2][tid] + s_red[3][tid]);
      }
      consumer_sync();
    }
    // q fragments (int8, K fragment order) of this thread's head r in every n-tile
    uint32_t qh[NT][4][2], ql[NT][4][2], jh[NT][QJL ? 4 : 1][2], jl[NT][QJL ? 4 : 1][2];
    float fq[NT][2], fj[NT][2], jsum[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t *qb = &s_q8[8 * nt + r][0][0];
#pragma unroll
      for (int st = 0; st < 4; ++st)
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int off = 32 * st + 16 * sl + 4 * q;
          qh[nt][st][sl] = *reinterpret_cast<const uint32_t *>(qb + off);
          ql[nt][st][sl] = *reinterpret_cast<const uint32_t *>(qb + D + off);
          if constexpr (QJL) {
            jh[nt][st][sl] = *reinterpret_cast<const uint32_t *>(qb + 2 * D + off);
            jl[nt][st][sl] = *reinterpret_cast<const uint32_t *>(qb + 3 * D + off);
          }
        }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int gg = 8 * nt + 2 * q + e;  // heads past G have zero q and zero factors
        fq[nt][e] = gg < G ? s_qs[gg][0] : 0.f;
        fj[nt][e] = gg < G && QJL ? s_qs[gg][1] : 0.f;
        jsum[nt][e] = gg < G && QJL ? s_qs[gg][2] : 0.f;
      }
    }
    const Lut lk = a.p.lut_k, lv = a.p.lut_v;

    float m_run[NT][2], l_run[NT][2], acc[NT][8][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        m_run[nt][e] = -INFINITY;
        l_run[nt][e] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
    }

    for (int it = 0; it < n_stage; ++it) {
      const int slot = it % kStages;
      if (!mbar_wait(smem_u32(&full_bar[slot]), (it / kStages) & 1)) {
        atomicOr(a.p.err, kErrWaitExpired);
        abort_flag = 1;
        break;
      }
      const unsigned char *st = smem + slot * St::bytes;
      const int tok0 = t0 + it * kStageTokens + kWarpTokens * warp;  // first token of this warp's tile
      if (tok0 < t1) {
        const int wt = kWarpTokens * warp;                             // tile row offset inside the stage
        // ---------------- scores: int8 MMA, two 16-token row blocks, 4 k-steps of 32
        int chh[2][NT][4], cmid[2][NT][4], cll[2][NT][4], cjh[2][NT][4], cjl[2][NT][4];
#pragma unroll
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) chh[rb][nt][e] = cmid[rb][nt][e] = cll[rb][nt][e] = cjh[rb][nt][e] = cjl[rb][nt][e] = 0;
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
          uint32_t wk0[BK], wk1[BK];
          const unsigned char *kr0 = st + St::kc + (wt + 16 * rb + r) * (D * BK / 8) + q * 4 * BK;
          const unsigned char *kr1 = kr0 + 8 * (D * BK / 8);
#pragma unroll
          for (int i = 0; i < BK; ++i) {
            wk0[i] = reinterpret_cast<const uint32_t *>(kr0)[i];
            wk1[i] = reinterpret_cast<const uint32_t *>(kr1)[i];
          }
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t alo[4], ahi[4];
            lookup<BK>(lk, k_selector<BK>(wk0, 2 * ks), alo[0], ahi[0]);
            lookup<BK>(lk, k_selector<BK>(wk1, 2 * ks), alo[1], ahi[1]);
            lookup<BK>(lk, k_selector<BK>(wk0, 2 * ks + 1), alo[2], ahi[2]);
            lookup<BK>(lk, k_selector<BK>(wk1, 2 * ks + 1), alo[3], ahi[3]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_i8<true, true>(chh[rb][nt], ahi[0], ahi[1], ahi[2], ahi[3], qh[nt][ks][0], qh[nt][ks][1]);
              mma_i8<true, false>(cmid[rb][nt], ahi[0], ahi[1], ahi[2], ahi[3], ql[nt][ks][0], ql[nt][ks][1]);
              mma_i8<false, true>(cmid[rb][nt], alo[0], alo[1], alo[2], alo[3], qh[nt][ks][0], qh[nt][ks][1]);
              mma_i8<false, false>(cll[rb][nt], alo[0], alo[1], alo[2], alo[3], ql[nt][ks][0], ql[nt][ks][1]);
            }
          }
          if constexpr (QJL) {
            const uint32_t w0 = reinterpret_cast<const uint32_t *>(st + St::jb + (wt + 16 * rb + r) * (D / 8))[q];
            const uint32_t w1 = reinterpret_cast<const uint32_t *>(st + St::jb + (wt + 16 * rb + r + 8) * (D / 8))[q];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              // bytes 0x00 / 0xFF (= -bit) for bits j, j+8, j+16, j+24 with j = 2 ks + slot
              const int j0 = 2 * ks, j1 = 2 * ks + 1;
              const uint32_t a0 = prmt(w0 << (7 - j0), 0u, 0xBA98u), a1 = prmt(w1 << (7 - j0), 0u, 0xBA98u);
              const uint32_t a2 = prmt(w0 << (7 - j1), 0u, 0xBA98u), a3 = prmt(w1 << (7 - j1), 0u, 0xBA98u);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_i8<true, true>(cjh[rb][nt], a0, a1, a2, a3, jh[nt][ks][0], jh[nt][ks][1]);
                mma_i8<true, false>(cjl[rb][nt], a0, a1, a2, a3, jl[nt][ks][0], jl[nt][ks][1]);
              }
            }
          }
        }
        // ---------------- scores -> online softmax over the 32 tokens
        // this thread's tokens: wt + 16 rb + r + 8 hf  (rb, hf in {0, 1})
        const __half *kn = reinterpret_cast<const __half *>(st + St::kn) + wt;
        const __half *vn = reinterpret_cast<const __half *>(st + St::vn) + wt;
        float nk[4], nv[4], gm[4];
        const bool partial = tok0 + kWarpTokens > t1;  // only the last tile of a split is ragged
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tt = 16 * (u >> 1) + r + 8 * (u & 1);
          nk[u] = __half2float(kn[tt]);
          nv[u] = __half2float(vn[tt]);
          gm[u] = 0.f;
          if constexpr (QJL) gm[u] = __half2float(reinterpret_cast<const __half *>(st + St::jg)[wt + tt]);
          if (partial && tok0 + tt >= t1) nk[u] = nv[u] = gm[u] = __int_as_float(0x7fc00000);  // NaN marks "masked"
        }
        uint32_t pb[2][NT][2];
        bool rescale = false;
        float alpha[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float sc[4][2];  // [token u][head hd]
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
              const int rb = u >> 1, e = 2 * (u & 1) + hd;
              // 65536 hh + 256 mid + ll = 256 (256 hh + mid) + ll; 256 hh + mid fits int32
              const int hm = (chh[rb][nt][e] << 8) + cmid[rb][nt][e];
              float v = fmaf(256.f, (float)hm, (float)cll[rb][nt][e]) * fq[nt][hd];
              if constexpr (QJL) {
                const float dj = fmaf(256.f, (float)cjh[rb][nt][e], (float)cjl[rb][nt][e]);
                v = fmaf(gm[u] * fj[nt][hd], fmaf(-2.f, dj, -jsum[nt][hd]), v);
              }
              sc[u][hd] = v * nk[u];
            }
          if (partial) {  // masked tokens carry NaN norms: their scores become -inf, their weights 0
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int hd = 0; hd < 2; ++hd)
                if (isnan(nv[u])) sc[u][hd] = -INFINITY;
          }
#pragma unroll
          for (int hd = 0; hd < 2; ++hd) {
            float mx = fmaxf(fmaxf(sc[0][hd], sc[1][hd]), fmaxf(sc[2][hd], sc[3][hd]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mn = fmaxf(m_run[nt][hd], mx);
            // a finite reference keeps exp2(-inf - ref) = 0 when nothing is unmasked yet
            const float ref = fmaxf(mn, -3.0e38f);
            const float al = fast_exp2(m_run[nt][hd] - ref);
            alpha[nt][hd] = al;
            rescale |= al != 1.f;
            m_run[nt][hd] = mn;
            float lsum = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float pv = fast_exp2(sc[u][hd] - ref);
              lsum += pv;
              sc[u][hd] = pv * nv[u];
            }
            if (partial) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (isnan(nv[u])) sc[u][hd] = 0.f;
            }
            l_run[nt][hd] = fmaf(l_run[nt][hd], al, lsum);
          }
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
            pb[rb][nt][0] = movmatrix_trans(pack_half2(sc[2 * rb][0], sc[2 * rb][1]));
            pb[rb][nt][1] = movmatrix_trans(pack_half2(sc[2 * rb + 1][0], sc[2 * rb + 1][1]));
          }
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
              acc[nt][mt][0] *= alpha[nt][0];
              acc[nt][mt][1] *= alpha[nt][1];
              acc[nt][mt][2] *= alpha[nt][0];
              acc[nt][mt][3] *= alpha[nt][1];
            }
        }
        // ---------------- values: fp16 MMA, k-step rb covers tokens 16 rb .. 16 rb + 15;
        // tokens (2q, 2q+1) and (2q+8, 2q+9) of each k-step, unit r of 16 coordinates
        constexpr int VB = D * BV / 8;
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
          const unsigned char *vt = st + St::vc + (wt + 16 * rb + 2 * q) * VB;
          if constexpr (BV == 3) {
            const int gofs = 12 * (r >> 1);
            const uint32_t gs = (r & 1) ? 0x7362u : 0x5140u;
            uint32_t ya[3], yb[3];
#pragma unroll
            for (int k = 0; k < 3; ++k) {
              const uint32_t A0 = reinterpret_cast<const uint32_t *>(vt + gofs)[k];
              const uint32_t B0 = reinterpret_cast<const uint32_t *>(vt + VB + gofs)[k];
              const uint32_t A1 = reinterpret_cast<const uint32_t *>(vt + 8 * VB + gofs)[k];
              const uint32_t B1 = reinterpret_cast<const uint32_t *>(vt + 9 * VB + gofs)[k];
              ya[k] = prmt(A0, B0, gs);
              yb[k] = prmt(A1, B1, gs);
            }
            const uint32_t spa = spare3(ya[0], ya[1], ya[2]), spb = spare3(yb[0], yb[1], yb[2]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t za = k < 3 ? (ya[k < 3 ? k : 0] & 0x77777777u) : spa;
              const uint32_t zb = k < 3 ? (yb[k < 3 ? k : 0] & 0x77777777u) : spb;
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                uint32_t a0, a1, a2, a3;
                v_pairs<3>(lv, hh ? za >> 16 : za, a0, a1);
                v_pairs<3>(lv, hh ? zb >> 16 : zb, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                  mma_f16(acc[nt][2 * k + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
              }
            }
          } else if constexpr (BV == 2) {
            const uint32_t A0 = reinterpret_cast<const uint32_t *>(vt)[r];
            const uint32_t B0 = reinterpret_cast<const uint32_t *>(vt + VB)[r];
            const uint32_t A1 = reinterpret_cast<const uint32_t *>(vt + 8 * VB)[r];
            const uint32_t B1 = reinterpret_cast<const uint32_t *>(vt + 9 * VB)[r];
#pragma unroll
            for (int yh = 0; yh < 2; ++yh) {
              const uint32_t gs = yh ? 0x7362u : 0x5140u;
              const uint32_t ya = prmt(A0, B0, gs), yb = prmt(A1, B1, gs);
#pragma unroll
              for (int par = 0; par < 2; ++par) {
                const uint32_t za = (ya >> (2 * par)) & 0x33333333u, zb = (yb >> (2 * par)) & 0x33333333u;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  uint32_t a0, a1, a2, a3;
                  v_pairs<2>(lv, hh ? za >> 16 : za, a0, a1);
                  v_pairs<2>(lv, hh ? zb >> 16 : zb, a2, a3);
#pragma unroll
                  for (int nt = 0; nt < NT; ++nt)
                    mma_f16(acc[nt][4 * yh + 2 * par + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
                }
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const uint32_t A0 = reinterpret_cast<const uint32_t *>(vt)[2 * r + u];
              const uint32_t B0 = reinterpret_cast<const uint32_t *>(vt + VB)[2 * r + u];
              const uint32_t A1 = reinterpret_cast<const uint32_t *>(vt + 8 * VB)[2 * r + u];
              const uint32_t B1 = reinterpret_cast<const uint32_t *>(vt + 9 * VB)[2 * r + u];
#pragma unroll
              for (int yh = 0; yh < 2; ++yh) {
                const uint32_t gs = yh ? 0x7362u : 0x5140u;
                const uint32_t ya = prmt(A0, B0, gs), yb = prmt(A1, B1, gs);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  uint32_t a0, a1, a2, a3;
                  v_pairs<4>(lv, hh ? ya >> 16 : ya, a0, a1);
                  v_pairs<4>(lv, hh ? yb >> 16 : yb, a2, a3);
#pragma unroll
                  for (int nt = 0; nt < NT; ++nt)
                    mma_f16(acc[nt][4 * u + 2 * yh + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
                }
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[slot]));
      if (*(volatile int *)&abort_flag) break;
    }

    // ---------------- all consumers are past the ring: park the state in smem
    consumer_sync();
    float *so = reinterpret_cast<float *>(smem);  // [warp][8 NT heads][D], V fragment order
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int hd = 0; hd < 2; ++hd) {
        float l = l_run[nt][hd];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (r == 0) {
          sm_m[warp][8 * nt + 2 * q + hd] = m_run[nt][hd];
          sm_l[warp][8 * nt + 2 * q + hd] = l;
        }
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        float *o0 = so + ((warp * 8 * NT) + 8 * nt + 2 * q) * D + 16 * mt + r;
        o0[0] = acc[nt][mt][0];
        o0[D] = acc[nt][mt][1];
        o0[8] = acc[nt][mt][2];
        o0[D + 8] = acc[nt][mt][3];
      }
    }
  }
  __syncthreads();
  // the merge kernel may start launching once every CTA is here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (*(volatile int *)&abort_flag) return;

  // ---------------- combine the consumer warps, write this split's partial
  const float *so = reinterpret_cast<const float *>(smem);
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int g = idx / D, i = idx % D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, sm_m[w][g]);
    float l = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float f = sm_m[w][g] == -INFINITY ? 0.f : exp2f(sm_m[w][g] - mx);
      l = fmaf(f, sm_l[w][g], l);
      o = fmaf(f, so[(w * 8 * NT + g) * D + i], o);
    }
    float *dst = a.partials + (((long)s * a.n_q_heads + h * G + g) * a.n_splits + split) * kPartialFloats;
    dst[4 + i] = o;
    if (i == 0) {
      dst[0] = mx;
      dst[1] = l;
    }
  }
}

// ---------------------------------------------------------------------------
// merge: per (sequence, query head) combine the splits (log-sum-exp in log2
// units) and apply Pi^T.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_max128(float v, float *red) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return r;
}

// A bf16 row of 128 entries (16-byte aligned) as 16 independent 16-byte loads.
__device__ __forceinline__ void load_bf16_row(const uint16_t *row, uint4 (&w)[16]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) w[c] = reinterpret_cast<const uint4 *>(row)[c];
}

// Dot product of a loaded bf16 row with a vector in shared memory, four
// partial sums.
__device__ __forceinline__ float dot_bf16_row(const uint4 (&w)[16], const float *x) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t u[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 8 * c + 2 * e;
      acc[e] = fmaf(__uint_as_float(u[e] << 16), x[j], acc[e]);
      acc[e] = fmaf(__uint_as_float(u[e] & 0xffff0000u), x[j + 1], acc[e]);
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// ---------------------------------------------------------------------------
// merge: per (sequence, query head) combine the splits (log-sum-exp in log2
// units) and apply Pi^T: o_i = sum_k Pi[vperm(k)][i] o~_k / L.
// ---------------------------------------------------------------------------
constexpr int kMergeMaxSplits = 1024;

__global__ void __launch_bounds__(128) merge_kernel(DeviceParams p, int n_q_heads, const int32_t *seq_lens,
                                                    int max_seq_len, int chunk, int n_splits,
                                                    const float *partials, float *out, float *lse) {
  __shared__ float s_ot[D];
  __shared__ float s_w[kMergeMaxSplits], s_l[kMergeMaxSplits];
  __shared__ __align__(16) float s_acc[4][D];
  __shared__ float red[4];
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this thread's row of Pi^T does not depend on the attention kernel: load it
  // before waiting for that kernel to complete
  uint4 pw[16];
  load_bf16_row(p.pivt + tid * D, pw);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel in the stream (an append, the next decode) may launch and
  // load its parameters now; it waits for this grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int s = row / n_q_heads;
  const float *src = partials + (long)row * n_splits * kPartialFloats;
  // One round of loads: the sequence length, and warp w's outputs of splits
  // w, w + 4, ... (lane j: outputs 4 j .. 4 j + 3) of every allocated split,
  // requested before any of them is used; splits past the used ones are
  // ignored below (their slots may hold anything).
  constexpr int kOPerWarp = 16;  // splits per warp held in registers
  float4 o4[kOPerWarp];
#pragma unroll
  for (int e = 0; e < kOPerWarp; ++e) {
    const int sp = warp + 4 * e;
    if (sp < n_splits) o4[e] = reinterpret_cast<const float4 *>(src + sp * kPartialFloats + 4)[lane];
  }
  // and thread t's (m, l) pair of split t, so that the pairs of the first 128
  // splits do not wait for the sequence length
  float2 ml0 = make_float2(-INFINITY, 0.f);
  if (tid < n_splits) ml0 = *reinterpret_cast<const float2 *>(src + tid * kPartialFloats);
  int len = seq_lens[s];
  len = len < 0 ? 0 : (len > max_seq_len ? max_seq_len : len);
  const int used = min((len + chunk - 1) / chunk, kMergeMaxSplits);
  float mloc = -INFINITY;
  if (tid < used) {
    s_w[tid] = ml0.x;
    s_l[tid] = ml0.y;
    mloc = ml0.x;
  }
  for (int sp = tid + 128; sp < used; sp += 128) {
    const float2 ml = *reinterpret_cast<const float2 *>(src + sp * kPartialFloats);
    s_w[sp] = ml.x;
    s_l[sp] = ml.y;
    mloc = fmaxf(mloc, ml.x);
  }
  const float mm = block_max128(mloc, red);  // split maxima in log2 units
  float lpart = 0.f;
  for (int sp = tid; sp < used; sp += 128) {
    const float w = s_w[sp] == -INFINITY ? 0.f : exp2f(s_w[sp] - mm);
    s_w[sp] = w;
    lpart = fmaf(w, s_l[sp], lpart);
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int e = 0; e < kOPerWarp; ++e) {
    const int sp = warp + 4 * e;
    if (sp < used) {
      const float w = s_w[sp];
      acc.x = fmaf(w, o4[e].x, acc.x);
      acc.y = fmaf(w, o4[e].y, acc.y);
      acc.z = fmaf(w, o4[e].z, acc.z);
      acc.w = fmaf(w, o4[e].w, acc.w);
    }
  }
  // splits beyond 4 * kOPerWarp (long sequences with short splits)
  for (int sp = warp + 4 * kOPerWarp; sp < used; sp += 4) {
    const float4 v = reinterpret_cast<const float4 *>(src + sp * kPartialFloats + 4)[lane];
    const float w = s_w[sp];
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  }
  reinterpret_cast<float4 *>(s_acc[warp])[lane] = acc;
  for (int o = 16; o; o >>= 1) lpart += __shfl_xor_sync(0xffffffffu, lpart, o);
  if (lane == 0) red[warp] = lpart;
  __syncthreads();
  const float ll = (red[0] + red[1]) + (red[2] + red[3]);
  const float oo = (s_acc[0][tid] + s_acc[1][tid]) + (s_acc[2][tid] + s_acc[3][tid]);
  s_ot[tid] = ll > 0.f ? oo / ll : 0.f;
  __syncthreads();
  // o_i = sum_k Pi^T[i][k] o~_k with Pi^T's columns in the V fragment order
  out[(long)row * D + tid] = dot_bf16_row(pw, s_ot);
  if (lse && tid == 0) lse[row] = ll > 0.f ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
}

template <int BK, int BV, bool QJL, int NT>
constexpr int decode_smem_bytes() {
  const int ring = kStages * Stage<BK, BV, QJL, kStageTokens>::bytes;
  const int park = kConsumerWarps * 8 * NT * D * 4;
  return ring > park ? ring : park;
}

using DecodeFn = void (*)(const DecodeArgs);

struct Variant {
  DecodeFn fn;
  int smem;
};

// Budgets: kShort (2 CTAs per SM), kLong (3 CTAs per SM) on the contiguous
// layout; kPaged, the paged layout, which always runs the 3-CTA budget (its
// callers decode batches of many sequences).
enum Build { kShort = 0, kLong = 1, kPaged = 2 };

template <int BK, int BV, bool QJL, int NT>
Variant variant_c(int build) {
  constexpr int smem = decode_smem_bytes<BK, BV, QJL, NT>();
  if (build == kPaged) return {decode_mma_kernel<BK, BV, QJL, NT, 3, true>, smem};
  if (build == kLong) return {decode_mma_kernel<BK, BV, QJL, NT, 3, false>, smem};
  return {decode_mma_kernel<BK, BV, QJL, NT, 2, false>, smem};
}

template <int BK, int BV, bool QJL>
Variant variant_q(int nt, int build) {
  return nt == 1 ? variant_c<BK, BV, QJL, 1>(build) : variant_c<BK, BV, QJL, 2>(build);
}

template <int BK, int BV>
Variant variant_v(bool qjl, int nt, int build) {
  return qjl ? variant_q<BK, BV, true>(nt, build) : variant_q<BK, BV, false>(nt, build);
}

template <int BK>
Variant variant_k(int bv, bool qjl, int nt, int build) {
  switch (bv) {
    case 2: return variant_v<BK, 2>(qjl, nt, build);
    case 3: return variant_v<BK, 3>(qjl, nt, build);
    default: return variant_v<BK, 4>(qjl, nt, build);
  }
}

Variant variant(int bk, int bv, bool qjl, int nt, int build) {
  switch (bk) {
    case 2: return variant_k<2>(bv, qjl, nt, build);
    case 3: return variant_k<3>(bv, qjl, nt, build);
    default: return variant_k<4>(bv, qjl, nt, build);
  }
}

int build_of(bool long_splits, bool paged) { return paged ? kPaged : long_splits ? kLong : kShort; }

}  // namespace

int decode_ctas_per_sm(int bits_k, int bits_v, int qjl, int group, bool long_splits, bool paged) {
  // cached per variant; atomically, as calls may come from several threads
  // (per device: the attribute and the occupancy query apply to the current one)
  static std::atomic<int> cache[kMaxDevices][3][3][2][2][3];
  const int nt = group > 8 ? 2 : 1;
  const int build = build_of(long_splits, paged);
  std::atomic<int> &slot = cache[current_device()][bits_k - 2][bits_v - 2][qjl ? 1 : 0][nt - 1][build];
  int c = slot.load(std::memory_order_relaxed);
  if (c == 0) {
    const Variant v = variant(bits_k, bits_v, qjl != 0, nt, build);
    cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem);
    cudaFuncSetAttribute(v.fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, v.fn, kThreads, v.smem) != cudaSuccess || n < 1) n = 1;
    c = n;
    slot.store(c, std::memory_order_relaxed);
  }
  return c;
}

int launch_decode(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype, int n_q_heads,
                  const int32_t *seq_lens, int max_seq_len, float scale, float *out, float *lse,
                  char *workspace, const DecodeSplit &split, const DecodeWorkspace &ws, void *stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int rows = c.n_seqs * n_q_heads;
  const int group = n_q_heads / c.n_kv_heads;
  float *partials = reinterpret_cast<float *>(workspace + ws.partials);

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;

  const Variant v = variant(p.bits_k, p.bits_v, p.qjl != 0, group > 8 ? 2 : 1,
                            build_of(split.long_splits, c.block_table != nullptr));
  DecodeArgs args{p, c, n_q_heads, max_seq_len, split.chunk, split.n_splits, seq_lens, q, q_dtype, scale, partials};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(split.n_splits, c.n_kv_heads, c.n_seqs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = v.smem;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, v.fn, args);
  if (e != cudaSuccess) return (int)e;

  cudaLaunchConfig_t mcfg = {};
  mcfg.gridDim = dim3(rows);
  mcfg.blockDim = dim3(128);
  mcfg.stream = st;
  mcfg.attrs = pdl;
  mcfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&mcfg, merge_kernel, p, n_q_heads, seq_lens, max_seq_len, split.chunk, split.n_splits,
                         (const float *)partials, out, lse);
  return (int)e;
}

}  // namespace tq
