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
//
// This header holds the attention kernel template and its instantiation
// helpers; tq_decode_variants.cu instantiates one slice of it per object
// (one head dimension and K width), tq_decode.cu holds the merge and the
// launch.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>

#include "tq_f32x2.cuh"
#include "tq_internal.h"
#include "tq_stream.cuh"

namespace tq {

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

using DecodeFn = void (*)(const DecodeArgs);

struct DecodeVariant {
  DecodeFn fn;
  int smem;  // dynamic shared memory bytes
};

// Budgets at d = 128: kShort (2 CTAs per SM), kLong (3 CTAs per SM) on the
// contiguous layout; kPaged, the paged layout, which always runs the 3-CTA
// budget (its callers decode batches of many sequences).  At d = 256 every
// build runs the 168-register budget (twice the value accumulators), at
// d = 64 the 128-register one; kShort and kLong are then the same kernel.
enum Build { kShort = 0, kLong = 1, kPaged = 2 };

// The instantiations for head dimension DH and K width BK (defined in
// tq_decode_variants.cu, one object per pair).
template <int DH, int BK>
DecodeVariant decode_variant(int bits_v, bool qjl, int nt, int build);

namespace {


constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kWarpTokens = 32;                            // tokens per consumer warp per stage
constexpr int kStageTokens = kWarpTokens * kConsumerWarps;  // 128
constexpr int kStages = 4;
constexpr int kPrefetchTokens = kStages * kStageTokens;  // L2 prefetch before the dependency wait
// ring depth: d = 256 stages are twice as large, so two of them
constexpr int stages_of(int dh) { return dh == 256 ? 2 : kStages; }

// Barrier of the four consumer warps only (the producer warp never joins).
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(32 * kConsumerWarps) : "memory");
}


// Per-thread K words and selectors of the score MMAs for head dimension DH.
// The int8 MMA's k index kappa = 32 s + 16 slot + 4 q + i is byte i of the
// A register (k-step s, slot) of the threads with q = lane % 4:
//   DH = 128: thread q holds coordinate group q (32 codes, BK words) and
//             register (s, slot) is selector 2 s + slot of that group;
//   DH = 256: groups q and q + 4 (2 BK words); k-steps 4 H .. 4 H + 3 read
//             group q + 4 H, selector 2 (s % 4) + slot;
//   DH = 64:  half q % 2 of group q / 2: selectors 4 (q % 2) + 2 s + slot.
template <int BK, int DH>
struct KWords {
  static constexpr int n = DH == 256 ? 2 * BK : BK;  // words loaded per token
  // byte offset of the thread's words inside a token's code row
  __device__ __forceinline__ static int offset(int q) {
    if constexpr (DH == 64) return BK == 3 ? 12 * (q >> 1) : q * 2 * BK;
    else return q * 4 * BK;
  }
  __device__ __forceinline__ static void load(const unsigned char *row, int q, uint32_t (&w)[n]) {
    const uint32_t *p = reinterpret_cast<const uint32_t *>(row + offset(q));
    if constexpr (DH == 256) {
      const uint32_t *p2 = reinterpret_cast<const uint32_t *>(row + 16 * BK + offset(q));
#pragma unroll
      for (int i = 0; i < BK; ++i) {
        w[i] = p[i];
        w[BK + i] = p2[i];
      }
    } else if constexpr (DH == 64 && BK != 3) {
#pragma unroll
      for (int i = 0; i < BK / 2; ++i) w[i] = p[i];
#pragma unroll
      for (int i = BK / 2; i < BK; ++i) w[i] = 0u;
    } else {
#pragma unroll
      for (int i = 0; i < BK; ++i) w[i] = p[i];
    }
  }
  // selector of register (s, slot); s and slot are compile-time after unrolling
  __device__ __forceinline__ static uint32_t sel(const uint32_t (&w)[n], int s, int slot, int q) {
    if constexpr (DH == 128) {
      return k_selector<BK>(w, 2 * s + slot);
    } else if constexpr (DH == 256) {
      uint32_t wh[BK];
#pragma unroll
      for (int i = 0; i < BK; ++i) wh[i] = w[(s >= 4 ? BK : 0) + i];
      return k_selector<BK>(wh, 2 * (s & 3) + slot);
    } else {
      const int j = 2 * s + slot;
      if constexpr (BK == 3) {
        const bool odd = (q & 1) != 0;
        const uint32_t x = j < 2 ? (odd ? w[2] & 0x77777777u : w[0] & 0x77777777u)
                                 : (odd ? spare3(w[0], w[1], w[2]) : w[1] & 0x77777777u);
        return (j & 1) ? x >> 16 : x;
      } else {
        return k_selector<BK>(w, j);
      }
    }
  }
};

// The QJL sign word of register (s, slot) and the bit inside its bytes: the
// register holds bits j, j + 8, j + 16, j + 24 of word `wd` of the token's
// sign row (DH / 32 words).
template <int DH>
__device__ __forceinline__ void qjl_pick(int s, int slot, int q, int &wd, int &j) {
  if constexpr (DH == 64) {
    wd = q >> 1;
    j = 4 * (q & 1) + 2 * s + slot;
  } else {
    wd = q + 4 * (s / 4);
    j = 2 * (s & 3) + slot;
  }
}

// Two register budgets of the same kernel, chosen per call from the split
// length (tq_api.cu): CTAS = 2 (168 registers) for short splits, where fewer
// CTAs amortise the per-CTA prologue and each warp has room for more
// independent work; CTAS = 3 (128 registers) for long splits, where twelve
// consumer warps per SM hide more latency in the steady state.
//
// PAGED selects the paged cache layout (the stage copies follow the block
// table); it is its own instantiation so that the contiguous kernels keep
// their code and register allocation.
template <int BK, int BV, bool QJL, int NT, int CTAS, bool PAGED, int DH>
__global__ void __maxnreg__(CTAS == 3 ? 128 : 168) decode_mma_kernel(const DecodeArgs a) {
  static_assert(kStageTokens % 64 == 0 && kWarpTokens == 32, "stages start on 64-token boundaries");
  static_assert(DH == 64 || DH == 128 || DH == 256, "head dimension");
  using St = Stage<BK, BV, QJL, kStageTokens, DH>;
  constexpr int kRows = 8 * NT;  // query-head rows of the score MMAs
  constexpr int KS = DH / 32;    // int8 k-steps of the scores
  constexpr int MT = DH / 16;    // m-tiles (16 coordinates) of the values
  constexpr int NTW = DH / 32;   // q-rotation n-tiles per consumer warp (DH / 4 positions)
  constexpr int KR = DH / 16;    // q-rotation k-steps
  constexpr bool kHoldPi = DH <= 128;  // Pi's fragments held in registers from before the dependency wait
  constexpr int D = DH;                // (shadows the library-wide 128 inside this kernel)
  constexpr int kStages = stages_of(DH);
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ int abort_flag;
  __shared__ float sm_m[kConsumerWarps][kRows], sm_l[kConsumerWarps][kRows];
  __shared__ __align__(16) uint8_t s_q8[kRows][QJL ? 4 : 2][DH];  // q_hat hi, lo; q_tilde hi, lo (fragment orders)
  // this KV head's query rows (fp32), read by the rotation; then (QJL) q_hat
  // in the K order, written once every consumer warp is past the rotation
  __shared__ __align__(16) float s_qf[kRows][DH];
  __shared__ float s_qs[kRows][4];                                // score factor, QJL factor, sum of q_tilde ints
  __shared__ float s_red[kConsumerWarps][kRows];

  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, q = lane & 3;
  const int G = a.n_q_heads / a.c.n_kv_heads;
  // B fragments of Pi (rows in the K fragment order) for this consumer warp's
  // DH / 4 output positions: parameters, loaded before waiting for the
  // previous kernel in the stream (DH = 256: read during the rotation)
  uint32_t bfr[kHoldPi ? NTW : 1][kHoldPi ? KR : 1][2];
  if (kHoldPi && warp < kConsumerWarps) {
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int j = 0; j < KR / 2; ++j) {
        const uint4 v = reinterpret_cast<const uint4 *>(a.p.pikf)[((warp * NTW + nt) * (KR / 2) + j) * 32 + lane];
        bfr[nt][2 * j][0] = v.x;
        bfr[nt][2 * j][1] = v.y;
        bfr[nt][2 * j + 1][0] = v.z;
        bfr[nt][2 * j + 1][1] = v.w;
      }
  }
  // While the previous kernel (typically the append) still runs, warm L2 with
  // the first four stages this CTA will stream (below the length bound and
  // the capacity).  A prefetch only moves lines into L2, the point of
  // coherence, so whatever the previous kernel writes there is what the
  // copies read after the wait.  The sequence length is not final yet.  The
  // 2-CTA (168-register) build, which at d = 128 runs short splits of one or
  // a few sequences (every split holds tokens, and the CTA's start is on the
  // critical path), fetches blind.  The 3-CTA build, which runs the long
  // splits of ragged batches, first reads the current length (a relaxed read,
  // one more memory round trip, amortised over a long split) and bounds the
  // prefetch by it, so that splits past their sequence's end fetch nothing; a
  // stale value costs at most a useless or a missing prefetch.
  if (warp == kConsumerWarps && lane == 0) {
    // this KV head's query rows (read right after the wait)
    const size_t qbytes = (size_t)G * DH * (a.q_dtype == TQ_F32 ? 4 : 2);
    prefetch_l2(static_cast<const char *>(a.q) + ((size_t)s * a.n_q_heads + (size_t)h * G) * DH *
                                                     (a.q_dtype == TQ_F32 ? 4 : 2),
                (uint32_t)qbytes);
    const int first = split * a.chunk;
    int last = min(min(first + a.chunk, a.max_seq_len), min(first + kPrefetchTokens, a.c.capacity));
    if constexpr (CTAS == 3) {
      int len_hint;
      asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(len_hint) : "l"(a.seq_lens + s));
      last = min(last, len_hint);
    } else {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a.seq_lens + s));
    }
    // (contiguous layout only: a paged cache's block table is not read before the wait)
    if (!PAGED && first < last) {
      const long tok = ((long)s * a.c.n_kv_heads + h) * a.c.capacity + first;
      const uint32_t n = (uint32_t)(last - first);
      prefetch_l2(a.c.codes_k + tok * (DH * BK / 8), n * (DH * BK / 8));
      prefetch_l2(a.c.codes_v + tok * (DH * BV / 8), n * (DH * BV / 8));
      prefetch_l2(a.c.norm_k + tok, (n * 2 + 15) & ~15u);
      prefetch_l2(a.c.norm_v + tok, (n * 2 + 15) & ~15u);
      if constexpr (QJL) {
        prefetch_l2(a.c.qjl_bits + tok * (DH / 8), n * (DH / 8));
        prefetch_l2(a.c.qjl_norm + tok, (n * 2 + 15) & ~15u);
      }
    }
  }
  // the stage barriers (shared memory only) are set up before the wait
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), kConsumerWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // launched as a programmatic dependent: the cache, q and seq_lens are final
  // once the previous kernel in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the consumers' loads of this KV head's G query rows (contiguous, 16-byte
  // aligned) go out first, beside the length's: they do not depend on it
  constexpr int kQIt = (kRows * DH / 4 + 32 * kConsumerWarps - 1) / (32 * kConsumerWarps);
  const int q_n4 = G * DH / 4;
  const bool q_f32 = a.q_dtype == TQ_F32;
  uint4 q_v[kQIt];  // raw: four fp32, or four bf16 in .x, .y (converted when stored)
  if (warp < kConsumerWarps) {
    const long q_off = ((long)s * a.n_q_heads + (long)h * G) * DH;
#pragma unroll
    for (int k = 0; k < kQIt; ++k) {
      const int i = tid + 32 * kConsumerWarps * k;
      if (i < q_n4) {
        if (q_f32) {
          q_v[k] = reinterpret_cast<const uint4 *>(static_cast<const float *>(a.q) + q_off)[i];
        } else {
          const uint2 u = reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(a.q) + q_off)[i];
          q_v[k] = make_uint4(u.x, u.y, 0u, 0u);
        }
      }
    }
  }
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
    // computes positions (D / 4) w .. (D / 4) w + D / 4 - 1.
    {
      const long qrow0 = (long)s * a.n_q_heads + (long)h * G;
      const bool f32 = a.q_dtype == TQ_F32;
      // the G query rows, loaded right after the dependency wait, into
      // shared memory
      {
        float4 *dst = reinterpret_cast<float4 *>(&s_qf[0][0]);
#pragma unroll
        for (int k = 0; k < kQIt; ++k) {
          const int i = tid + 32 * kConsumerWarps * k;
          if (i < q_n4) {
            const uint4 u = q_v[k];
            dst[i] = q_f32 ? make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z),
                                         __uint_as_float(u.w))
                           : make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                         __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
          }
        }
        consumer_sync();
      }
      float c[NTW][4];
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KR; ++ks) {
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // a0: row r; a1: row r + 8; a2, a3: the same rows, columns + 8
          const int row = r + 8 * (e & 1), col = 16 * ks + 8 * (e >> 1) + 2 * q;
          float x0 = 0.f, x1 = 0.f;
          if (row < G) {
            const float2 v = *reinterpret_cast<const float2 *>(&s_qf[row][col]);
            x0 = v.x;
            x1 = v.y;
          }
          split_bf16x2(x0, x1, ahi[e], alo[e]);
        }
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
          uint32_t b0, b1;
          if constexpr (kHoldPi) {
            b0 = bfr[nt][ks][0];
            b1 = bfr[nt][ks][1];
          } else {
            const uint2 v = reinterpret_cast<const uint2 *>(
                a.p.pikf)[(((warp * NTW + nt) * (KR / 2) + ks / 2) * 32 + lane) * 2 + (ks & 1)];
            b0 = v.x;
            b1 = v.y;
          }
          mma_bf16(c[nt], ahi[0], ahi[1], ahi[2], ahi[3], b0, b1);
          if (f32) mma_bf16(c[nt], alo[0], alo[1], alo[2], alo[3], b0, b1);
        }
      }
      // per head: mu = 32767 / max |q_hat|, q_hat as 16-bit fixed point (hi, lo bytes)
      float mx0 = 0.f, mx1 = 0.f;  // rows r, r + 8
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
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
      float mu[2], qmax[2] = {0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (kRows <= 8 && e == 1) break;
        const int row = r + 8 * e;
        const float m = fmaxf(fmaxf(s_red[0][row], s_red[1][row]), fmaxf(s_red[2][row], s_red[3][row]));
        mu[e] = m > 0.f ? 32767.f / m : 1.f;
        qmax[e] = m;
      }
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        const int kap = (D / 4) * warp + 8 * nt + 2 * q;
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
        s_qs[r][0] = a.scale * kLog2e / (mu[0] * ldexpf(1.f, a.p.k_shift));
        if constexpr (kRows > 8) s_qs[r + 8][0] = a.scale * kLog2e / (mu[1] * ldexpf(1.f, a.p.k_shift));
      }
      if constexpr (QJL) {
        // q_tilde = S' q_hat (rows of S in the QJL fragment order, columns in
        // the K order) on the tensor cores: q_hat, scaled per head by a power
        // of two that puts max |q_hat| in [2^13, 2^14), and S' 2^sigma as fp16
        // hi + lo parts (hi hi + hi lo + lo hi, about 22 significant bits,
        // fp32 sums); warp w takes the output n-tiles w NTQ .. w NTQ + NTQ - 1
        consumer_sync();  // q_hat is complete in s_qf
        constexpr int NTQ = D / 32, CHQ = D / 32;  // n-tiles per warp; chunks of two k-steps
        float sc[2];  // the power-of-two scales of rows r and r + 8
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          int ex = 0;
          if (qmax[e] > 0.f) frexpf(qmax[e], &ex);
          sc[e] = qmax[e] > 0.f ? ldexpf(1.f, 14 - ex) : 1.f;
        }
        float cq[NTQ][4];
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) cq[nt][e] = 0.f;
        const uint4 *sjf = reinterpret_cast<const uint4 *>(a.p.sjkf);
        constexpr int kPart = (D / 8) * CHQ * 32;  // uint4 per part
#pragma unroll 2
        for (int j = 0; j < CHQ; ++j) {
          uint32_t ah[2][4], al[2][4];  // A fragments of k-steps 2 j, 2 j + 1
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = r + 8 * (e & 1), col = 16 * (2 * j + kk) + 8 * (e >> 1) + 2 * q;
              if (row < kRows) {
                const float f = sc[e & 1];
                split_f16x2(s_qf[row][col] * f, s_qf[row][col + 1] * f, ah[kk][e], al[kk][e]);
              } else {
                ah[kk][e] = al[kk][e] = 0u;
              }
            }
#pragma unroll
          for (int nt = 0; nt < NTQ; ++nt) {
            const int idx = ((warp * NTQ + nt) * CHQ + j) * 32 + lane;
            const uint4 bh = sjf[idx], bl = sjf[kPart + idx];
            mma_f16(cq[nt], ah[0][0], ah[0][1], ah[0][2], ah[0][3], bh.x, bh.y);
            mma_f16(cq[nt], ah[0][0], ah[0][1], ah[0][2], ah[0][3], bl.x, bl.y);
            mma_f16(cq[nt], al[0][0], al[0][1], al[0][2], al[0][3], bh.x, bh.y);
            mma_f16(cq[nt], ah[1][0], ah[1][1], ah[1][2], ah[1][3], bh.z, bh.w);
            mma_f16(cq[nt], ah[1][0], ah[1][1], ah[1][2], ah[1][3], bl.z, bl.w);
            mma_f16(cq[nt], al[1][0], al[1][1], al[1][2], al[1][3], bh.z, bh.w);
          }
        }
        consumer_sync();  // every warp has read q_hat: s_qf takes q_tilde
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt) {
          const int pos = 8 * (warp * NTQ + nt) + 2 * q;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int row = r + 8 * e;
            if (row < kRows) {
              const float u = ldexpf(1.f, -a.p.s_shift) / sc[e];  // exact: powers of two
              *reinterpret_cast<float2 *>(&s_qf[row][pos]) = make_float2(cq[nt][2 * e] * u, cq[nt][2 * e + 1] * u);
            }
          }
        }
        consumer_sync();
        constexpr int PP = D >= 128 ? D / 128 : 1;  // positions per consumer thread
        float qt[PP][kRows];
#pragma unroll
        for (int pp = 0; pp < PP; ++pp) {
          const int pos = tid + 128 * pp;
#pragma unroll
          for (int g = 0; g < kRows; ++g) qt[pp][g] = pos < D ? s_qf[g][pos] : 0.f;
        }
        // nu = 32767 / max |q_tilde| per head, then the ints and their sum
#pragma unroll
        for (int g = 0; g < kRows; ++g) {
          float m = 0.f;
#pragma unroll
          for (int pp = 0; pp < PP; ++pp) m = fmaxf(m, fabsf(qt[pp][g]));
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
          int sum = 0;
#pragma unroll
          for (int pp = 0; pp < PP; ++pp) {
            const int pos = tid + 128 * pp;
            if (pos < D) {
              const int vi = (int)rintf(qt[pp][g] * nu[g]);
              s_q8[g][2][pos] = (uint8_t)(vi >> 8);
              s_q8[g][3][pos] = (uint8_t)(vi & 0xFF);
              sum += vi;
            }
          }
#pragma unroll
          for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) s_red[warp][g] = (float)sum;  // |sum| < 2^23: exact
        }
        consumer_sync();
        if (tid < kRows) s_qs[tid][2] = (s_red[0][tid] + s_red[1][tid]) + (s_red[2][tid] + s_red[3][tid]);
      }
      consumer_sync();
    }
    // q fragments (int8, K fragment order) of this thread's head r in every n-tile
    uint32_t qh[NT][KS][2], ql[NT][KS][2], jh[NT][QJL ? KS : 1][2], jl[NT][QJL ? KS : 1][2];
    float fq[NT][2], fj[NT][2], jsum[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t *qb = &s_q8[8 * nt + r][0][0];
#pragma unroll
      for (int st = 0; st < KS; ++st)
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

    float m_run[NT][2], l_run[NT][2], acc[NT][MT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        m_run[nt][e] = -INFINITY;
        l_run[nt][e] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
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
        // ---------------- scores: int8 MMA, two 16-token row blocks, D / 32 k-steps of 32
        int chh[2][NT][4], cmid[2][NT][4], cll[2][NT][4], cjh[2][NT][4], cjl[2][NT][4];
#pragma unroll
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) chh[rb][nt][e] = cmid[rb][nt][e] = cll[rb][nt][e] = cjh[rb][nt][e] = cjl[rb][nt][e] = 0;
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
          using KW = KWords<BK, D>;
          uint32_t wk0[KW::n], wk1[KW::n];
          const unsigned char *kr0 = st + St::kc + (wt + 16 * rb + r) * (D * BK / 8);
          KW::load(kr0, q, wk0);
          KW::load(kr0 + 8 * (D * BK / 8), q, wk1);
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            uint32_t alo[4], ahi[4];
            lookup<BK>(lk, KW::sel(wk0, ks, 0, q), alo[0], ahi[0]);
            lookup<BK>(lk, KW::sel(wk1, ks, 0, q), alo[1], ahi[1]);
            lookup<BK>(lk, KW::sel(wk0, ks, 1, q), alo[2], ahi[2]);
            lookup<BK>(lk, KW::sel(wk1, ks, 1, q), alo[3], ahi[3]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_i8<true, true>(chh[rb][nt], ahi[0], ahi[1], ahi[2], ahi[3], qh[nt][ks][0], qh[nt][ks][1]);
              mma_i8<true, false>(cmid[rb][nt], ahi[0], ahi[1], ahi[2], ahi[3], ql[nt][ks][0], ql[nt][ks][1]);
              mma_i8<false, true>(cmid[rb][nt], alo[0], alo[1], alo[2], alo[3], qh[nt][ks][0], qh[nt][ks][1]);
              mma_i8<false, false>(cll[rb][nt], alo[0], alo[1], alo[2], alo[3], ql[nt][ks][0], ql[nt][ks][1]);
            }
          }
          if constexpr (QJL) {
            const uint32_t *jr0 = reinterpret_cast<const uint32_t *>(st + St::jb + (wt + 16 * rb + r) * (D / 8));
            const uint32_t *jr1 = jr0 + 8 * (D / 32);  // token + 8 (D / 32 words per token)
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              // bytes 0x00 / 0xFF (= -bit) for bits j, j+8, j+16, j+24 of word wd
              int wd0, j0, wd1, j1;
              qjl_pick<D>(ks, 0, q, wd0, j0);
              qjl_pick<D>(ks, 1, q, wd1, j1);
              const uint32_t a0 = prmt(jr0[wd0] << (7 - j0), 0u, 0xBA98u), a1 = prmt(jr1[wd0] << (7 - j0), 0u, 0xBA98u);
              const uint32_t a2 = prmt(jr0[wd1] << (7 - j1), 0u, 0xBA98u), a3 = prmt(jr1[wd1] << (7 - j1), 0u, 0xBA98u);
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
          if constexpr (CTAS == 3) {
            // the two heads of a token as one packed fp32 pair (f32x2 rounds
            // each lane as the scalar form would)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int rb = u >> 1, e = 2 * (u & 1);
              // 65536 hh + 256 mid + ll = 256 (256 hh + mid) + ll; 256 hh + mid fits int32
              const float2 hm = make_float2((float)((chh[rb][nt][e] << 8) + cmid[rb][nt][e]),
                                            (float)((chh[rb][nt][e + 1] << 8) + cmid[rb][nt][e + 1]));
              float2 v = mul2(fma2(make_float2(256.f, 256.f), hm,
                                   make_float2((float)cll[rb][nt][e], (float)cll[rb][nt][e + 1])),
                              make_float2(fq[nt][0], fq[nt][1]));
              if constexpr (QJL) {
                const float dj0 = fmaf(256.f, (float)cjh[rb][nt][e], (float)cjl[rb][nt][e]);
                const float dj1 = fmaf(256.f, (float)cjh[rb][nt][e + 1], (float)cjl[rb][nt][e + 1]);
                v.x = fmaf(gm[u] * fj[nt][0], fmaf(-2.f, dj0, -jsum[nt][0]), v.x);
                v.y = fmaf(gm[u] * fj[nt][1], fmaf(-2.f, dj1, -jsum[nt][1]), v.y);
              }
              v = mul2(v, make_float2(nk[u], nk[u]));
              sc[u][0] = v.x;
              sc[u][1] = v.y;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int hd = 0; hd < 2; ++hd) {
                const int rb = u >> 1, e = 2 * (u & 1) + hd;
                const int hm = (chh[rb][nt][e] << 8) + cmid[rb][nt][e];
                float v = fmaf(256.f, (float)hm, (float)cll[rb][nt][e]) * fq[nt][hd];
                if constexpr (QJL) {
                  const float dj = fmaf(256.f, (float)cjh[rb][nt][e], (float)cjl[rb][nt][e]);
                  v = fmaf(gm[u] * fj[nt][hd], fmaf(-2.f, dj, -jsum[nt][hd]), v);
                }
                sc[u][hd] = v * nk[u];
              }
          }
          if (partial) {  // masked tokens carry NaN norms: their scores become -inf, their weights 0
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int hd = 0; hd < 2; ++hd)
                if (isnan(nv[u])) sc[u][hd] = -INFINITY;
          }
          if constexpr (CTAS == 3) {
            // both heads' maxima first, then their weights as packed pairs
            float nref[2];
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
              float mx = fmaxf(max3(sc[0][hd], sc[1][hd], sc[2][hd]), sc[3][hd]);
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
              nref[hd] = -ref;
            }
            float2 lsum = make_float2(0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 t = add2(make_float2(sc[u][0], sc[u][1]), make_float2(nref[0], nref[1]));
              const float2 pe = make_float2(fast_exp2(t.x), fast_exp2(t.y));
              lsum = add2(lsum, pe);
              const float2 pv = mul2(pe, make_float2(nv[u], nv[u]));
              sc[u][0] = pv.x;
              sc[u][1] = pv.y;
            }
            if (partial) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (isnan(nv[u])) sc[u][0] = sc[u][1] = 0.f;
            }
            l_run[nt][0] = fmaf(l_run[nt][0], alpha[nt][0], lsum.x);
            l_run[nt][1] = fmaf(l_run[nt][1], alpha[nt][1], lsum.y);
          } else {
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
              float mx = fmaxf(fmaxf(sc[0][hd], sc[1][hd]), fmaxf(sc[2][hd], sc[3][hd]));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
              const float mn = fmaxf(m_run[nt][hd], mx);
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
          }
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
            pb[rb][nt][0] = movmatrix_trans(pack_half2(sc[2 * rb][0], sc[2 * rb][1]));
            pb[rb][nt][1] = movmatrix_trans(pack_half2(sc[2 * rb + 1][0], sc[2 * rb + 1][1]));
          }
        }
        // with 3-bit V the long-split build, and the d = 256 build without
        // QJL, rescale unconditionally (alpha = 1 is exact): no vote, and no
        // branch between the softmax and the value expansion (longest at 3
        // bits, with the spare-column gather) to stop the scheduler from
        // interleaving them.  Elsewhere the vote, which skips the multiplies,
        // measured faster: at 2/2 and 4/4 bits, 4/4 with QJL, and d = 256 with
        // QJL (2/2 with QJL: 0.5 % slower, within the rule's simplicity)
        constexpr bool kNoVote = BV == 3 && (CTAS == 3 || (DH == 256 && !QJL));
        if (kNoVote || __any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              acc[nt][mt][0] *= alpha[nt][0];
              acc[nt][mt][1] *= alpha[nt][1];
              acc[nt][mt][2] *= alpha[nt][0];
              acc[nt][mt][3] *= alpha[nt][1];
            }
        }
        // ---------------- values: fp16 MMA, k-step rb covers tokens 16 rb .. 16 rb + 15;
        // tokens (2q, 2q+1) and (2q+8, 2q+9) of each k-step; per 128-coordinate
        // half, unit r of 16 coordinates (D = 64: unit r of 8 coordinates)
        constexpr int VB = D * BV / 8;
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
          const unsigned char *vt0 = st + St::vc + (wt + 16 * rb + 2 * q) * VB;
          if constexpr (D == 64) {
            if constexpr (BV == 3) {
              // byte r % 4 of each word of group r / 4: codes 8 k + 2 (r % 4) (x) and + 1 (y)
              const int gofs = 12 * (r >> 2), b = r & 3;
              const uint32_t gs = (uint32_t)(b | ((4 + b) << 4));
              uint32_t ya[3], yb[3];
#pragma unroll
              for (int k = 0; k < 3; ++k) {
                const uint32_t A0 = reinterpret_cast<const uint32_t *>(vt0 + gofs)[k];
                const uint32_t B0 = reinterpret_cast<const uint32_t *>(vt0 + VB + gofs)[k];
                const uint32_t A1 = reinterpret_cast<const uint32_t *>(vt0 + 8 * VB + gofs)[k];
                const uint32_t B1 = reinterpret_cast<const uint32_t *>(vt0 + 9 * VB + gofs)[k];
                ya[k] = prmt(A0, B0, gs);
                yb[k] = prmt(A1, B1, gs);
              }
              const uint32_t spa = spare3(ya[0], ya[1], ya[2]), spb = spare3(yb[0], yb[1], yb[2]);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t za = k < 3 ? (ya[k < 3 ? k : 0] & 0x77777777u) : spa;
                const uint32_t zb = k < 3 ? (yb[k < 3 ? k : 0] & 0x77777777u) : spb;
                uint32_t a0, a1, a2, a3;
                v_pairs<3>(lv, za, a0, a1);
                v_pairs<3>(lv, zb, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                  mma_f16(acc[nt][k], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
              }
            } else {
              // 2 bits: bytes 2 (r % 2), + 1 of word r / 2; 4 bits: word r
              const int wd = BV == 2 ? (r >> 1) : r;
              const uint32_t A0 = reinterpret_cast<const uint32_t *>(vt0)[wd];
              const uint32_t B0 = reinterpret_cast<const uint32_t *>(vt0 + VB)[wd];
              const uint32_t A1 = reinterpret_cast<const uint32_t *>(vt0 + 8 * VB)[wd];
              const uint32_t B1 = reinterpret_cast<const uint32_t *>(vt0 + 9 * VB)[wd];
#pragma unroll
              for (int yh = 0; yh < 2; ++yh) {
                if (BV == 2 && yh == 1) break;
                const uint32_t gs = (BV == 2 ? (r & 1) : yh) ? 0x7362u : 0x5140u;
                const uint32_t ya = prmt(A0, B0, gs), yb = prmt(A1, B1, gs);
#pragma unroll
                for (int par = 0; par < (BV == 2 ? 2 : 1); ++par) {
                  const uint32_t za = BV == 2 ? (ya >> (2 * par)) & 0x33333333u : ya;
                  const uint32_t zb = BV == 2 ? (yb >> (2 * par)) & 0x33333333u : yb;
#pragma unroll
                  for (int hh = 0; hh < 2; ++hh) {
                    uint32_t a0, a1, a2, a3;
                    v_pairs<BV>(lv, hh ? za >> 16 : za, a0, a1);
                    v_pairs<BV>(lv, hh ? zb >> 16 : zb, a2, a3);
                    const int mt = BV == 2 ? 2 * par + hh : 2 * yh + hh;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                      mma_f16(acc[nt][mt], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
                  }
                }
              }
            }
          } else {
#pragma unroll
          for (int hv = 0; hv < D / 128; ++hv) {
            const unsigned char *vt = vt0 + hv * 16 * BV;
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
                    mma_f16(acc[nt][8 * hv + 2 * k + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
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
                      mma_f16(acc[nt][8 * hv + 4 * yh + 2 * par + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
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
                      mma_f16(acc[nt][8 * hv + 4 * u + 2 * yh + hh], a0, a1, a2, a3, pb[rb][nt][0], pb[rb][nt][1]);
                  }
                }
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
      for (int mt = 0; mt < MT; ++mt) {
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
    float *dst = a.partials + (((long)s * a.n_q_heads + h * G + g) * a.n_splits + split) * (D + 4);
    dst[4 + i] = o;
    if (i == 0) {
      dst[0] = mx;
      dst[1] = l;
    }
  }
}


template <int BK, int BV, bool QJL, int NT, int DH>
constexpr int decode_smem_bytes() {
  const int ring = stages_of(DH) * Stage<BK, BV, QJL, kStageTokens, DH>::bytes;
  const int park = kConsumerWarps * 8 * NT * DH * 4;
  return ring > park ? ring : park;
}



template <int BK, int BV, bool QJL, int NT, int DH>
DecodeVariant variant_c(int build) {
  constexpr int smem = decode_smem_bytes<BK, BV, QJL, NT, DH>();
  if constexpr (DH == 128) {
    if (build == kPaged) return {decode_mma_kernel<BK, BV, QJL, NT, 3, true, DH>, smem};
    if (build == kLong) return {decode_mma_kernel<BK, BV, QJL, NT, 3, false, DH>, smem};
    return {decode_mma_kernel<BK, BV, QJL, NT, 2, false, DH>, smem};
  } else {
    constexpr int C = DH == 256 ? 2 : 3;
    if (build == kPaged) return {decode_mma_kernel<BK, BV, QJL, NT, C, true, DH>, smem};
    return {decode_mma_kernel<BK, BV, QJL, NT, C, false, DH>, smem};
  }
}

template <int BK, int BV, bool QJL, int DH>
DecodeVariant variant_q(int nt, int build) {
  return nt == 1 ? variant_c<BK, BV, QJL, 1, DH>(build) : variant_c<BK, BV, QJL, 2, DH>(build);
}

template <int BK, int BV, int DH>
DecodeVariant variant_v(bool qjl, int nt, int build) {
  return qjl ? variant_q<BK, BV, true, DH>(nt, build) : variant_q<BK, BV, false, DH>(nt, build);
}

template <int BK, int DH>
DecodeVariant variant_k(int bv, bool qjl, int nt, int build) {
  switch (bv) {
    case 2: return variant_v<BK, 2, DH>(qjl, nt, build);
    case 3: return variant_v<BK, 3, DH>(qjl, nt, build);
    default: return variant_v<BK, 4, DH>(qjl, nt, build);
  }
}

}  // namespace
}  // namespace tq
