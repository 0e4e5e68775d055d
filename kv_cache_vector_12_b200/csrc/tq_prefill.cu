// Causal prefill attention over the packed TurboQuant cache, sm_100a.
//
// Prompt processing is where a compressed cache costs the most
// (qxai.app, "Tether QVACのTurboQuant実装", fifth paragraph): the prompt's K
// and V are quantized into the cache (tq_quantize), then every prompt token
// attends over the cached positions up to its own, reading the packed codes
// exactly as decode does ("TurboQuantの仕組み", ai-accelerate.xyz explainer:
// scores from the rotated query and the per-coordinate codes, values
// accumulated in rotated space, one inverse rotation at the end).  The bf16
// K/V of the prompt is never read again.
//
// One CTA per (block of query positions, KV head, sequence): four consumer
// warps of 16 query rows each (a row is one (position, query head) pair of
// the KV head's group) and one producer warp that streams the cache with 1-D
// TMA bulk copies into a ring of 128-token stages (mbarriers, bounded waits).
// Every consumer warp takes every key of every stage it needs:
//
//   q_hat   Pi q per row on the tensor cores (mma m16n8k16 bf16, fp32 q as an
//           exact hi + lo pair), then 16-bit fixed point (hi/lo bytes) in the
//           decode's K fragment order; with QJL q_tilde = S q_hat (three fp16
//           products of two-part splits) in the QJL fragment order.
//   scores  S[row][key] = q_hat . c_K[code]: int8 tensor cores (m16n8k32) with
//           q_hat as the A operand and the key's codes, expanded by byte
//           permutes into the exact 16-bit fixed-point centroids (hi/lo
//           bytes), as the B operand; QJL signs as 0/-1 bytes against
//           q_tilde.  The four products make the dot product exact up to
//           q_hat's rounding.
//   softmax online per row (exp2), causal mask key <= position.
//   values  O[row][coord] += P'[row][key] V~[key][coord]: fp16 tensor cores
//           (m16n8k16); P' = p ||v|| comes straight from the score
//           accumulators, V~ from byte-permute lookups of the fp16 centroids.
//   output  o = Pi^T (O / l) on the tensor cores (bf16 hi + lo split of O),
//           and the log-sum-exp of the scores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>

#include "tq_f32x2.cuh"
#include "tq_internal.h"
#include "tq_stream.cuh"

namespace tq {
namespace {

constexpr int kPWarps = 4;                      // consumer warps
constexpr int kPThreads = 32 * (kPWarps + 1);   // + the producer warp
constexpr int kPRows = 16 * kPWarps;            // query rows per CTA
constexpr int kPStageTokens = 128;              // keys per stage
constexpr int kPStages = 3;
constexpr int kChunk = 32;                      // keys per softmax step of a warp

struct PrefillArgs {
  DeviceParams p;
  tq_cache c;
  int n_q_heads, max_seq_len, max_q;
  const int32_t *cu_q;      // [n_seqs + 1] first query row of each sequence
  const int32_t *seq_lens;  // [n_seqs] cached length, the queries' tokens included
  const void *q;            // [rows][n_q_heads][d], fp32 or bf16 (q_dtype)
  int q_dtype;
  float scale;
  float *out;               // [rows][n_q_heads][d]
  float *lse;               // [rows][n_q_heads] or null
};

template <int BK, int BV, bool QJL>
constexpr int prefill_smem_bytes() {
  constexpr int ring = kPStages * Stage<BK, BV, QJL, kPStageTokens>::bytes;
  constexpr int scratch = kPRows * D * 4 * (QJL ? 2 : 1);  // q_hat (and q_tilde), fp32, prologue only
  return ring > scratch ? ring : scratch;
}

template <int BK, int BV, bool QJL>
__global__ void __launch_bounds__(kPThreads, 2) prefill_attn_kernel(const PrefillArgs a) {
  using St = Stage<BK, BV, QJL, kPStageTokens>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kPStages], empty_bar[kPStages];
  __shared__ int abort_flag;
  __shared__ __align__(16) uint8_t s_q8[kPRows][QJL ? 4 : 2][D];  // q_hat hi, lo; q_tilde hi, lo
  __shared__ float s_qs[kPRows][4];                               // score factor, QJL factor, sum of q_tilde ints
  __shared__ int s_pos[kPRows];                                   // position of each row, -1 if none

  const int s = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = lane >> 2, q = lane & 3;
  const int G = a.n_q_heads / a.c.n_kv_heads;
  const int PW = 16 / G;                       // positions per warp (G <= 16)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the longest blocks (the last positions) first
  const int blk = gridDim.x - 1 - blockIdx.x;
  const int q0 = a.cu_q[s], n_q = a.cu_q[s + 1] - q0;
  int len = a.seq_lens[s];
  if (len < 0 || len > a.max_seq_len || n_q < 0 || n_q > len || n_q > a.max_q) {
    if (tid == 0 && blk == 0 && h == 0) atomicOr(a.p.err, kErrSeqLen);
    return;
  }
  const int first_q = blk * kPWarps * PW;      // first query index (within the sequence) of this CTA
  if (first_q >= n_q) return;
  const int p0 = len - n_q;                    // position of query 0
  const int last_q = min(n_q, first_q + kPWarps * PW) - 1;
  const int kend = p0 + last_q + 1;            // keys [0, kend) feed this CTA
  const int n_stage = (kend + kPStageTokens - 1) / kPStageTokens;
  const long base = ((long)s * a.c.n_kv_heads + h) * a.c.capacity;
  const long qrow0 = (long)q0 * a.n_q_heads + (long)h * G;  // row (query 0, head 0 of this KV head)

  if (tid < kPRows) {  // row -> (query, head)
    const int w = tid >> 4, rho = tid & 15;
    const int qi = first_q + w * PW + rho / G;
    s_pos[tid] = (rho < PW * G && qi < n_q) ? p0 + qi : -1;
  }
  if (tid == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), kPWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // ------------------------------------------------ prologue: q_hat, q_tilde
  float *s_qf = reinterpret_cast<float *>(smem);        // [kPRows][D] q_hat, natural order
  float *s_qt = s_qf + kPRows * D;                      // [kPRows][D] q_tilde (times a per-row power of 2)
  if (warp < kPWarps) {
    // A fragments of this warp's 16 rows (q, split into bf16 hi + lo)
    const bool f32 = a.q_dtype == TQ_F32;
    uint32_t ahi[8][4], alo[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 16 * warp + r + 8 * (e & 1), col = 16 * ks + 8 * (e >> 1) + 2 * q;
        const int pr = s_pos[row];
        float x0 = 0.f, x1 = 0.f;
        if (pr >= 0) {
          const int rho = row & 15;
          const long qr = qrow0 + (long)(pr - p0) * a.n_q_heads + (rho % G);
          if (f32) {
            const float2 v = *reinterpret_cast<const float2 *>(static_cast<const float *>(a.q) + qr * D + col);
            x0 = v.x;
            x1 = v.y;
          } else {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(a.q) + qr * D + col);
            x0 = __uint_as_float(v << 16);
            x1 = __uint_as_float(v & 0xffff0000u);
          }
        }
        split_bf16x2(x0, x1, ahi[ks][e], alo[ks][e]);
      }
    // q_hat = q Pi^T, natural coordinate order, n-tile by n-tile
#pragma unroll 1
    for (int nt = 0; nt < 16; ++nt) {
      uint32_t bfr[8][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = reinterpret_cast<const uint4 *>(a.p.pif)[(nt * 4 + j) * 32 + lane];
        bfr[2 * j][0] = v.x;
        bfr[2 * j][1] = v.y;
        bfr[2 * j + 1][0] = v.z;
        bfr[2 * j + 1][1] = v.w;
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        mma_bf16(c, ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], bfr[ks][0], bfr[ks][1]);
        mma_bf16(c, alo[ks][0], alo[ks][1], alo[ks][2], alo[ks][3], bfr[ks][0], bfr[ks][1]);
      }
      float *d0 = s_qf + (16 * warp + r) * D + 8 * nt + 2 * q;
      d0[0] = c[0];
      d0[1] = c[1];
      d0[8 * D] = c[2];
      d0[8 * D + 1] = c[3];
    }
    __syncwarp();
    if constexpr (QJL) {
      // q_tilde = q_hat S^T on fp16 tensor cores: q_hat 2^e (per row, max
      // in [2^13, 2^14)) and S 2^sigma as two-part fp16 splits, three
      // products; the per-row factor 2^(e + sigma) is divided out below
      float mrow[2] = {0.f, 0.f};
      for (int j = 0; j < D; j += 4) {
        mrow[0] = fmaxf(mrow[0], fabsf(s_qf[(16 * warp + r) * D + j + q]));
        mrow[1] = fmaxf(mrow[1], fabsf(s_qf[(16 * warp + r + 8) * D + j + q]));
      }
      float sc[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        mrow[e] = fmaxf(mrow[e], __shfl_xor_sync(0xffffffffu, mrow[e], 1));
        mrow[e] = fmaxf(mrow[e], __shfl_xor_sync(0xffffffffu, mrow[e], 2));
        int ex = 0;
        if (mrow[e] > 0.f) frexpf(mrow[e], &ex);      // mrow in [2^(ex-1), 2^ex)
        sc[e] = mrow[e] > 0.f ? ldexpf(1.f, 14 - ex) : 1.f;
      }
      uint32_t qh16[8][4], ql16[8][4];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = 16 * warp + r + 8 * (e & 1), col = 16 * ks + 8 * (e >> 1) + 2 * q;
          const float f = sc[e & 1];
          split_f16x2(s_qf[row * D + col] * f, s_qf[row * D + col + 1] * f, qh16[ks][e], ql16[ks][e]);
        }
      const uint4 *sf = reinterpret_cast<const uint4 *>(a.p.sf);
#pragma unroll 1
      for (int nt = 0; nt < 16; ++nt) {
        uint32_t bh[8][2], bl[8][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = sf[(nt * 4 + j) * 32 + lane];
          const uint4 w = sf[16 * 4 * 32 + (nt * 4 + j) * 32 + lane];
          bh[2 * j][0] = v.x, bh[2 * j][1] = v.y, bh[2 * j + 1][0] = v.z, bh[2 * j + 1][1] = v.w;
          bl[2 * j][0] = w.x, bl[2 * j][1] = w.y, bl[2 * j + 1][0] = w.z, bl[2 * j + 1][1] = w.w;
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          mma_f16(c, qh16[ks][0], qh16[ks][1], qh16[ks][2], qh16[ks][3], bh[ks][0], bh[ks][1]);
          mma_f16(c, qh16[ks][0], qh16[ks][1], qh16[ks][2], qh16[ks][3], bl[ks][0], bl[ks][1]);
          mma_f16(c, ql16[ks][0], ql16[ks][1], ql16[ks][2], ql16[ks][3], bh[ks][0], bh[ks][1]);
        }
        // q_tilde (natural projection order) times 2^sigma sc[row]
        float *d0 = s_qt + (16 * warp + r) * D + 8 * nt + 2 * q;
        d0[0] = c[0];
        d0[1] = c[1];
        d0[8 * D] = c[2];
        d0[8 * D + 1] = c[3];
      }
      if (q == 0) {
        s_qs[16 * warp + r][3] = sc[0];
        s_qs[16 * warp + r + 8][3] = sc[1];
      }
    }
    __syncwarp();
    // per row: mu = 32767 / max |q_hat|, q_hat in 16-bit fixed point (hi, lo
    // bytes) in the K fragment order; with QJL the same for q_tilde in the
    // QJL fragment order, and the factors.  Lane pair (2 lanes per row).
    {
      const int row = 16 * warp + (lane >> 1), half = lane & 1;
      const float *qf = s_qf + row * D;
      float m = 0.f;
      for (int j = half; j < D; j += 2) m = fmaxf(m, fabsf(qf[j]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      const float mu = m > 0.f ? 32767.f / m : 1.f;
      for (int kap = half; kap < D; kap += 2) {
        const int v = (int)rintf(qf[a.p.kperm[kap]] * mu);
        s_q8[row][0][kap] = (uint8_t)((v >> 8) & 0xFF);
        s_q8[row][1][kap] = (uint8_t)(v & 0xFF);
      }
      if (half == 0) s_qs[row][0] = a.scale * kLog2e / (mu * ldexpf(1.f, a.p.k_shift));
      if constexpr (QJL) {
        const float *qt = s_qt + row * D;
        float mt = 0.f;
        for (int j = half; j < D; j += 2) mt = fmaxf(mt, fabsf(qt[j]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        const float nu = mt > 0.f ? 32767.f / mt : 1.f;
        int sum = 0;
        for (int kap = half; kap < D; kap += 2) {
          const int v = (int)rintf(qt[a.p.jperm[kap]] * nu);
          s_q8[row][2][kap] = (uint8_t)((v >> 8) & 0xFF);
          s_q8[row][3][kap] = (uint8_t)(v & 0xFF);
          sum += v;
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        // s_qt = q_tilde 2^sigma sc, so the ints are q_tilde (2^sigma sc nu)
        const float inv_nu = 1.f / (ldexpf(s_qs[row][3], a.p.s_shift) * nu);
        if (half == 0) {
          s_qs[row][1] = a.scale * kLog2e * kSqrtHalfPi * inv_nu / (float)D;
          s_qs[row][2] = (float)sum;  // |sum| < 2^22: exact
        }
      }
    }
  }
  __syncthreads();  // the prologue scratch (the ring's memory) is free from here on

  if (warp == kPWarps) {
    // ---------------- producer: one elected lane issues the bulk copies
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_stage; ++it) {
        const int slot = it % kPStages;
        if (it >= kPStages && !mbar_wait(smem_u32(&empty_bar[slot]), ((it / kPStages) - 1) & 1)) {
          atomicOr(a.p.err, kErrWaitExpired);
          abort_flag = 1;
          break;
        }
        if (*(volatile int *)&abort_flag) break;
        unsigned char *st = smem + slot * St::bytes;
        const uint32_t bar = smem_u32(&full_bar[slot]);
        const int first = it * kPStageTokens;
        // the stage's keys below kend rounded up to 64: never past the
        // capacity, nor into a block that holds no key below kend
        const uint32_t n = (uint32_t)min(kPStageTokens, (kend - first + 63) & ~63);
        mbar_arrive_expect_tx(bar, n * (D * BK / 8 + D * BV / 8 + 4 + (QJL ? D / 8 + 2 : 0)));
        for (uint32_t done = 0; done < n;) {
          long tok;
          uint32_t run = n - done;
          if (a.c.block_table) {  // paged: runs that stay inside one block
            const int pp = first + (int)done, j = pp / a.c.block_size, off = pp - j * a.c.block_size;
            run = min(run, (uint32_t)(a.c.block_size - off));
            int bl = a.c.block_table[(long)s * (a.c.capacity / a.c.block_size) + j];
            if (bl < 0 || bl >= a.c.n_blocks) {
              atomicOr(a.p.err, kErrTokenRange);
              bl = 0;
            }
            tok = ((long)bl * a.c.n_kv_heads + h) * a.c.block_size + off;
          } else {
            tok = base + first + done;
          }
          bulk_g2s(smem_u32(st + St::kc + done * (D * BK / 8)), a.c.codes_k + tok * (D * BK / 8), run * (D * BK / 8),
                   bar);
          bulk_g2s(smem_u32(st + St::vc + done * (D * BV / 8)), a.c.codes_v + tok * (D * BV / 8), run * (D * BV / 8),
                   bar);
          bulk_g2s(smem_u32(st + St::kn + done * 2), a.c.norm_k + tok, run * 2, bar);
          bulk_g2s(smem_u32(st + St::vn + done * 2), a.c.norm_v + tok, run * 2, bar);
          if constexpr (QJL) {
            bulk_g2s(smem_u32(st + St::jb + done * (D / 8)), a.c.qjl_bits + tok * (D / 8), run * (D / 8), bar);
            bulk_g2s(smem_u32(st + St::jg + done * 2), a.c.qjl_norm + tok, run * 2, bar);
          }
          done += run;
        }
        issued = it + 1;
      }
      if (*(volatile int *)&abort_flag) {
        for (int it = max(0, issued - kPStages); it < issued; ++it)
          mbar_wait(smem_u32(&full_bar[it % kPStages]), (it / kPStages) & 1);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int row0 = 16 * warp + r, row1 = row0 + 8;
  const int pos0 = s_pos[row0], pos1 = s_pos[row1];
  // keys this warp needs: up to its last row's position
  int kend_w = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) kend_w = max(kend_w, s_pos[16 * warp + i] + 1);
  uint32_t qh[4][4], ql[4][4], jh[QJL ? 4 : 1][4], jl[QJL ? 4 : 1][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int e = 0; e < 4; ++e) {  // a0: row r, a1: row r + 8; a2, a3: k + 16
      const int row = (e & 1) ? row1 : row0, off = 32 * ks + 16 * (e >> 1) + 4 * q;
      qh[ks][e] = *reinterpret_cast<const uint32_t *>(&s_q8[row][0][off]);
      ql[ks][e] = *reinterpret_cast<const uint32_t *>(&s_q8[row][1][off]);
      if constexpr (QJL) {
        jh[ks][e] = *reinterpret_cast<const uint32_t *>(&s_q8[row][2][off]);
        jl[ks][e] = *reinterpret_cast<const uint32_t *>(&s_q8[row][3][off]);
      }
    }
  const float fq0 = s_qs[row0][0], fq1 = s_qs[row1][0];
  const float fj0 = QJL ? s_qs[row0][1] : 0.f, fj1 = QJL ? s_qs[row1][1] : 0.f;
  const float js0 = QJL ? s_qs[row0][2] : 0.f, js1 = QJL ? s_qs[row1][2] : 0.f;
  const Lut lk = a.p.lut_k, lv = a.p.lut_v;

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;

  for (int it = 0; it < n_stage; ++it) {
    const int slot = it % kPStages;
    if (!mbar_wait(smem_u32(&full_bar[slot]), (it / kPStages) & 1)) {
      atomicOr(a.p.err, kErrWaitExpired);
      abort_flag = 1;
      break;
    }
    const unsigned char *st = smem + slot * St::bytes;
    const int first = it * kPStageTokens;
#pragma unroll 1
    for (int ch = 0; ch < kPStageTokens / kChunk; ++ch) {
      const int kbase = first + ch * kChunk;  // position of the chunk's first key
      if (kbase >= kend_w) break;
      const int kc0 = ch * kChunk;             // its row inside the stage
      // ---------------- scores of 4 key n-tiles (keys kbase + 8 j + r as B
      // rows), each turned into floats at once; element (j, e): row r (e < 2)
      // or r + 8, key kbase + 8 j + 2 q + (e & 1)
      const __half *kn = reinterpret_cast<const __half *>(st + St::kn) + kc0;
      const __half *vn = reinterpret_cast<const __half *>(st + St::vn) + kc0;
      const __half *gn = reinterpret_cast<const __half *>(st + St::jg) + kc0;
      float sc[4][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int chh[4] = {0, 0, 0, 0}, cmid[4] = {0, 0, 0, 0}, cll[4] = {0, 0, 0, 0};
        int cjh[4] = {0, 0, 0, 0}, cjl[4] = {0, 0, 0, 0};
        uint32_t wk[BK];
        const unsigned char *kr = st + St::kc + (kc0 + 8 * j + r) * (D * BK / 8) + q * 4 * BK;
#pragma unroll
        for (int i = 0; i < BK; ++i) wk[i] = reinterpret_cast<const uint32_t *>(kr)[i];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t blo0, bhi0, blo1, bhi1;
          lookup<BK>(lk, k_selector<BK>(wk, 2 * ks), blo0, bhi0);
          lookup<BK>(lk, k_selector<BK>(wk, 2 * ks + 1), blo1, bhi1);
          mma_i8<true, true>(chh, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], bhi0, bhi1);
          mma_i8<true, false>(cmid, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], blo0, blo1);
          mma_i8<false, true>(cmid, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3], bhi0, bhi1);
          mma_i8<false, false>(cll, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3], blo0, blo1);
        }
        if constexpr (QJL) {
          const uint32_t sw = reinterpret_cast<const uint32_t *>(st + St::jb + (kc0 + 8 * j + r) * (D / 8))[q];
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint32_t b0 = prmt(sw << (7 - 2 * ks), 0u, 0xBA98u), b1 = prmt(sw << (6 - 2 * ks), 0u, 0xBA98u);
            mma_i8<true, true>(cjh, jh[ks][0], jh[ks][1], jh[ks][2], jh[ks][3], b0, b1);
            mma_i8<false, true>(cjl, jl[ks][0], jl[ks][1], jl[ks][2], jl[ks][3], b0, b1);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = 8 * j + 2 * q + (e & 1);
          const bool top = e < 2;
          const int hm = (chh[e] << 8) + cmid[e];
          float v = fmaf(256.f, (float)hm, (float)cll[e]) * (top ? fq0 : fq1);
          if constexpr (QJL) {
            const float dj = fmaf(256.f, (float)cjh[e], (float)cjl[e]);
            v = fmaf(__half2float(gn[kk]) * (top ? fj0 : fj1), fmaf(-2.f, dj, -(top ? js0 : js1)), v);
          }
          v *= __half2float(kn[kk]);
          const bool live = kbase + kk <= (top ? pos0 : pos1);
          sc[j][e] = live ? v : -INFINITY;
          if (top) mx0 = fmaxf(mx0, sc[j][e]);
          else mx1 = fmaxf(mx1, sc[j][e]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
      // a finite reference keeps exp2(-inf - ref) = 0 while a row has no live key
      const float ref0 = fmaxf(mn0, -3.0e38f), ref1 = fmaxf(mn1, -3.0e38f);
      const float al0 = fast_exp2(m_run[0] - ref0), al1 = fast_exp2(m_run[1] - ref1);
      m_run[0] = mn0;
      m_run[1] = mn1;
      float ls0 = 0.f, ls1 = 0.f;
      uint32_t pa[2][4];  // A fragments of P' for the two k16 steps
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = 8 * j + 2 * q + (e & 1);
          const bool top = e < 2;
          const float pe = fast_exp2(sc[j][e] - (top ? ref0 : ref1));
          if (top) ls0 += pe;
          else ls1 += pe;
          pv[e] = sc[j][e] == -INFINITY ? 0.f : pe * __half2float(vn[kk]);
        }
        // n-tile j is k-half (j & 1) of k16 step j / 2: a0/a1 (keys 0..7) or a2/a3
        pa[j >> 1][2 * (j & 1)] = pack_half2(pv[0], pv[1]);
        pa[j >> 1][2 * (j & 1) + 1] = pack_half2(pv[2], pv[3]);
      }
      l_run[0] = fmaf(l_run[0], al0, ls0);
      l_run[1] = fmaf(l_run[1], al1, ls1);
      if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          acc[nt][0] *= al0;
          acc[nt][1] *= al0;
          acc[nt][2] *= al1;
          acc[nt][3] *= al1;
        }
      }
      // ---------------- values: fp16 MMA per k16 step (keys kc0 + 16 t ..),
      // V expanded as in decode (tokens 2q, 2q+1 and 2q+8, 2q+9; coordinate
      // units of 16): B of n-tile 2 mt = (a0, a2), of n-tile 2 mt + 1 = (a1, a3)
      constexpr int VB = D * BV / 8;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const unsigned char *vt = st + St::vc + (kc0 + 16 * t + 2 * q) * VB;
        const uint32_t *P = pa[t];
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
              const int mt = 2 * k + hh;
              mma_f16(acc[2 * mt], P[0], P[1], P[2], P[3], a0, a2);
              mma_f16(acc[2 * mt + 1], P[0], P[1], P[2], P[3], a1, a3);
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
                const int mt = 4 * yh + 2 * par + hh;
                mma_f16(acc[2 * mt], P[0], P[1], P[2], P[3], a0, a2);
                mma_f16(acc[2 * mt + 1], P[0], P[1], P[2], P[3], a1, a3);
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
                const int mt = 4 * u + 2 * yh + hh;
                mma_f16(acc[2 * mt], P[0], P[1], P[2], P[3], a0, a2);
                mma_f16(acc[2 * mt + 1], P[0], P[1], P[2], P[3], a1, a3);
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
  if (*(volatile int *)&abort_flag) return;

  // ---------------- o = Pi^T (O / l): A = O (bf16 hi + lo), B from Pi^T's
  // rows in the V fragment order (pivt[i][k] = Pi[vperm(k)][i])
  float l0 = l_run[0], l1 = l_run[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float il0 = l0 > 0.f ? 1.f / l0 : 0.f, il1 = l1 > 0.f ? 1.f / l1 : 0.f;
  uint32_t ohi[8][4], olo[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    split_bf16x2(acc[2 * ks][0] * il0, acc[2 * ks][1] * il0, ohi[ks][0], olo[ks][0]);
    split_bf16x2(acc[2 * ks][2] * il1, acc[2 * ks][3] * il1, ohi[ks][1], olo[ks][1]);
    split_bf16x2(acc[2 * ks + 1][0] * il0, acc[2 * ks + 1][1] * il0, ohi[ks][2], olo[ks][2]);
    split_bf16x2(acc[2 * ks + 1][2] * il1, acc[2 * ks + 1][3] * il1, ohi[ks][3], olo[ks][3]);
  }
  const int rho0 = row0 & 15, rho1 = row1 & 15;
  float *o0 = pos0 >= 0 ? a.out + (qrow0 + (long)(pos0 - p0) * a.n_q_heads + rho0 % G) * D : nullptr;
  float *o1 = pos1 >= 0 ? a.out + (qrow0 + (long)(pos1 - p0) * a.n_q_heads + rho1 % G) * D : nullptr;
#pragma unroll 2
  for (int nt = 0; nt < 16; ++nt) {
    // this n-tile's B fragments: four coalesced 16-byte loads (two k-steps each)
    uint4 bf[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) bf[j] = reinterpret_cast<const uint4 *>(a.p.pvf)[(nt * 4 + j) * 32 + lane];
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint4 &v = bf[ks / 2];
      const uint32_t b0 = (ks & 1) ? v.z : v.x, b1 = (ks & 1) ? v.w : v.y;
      mma_bf16(c, ohi[ks][0], ohi[ks][1], ohi[ks][2], ohi[ks][3], b0, b1);
      mma_bf16(c, olo[ks][0], olo[ks][1], olo[ks][2], olo[ks][3], b0, b1);
    }
    if (o0) *reinterpret_cast<float2 *>(o0 + 8 * nt + 2 * q) = make_float2(c[0], c[1]);
    if (o1) *reinterpret_cast<float2 *>(o1 + 8 * nt + 2 * q) = make_float2(c[2], c[3]);
  }
  if (a.lse && q == 0) {
    constexpr float kLn2 = 0.6931471805599453f;
    if (pos0 >= 0) a.lse[qrow0 + (long)(pos0 - p0) * a.n_q_heads + rho0 % G] = (m_run[0] + log2f(l0)) * kLn2;
    if (pos1 >= 0) a.lse[qrow0 + (long)(pos1 - p0) * a.n_q_heads + rho1 % G] = (m_run[1] + log2f(l1)) * kLn2;
  }
}

using PrefillFn = void (*)(const PrefillArgs);

template <int BK, int BV>
PrefillFn pick_q(bool qjl) {
  return qjl ? prefill_attn_kernel<BK, BV, true> : prefill_attn_kernel<BK, BV, false>;
}

template <int BK>
PrefillFn pick_v(int bv, bool qjl) {
  return bv == 2 ? pick_q<BK, 2>(qjl) : bv == 3 ? pick_q<BK, 3>(qjl) : pick_q<BK, 4>(qjl);
}

PrefillFn pick(int bk, int bv, bool qjl) {
  return bk == 2 ? pick_v<2>(bv, qjl) : bk == 3 ? pick_v<3>(bv, qjl) : pick_v<4>(bv, qjl);
}

int smem_of(int bk, int bv, bool qjl) {
  static constexpr int t[3][3][2] = {
      {{prefill_smem_bytes<2, 2, false>(), prefill_smem_bytes<2, 2, true>()},
       {prefill_smem_bytes<2, 3, false>(), prefill_smem_bytes<2, 3, true>()},
       {prefill_smem_bytes<2, 4, false>(), prefill_smem_bytes<2, 4, true>()}},
      {{prefill_smem_bytes<3, 2, false>(), prefill_smem_bytes<3, 2, true>()},
       {prefill_smem_bytes<3, 3, false>(), prefill_smem_bytes<3, 3, true>()},
       {prefill_smem_bytes<3, 4, false>(), prefill_smem_bytes<3, 4, true>()}},
      {{prefill_smem_bytes<4, 2, false>(), prefill_smem_bytes<4, 2, true>()},
       {prefill_smem_bytes<4, 3, false>(), prefill_smem_bytes<4, 3, true>()},
       {prefill_smem_bytes<4, 4, false>(), prefill_smem_bytes<4, 4, true>()}}};
  return t[bk - 2][bv - 2][qjl ? 1 : 0];
}

}  // namespace

}  // namespace tq


// ===========================================================================
// The tcgen05 form (contexts without QJL).  Per CTA 128 query rows (the MMA's
// M) and, per tile of 128 keys, four roles that overlap across tiles:
//   expand   (warps 8-11) the keys' codes into two fp16 shared-memory
//            operands in the 128-byte-swizzled K-major layout,
//            double-buffered: K~[key][kappa] (the exact fp16 K centroids, K
//            fragment order) and V~^T[kappa_v][key] (fp16 V centroids, V
//            fragment order), and the key norms as fp32;
//   MMA      (warp 13, one thread) S = Q^_hi K~^T + Q^_lo K~^T with the
//            two-part fp16 q_hat (scaled per row by a power of two) as the A
//            operand in tensor memory, and O += P' V~ with P' as the A
//            operand in tensor memory; fp32 accumulators in tensor memory;
//            the next tile's scores are issued as soon as the softmax has
//            read the current ones;
//   softmax  (warps 0-7) two threads per row, one per half of the keys and
//            of the output coordinates: S from tensor memory, times the row's
//            factor and the key norms, causal mask (on the diagonal tiles
//            only), the tile maximum exchanged between the halves, online max
//            and sum (exp2), P' = p ||v|| as fp16 into tensor memory; a moved
//            max rescales the row of O;
//   producer (warp 12) streams the codes with 1-D bulk copies.
// At the end o = Pi^T (O / l) is one more pair of MMAs (O as bf16 hi + lo,
// Pi^T's rows in the V fragment order as the B operand), and the lse.
// Tensor memory: S at columns 0-127, O at 128-255, q_hat hi and lo at
// 256-319 and 320-383, P' at 384-447 and 448-511 (tiles alternate, so the
// softmax of a tile does not wait for the previous tile's value MMAs unless
// it rescales O).  Every mbarrier wait is bounded.
// ===========================================================================
namespace tq {
namespace {

constexpr int kTcRows = 128;                      // query rows per CTA
constexpr int kTcKeys = 128;                      // keys per tile
constexpr int kTcExpWarp0 = 8;                    // warps 8-11 expand (0-7: softmax)
constexpr int kTcProdWarp = 12, kTcMmaWarp = 13;
constexpr int kTcThreads = 32 * 14;
constexpr int kTcStages = 2;
constexpr int kOpBytes = 128 * kHeadDim * 2;      // one 128 x 128 16-bit operand: two 128 x 64 swizzled boxes
constexpr int kOpBox = kOpBytes / 2;
constexpr uint32_t kTcCols = 512;
constexpr uint32_t kTcS = 0, kTcO = 128, kTcQ = 256, kTcP = 384;  // tensor-memory columns

template <int BK, int BV>
struct TcLayout {
  // K~ buffers 0, 1; V~ buffers 0, 1 (the prologue's fp32 q_hat scratch
  // spans both K~ buffers; the epilogue's operands reuse K~ and V~ 0)
  static constexpr int kt0 = 0, kt1 = kOpBytes, vt0 = 2 * kOpBytes, vt1 = 3 * kOpBytes;
  static constexpr int ring = 4 * kOpBytes;
  static constexpr int stage = Stage<BK, BV, false, kTcKeys>::bytes;
  // the tile's key norms as fp32, per K~ / V~ buffer: nf[buffer][k or v][key]
  static constexpr int nf = ring + kTcStages * stage;
  static constexpr int bytes = nf + 2 * 2 * kTcKeys * 4 + 1024;  // + alignment slack
};

__device__ __forceinline__ void tcx_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tcx_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Byte offset of element (row, col) of a 128 x 128 16-bit operand stored as
// two boxes of 128 rows x 64 columns, 128-byte rows, 16-byte chunks swizzled
// by the row within each 8-row (1024-byte) atom.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  const int box = col >> 6, cc = col & 63;
  return (uint32_t)(box * kOpBox + row * 128 + ((((cc >> 3) ^ (row & 7)) & 7) << 4) + ((cc & 7) << 1));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t swdesc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptors, kind::f16, fp32 accumulator, A and B K-major,
// M = N = 128: fp16 inputs, and bf16 inputs.
constexpr uint32_t kIdescF16 = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescBF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// D += A B with A and B in shared memory.
__device__ __forceinline__ void tcx_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
               : "memory");
}
// D += A B with A in tensor memory (fp16, two elements per 32-bit column)
// and B in shared memory.
__device__ __forceinline__ void tcx_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t accumulate) {
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
                   tmem_d),
               "r"(tmem_a), "l"(b), "r"(kIdescF16), "r"(accumulate)
               : "memory");
}
__device__ __forceinline__ void tcx_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld16x(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st16x(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// After tmem_wait_ld: passes the loaded registers through an empty asm, so
// that no use of them is scheduled above the wait.
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// fp16 pairs (codes 0, 1) and (codes 2, 3) of one lookup's low and high bytes.
__device__ __forceinline__ void f16_pairs(uint32_t lo, uint32_t hi, uint32_t &p01, uint32_t &p23) {
  p01 = prmt(lo, hi, 0x5140u);
  p23 = prmt(lo, hi, 0x7362u);
}

// K~ and V~^T of one tile of keys (ew: the expanding warp 0-3, keys
// 32 ew .. 32 ew + 31) into the operand buffers kt and vt.
template <int BK, int BV>
__device__ __forceinline__ void expand_tile(const unsigned char *st, unsigned char *kt, unsigned char *vt,
                                            const Lut &lkf, const Lut &lv, int ew, int r, int q) {
  using St = Stage<BK, BV, false, kTcKeys>;
#pragma unroll
  for (int rb = 0; rb < 2; ++rb) {
    const int k0 = 32 * ew + 16 * rb + r, k1 = k0 + 8;
    uint32_t wk0[BK], wk1[BK];
    const unsigned char *kr0 = st + St::kc + k0 * (D * BK / 8) + q * 4 * BK;
    const unsigned char *kr1 = st + St::kc + k1 * (D * BK / 8) + q * 4 * BK;
#pragma unroll
    for (int i = 0; i < BK; ++i) {
      wk0[i] = reinterpret_cast<const uint32_t *>(kr0)[i];
      wk1[i] = reinterpret_cast<const uint32_t *>(kr1)[i];
    }
#pragma unroll
    for (int sg = 0; sg < 8; ++sg) {
      const int kap = 32 * (sg >> 1) + 16 * (sg & 1) + 4 * q;
      uint32_t lo, hi, p01, p23;
      lookup<BK>(lkf, k_selector<BK>(wk0, sg), lo, hi);
      f16_pairs(lo, hi, p01, p23);
      *reinterpret_cast<uint2 *>(kt + sw_off(k0, kap)) = make_uint2(p01, p23);
      lookup<BK>(lkf, k_selector<BK>(wk1, sg), lo, hi);
      f16_pairs(lo, hi, p01, p23);
      *reinterpret_cast<uint2 *>(kt + sw_off(k1, kap)) = make_uint2(p01, p23);
    }
  }
#pragma unroll
  for (int rb = 0; rb < 2; ++rb) {
    // V~^T: rows in the V fragment order, keys as columns (decode's A
    // fragments: a0 = row 16 mt + r, keys 2q, 2q+1; a1 = row + 8; a2, a3:
    // keys + 8)
    constexpr int VB = D * BV / 8;
    const int kb = 32 * ew + 16 * rb;  // first key of the 16-key block
    const unsigned char *vc = st + St::vc + (kb + 2 * q) * VB;
    auto put = [&](int mt, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
      *reinterpret_cast<uint32_t *>(vt + sw_off(16 * mt + r, kb + 2 * q)) = a0;
      *reinterpret_cast<uint32_t *>(vt + sw_off(16 * mt + r + 8, kb + 2 * q)) = a1;
      *reinterpret_cast<uint32_t *>(vt + sw_off(16 * mt + r, kb + 8 + 2 * q)) = a2;
      *reinterpret_cast<uint32_t *>(vt + sw_off(16 * mt + r + 8, kb + 8 + 2 * q)) = a3;
    };
    if constexpr (BV == 3) {
      const int gofs = 12 * (r >> 1);
      const uint32_t gs = (r & 1) ? 0x7362u : 0x5140u;
      uint32_t ya[3], yb[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        ya[k] = prmt(reinterpret_cast<const uint32_t *>(vc + gofs)[k],
                     reinterpret_cast<const uint32_t *>(vc + VB + gofs)[k], gs);
        yb[k] = prmt(reinterpret_cast<const uint32_t *>(vc + 8 * VB + gofs)[k],
                     reinterpret_cast<const uint32_t *>(vc + 9 * VB + gofs)[k], gs);
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
          put(2 * k + hh, a0, a1, a2, a3);
        }
      }
    } else if constexpr (BV == 2) {
      const uint32_t A0 = reinterpret_cast<const uint32_t *>(vc)[r];
      const uint32_t B0 = reinterpret_cast<const uint32_t *>(vc + VB)[r];
      const uint32_t A1 = reinterpret_cast<const uint32_t *>(vc + 8 * VB)[r];
      const uint32_t B1 = reinterpret_cast<const uint32_t *>(vc + 9 * VB)[r];
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
            put(4 * yh + 2 * par + hh, a0, a1, a2, a3);
          }
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t A0 = reinterpret_cast<const uint32_t *>(vc)[2 * r + u];
        const uint32_t B0 = reinterpret_cast<const uint32_t *>(vc + VB)[2 * r + u];
        const uint32_t A1 = reinterpret_cast<const uint32_t *>(vc + 8 * VB)[2 * r + u];
        const uint32_t B1 = reinterpret_cast<const uint32_t *>(vc + 9 * VB)[2 * r + u];
#pragma unroll
        for (int yh = 0; yh < 2; ++yh) {
          const uint32_t gs = yh ? 0x7362u : 0x5140u;
          const uint32_t ya = prmt(A0, B0, gs), yb = prmt(A1, B1, gs);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t a0, a1, a2, a3;
            v_pairs<4>(lv, hh ? ya >> 16 : ya, a0, a1);
            v_pairs<4>(lv, hh ? yb >> 16 : yb, a2, a3);
            put(4 * u + 2 * yh + hh, a0, a1, a2, a3);
          }
        }
      }
    }
  }
}

// A wait on the kernel's flag or on a barrier; false (and the error flagged,
// the kernel told to stop) once the barrier's bounded wait expires.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, unsigned *err, int *abort_flag) {
  if (mbar_wait(smem_u32(bar), parity)) return true;
  atomicOr(err, kErrWaitExpired);
  *(volatile int *)abort_flag = 1;
  return false;
}

template <int BK, int BV>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const PrefillArgs a) {
  using L = TcLayout<BK, BV>;
  using St = Stage<BK, BV, false, kTcKeys>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full_bar[kTcStages], empty_bar[kTcStages];
  __shared__ __align__(8) uint64_t kv_full[2], kv_empty[2], s_full, s_empty, p_full, pv_done[2];
  __shared__ __align__(8) uint64_t q_ready, scratch_done, scratch_free, o_ready, fin_bar, mma_done;
  __shared__ __align__(8) uint64_t mx_bar[2], l_bar;
  __shared__ float s_max[2][2][kTcRows], s_l[2][kTcRows];  // the half rows' maxima (by tile parity) and sums
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int s_pos[kTcRows];

  const int s = blockIdx.z, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, r = lane >> 2, q = lane & 3;
  const int G = a.n_q_heads / a.c.n_kv_heads;
  const int PC = kTcRows / G;                  // positions per CTA
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int blk = gridDim.x - 1 - blockIdx.x;  // the longest blocks first
  const int q0 = a.cu_q[s], n_q = a.cu_q[s + 1] - q0;
  const int len = a.seq_lens[s];
  if (len < 0 || len > a.max_seq_len || n_q < 0 || n_q > len || n_q > a.max_q) {
    if (tid == 0 && blk == 0 && h == 0) atomicOr(a.p.err, kErrSeqLen);
    return;
  }
  const int first_q = blk * PC;
  if (first_q >= n_q) return;
  const int p0 = len - n_q;
  const int last_q = min(n_q, first_q + PC) - 1;
  const int kend = p0 + last_q + 1;
  const int n_tiles = (kend + kTcKeys - 1) / kTcKeys;
  const long base = ((long)s * a.c.n_kv_heads + h) * a.c.capacity;
  const long qrow0 = (long)q0 * a.n_q_heads + (long)h * G;
  unsigned *err = a.p.err;

  if (tid < kTcRows) {
    const int qi = first_q + tid / G;
    s_pos[tid] = (tid < PC * G && qi < n_q) ? p0 + qi : -1;
  }
  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 4);  // the expanding warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&kv_full[b]), 4);
      mbar_init(smem_u32(&kv_empty[b]), 1);
    }
    mbar_init(smem_u32(&s_full), 1);
    mbar_init(smem_u32(&s_empty), 8);  // the eight softmax warps
    mbar_init(smem_u32(&p_full), 8);
    mbar_init(smem_u32(&pv_done[0]), 1);
    mbar_init(smem_u32(&pv_done[1]), 1);
    mbar_init(smem_u32(&q_ready), 8);
    mbar_init(smem_u32(&scratch_done), 8);
    mbar_init(smem_u32(&scratch_free), 8);
    mbar_init(smem_u32(&o_ready), 8);
    mbar_init(smem_u32(&mx_bar[0]), 8);
    mbar_init(smem_u32(&mx_bar[1]), 8);
    mbar_init(smem_u32(&l_bar), 8);
    mbar_init(smem_u32(&fin_bar), 1);
    mbar_init(smem_u32(&mma_done), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTcMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tcx_fence_before();
  __syncthreads();
  tcx_fence_after();
  const uint32_t tmem = tmem_slot;
  int *abf = &abort_flag;

  if (warp == kTcProdWarp) {
    // ---------------- producer: the codes of one tile of keys per stage
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int slot = it % kTcStages;
        if (it >= kTcStages && !tc_wait(&empty_bar[slot], ((it / kTcStages) - 1) & 1, err, abf)) break;
        if (*(volatile int *)abf) break;
        unsigned char *st = sm + L::ring + slot * L::stage;
        const uint32_t bar = smem_u32(&full_bar[slot]);
        const int first = it * kTcKeys;
        const uint32_t n = (uint32_t)min(kTcKeys, (kend - first + 63) & ~63);
        mbar_arrive_expect_tx(bar, n * (D * BK / 8 + D * BV / 8 + 4));
        for (uint32_t done = 0; done < n;) {
          long tok;
          uint32_t run = n - done;
          if (a.c.block_table) {
            const int pp = first + (int)done, j = pp / a.c.block_size, off = pp - j * a.c.block_size;
            run = min(run, (uint32_t)(a.c.block_size - off));
            int bl = a.c.block_table[(long)s * (a.c.capacity / a.c.block_size) + j];
            if (bl < 0 || bl >= a.c.n_blocks) {
              atomicOr(err, kErrTokenRange);
              bl = 0;
            }
            tok = ((long)bl * a.c.n_kv_heads + h) * a.c.block_size + off;
          } else {
            tok = base + first + done;
          }
          bulk_g2s(smem_u32(st + St::kc + done * (D * BK / 8)), a.c.codes_k + tok * (D * BK / 8), run * (D * BK / 8),
                   bar);
          bulk_g2s(smem_u32(st + St::vc + done * (D * BV / 8)), a.c.codes_v + tok * (D * BV / 8), run * (D * BV / 8),
                   bar);
          bulk_g2s(smem_u32(st + St::kn + done * 2), a.c.norm_k + tok, run * 2, bar);
          bulk_g2s(smem_u32(st + St::vn + done * 2), a.c.norm_v + tok, run * 2, bar);
          done += run;
        }
        issued = it + 1;
      }
      if (*(volatile int *)abf) {  // never leave copies in flight
        for (int it = max(0, issued - kTcStages); it < issued; ++it)
          mbar_wait(smem_u32(&full_bar[it % kTcStages]), (it / kTcStages) & 1);
      }
    }
  } else if (warp == kTcMmaWarp) {
    // ---------------- MMA issuer: S(it + 1) as soon as the softmax has read
    // S(it), then O += P'(it) V~(it)
    if (lane == 0) {
      const uint32_t t_s = tmem + kTcS, t_o = tmem + kTcO, t_q = tmem + kTcQ, t_p = tmem + kTcP;
      auto scores = [&](int it) {
        const uint32_t bk = smem_u32(sm + ((it & 1) ? L::kt1 : L::kt0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kOpBox + (kk & 3) * 32;
          tcx_mma_ts(t_s, t_q + 8 * kk, swdesc(bk + off), kk > 0);  // q_hat hi
          tcx_mma_ts(t_s, t_q + 64 + 8 * kk, swdesc(bk + off), 1);  // q_hat lo
        }
        tcx_commit(smem_u32(&s_full));
      };
      bool ok = tc_wait(&q_ready, 0, err, abf) && tc_wait(&kv_full[0], 0, err, abf);
      if (ok) {
        tcx_fence_after();
        scores(0);
      }
      for (int it = 0; ok && it < n_tiles; ++it) {
        if (it + 1 < n_tiles) {
          ok = tc_wait(&kv_full[(it + 1) & 1], ((it + 1) >> 1) & 1, err, abf) && tc_wait(&s_empty, it & 1, err, abf);
          if (!ok || *(volatile int *)abf) break;
          tcx_fence_after();
          scores(it + 1);
        }
        ok = tc_wait(&p_full, it & 1, err, abf);
        if (!ok || *(volatile int *)abf) break;
        tcx_fence_after();
        const uint32_t bv = smem_u32(sm + ((it & 1) ? L::vt1 : L::vt0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kOpBox + (kk & 3) * 32;
          tcx_mma_ts(t_o, t_p + 64 * (it & 1) + 8 * kk, swdesc(bv + off), (it > 0 || kk > 0) ? 1u : 0u);
        }
        tcx_commit(smem_u32(&pv_done[it & 1]));
        tcx_commit(smem_u32(&kv_empty[it & 1]));
      }
      // o = Pi^T (O / l): A = O as bf16 hi + lo (over K~ 0 and 1), B = Pi^T's
      // rows in the V fragment order (over V~ 0)
      if (ok && !*(volatile int *)abf) {
        ok = tc_wait(&o_ready, 0, err, abf);
        if (ok) {
          tcx_fence_after();
          const uint32_t ah = smem_u32(sm + L::kt0), alo = smem_u32(sm + L::kt1), bp = smem_u32(sm + L::vt0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kOpBox + (kk & 3) * 32;
            tcx_mma(t_s, swdesc(ah + off), swdesc(bp + off), kIdescBF16, kk > 0);
            tcx_mma(t_s, swdesc(alo + off), swdesc(bp + off), kIdescBF16, 1);
          }
          tcx_commit(smem_u32(&fin_bar));
        }
      }
      // every MMA issued here has completed before the tensor memory is released
      tcx_commit(smem_u32(&mma_done));
      mbar_wait(smem_u32(&mma_done), 0);
    }
  } else if (warp >= kTcExpWarp0) {
    // ---------------- expansion: K~ and V~ of every tile, double-buffered
    const int ew = warp - kTcExpWarp0;
    Lut lkf;  // the K centroids as fp16 byte tables (exact: the centroids are fp16 values)
#pragma unroll
    for (int i = 0; i < 4; ++i) lkf.lo[i] = lkf.hi[i] = 0u;
    for (int e = 0; e < (1 << BK); ++e) {
      const uint16_t hb = __half_as_ushort(__float2half_rn(a.p.cb[e]));
      lkf.lo[e / 4] |= (uint32_t)(hb & 0xff) << (8 * (e % 4));
      lkf.hi[e / 4] |= (uint32_t)(hb >> 8) << (8 * (e % 4));
    }
    const Lut lv = a.p.lut_v;
    // the first expansion overwrites the softmax warps' q_hat scratch
    bool ok = tc_wait(&scratch_free, 0, err, abf);
    for (int it = 0; ok && it < n_tiles; ++it) {
      const int slot = it % kTcStages, b = it & 1;
      ok = tc_wait(&full_bar[slot], (it / kTcStages) & 1, err, abf);
      if (ok && it >= 2) ok = tc_wait(&kv_empty[b], ((it >> 1) - 1) & 1, err, abf);
      if (!ok || *(volatile int *)abf) break;
      tcx_fence_after();
      const unsigned char *st = sm + L::ring + slot * L::stage;
      expand_tile<BK, BV>(st, sm + (b ? L::kt1 : L::kt0), sm + (b ? L::vt1 : L::vt0), lkf, lv, ew, r, q);
      {  // the key norms as fp32 for the softmax warps (keys past the copied ones are masked there)
        const int key = tid - 32 * kTcExpWarp0;
        float *nf = reinterpret_cast<float *>(sm + L::nf) + b * 2 * kTcKeys;
        nf[key] = __half2float(reinterpret_cast<const __half *>(st + St::kn)[key]);
        nf[kTcKeys + key] = __half2float(reinterpret_cast<const __half *>(st + St::vn)[key]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&kv_full[b]));
        mbar_arrive(smem_u32(&empty_bar[slot]));  // the codes are read
      }
    }
  } else {
    // ---------------- softmax warps: row 32 (warp % 4) + lane, half
    // h = warp / 4 of its keys (64 h .. 64 h + 63 of every tile) and of its
    // output coordinates; the two halves of a row meet on mbarriers for the
    // tile maximum and, at the end, for the sum
    const int h2 = warp >> 2, quarter = warp & 3;
    const int row = 32 * quarter + lane, pos = s_pos[row];
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;  // this warp's TMEM lane quarter
    const uint32_t t_s = tmem + kTcS + lane_off + 64 * h2, t_o = tmem + kTcO + lane_off + 64 * h2;
    const uint32_t t_q = tmem + kTcQ + lane_off + 32 * h2, t_p = tmem + kTcP + lane_off + 32 * h2;
    // q_hat = Pi q in the K fragment order (Pi's rows stored in that order),
    // mma m16n8k16 bf16, fp32 q as hi + lo; warp w computes rows 16 w ..
    // 16 w + 15 into a fp32 scratch over the K~ buffers
    float *scr = reinterpret_cast<float *>(sm + L::kt0);  // [128 rows][128], 64 KB
    {
      const bool f32 = a.q_dtype == TQ_F32;
      uint32_t ahi[8][4], alo[8][4];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = 16 * warp + r + 8 * (e & 1), col = 16 * ks + 8 * (e >> 1) + 2 * q;
          const int pr = s_pos[rr];
          float x0 = 0.f, x1 = 0.f;
          if (pr >= 0) {
            const long qr = qrow0 + (long)(pr - p0) * a.n_q_heads + (rr % G);
            if (f32) {
              const float2 v = *reinterpret_cast<const float2 *>(static_cast<const float *>(a.q) + qr * D + col);
              x0 = v.x;
              x1 = v.y;
            } else {
              const uint32_t v =
                  *reinterpret_cast<const uint32_t *>(static_cast<const uint16_t *>(a.q) + qr * D + col);
              x0 = __uint_as_float(v << 16);
              x1 = __uint_as_float(v & 0xffff0000u);
            }
          }
          split_bf16x2(x0, x1, ahi[ks][e], alo[ks][e]);
        }
#pragma unroll 1
      for (int nt = 0; nt < 16; ++nt) {
        uint32_t bfr[8][2];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint4 v = reinterpret_cast<const uint4 *>(a.p.pikf)[(nt * 4 + jj) * 32 + lane];
          bfr[2 * jj][0] = v.x, bfr[2 * jj][1] = v.y, bfr[2 * jj + 1][0] = v.z, bfr[2 * jj + 1][1] = v.w;
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          mma_bf16(c, ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3], bfr[ks][0], bfr[ks][1]);
          mma_bf16(c, alo[ks][0], alo[ks][1], alo[ks][2], alo[ks][3], bfr[ks][0], bfr[ks][1]);
        }
        float *d0 = scr + (16 * warp + r) * D + 8 * nt + 2 * q;
        *reinterpret_cast<float2 *>(d0) = make_float2(c[0], c[1]);
        *reinterpret_cast<float2 *>(d0 + 8 * D) = make_float2(c[2], c[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&scratch_done));
    bool ok = tc_wait(&scratch_done, 0, err, abf);
    // per row: a power-of-two scale puts max |q_hat| in [2^13, 2^14), then
    // this half's coordinates of q_hat = hi + lo in fp16 into tensor memory
    // (the scores' A operand)
    float fq = 0.f;
    if (ok) {
      const float *qr = scr + row * D;
      float m = 0.f;
      for (int k = 0; k < D; ++k) m = fmaxf(m, fabsf(qr[(k + lane) & (D - 1)]));
      int ex = 0;
      if (m > 0.f) frexpf(m, &ex);
      const float sc = m > 0.f ? ldexpf(1.f, 14 - ex) : 1.f;
      fq = a.scale * kLog2e / sc;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int k0 = 64 * h2 + 32 * c;
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) split_f16x2(qr[k0 + 2 * e] * sc, qr[k0 + 2 * e + 1] * sc, hi[e], lo[e]);
        tmem_st16x(t_q + 16 * c, hi);
        tmem_st16x(t_q + 64 + 16 * c, lo);
      }
      tmem_wait_st();
    }
    tcx_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(smem_u32(&q_ready));
      mbar_arrive(smem_u32(&scratch_free));  // this thread's scratch reads are done
    }
    float m_run = -INFINITY, l_run = 0.f;
    const int min_pos = p0 + first_q;  // the CTA's first query position
    for (int it = 0; ok && it < n_tiles; ++it) {
      const int b = it & 1;
      // the tile's key norms (published with K~ and V~) and S(it)
      ok = tc_wait(&kv_full[b], (it >> 1) & 1, err, abf) && tc_wait(&s_full, it & 1, err, abf);
      if (!ok) break;
      tcx_fence_after();
      const float4 *kn4 = reinterpret_cast<const float4 *>(sm + L::nf) + b * 2 * (kTcKeys / 4) + 16 * h2;
      const float4 *vn4 = kn4 + kTcKeys / 4;
      const int kfirst = it * kTcKeys + 64 * h2;  // this half's first key
      // tiles wholly below the CTA's first query position need no causal mask
      const bool masked = it * kTcKeys + kTcKeys - 1 > min_pos;
      // this half of the row of S: four loads in flight before one wait
      uint32_t sv[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16x(t_s + 16 * c, sv[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence16(sv[c]);
      // S is read: the next tile's scores may overwrite it
      tcx_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_empty));
      // x' = S ||k||, two keys per instruction; the row factor fq (> 0)
      // enters in the exponent below, so max x = fq max x'
      float mx = -INFINITY;
#pragma unroll
      for (int j4 = 0; j4 < 16; ++j4) {
        const float4 kf = kn4[j4];
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int j = 4 * j4 + e;  // even: keys j, j + 1 sit in one 16-column load
          uint32_t &c0 = sv[j >> 4][j & 15], &c1 = sv[j >> 4][(j & 15) + 1];
          float2 x = mul2(make_float2(__uint_as_float(c0), __uint_as_float(c1)),
                          e ? make_float2(kf.z, kf.w) : make_float2(kf.x, kf.y));
          if (masked) {
            if (kfirst + j > pos) x.x = -INFINITY;
            if (kfirst + j + 1 > pos) x.y = -INFINITY;
          }
          c0 = __float_as_uint(x.x);
          c1 = __float_as_uint(x.y);
          mx = max3(mx, x.x, x.y);
        }
      }
      // the row's maximum from both halves (double-buffered by tile parity)
      s_max[b][h2][row] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&mx_bar[b]));
      ok = tc_wait(&mx_bar[b], (it >> 1) & 1, err, abf);
      if (!ok) break;
      mx = fmaxf(s_max[b][0][row], s_max[b][1][row]) * fq;
      const float mn = fmaxf(m_run, mx);
      const float ref = fmaxf(mn, -3.0e38f);
      const float al = fast_exp2(m_run - ref);
      m_run = mn;
      // P' is double-buffered in tensor memory: this tile's buffer was last
      // read by the value MMAs of tile it - 2, while those of tile it - 1 may
      // still be accumulating into O.  A moved maximum in the warp's rows
      // waits for tile it - 1 and rescales this half of O; otherwise only
      // tile it - 2 is waited for.  (Waiting on every tile's barrier phase
      // in turn, at most one phase apart, keeps the parity waits exact.)
      if (it > 0) {
        const bool rescale = __any_sync(0xffffffffu, al != 1.f);
        if (rescale) ok = tc_wait(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, err, abf);
        else if (it >= 2) ok = tc_wait(&pv_done[it & 1], ((it - 2) >> 1) & 1, err, abf);
        if (!ok) break;
        tcx_fence_after();
        if (rescale) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[16];
            tmem_ld16x(t_o + 16 * c, v);
            tmem_wait_ld();
            reg_fence16(v);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const float2 w = mul2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), make_float2(al, al));
              v[e] = __float_as_uint(w.x);
              v[e + 1] = __float_as_uint(w.y);
            }
            tmem_st16x(t_o + 16 * c, v);
          }
        }
      }
      // p = 2^(fq x' - ref), P' = p ||v||, two keys per instruction
      float2 ls2 = make_float2(0.f, 0.f);
      const float2 fq2 = make_float2(fq, fq), nref2 = make_float2(-ref, -ref);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 vf = vn4[8 * c + j4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 32 * c + 4 * j4 + 2 * e;
            const float sa = __uint_as_float(sv[j >> 4][j & 15]), sb = __uint_as_float(sv[j >> 4][(j & 15) + 1]);
            const float2 t = fma2(make_float2(sa, sb), fq2, nref2);
            const float2 pe = make_float2(fast_exp2(t.x), fast_exp2(t.y));
            ls2 = add2(ls2, pe);
            float2 pv = mul2(pe, e ? make_float2(vf.z, vf.w) : make_float2(vf.x, vf.y));
            if (masked) {  // masked keys (and keys past the copied ones, whose norms are not set) contribute 0
              if (sa == -INFINITY) pv.x = 0.f;
              if (sb == -INFINITY) pv.y = 0.f;
            }
            pk[2 * j4 + e] = pack_half2(pv.x, pv.y);
          }
        }
        tmem_st16x(t_p + 64 * (it & 1) + 16 * c, pk);
      }
      l_run = fmaf(l_run, al, ls2.x + ls2.y);
      tmem_wait_st();
      tcx_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full));
    }
    // ---------------- o = Pi^T (O / l)
    if (ok) ok = tc_wait(&pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, err, abf);
    if (ok) {
      s_l[h2][row] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_bar));
      ok = tc_wait(&l_bar, 0, err, abf);
    }
    if (ok) {
      tcx_fence_after();
      const float l = s_l[0][row] + s_l[1][row];
      const float il = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int col = 64 * h2 + 16 * c;
        uint32_t v[16];
        tmem_ld16x(t_o + 16 * c, v);
        tmem_wait_ld();
        reg_fence16(v);
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          split_bf16x2(__uint_as_float(v[2 * e]) * il, __uint_as_float(v[2 * e + 1]) * il, hi[e], lo[e]);
        *reinterpret_cast<uint4 *>(sm + L::kt0 + sw_off(row, col)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(sm + L::kt0 + sw_off(row, col + 8)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        *reinterpret_cast<uint4 *>(sm + L::kt1 + sw_off(row, col)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4 *>(sm + L::kt1 + sw_off(row, col + 8)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      }
      // this half of row `row` of Pi^T (pivt[i][k] = Pi[vperm k][i]) into the B operand
      const uint4 *prow = reinterpret_cast<const uint4 *>(a.p.pivt + (size_t)row * D + 64 * h2);
#pragma unroll 4
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(sm + L::vt0 + sw_off(row, 64 * h2 + 8 * c)) = prow[c];
      fence_async_smem();
      tcx_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&o_ready));
      ok = tc_wait(&fin_bar, 0, err, abf);
      if (ok) {
        tcx_fence_after();
        const int rho = row % G;
        float *orow = pos >= 0 ? a.out + (qrow0 + (long)(pos - p0) * a.n_q_heads + rho) * D + 64 * h2 : nullptr;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[16];
          tmem_ld16x(t_s + 16 * c, v);
          tmem_wait_ld();
          reg_fence16(v);
          if (orow) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              reinterpret_cast<float4 *>(orow + 16 * c)[e] =
                  make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]), __uint_as_float(v[4 * e + 2]),
                              __uint_as_float(v[4 * e + 3]));
          }
        }
        if (a.lse && pos >= 0 && h2 == 0)
          a.lse[qrow0 + (long)(pos - p0) * a.n_q_heads + rho] = (m_run + log2f(l)) * 0.6931471805599453f;
      }
    }
  }
  // release the tensor memory once every MMA and tcgen05 access is finished
  tcx_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tcx_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols) : "memory");
  }
}

}  // namespace
}  // namespace tq

namespace tq {
namespace {

using PrefillTcFn = void (*)(const PrefillArgs);

template <int BK>
PrefillTcFn pick_tc_v(int bv) {
  return bv == 2 ? prefill_tc_kernel<BK, 2> : bv == 3 ? prefill_tc_kernel<BK, 3> : prefill_tc_kernel<BK, 4>;
}

PrefillTcFn pick_tc(int bk, int bv) { return bk == 2 ? pick_tc_v<2>(bv) : bk == 3 ? pick_tc_v<3>(bv) : pick_tc_v<4>(bv); }

template <int BK>
int tc_bytes_v(int bv) {
  return bv == 2 ? TcLayout<BK, 2>::bytes : bv == 3 ? TcLayout<BK, 3>::bytes : TcLayout<BK, 4>::bytes;
}

int tc_bytes(int bk, int bv) { return bk == 2 ? tc_bytes_v<2>(bv) : bk == 3 ? tc_bytes_v<3>(bv) : tc_bytes_v<4>(bv); }

}  // namespace

// Contexts without QJL run the tcgen05 kernel (128 query rows per CTA);
// with QJL, the mma.sync kernel (64 rows per CTA).
int launch_prefill(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype, int n_q_heads,
                   const int32_t *cu_q, const int32_t *seq_lens, int max_q, int max_seq_len, float scale,
                   float *out, float *lse, void *stream) {
  const bool qjl = p.qjl != 0;
  const int G = n_q_heads / c.n_kv_heads;
  PrefillArgs args{p, c, n_q_heads, max_seq_len, max_q, cu_q, seq_lens, q, q_dtype, scale, out, lse};
  cudaLaunchConfig_t cfg = {};
  cfg.stream = (cudaStream_t)stream;
  if (!qjl) {
    const PrefillTcFn fn = pick_tc(p.bits_k, p.bits_v);
    const int smem = tc_bytes(p.bits_k, p.bits_v);
    static std::atomic<bool> configured_tc[kMaxDevices][3][3];
    std::atomic<bool> &done = configured_tc[current_device()][p.bits_k - 2][p.bits_v - 2];
    if (!done.load(std::memory_order_acquire)) {
      const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return (int)e;
      done.store(true, std::memory_order_release);
    }
    const int per_cta = kTcRows / G;
    cfg.gridDim = dim3((unsigned)((max_q + per_cta - 1) / per_cta), c.n_kv_heads, c.n_seqs);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    return (int)cudaLaunchKernelEx(&cfg, fn, args);
  }
  const PrefillFn fn = pick(p.bits_k, p.bits_v, qjl);
  const int smem = smem_of(p.bits_k, p.bits_v, qjl);
  // the dynamic shared-memory limit is set once per device and variant
  static std::atomic<bool> configured[kMaxDevices][3][3][2];
  std::atomic<bool> &done = configured[current_device()][p.bits_k - 2][p.bits_v - 2][qjl ? 1 : 0];
  if (!done.load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    done.store(true, std::memory_order_release);
  }
  const int per_cta = kPWarps * (16 / G);
  cfg.gridDim = dim3((unsigned)((max_q + per_cta - 1) / per_cta), c.n_kv_heads, c.n_seqs);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = smem;
  return (int)cudaLaunchKernelEx(&cfg, fn, args);
}

}  // namespace tq
