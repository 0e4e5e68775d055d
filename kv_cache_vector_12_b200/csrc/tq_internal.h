// Internal declarations shared by the host code, the API layer and the
// kernels of the TurboQuant library.  Nothing here is part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

constexpr int kHeadDim = 128;  // the head dimension of the tensor-core quantize and prefill kernels
// Head dimensions the library takes: 64, 128, 256.
inline bool supported_head_dim(int d) { return d == 64 || d == 128 || d == 256; }
constexpr int kMaxLevels = 16;  // 2^4 centroids at most

// Sticky device-side error flags (tq_check_device_errors).
constexpr unsigned kErrTokenRange = 1u;
constexpr unsigned kErrSeqLen = 2u;
constexpr unsigned kErrWaitExpired = 4u;

// --- host parameter construction (tq_host.cpp) ---
void gaussian_stream(uint64_t seed, uint32_t stream, size_t count, double *out);
uint16_t double_to_bf16_bits(double x);
float bf16_bits_to_float(uint16_t h);
uint16_t double_to_half_bits(double x);  // round to nearest even, subnormals kept
double half_bits_to_double(uint16_t h);  // finite halves
void rotation_bf16(int d, uint64_t seed, uint16_t *pi_bits);
void qjl_matrix(int d, uint64_t seed, float *s);
void lloyd_max_gaussian(int bits, double *c);
void lloyd_max_sphere(int bits, int d, double *c);
void codebook(int bits, int d, int law, float *centroids, float *thresholds);
// Whether the quantize kernel's binary search over these thresholds selects
// every threshold exactly in fp32 (tq_host.cpp).
bool threshold_search_exact(int bits, const float *thresholds);

// Bytes of one packed vector of d codes.
inline int code_bytes(int bits, int d) { return d * bits / 8; }

// Byte tables for the byte-permute lookups of the decode kernel: lo[i] packs
// the low bytes of entries 4i..4i+3, hi[i] their high bytes.  K entries are
// the centroids as 16-bit fixed point (c * 2^k_shift, exact; k_shift is the
// largest shift up to 17 that keeps every entry in [-32767, 32767], 17 at
// d = 128); V entries are the fp16 bit patterns of the centroids.
struct Lut {
  uint32_t lo[4], hi[4];
};

// Device-resident parameters of one context (all pointers device memory).
struct DeviceParams {
  const uint16_t *pi;     // Pi  [d][d] bf16 bits, row-major (z = Pi x)
  const uint32_t *pikf;   // Pi with rows in K fragment order, as the decode kernel's bf16 MMA B fragments:
                          // [warp 4][n-tile 4][chunk 4][lane 32][4 words] (16-byte aligned; see tq_api.cu)
  const float *s;         // S   [d][d] fp32 (qjl only)
  const uint32_t *sjkf;   // S' 2^sigma, S'[kappa][kappa'] = S[jperm[kappa]][kperm[kappa']], split into two fp16
                          // parts (hi + lo), each as fp16 MMA B fragments laid out like pif (qjl only)
  const uint32_t *pif;    // Pi (natural row order) as bf16 MMA B fragments [n-tile 16][chunk 4][lane 32][4 words]
  const uint32_t *sf;     // S 2^sigma split into two fp16 parts (hi + lo), each as B fragments like pif:
                          // [part 2][n-tile 16][chunk 4][lane 32][4 words] (qjl only; sigma chosen on the host)
  const uint16_t *ssplit; // the same two parts as plain row-major fp16 matrices [part 2][d][d] (qjl only)
  const float *cb;        // [4][16]: centroids_k, thresholds_k, centroids_v, thresholds_v
  unsigned *err;          // sticky error flags
  const uint8_t *kperm;   // [d] K fragment order -> coordinate
  const uint8_t *jperm;   // [d] QJL fragment order -> projection index
  const uint16_t *pivt;   // [d][d] bf16: pivt[i][k] = Pi[vperm[k]][i] (Pi^T, columns in V fragment order)
  const uint32_t *pvf;    // pivt as bf16 MMA B fragments, laid out like pif (the product O pivt^T)
  Lut lut_k, lut_v;
  int d, bits_k, bits_v, qjl;
  int k_shift;            // K centroids are exact integers times 2^-k_shift (Lut)
  int s_shift;            // sigma of sf: the fragment tables hold S 2^sigma (qjl only)
};

// Fragment orders of the decode kernel for head dimension d (host,
// tq_fragments.cpp): permutations of 0 .. d - 1.
void kperm_of(int bits, int d, uint8_t *perm);
void vperm_of(int bits, int d, uint8_t *perm);
void jperm_of(int d, uint8_t *perm);

// Split of the sequence axis used by decode attention.
struct DecodeSplit {
  int chunk;         // tokens per split (multiple of 64)
  int n_splits;      // ceil(max_seq_len / chunk), at least 1
  bool long_splits;  // run the 3-CTA-per-SM register budget of the attention kernel
};
DecodeSplit decode_split(int n_seqs, int n_kv_heads, int max_seq_len, int ctas_per_sm);
// CTAs per SM of the attention kernel for these bit widths and query heads per
// KV head, with the long-split (128-register) or short-split (168) budget, or
// the paged-layout build (128 registers).
int decode_ctas_per_sm(int d, int bits_k, int bits_v, int qjl, int group, bool long_splits, bool paged);
// The split and register budget of one decode call (tq_api.cu).
DecodeSplit plan_decode(int d, int bits_k, int bits_v, int qjl, int group, int n_seqs, int n_kv_heads,
                        int max_seq_len, bool paged);

// Workspace layout of decode attention (byte offsets, 256-aligned): the split
// partials [rows][splits][d+4] (m, l, two unused floats, then the d outputs,
// so every output block is 16-byte aligned).
struct DecodeWorkspace {
  size_t partials, total;
};
DecodeWorkspace decode_workspace(int n_seqs, int n_q_heads, DecodeSplit split, int d);

// Record a message for tq_last_error() and return `st` (tq_api.cu).
tq_status report_error(tq_status st, const char *fmt, ...);

// TQ_OK when the current CUDA device is the one the context was created on;
// otherwise TQ_ERR_INVALID (or TQ_ERR_CUDA) with a message (tq_api.cu).
tq_status check_context_device(const tq_ctx *ctx);

// Host-side caches of per-device facts (SM count, kernel attributes,
// occupancy) are indexed by the device ordinal: cudaFuncSetAttribute and the
// occupancy queries apply to the current device only.
constexpr int kMaxDevices = 64;
// The current device's ordinal, clamped into [0, kMaxDevices).
int current_device();

// --- launches (tq_kernels.cu, tq_decode.cu); return a cudaError_t as int ---
int launch_quantize(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                    const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream);
// MSE codes of K and / or V rows on tcgen05 for head dimension 128 or 64
// (tq_quantize_tc.cu).  seq_idx and pos may both be null: token t then goes
// to position t of sequence 0 (the row layout of tq_weight_quantize).
// include_k / include_v select the matrices quantized here.
int launch_quantize_tc(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                       const int32_t *seq_idx, const int32_t *pos, int n_tok, bool include_k, bool include_v,
                       void *stream);
// K and / or V rows for head dimension 256 on tcgen05 (tq_quantize_tc256.cu),
// the same index convention as launch_quantize_tc.
int launch_quantize_tc256(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                          const int32_t *seq_idx, const int32_t *pos, int n_tok, bool include_k, bool include_v,
                          void *stream);
// K rows only, the same index convention: the per-row kernel (batches of at
// most 1024 rows), or at d = 256 with QJL the batched QJL kernel.
int launch_quantize_rows_k(const DeviceParams &p, const tq_cache &c, const void *k, const int32_t *seq_idx,
                           const int32_t *pos, int n_tok, void *stream);
// K with QJL and V (MSE codes) on tcgen05 (d = 128 or 64), tiles of 128
// rows, one launch (tq_quantize_qjl_tc.cu).
int launch_quantize_qjl_tc(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                           const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream);

// B fragments of mma m16n8k16 for a d x d row-major 16-bit matrix M (the
// product is X M^T), laid out [n-tile d / 8][chunk d / 32][lane 32][4 words]:
// word 4 j + e of lane (r = lane / 4, qq = lane % 4) in n-tile nt holds the
// pair M[8 nt + r][16 ks + 8 b + 2 qq (+1)] with ks = (4 j + e) / 2 and
// b = (4 j + e) % 2, so a thread loads a chunk with one coalesced 16-byte
// load (tq_api.cu).
void mma_b_fragments(const uint16_t *m_bits, int d, uint32_t *out);
// Causal prefill attention over the packed cache (tq_prefill.cu): the queries
// of sequence s are rows cu_q[s] .. cu_q[s + 1] - 1 of q, at the last
// cu_q[s + 1] - cu_q[s] positions below seq_lens[s].
int launch_prefill(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype, int n_q_heads,
                   const int32_t *cu_q, const int32_t *seq_lens, int max_q, int max_seq_len, float scale,
                   float *out, float *lse, void *stream);
// Weight rows (tq_weight.cu): workspace of the product and its launch
// (y zeroed, x rotated, the packed rows streamed).
size_t weight_workspace_bytes(int n_tok, int n_in);
int launch_weight_gemm(const DeviceParams &p, const tq_cache &w, int n_out, int n_in, const void *x, int x_dtype,
                       int n_tok, float *y, char *workspace, void *stream);
int launch_decode(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype,
                  int n_q_heads, const int32_t *seq_lens, int max_seq_len, float scale,
                  float *out, float *lse, char *workspace, const DecodeSplit &split,
                  const DecodeWorkspace &ws, void *stream);

}  // namespace tq
