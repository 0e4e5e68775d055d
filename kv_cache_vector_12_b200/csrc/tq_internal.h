// Internal declarations shared by the host code, the API layer and the
// kernels of the TurboQuant library.  Nothing here is part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

constexpr int kHeadDim = 128;
constexpr int kMaxLevels = 16;  // 2^4 centroids at most

// Sticky device-side error flags (tq_check_device_errors).
constexpr unsigned kErrTokenRange = 1u;
constexpr unsigned kErrSeqLen = 2u;
constexpr unsigned kErrWaitExpired = 4u;

// --- host parameter construction (tq_host.cpp) ---
void gaussian_stream(uint64_t seed, uint32_t stream, size_t count, double *out);
uint16_t double_to_bf16_bits(double x);
float bf16_bits_to_float(uint16_t h);
void rotation_bf16(int d, uint64_t seed, uint16_t *pi_bits);
void qjl_matrix(int d, uint64_t seed, float *s);
void lloyd_max_gaussian(int bits, double *c);
void codebook(int bits, int d, float *centroids, float *thresholds);

// Bytes of one packed vector of codes.
inline int code_bytes(int bits) { return kHeadDim * bits / 8; }

// Device-resident parameters of one context (all pointers device memory).
struct DeviceParams {
  const uint16_t *pi;     // Pi  [d][d] bf16 bits, row-major (z = Pi x)
  const uint16_t *pit;    // Pi^T [d][d] bf16 bits
  const float *s;         // S   [d][d] fp32 (qjl only)
  const float *st;        // S^T [d][d] fp32 (qjl only)
  const float *cb;        // [4][16]: centroids_k, thresholds_k, centroids_v, thresholds_v
  unsigned *err;          // sticky error flags
  int bits_k, bits_v, qjl;
};

// Split of the sequence axis used by decode attention.
struct DecodeSplit {
  int chunk;     // tokens per split (multiple of 64)
  int n_splits;  // ceil(max_seq_len / chunk), at least 1
};
DecodeSplit decode_split(int n_seqs, int n_kv_heads, int max_seq_len);

// Workspace layout of decode attention (byte offsets, 256-aligned).
struct DecodeWorkspace {
  size_t q_hat, q_tilde, partials, total;
};
DecodeWorkspace decode_workspace(int n_seqs, int n_q_heads, int qjl, DecodeSplit split);

// --- launches (tq_kernels.cu); return cudaGetLastError() as int ---
int launch_quantize(const DeviceParams &p, const tq_cache &c, const void *k, const void *v,
                    const int32_t *seq_idx, const int32_t *pos, int n_tok, void *stream);
int launch_decode(const DeviceParams &p, const tq_cache &c, const void *q, int q_dtype,
                  int n_q_heads, const int32_t *seq_lens, int max_seq_len, float scale,
                  float *out, float *lse, char *workspace, const DecodeSplit &split,
                  const DecodeWorkspace &ws, void *stream);

}  // namespace tq
