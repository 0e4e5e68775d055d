/*
 * tq.h - TurboQuant KV-cache compression on NVIDIA B200 (sm_100a): C ABI.
 *
 * The method (ai-accelerate.xyz TurboQuant explainer, "TurboQuantの仕組み";
 * qxai.app, "Tether QVACのTurboQuant実装"): every K/V head vector is split
 * into its L2 norm and its direction; the direction is rotated by a seeded
 * random orthogonal matrix Pi, each rotated coordinate is quantized on its own
 * with the Lloyd-Max quantizer of its (near-Gaussian) law, and no per-block
 * scale or centroid is stored ("ステップ1: PolarQuant").  An optional second
 * stage keeps one sign bit per coordinate of S r, the Gaussian projection of
 * the stage-1 residual r, plus ||r||, which makes inner products unbiased
 * ("ステップ2: QJL").  Decode attention reads the packed cache directly.
 *
 * Conventions for every call below
 *  - All pointers named "device" are CUDA device pointers on the current
 *    device; "host" pointers are ordinary host memory.  The caller owns every
 *    buffer; the library never frees, keeps or allocates caller memory.
 *  - A context belongs to the device that was current when it was created.
 *    The compute calls (tq_quantize, tq_decode_attention,
 *    tq_decode_attention_noalloc, tq_prefill_attention, tq_weight_quantize,
 *    tq_weight_gemm) check that this device is current and return
 *    TQ_ERR_INVALID, launching nothing, when it is not.  One process may hold
 *    contexts on several devices.
 *  - The compute calls are asynchronous on the given stream (a cudaStream_t
 *    passed as void*; NULL = legacy default stream), allocate nothing, never
 *    synchronise and never read device data on the host.
 *  - On any non-TQ_OK status nothing has been launched (argument errors) or a
 *    CUDA call failed (TQ_ERR_CUDA); tq_last_error() returns a thread-local
 *    message.  Device-side range errors (a seq_idx, pos or seq_len outside the
 *    cache) skip the offending token or sequence and set a sticky flag that
 *    tq_check_device_errors() reports.
 *  - Head dimension d in {64, 128, 256} for the cache (tq_quantize,
 *    tq_decode_attention); prefill attention and weight rows take d = 128
 *    only.  bits_k, bits_v in {2, 3, 4}.  qjl in {0, 1} (applies to K only).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_ctx tq_ctx; /* opaque: Pi, Pi^T, S, codebooks on one device */

typedef enum tq_status {
  TQ_OK = 0,
  TQ_ERR_INVALID = 1,     /* bad argument; nothing launched */
  TQ_ERR_CUDA = 2,        /* a CUDA runtime call failed */
  TQ_ERR_NOMEM = 3,       /* device allocation in tq_create failed */
  TQ_ERR_UNSUPPORTED = 4, /* valid but not implemented (e.g. d = 96) */
  TQ_ERR_DEVICE = 5       /* a kernel recorded a device-side range error */
} tq_status;

typedef enum tq_dtype { TQ_BF16 = 0, TQ_F32 = 1 } tq_dtype;

/*
 * Coordinate law the Lloyd-Max codebook is optimised for.  After the random
 * rotation every coordinate of a unit direction follows one fixed law, which
 * the method describes as close to Gaussian ("ステップ1: PolarQuant",
 * ai-accelerate.xyz TurboQuant explainer).
 *  TQ_LAW_GAUSSIAN  N(0, 1/d): Lloyd-Max centroids of N(0,1) / sqrt(d) (the
 *                   default, and what tq_create uses).
 *  TQ_LAW_SPHERE    the exact law of one coordinate of a uniform unit vector
 *                   in R^d, density (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on
 *                   (-1, 1), of which N(0, 1/d) is the large-d limit.
 * Either way the centroids are rounded to fp16 and the thresholds are the
 * exact midpoints; the kernels, layouts and the decode are the same.
 */
typedef enum tq_law { TQ_LAW_GAUSSIAN = 0, TQ_LAW_SPHERE = 1 } tq_law;

/* Plane indices of tq_layout(). */
enum {
  TQ_PLANE_CODES_K = 0,
  TQ_PLANE_NORM_K = 1,
  TQ_PLANE_QJL_BITS = 2,
  TQ_PLANE_QJL_NORM = 3,
  TQ_PLANE_CODES_V = 4,
  TQ_PLANE_NORM_V = 5
};

/*
 * The packed cache of one attention layer: six planes of caller-owned device
 * memory, each laid out [n_seqs][n_kv_heads][capacity][bytes_per_token_head]
 * (so the tokens of one (sequence, KV head) are contiguous).
 *  codes_k  d*bits_k/8 bytes per vector.  2 and 4 bits: LSB-first stream,
 *           code i at bits [i*b, i*b+b).  3 bits: groups of 32 coordinates in
 *           three little-endian 32-bit words w0..w2; local coordinate l < 24
 *           occupies bits [4(l%8), 4(l%8)+3) of word l/8, and bit k of the
 *           code of l >= 24 is bit 4(l-24)+3 of word k.  A code is the index
 *           of its centroid in ascending order.
 *  norm_k   ||k|| as IEEE fp16 bits (round to nearest even, saturating).
 *  qjl_bits d/8 bytes, bit m = [(S r)_m >= 0], LSB first (NULL if qjl == 0).
 *  qjl_norm ||r|| as fp16 bits (NULL if qjl == 0).
 *  codes_v, norm_v as codes_k, norm_k with bits_v.
 * capacity must be a positive multiple of 64; every plane pointer 16-byte
 * aligned.
 *
 * Paged layout (block_table != NULL), as serving engines keep their KV
 * caches: the planes hold n_blocks physical blocks of block_size tokens,
 * laid out [n_blocks][n_kv_heads][block_size][bytes_per_token_head], and
 * block_table (device int32, [n_seqs][capacity / block_size], 4-byte
 * aligned) maps logical block j of sequence s to its physical block.
 * Position p of sequence s is token p % block_size of physical block
 * block_table[s][p / block_size].  capacity (the logical length per
 * sequence) must be a multiple of block_size, and block_size a positive
 * multiple of 64.  Only the entries a call needs are read: quantize reads
 * the entry of each position it writes, decode the entries of the blocks
 * that hold positions below each sequence's length.  Entries past a
 * sequence's length may therefore hold anything (an engine's -1 for an
 * unassigned block, say).  An entry that is read and lies outside
 * [0, n_blocks) is a device-side range error: quantize skips the token,
 * decode reads block 0 instead, and both set the token-range flag that
 * tq_check_device_errors reports.  With block_table == NULL, block_size and
 * n_blocks are ignored.
 */
typedef struct tq_cache {
  uint8_t *codes_k;
  uint16_t *norm_k;
  uint8_t *qjl_bits;
  uint16_t *qjl_norm;
  uint8_t *codes_v;
  uint16_t *norm_v;
  int32_t capacity;
  int32_t n_seqs;
  int32_t n_kv_heads;
  const int32_t *block_table;
  int32_t block_size;
  int32_t n_blocks;
} tq_cache;

/*
 * Create a context on the current CUDA device.  Pi is the QR factor of a
 * d x d Gaussian (SplitMix64 counters 1.. from `seed`, Box-Muller), columns
 * signed so that R has a positive diagonal, rounded to bf16 (the random
 * orthogonal matrix of section "ステップ1: PolarQuant").  The codebook of b
 * bits is the Lloyd-Max quantizer of N(0,1) scaled by 1/sqrt(d) (the same
 * section's optimal scalar quantizer, for the N(0,1/d) reading of its
 * near-Gaussian coordinate law), its centroids rounded to fp16 and the exact
 * midpoints (fp32) as thresholds.  With qjl, S is a second d x d Gaussian
 * from counters 2^32+1.. (fp32).  Allocates and uploads the parameters
 * (synchronous); the only call that allocates device memory.
 * Errors: TQ_ERR_INVALID (null out, bits outside {2,3,4}, qjl outside {0,1}),
 * TQ_ERR_UNSUPPORTED (d outside {64, 128, 256}, or a codebook whose
 * thresholds the quantize kernels could not select exactly in fp32; the host
 * checks this, and it holds for every codebook of those d), TQ_ERR_NOMEM,
 * TQ_ERR_CUDA.
 */
tq_status tq_create(tq_ctx **out, int32_t d, int32_t bits_k, int32_t bits_v,
                    int32_t qjl, uint64_t seed);

/*
 * tq_create with the codebook's coordinate law chosen (tq_law); law =
 * TQ_LAW_GAUSSIAN is tq_create.  Errors: those of tq_create, and
 * TQ_ERR_INVALID for a law outside tq_law.
 */
tq_status tq_create_ex(tq_ctx **out, int32_t d, int32_t bits_k, int32_t bits_v,
                       int32_t qjl, uint64_t seed, int32_t law);

/* Free the context's device memory.  NULL is a no-op. */
void tq_destroy(tq_ctx *ctx);

/* Bytes per (token, KV head) of each plane, indexed by TQ_PLANE_* (0 for the
 * QJL planes when qjl == 0).  Host array of 6. */
tq_status tq_layout(const tq_ctx *ctx, size_t bytes_per_token_head[6]);

/*
 * Copy the method's parameters to host memory (any pointer may be NULL):
 * pi [d*d] row-major (z = Pi x), values exactly representable in bf16;
 * s [d*d] row-major (NULL result if qjl == 0); centroids_* [2^bits]
 * ascending; thresholds_* [2^bits - 1].
 */
tq_status tq_get_params(const tq_ctx *ctx, float *pi, float *s,
                        float *centroids_k, float *thresholds_k,
                        float *centroids_v, float *thresholds_v);

/*
 * The same parameters computed on the host only (no CUDA call): what
 * tq_create(d, bits_k, bits_v, qjl, seed) would upload.  Same output layout
 * as tq_get_params; s is left untouched when qjl == 0.  Errors: those of
 * tq_create's host checks (TQ_ERR_INVALID, TQ_ERR_UNSUPPORTED).
 */
tq_status tq_host_params(int32_t d, int32_t bits_k, int32_t bits_v,
                         int32_t qjl, uint64_t seed, float *pi, float *s,
                         float *centroids_k, float *thresholds_k,
                         float *centroids_v, float *thresholds_v);

/* tq_host_params for tq_create_ex(d, bits_k, bits_v, qjl, seed, law). */
tq_status tq_host_params_ex(int32_t d, int32_t bits_k, int32_t bits_v,
                            int32_t qjl, uint64_t seed, int32_t law,
                            float *pi, float *s,
                            float *centroids_k, float *thresholds_k,
                            float *centroids_v, float *thresholds_v);

/*
 * Quantize-on-append ("ステップ1" and, with qjl, "ステップ2"): for each of
 * n_tok tokens t and KV head h, k[t][h][:] and v[t][h][:] (device, bf16,
 * contiguous [n_tok][n_kv_heads][d]) are normed, rotated by Pi, quantized,
 * packed and written at position pos[t] of sequence seq_idx[t] (device int32
 * arrays of n_tok).  Rows whose (seq_idx, pos) falls outside the cache, or
 * whose block-table entry is out of range in a paged cache, are skipped and
 * flagged.  Tokens may arrive in any order; two tokens with the
 * same (seq_idx, pos) race.  n_tok == 0 is a no-op.
 */
tq_status tq_quantize(tq_ctx *ctx, const tq_cache *cache, const void *k,
                      const void *v, const int32_t *seq_idx,
                      const int32_t *pos, int32_t n_tok, void *stream);

/* Device workspace (bytes) that tq_decode_attention needs for this shape. */
size_t tq_workspace_bytes(const tq_ctx *ctx, int32_t n_seqs,
                          int32_t n_q_heads, int32_t max_seq_len);

/*
 * Decode attention over the packed cache: for every sequence s and query
 * head g (KV head g / (n_q_heads / n_kv_heads)),
 *   q_hat = Pi q, q_tilde = S q_hat,
 *   score_j = scale * ||k_j|| * (q_hat . c_K[code_j]
 *             + [qjl] sqrt(pi/2)/d * ||r_j|| * sum_m q_tilde_m (2 s_jm - 1)),
 *   o = Pi^T sum_j softmax(score)_j ||v_j|| c_V[codeV_j]
 * over the positions [0, seq_lens[s]).  q: device [n_seqs][n_q_heads][d] of
 * q_dtype (TQ_BF16 or TQ_F32).  seq_lens: device int32 [n_seqs], each at most
 * max_seq_len (a host bound used to size the grid; <= capacity).
 * scale <= 0 means 1/sqrt(d).  out: device fp32 [n_seqs][n_q_heads][d].
 * lse: device fp32 [n_seqs][n_q_heads] log-sum-exp of the scores, or NULL.
 * A sequence of length 0 yields out = 0 and lse = -inf.  workspace: device,
 * at least tq_workspace_bytes(ctx, n_seqs, n_q_heads, max_seq_len) bytes,
 * 256-byte aligned; its contents need no initialisation.
 */
tq_status tq_decode_attention(tq_ctx *ctx, const tq_cache *cache,
                              const void *q, int32_t q_dtype,
                              int32_t n_q_heads, const int32_t *seq_lens,
                              int32_t max_seq_len, float scale, float *out,
                              float *lse, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Causal prefill (prompt) attention over the packed cache, the step that
 * qxai.app ("Tether QVACのTurboQuant実装", fifth paragraph) names as where a
 * compressed cache costs the most: the prompt's K and V are first quantized
 * into the cache with tq_quantize, then every prompt token attends over the
 * cached positions up to and including its own, reading the packed codes
 * exactly as tq_decode_attention does (q_hat = Pi q, the same scores,
 * softmax, V accumulation in rotated space, o = Pi^T o_tilde).  The bf16 K/V
 * of the prompt is not read.  The queries of sequence s are rows
 * cu_q[s] .. cu_q[s+1]-1 of q and sit at the last n_s = cu_q[s+1] - cu_q[s]
 * positions of the sequence, seq_lens[s] - n_s .. seq_lens[s] - 1 (a whole
 * prompt when n_s == seq_lens[s], a chunk of one otherwise); the query at
 * position p attends over positions [0, p].
 *  q        device [total][n_q_heads][d] of q_dtype, total = cu_q[n_seqs].
 *  cu_q     device int32 [n_seqs + 1], cu_q[0] = 0, non-decreasing.
 *  seq_lens device int32 [n_seqs], each at most max_seq_len (<= capacity).
 *  max_q    host bound on every n_s (sizes the grid); max_seq_len likewise.
 *  out      device fp32 [total][n_q_heads][d]; lse device fp32
 *           [total][n_q_heads] or NULL.
 * No workspace.  A sequence whose n_s or seq_lens is out of range gets no
 * output and sets the seq_len flag of tq_check_device_errors.  Query heads
 * per KV head at most 16.
 */
tq_status tq_prefill_attention(tq_ctx *ctx, const tq_cache *cache,
                               const void *q, int32_t q_dtype,
                               int32_t n_q_heads, const int32_t *cu_q,
                               const int32_t *seq_lens, int32_t max_q,
                               int32_t max_seq_len, float scale, float *out,
                               float *lse, void *stream);

/*
 * Weight quantization with the same method (ai-accelerate.xyz TurboQuant
 * explainer, "重みの量子化にも応用できる": the algorithm applied to the
 * weights of a linear layer).  Every row of W (device, bf16, row-major
 * [n_out][n_in]) is cut into n_in / d blocks of d coordinates, and every
 * block is quantized as one vector with the context's K codebook (its norm,
 * the rotation by Pi, bits_k-bit codes; no QJL, whatever the context's qjl).
 * The packed rows go to a tq_cache `w` of one sequence whose KV heads are the
 * blocks and whose positions are the rows: n_seqs = 1, n_kv_heads = n_in / d,
 * capacity >= n_out (a multiple of 64), block_table NULL; only codes_k and
 * norm_k are used (the other planes may be NULL).  Block b of row i is at
 * position i of KV head b, in the cache's K layout.  d must be 128 and n_in
 * a positive multiple of it.  Asynchronous on `stream`, allocates nothing.
 */
tq_status tq_weight_quantize(tq_ctx *ctx, const tq_cache *w, const void *w_rows,
                             int32_t n_out, int32_t n_in, void *stream);

/* Device workspace (bytes) that tq_weight_gemm needs for n_tok rows of x. */
size_t tq_weight_workspace_bytes(const tq_ctx *ctx, int32_t n_tok, int32_t n_in);

/*
 * y = x W~^T over weights packed by tq_weight_quantize, W~ being the rows as
 * the method reconstructs them (each block n_b Pi^T c[codes_b]).  The product
 * runs in rotated space and never rebuilds W~:
 *   y[t][i] = sum_b n_ib (Pi x[t][block b]) . c[code_ib].
 *  x         device [n_tok][n_in] of x_dtype (TQ_BF16 or TQ_F32).
 *  y         device fp32 [n_tok][n_out] (overwritten).
 *  workspace device, at least tq_weight_workspace_bytes(ctx, n_tok, n_in)
 *            bytes, 256-byte aligned; contents need no initialisation.
 * n_tok at most 65520.  Sums over blocks are fp32 and combined with atomic
 * adds, so the last bits of y may differ between runs.
 */
tq_status tq_weight_gemm(tq_ctx *ctx, const tq_cache *w, int32_t n_out,
                         int32_t n_in, const void *x, int32_t x_dtype,
                         int32_t n_tok, float *y, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Allocation-free decode attention (no counterpart in the method's sources;
 * it is a deployment variant of tq_decode_attention).  For callers that cannot
 * allocate device memory while they decode: code inside CUDA graph stream
 * capture, engines restricted to their own memory pool, latency-critical
 * loops that cannot absorb cudaMalloc's implicit synchronisation.  Same
 * arguments and results as tq_decode_attention, minus the workspace: the
 * workspace is a static device array of TQ_NOALLOC_SCRATCH_BYTES built into
 * the library (held by every GPU that loads it until exit).  Calls that need
 * more than that (see tq_workspace_bytes) fail with TQ_ERR_INVALID and launch
 * nothing.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the array, so calls whose kernels overlap on the GPU
 * (other streams, other threads) race; it allocates nothing itself.
 */
#define TQ_NOALLOC_SCRATCH_BYTES (8 * 1024 * 1024)
tq_status tq_decode_attention_noalloc(tq_ctx *ctx, const tq_cache *cache,
                                      const void *q, int32_t q_dtype,
                                      int32_t n_q_heads,
                                      const int32_t *seq_lens,
                                      int32_t max_seq_len, float scale,
                                      float *out, float *lse, void *stream);

/*
 * Synchronise `stream`, then report and clear the context's sticky
 * device-side error flags: TQ_OK, or TQ_ERR_DEVICE with a message naming the
 * flags (bit 0: a token outside the cache in tq_quantize, or a paged
 * cache's block-table entry outside [0, n_blocks) in either call; bit 1:
 * seq_len outside [0, max_seq_len] in tq_decode_attention; bit 2: a bounded
 * wait in a kernel expired).
 */
tq_status tq_check_device_errors(tq_ctx *ctx, void *stream);

/* Thread-local message describing the last non-TQ_OK status ("" if none). */
const char *tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
