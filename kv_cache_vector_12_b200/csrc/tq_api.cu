// C ABI of the TurboQuant library: context lifetime, argument validation and
// the dispatch of the compute calls to their kernels.  Validation happens
// entirely on the host, before anything is launched; device-side range
// problems are recorded in a sticky flag word instead of faulting.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "tq_internal.h"

struct tq_ctx {
  int device;
  int d, bits_k, bits_v, qjl, law;
  uint64_t seed;
  std::vector<uint16_t> pi_bits;  // host copies of the uploaded parameters
  std::vector<float> s, ck, tk, cv, tv;
  void *dev_block;                // one allocation holding every device parameter
  tq::DeviceParams dp;
};

namespace {

// fp16 bit pattern of a float that is exactly representable in fp16's normal
// range (every centroid is).
uint16_t exact_half_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) == 0) return (uint16_t)(u >> 16);
  const uint32_t sign = (u >> 16) & 0x8000u;
  const int exp = (int)((u >> 23) & 0xff) - 127 + 15;
  return (uint16_t)(sign | ((uint32_t)exp << 10) | ((u & 0x7fffffu) >> 13));
}

// The largest shift k <= 17 with every K centroid c 2^k an integer in
// [-32767, 32767] (exact 16-bit fixed point), or -1 if none from 17 down to 8.
int k_fixed_shift(const float *ck, int bits_k) {
  for (int k = 17; k >= 8; --k) {
    bool ok = true;
    for (int e = 0; e < (1 << bits_k) && ok; ++e) {
      const double scaled = std::ldexp((double)ck[e], k);
      ok = std::nearbyint(scaled) == scaled && std::fabs(scaled) <= 32767.0;
    }
    if (ok) return k;
  }
  return -1;
}

// Byte tables of the decode kernel's lookups (see tq_internal.h).
bool build_luts(const float *ck, int bits_k, int k_shift, const float *cv, int bits_v, tq::Lut &lk, tq::Lut &lv) {
  std::memset(&lk, 0, sizeof lk);
  std::memset(&lv, 0, sizeof lv);
  if (k_shift < 0) return false;
  for (int e = 0; e < (1 << bits_k); ++e) {
    const double scaled = std::ldexp((double)ck[e], k_shift);
    const long v = std::lrint(scaled);
    if ((double)v != scaled || v > 32767 || v < -32767) return false;  // not exact 16-bit fixed point
    lk.lo[e / 4] |= (uint32_t)(v & 0xff) << (8 * (e % 4));
    lk.hi[e / 4] |= (uint32_t)((v >> 8) & 0xff) << (8 * (e % 4));
  }
  for (int e = 0; e < (1 << bits_v); ++e) {
    const uint16_t hb = exact_half_bits(cv[e]);
    lv.lo[e / 4] |= (uint32_t)(hb & 0xff) << (8 * (e % 4));
    lv.hi[e / 4] |= (uint32_t)(hb >> 8) << (8 * (e % 4));
  }
  return true;
}

bool is_permutation(const uint8_t *p, int d) {
  bool seen[256] = {};
  for (int i = 0; i < d; ++i) {
    if (p[i] >= d || seen[p[i]]) return false;
    seen[p[i]] = true;
  }
  return true;
}

}  // namespace

namespace {

thread_local char g_last_error[512] = "";

tq_status fail(tq_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

tq_status cuda_fail(cudaError_t e, const char *what) {
  return fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

tq_status check_params(int d, int bits_k, int bits_v, int qjl, int law) {
  if (law != TQ_LAW_GAUSSIAN && law != TQ_LAW_SPHERE)
    return fail(TQ_ERR_INVALID, "law=%d must be TQ_LAW_GAUSSIAN (0) or TQ_LAW_SPHERE (1)", law);
  if (bits_k < 2 || bits_k > 4 || bits_v < 2 || bits_v > 4)
    return fail(TQ_ERR_INVALID, "bits_k=%d bits_v=%d: each must be 2, 3 or 4", bits_k, bits_v);
  if (qjl != 0 && qjl != 1) return fail(TQ_ERR_INVALID, "qjl=%d must be 0 or 1", qjl);
  if (!tq::supported_head_dim(d)) return fail(TQ_ERR_UNSUPPORTED, "d=%d: the head dimension must be 64, 128 or 256", d);
  return TQ_OK;
}

tq_status check_cache(const tq_ctx *ctx, const tq_cache *c) {
  if (!c) return fail(TQ_ERR_INVALID, "cache is NULL");
  if (c->capacity <= 0 || c->capacity % 64 != 0)
    return fail(TQ_ERR_INVALID, "capacity=%d must be a positive multiple of 64", c->capacity);
  if (c->n_seqs <= 0 || c->n_kv_heads <= 0)
    return fail(TQ_ERR_INVALID, "n_seqs=%d n_kv_heads=%d must be positive", c->n_seqs, c->n_kv_heads);
  const void *planes[6] = {c->codes_k, c->norm_k, c->qjl_bits, c->qjl_norm, c->codes_v, c->norm_v};
  for (int i = 0; i < 6; ++i) {
    const bool needed = (i != 2 && i != 3) || ctx->qjl;
    if (needed && !planes[i]) return fail(TQ_ERR_INVALID, "cache plane %d is NULL", i);
    if (planes[i] && !aligned16(planes[i]))
      return fail(TQ_ERR_INVALID, "cache plane %d is not 16-byte aligned", i);
  }
  if (c->block_table) {  // paged layout
    if (((uintptr_t)c->block_table & 3u) != 0) return fail(TQ_ERR_INVALID, "block_table must be 4-byte aligned");
    if (c->block_size <= 0 || c->block_size % 64 != 0)
      return fail(TQ_ERR_INVALID, "block_size=%d must be a positive multiple of 64", c->block_size);
    if (c->capacity % c->block_size != 0)
      return fail(TQ_ERR_INVALID, "capacity=%d must be a multiple of block_size=%d", c->capacity, c->block_size);
    if (c->n_blocks <= 0) return fail(TQ_ERR_INVALID, "n_blocks=%d must be positive", c->n_blocks);
  }
  return TQ_OK;
}

}  // namespace

namespace tq {

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  return dev;
}

tq_status check_context_device(const tq_ctx *ctx) {
  int cur = -1;
  const cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != ctx->device)
    return fail(TQ_ERR_INVALID, "the current CUDA device is %d but the context was created on device %d", cur,
                ctx->device);
  return TQ_OK;
}

// Cached once per device (atomically: calls may come from several threads).
static int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Splits of the sequence axis.  Start from one wave of resident CTAs (SMs x
// CTAs per SM) spread over the (sequence, KV head) units; take at least
// min(8, four waves / units) splits per unit, so that ragged batches balance;
// when the units hold fewer than four slots each (batches of many sequences,
// whose lengths the host does not see), at least min(12, six waves / units)
// (on the 32-sequence serving batch 11 splits decode 4.5 % faster than 7);
// and at least 256 tokens per split.
DecodeSplit decode_split(int n_seqs, int n_kv_heads, int max_seq_len, int ctas_per_sm) {
  if (ctas_per_sm > 4) ctas_per_sm = 4;
  if (ctas_per_sm < 1) ctas_per_sm = 1;
  const long units = (long)n_seqs * n_kv_heads;
  const long slots = (long)sm_count() * ctas_per_sm;
  long n = slots / units;
  const long per_unit = n;
  const long balance = (4 * slots + units - 1) / units;
  if (n < (balance < 8 ? balance : 8)) n = balance < 8 ? balance : 8;
  if (per_unit < 4) {
    const long ragged = (6 * slots + units - 1) / units;
    if (n < (ragged < 12 ? ragged : 12)) n = ragged < 12 ? ragged : 12;
  }
  if (n < 1) n = 1;
  long chunk = ((long)max_seq_len + n - 1) / n;
  if (chunk < 256) chunk = 256;
  chunk = (chunk + 63) / 64 * 64;
  DecodeSplit sp;
  sp.chunk = (int)chunk;
  sp.n_splits = max_seq_len > 0 ? (int)(((long)max_seq_len + chunk - 1) / chunk) : 1;
  sp.long_splits = false;
  return sp;
}

// The attention kernel has two register budgets.  With 128 registers (3 CTAs
// per SM) twelve consumer warps per SM hide more latency; with 168 (2 CTAs per
// SM, where the code needs more than 128) each CTA is longer and fewer CTAs
// pay the per-CTA prologue.  Measured on the 3/3-bit kernel, the 3-CTA budget
// wins when the split grid fills at least two waves (a batch of many
// sequences) or a split streams at least kLongSplitTokens tokens; the 2-CTA
// budget wins for one wave of short splits (one or a few sequences).
constexpr int kLongSplitTokens = 8192;

// The split is planned for the 3-CTA budget first; a call that meets neither
// condition runs the 2-CTA budget instead, re-split for that occupancy.
DecodeSplit plan_decode(int d, int bits_k, int bits_v, int qjl, int group, int n_seqs, int n_kv_heads,
                        int max_seq_len, bool paged) {
  if (paged) {  // the paged build has one budget
    DecodeSplit sp = decode_split(n_seqs, n_kv_heads, max_seq_len,
                                  decode_ctas_per_sm(d, bits_k, bits_v, qjl, group, true, true));
    sp.long_splits = true;
    return sp;
  }
  const int ctas = decode_ctas_per_sm(d, bits_k, bits_v, qjl, group, true, false);
  DecodeSplit sp = decode_split(n_seqs, n_kv_heads, max_seq_len, ctas);
  const long grid = (long)sp.n_splits * n_seqs * n_kv_heads;
  if (grid >= 2L * sm_count() * ctas || sp.chunk >= kLongSplitTokens) {
    sp.long_splits = true;
    return sp;
  }
  return decode_split(n_seqs, n_kv_heads, max_seq_len,
                      decode_ctas_per_sm(d, bits_k, bits_v, qjl, group, false, false));
}

tq_status report_error(tq_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

void mma_b_fragments(const uint16_t *m_bits, int d, uint32_t *out) {
  const int chunks = d / 32;
  for (int nt = 0; nt < d / 8; ++nt)
    for (int j = 0; j < chunks; ++j)
      for (int lane = 0; lane < 32; ++lane)
        for (int e = 0; e < 4; ++e) {
          const int ks = (4 * j + e) / 2, b = (4 * j + e) % 2;
          const uint16_t *src = m_bits + (size_t)(8 * nt + lane / 4) * d + 16 * ks + 8 * b + 2 * (lane % 4);
          out[((nt * chunks + j) * 32 + lane) * 4 + e] = (uint32_t)src[0] | ((uint32_t)src[1] << 16);
        }
}

DecodeWorkspace decode_workspace(int n_seqs, int n_q_heads, DecodeSplit split, int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t rows = (size_t)n_seqs * n_q_heads;
  DecodeWorkspace w;
  w.partials = 0;
  w.total = up(rows * (size_t)split.n_splits * (size_t)(d + 4) * sizeof(float));
  return w;
}

}  // namespace tq

extern "C" {

const char *tq_last_error(void) { return g_last_error; }

tq_status tq_host_params(int32_t d, int32_t bits_k, int32_t bits_v, int32_t qjl, uint64_t seed,
                         float *pi, float *s, float *centroids_k, float *thresholds_k,
                         float *centroids_v, float *thresholds_v) {
  return tq_host_params_ex(d, bits_k, bits_v, qjl, seed, TQ_LAW_GAUSSIAN, pi, s, centroids_k, thresholds_k,
                           centroids_v, thresholds_v);
}

tq_status tq_host_params_ex(int32_t d, int32_t bits_k, int32_t bits_v, int32_t qjl, uint64_t seed, int32_t law,
                            float *pi, float *s, float *centroids_k, float *thresholds_k,
                            float *centroids_v, float *thresholds_v) {
  tq_status st = check_params(d, bits_k, bits_v, qjl, law);
  if (st != TQ_OK) return st;
  if (pi) {
    std::vector<uint16_t> bits((size_t)d * d);
    tq::rotation_bf16(d, seed, bits.data());
    for (size_t i = 0; i < bits.size(); ++i) pi[i] = tq::bf16_bits_to_float(bits[i]);
  }
  if (s && qjl) tq::qjl_matrix(d, seed, s);
  float c[tq::kMaxLevels], t[tq::kMaxLevels];
  for (const int b : {bits_k, bits_v}) {
    tq::codebook(b, d, law, c, t);
    if (d == tq::kHeadDim && !tq::threshold_search_exact(b, t))
      return fail(TQ_ERR_UNSUPPORTED, "%d-bit thresholds: the quantize search is not exact in fp32", b);
  }
  if (centroids_k || thresholds_k) {
    tq::codebook(bits_k, d, law, c, t);
    if (centroids_k) std::memcpy(centroids_k, c, sizeof(float) << bits_k);
    if (thresholds_k) std::memcpy(thresholds_k, t, sizeof(float) * ((1 << bits_k) - 1));
  }
  if (centroids_v || thresholds_v) {
    tq::codebook(bits_v, d, law, c, t);
    if (centroids_v) std::memcpy(centroids_v, c, sizeof(float) << bits_v);
    if (thresholds_v) std::memcpy(thresholds_v, t, sizeof(float) * ((1 << bits_v) - 1));
  }
  return TQ_OK;
}

tq_status tq_create(tq_ctx **out, int32_t d, int32_t bits_k, int32_t bits_v, int32_t qjl,
                    uint64_t seed) {
  return tq_create_ex(out, d, bits_k, bits_v, qjl, seed, TQ_LAW_GAUSSIAN);
}

tq_status tq_create_ex(tq_ctx **out, int32_t d, int32_t bits_k, int32_t bits_v, int32_t qjl,
                       uint64_t seed, int32_t law) {
  if (!out) return fail(TQ_ERR_INVALID, "out is NULL");
  *out = nullptr;
  tq_status st = check_params(d, bits_k, bits_v, qjl, law);
  if (st != TQ_OK) return st;

  tq_ctx *ctx = new tq_ctx();
  ctx->d = d;
  ctx->bits_k = bits_k;
  ctx->bits_v = bits_v;
  ctx->qjl = qjl;
  ctx->law = law;
  ctx->seed = seed;
  ctx->dev_block = nullptr;
  ctx->dp.s_shift = 0;
  ctx->pi_bits.resize((size_t)d * d);
  tq::rotation_bf16(d, seed, ctx->pi_bits.data());
  ctx->ck.assign(tq::kMaxLevels, 0.f);
  ctx->tk.assign(tq::kMaxLevels, 0.f);
  ctx->cv.assign(tq::kMaxLevels, 0.f);
  ctx->tv.assign(tq::kMaxLevels, 0.f);
  tq::codebook(bits_k, d, law, ctx->ck.data(), ctx->tk.data());
  tq::codebook(bits_v, d, law, ctx->cv.data(), ctx->tv.data());
  if (d == tq::kHeadDim &&
      (!tq::threshold_search_exact(bits_k, ctx->tk.data()) || !tq::threshold_search_exact(bits_v, ctx->tv.data()))) {
    delete ctx;
    return fail(TQ_ERR_UNSUPPORTED, "thresholds: the quantize search is not exact in fp32");
  }
  if (qjl) {
    ctx->s.resize((size_t)d * d);
    tq::qjl_matrix(d, seed, ctx->s.data());
  }

  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e != cudaSuccess) {
    delete ctx;
    return cuda_fail(e, "cudaGetDevice");
  }
  uint8_t kperm[256], vperm[256], jperm[256];
  tq::kperm_of(bits_k, d, kperm);
  tq::vperm_of(bits_v, d, vperm);
  tq::jperm_of(d, jperm);
  ctx->dp.k_shift = k_fixed_shift(ctx->ck.data(), bits_k);
  if (!is_permutation(kperm, d) || !is_permutation(vperm, d) || !is_permutation(jperm, d) ||
      !build_luts(ctx->ck.data(), bits_k, ctx->dp.k_shift, ctx->cv.data(), bits_v, ctx->dp.lut_k, ctx->dp.lut_v)) {
    delete ctx;
    return fail(TQ_ERR_UNSUPPORTED, "internal: fragment orders or codebook tables could not be built");
  }
  // One block: pi | pik | pivt | pif | pvf | s | sjkf | sf | ssplit | codebooks | kperm | jperm | error word.
  const size_t dd = (size_t)d * d;
  const size_t off_pi = 0, off_pik = off_pi + dd * 2, off_piv = off_pik + dd * 2, off_pif = off_piv + dd * 2;
  const size_t off_pvf = off_pif + dd * 2, off_s = off_pvf + dd * 2;
  const size_t off_sjk = off_s + dd * 4, off_sf = off_sjk + dd * 4, off_ss = off_sf + 2 * dd * 2;
  const size_t off_cb = off_ss + 2 * dd * 2;
  const size_t off_kperm = off_cb + 4 * tq::kMaxLevels * 4, off_jperm = off_kperm + 256;
  const size_t off_err = off_jperm + 256, total = off_err + 256;
  e = cudaMalloc(&ctx->dev_block, total);
  if (e != cudaSuccess) {
    delete ctx;
    return fail(TQ_ERR_NOMEM, "cudaMalloc(%zu): %s", total, cudaGetErrorString(e));
  }
  std::vector<char> h(total, 0);
  std::memcpy(h.data() + off_pi, ctx->pi_bits.data(), dd * 2);
  // Pi with its rows in the K fragment order (q_hat = Pi q then comes out of
  // the decode kernel's MMA in that order), as B fragments: consumer warp w
  // reads n-tiles 4 w .. 4 w + 3.
  {
    std::vector<uint16_t> pik(dd);
    for (int kap = 0; kap < d; ++kap)
      std::memcpy(pik.data() + (size_t)kap * d, ctx->pi_bits.data() + (size_t)kperm[kap] * d, (size_t)d * 2);
    tq::mma_b_fragments(pik.data(), d, (uint32_t *)(h.data() + off_pik));
  }
  tq::mma_b_fragments(ctx->pi_bits.data(), d, (uint32_t *)(h.data() + off_pif));
  if (qjl) {
    std::memcpy(h.data() + off_s, ctx->s.data(), dd * 4);
    // S 2^sigma = hi + lo with two fp16 parts (22 significant bits; only the
    // signs of S r are kept, so the power-of-two scale is free).  sigma puts
    // the largest entry at or below 2^15: hi never overflows, and lo stays in
    // fp16's normal range for every entry above 2^-(sigma - 3).
    double smax = 0.0;
    for (size_t i = 0; i < dd; ++i) smax = std::max(smax, (double)std::fabs(ctx->s[i]));
    const int sigma = smax > 0.0 ? (int)std::floor(std::log2(32768.0 / smax)) : 0;
    ctx->dp.s_shift = sigma;
    std::vector<uint16_t> part(dd);
    std::vector<double> rest(dd);
    for (size_t i = 0; i < dd; ++i) rest[i] = std::ldexp((double)ctx->s[i], sigma);
    for (int k = 0; k < 2; ++k) {
      for (size_t i = 0; i < dd; ++i) {
        part[i] = tq::double_to_half_bits(rest[i]);
        rest[i] -= tq::half_bits_to_double(part[i]);
      }
      tq::mma_b_fragments(part.data(), d, (uint32_t *)(h.data() + off_sf) + (size_t)k * dd / 2);
      std::memcpy(h.data() + off_ss + (size_t)k * dd * 2, part.data(), dd * 2);
    }
    // the same two parts with S's rows in the QJL fragment order and its
    // columns in the K fragment order (S'[i][j] = S[jperm i][kperm j]), as
    // fp16 MMA B fragments: the decode kernel's q_tilde = S' q_hat
    std::vector<uint16_t> perm_part(dd);
    for (size_t i = 0; i < dd; ++i) rest[i] = std::ldexp((double)ctx->s[(size_t)jperm[i / d] * d + kperm[i % d]], sigma);
    for (int k = 0; k < 2; ++k) {
      for (size_t i = 0; i < dd; ++i) {
        perm_part[i] = tq::double_to_half_bits(rest[i]);
        rest[i] -= tq::half_bits_to_double(perm_part[i]);
      }
      tq::mma_b_fragments(perm_part.data(), d, (uint32_t *)(h.data() + off_sjk) + (size_t)k * dd / 2);
    }
  }
  uint16_t *pivt = (uint16_t *)(h.data() + off_piv);
  for (int i = 0; i < d; ++i)
    for (int k = 0; k < d; ++k) pivt[(size_t)i * d + k] = ctx->pi_bits[(size_t)vperm[k] * d + i];
  tq::mma_b_fragments(pivt, d, (uint32_t *)(h.data() + off_pvf));
  std::memcpy(h.data() + off_kperm, kperm, (size_t)d);
  std::memcpy(h.data() + off_jperm, jperm, (size_t)d);
  float *cb = (float *)(h.data() + off_cb);
  std::memcpy(cb + 0 * tq::kMaxLevels, ctx->ck.data(), tq::kMaxLevels * 4);
  std::memcpy(cb + 1 * tq::kMaxLevels, ctx->tk.data(), tq::kMaxLevels * 4);
  std::memcpy(cb + 2 * tq::kMaxLevels, ctx->cv.data(), tq::kMaxLevels * 4);
  std::memcpy(cb + 3 * tq::kMaxLevels, ctx->tv.data(), tq::kMaxLevels * 4);
  e = cudaMemcpy(ctx->dev_block, h.data(), total, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(ctx->dev_block);
    delete ctx;
    return cuda_fail(e, "cudaMemcpy(params)");
  }
  char *base = (char *)ctx->dev_block;
  ctx->dp.pi = (const uint16_t *)(base + off_pi);
  ctx->dp.pikf = (const uint32_t *)(base + off_pik);
  ctx->dp.s = (const float *)(base + off_s);
  ctx->dp.sjkf = (const uint32_t *)(base + off_sjk);
  ctx->dp.pif = (const uint32_t *)(base + off_pif);
  ctx->dp.sf = (const uint32_t *)(base + off_sf);
  ctx->dp.ssplit = (const uint16_t *)(base + off_ss);
  ctx->dp.cb = (const float *)(base + off_cb);
  ctx->dp.err = (unsigned *)(base + off_err);
  ctx->dp.pivt = (const uint16_t *)(base + off_piv);
  ctx->dp.pvf = (const uint32_t *)(base + off_pvf);
  ctx->dp.kperm = (const uint8_t *)(base + off_kperm);
  ctx->dp.jperm = (const uint8_t *)(base + off_jperm);
  ctx->dp.d = d;
  ctx->dp.bits_k = bits_k;
  ctx->dp.bits_v = bits_v;
  ctx->dp.qjl = qjl;
  // resolve the decode kernels' occupancy now, outside any stream capture
  for (const bool long_splits : {false, true})
    for (const bool paged : {false, true}) {
      tq::decode_ctas_per_sm(d, bits_k, bits_v, qjl, 8, long_splits, paged);
      tq::decode_ctas_per_sm(d, bits_k, bits_v, qjl, 16, long_splits, paged);
    }
  *out = ctx;
  return TQ_OK;
}

void tq_destroy(tq_ctx *ctx) {
  if (!ctx) return;
  if (ctx->dev_block) cudaFree(ctx->dev_block);
  delete ctx;
}

tq_status tq_layout(const tq_ctx *ctx, size_t b[6]) {
  if (!ctx || !b) return fail(TQ_ERR_INVALID, "ctx or output is NULL");
  b[TQ_PLANE_CODES_K] = (size_t)tq::code_bytes(ctx->bits_k, ctx->d);
  b[TQ_PLANE_NORM_K] = 2;
  b[TQ_PLANE_QJL_BITS] = ctx->qjl ? (size_t)ctx->d / 8 : 0;
  b[TQ_PLANE_QJL_NORM] = ctx->qjl ? 2 : 0;
  b[TQ_PLANE_CODES_V] = (size_t)tq::code_bytes(ctx->bits_v, ctx->d);
  b[TQ_PLANE_NORM_V] = 2;
  return TQ_OK;
}

tq_status tq_get_params(const tq_ctx *ctx, float *pi, float *s, float *centroids_k,
                        float *thresholds_k, float *centroids_v, float *thresholds_v) {
  if (!ctx) return fail(TQ_ERR_INVALID, "ctx is NULL");
  const size_t dd = (size_t)ctx->d * ctx->d;
  if (pi)
    for (size_t i = 0; i < dd; ++i) pi[i] = tq::bf16_bits_to_float(ctx->pi_bits[i]);
  if (s && ctx->qjl) std::memcpy(s, ctx->s.data(), dd * 4);
  if (centroids_k) std::memcpy(centroids_k, ctx->ck.data(), sizeof(float) << ctx->bits_k);
  if (thresholds_k) std::memcpy(thresholds_k, ctx->tk.data(), sizeof(float) * ((1 << ctx->bits_k) - 1));
  if (centroids_v) std::memcpy(centroids_v, ctx->cv.data(), sizeof(float) << ctx->bits_v);
  if (thresholds_v) std::memcpy(thresholds_v, ctx->tv.data(), sizeof(float) * ((1 << ctx->bits_v) - 1));
  return TQ_OK;
}

tq_status tq_quantize(tq_ctx *ctx, const tq_cache *cache, const void *k, const void *v,
                      const int32_t *seq_idx, const int32_t *pos, int32_t n_tok, void *stream) {
  if (!ctx) return fail(TQ_ERR_INVALID, "ctx is NULL");
  tq_status st = tq::check_context_device(ctx);
  if (st != TQ_OK) return st;
  st = check_cache(ctx, cache);
  if (st != TQ_OK) return st;
  if (n_tok < 0) return fail(TQ_ERR_INVALID, "n_tok=%d is negative", n_tok);
  if (n_tok == 0) return TQ_OK;
  if (!k || !v || !seq_idx || !pos) return fail(TQ_ERR_INVALID, "k, v, seq_idx and pos must be non-NULL");
  if (!aligned16(k) || !aligned16(v)) return fail(TQ_ERR_INVALID, "k and v must be 16-byte aligned");
  if (((uintptr_t)seq_idx & 3u) || ((uintptr_t)pos & 3u))
    return fail(TQ_ERR_INVALID, "seq_idx and pos must be 4-byte aligned");
  const int e = tq::launch_quantize(ctx->dp, *cache, k, v, seq_idx, pos, n_tok, stream);
  if (e != 0) return cuda_fail((cudaError_t)e, "tq_quantize launch");
  return TQ_OK;
}

size_t tq_workspace_bytes(const tq_ctx *ctx, int32_t n_seqs, int32_t n_q_heads, int32_t max_seq_len) {
  if (!ctx || n_seqs <= 0 || n_q_heads <= 0 || max_seq_len < 0) return 0;
  // The split count falls as the (sequence, KV head) units grow and rises with
  // CTAs per SM; one KV head and the largest occupancy bound it from above.
  const tq::DecodeSplit sp = tq::decode_split(n_seqs, 1, max_seq_len, 4);
  return tq::decode_workspace(n_seqs, n_q_heads, sp, ctx->d).total;
}

tq_status tq_decode_attention(tq_ctx *ctx, const tq_cache *cache, const void *q, int32_t q_dtype,
                              int32_t n_q_heads, const int32_t *seq_lens, int32_t max_seq_len,
                              float scale, float *out, float *lse, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (!ctx) return fail(TQ_ERR_INVALID, "ctx is NULL");
  tq_status st = tq::check_context_device(ctx);
  if (st != TQ_OK) return st;
  st = check_cache(ctx, cache);
  if (st != TQ_OK) return st;
  if (!q || !seq_lens || !out || !workspace)
    return fail(TQ_ERR_INVALID, "q, seq_lens, out and workspace must be non-NULL");
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID, "q_dtype=%d", q_dtype);
  if (n_q_heads <= 0 || n_q_heads % cache->n_kv_heads != 0)
    return fail(TQ_ERR_INVALID, "n_q_heads=%d must be a positive multiple of n_kv_heads=%d",
                n_q_heads, cache->n_kv_heads);
  if (n_q_heads / cache->n_kv_heads > 16)
    return fail(TQ_ERR_UNSUPPORTED, "query heads per KV head = %d > 16", n_q_heads / cache->n_kv_heads);
  if (max_seq_len < 0 || max_seq_len > cache->capacity)
    return fail(TQ_ERR_INVALID, "max_seq_len=%d outside [0, capacity=%d]", max_seq_len, cache->capacity);
  if (!aligned16(q) || !aligned16(out) || ((uintptr_t)workspace & 255u) || ((uintptr_t)seq_lens & 3u) ||
      (lse && ((uintptr_t)lse & 3u)))
    return fail(TQ_ERR_INVALID, "misaligned q/out (16 B), workspace (256 B) or seq_lens/lse (4 B)");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID, "scale is not finite");
  const int group = n_q_heads / cache->n_kv_heads;
  const tq::DecodeSplit sp = tq::plan_decode(ctx->d, ctx->bits_k, ctx->bits_v, ctx->qjl, group, cache->n_seqs,
                                             cache->n_kv_heads, max_seq_len, cache->block_table != nullptr);
  const tq::DecodeWorkspace ws = tq::decode_workspace(cache->n_seqs, n_q_heads, sp, ctx->d);
  if (workspace_bytes < ws.total)
    return fail(TQ_ERR_INVALID, "workspace_bytes=%zu < required %zu", workspace_bytes, ws.total);
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)ctx->d);
  const int e = tq::launch_decode(ctx->dp, *cache, q, q_dtype, n_q_heads, seq_lens, max_seq_len, scale,
                                  out, lse, (char *)workspace, sp, ws, stream);
  if (e != 0) return cuda_fail((cudaError_t)e, "tq_decode_attention launch");
  return TQ_OK;
}

tq_status tq_prefill_attention(tq_ctx *ctx, const tq_cache *cache, const void *q, int32_t q_dtype,
                               int32_t n_q_heads, const int32_t *cu_q, const int32_t *seq_lens, int32_t max_q,
                               int32_t max_seq_len, float scale, float *out, float *lse, void *stream) {
  if (!ctx) return fail(TQ_ERR_INVALID, "ctx is NULL");
  tq_status st = tq::check_context_device(ctx);
  if (st != TQ_OK) return st;
  st = check_cache(ctx, cache);
  if (st != TQ_OK) return st;
  if (!q || !cu_q || !seq_lens || !out) return fail(TQ_ERR_INVALID, "q, cu_q, seq_lens and out must be non-NULL");
  if (ctx->d != tq::kHeadDim)
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: prefill attention is implemented for d = 128", ctx->d);
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID, "q_dtype=%d", q_dtype);
  if (n_q_heads <= 0 || n_q_heads % cache->n_kv_heads != 0)
    return fail(TQ_ERR_INVALID, "n_q_heads=%d must be a positive multiple of n_kv_heads=%d",
                n_q_heads, cache->n_kv_heads);
  if (n_q_heads / cache->n_kv_heads > 16)
    return fail(TQ_ERR_UNSUPPORTED, "query heads per KV head = %d > 16", n_q_heads / cache->n_kv_heads);
  if (max_seq_len < 0 || max_seq_len > cache->capacity)
    return fail(TQ_ERR_INVALID, "max_seq_len=%d outside [0, capacity=%d]", max_seq_len, cache->capacity);
  if (max_q < 0 || max_q > max_seq_len)
    return fail(TQ_ERR_INVALID, "max_q=%d outside [0, max_seq_len=%d]", max_q, max_seq_len);
  if (!aligned16(q) || !aligned16(out) || ((uintptr_t)cu_q & 3u) || ((uintptr_t)seq_lens & 3u) ||
      (lse && ((uintptr_t)lse & 3u)))
    return fail(TQ_ERR_INVALID, "misaligned q/out (16 B) or cu_q/seq_lens/lse (4 B)");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID, "scale is not finite");
  if (max_q == 0) return TQ_OK;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)ctx->d);
  const int e = tq::launch_prefill(ctx->dp, *cache, q, q_dtype, n_q_heads, cu_q, seq_lens, max_q, max_seq_len,
                                   scale, out, lse, stream);
  if (e != 0) return cuda_fail((cudaError_t)e, "tq_prefill_attention launch");
  return TQ_OK;
}

namespace {

tq_status check_weight_args(const tq_ctx *ctx, const tq_cache *w, int32_t n_out, int32_t n_in) {
  if (!ctx || !w) return fail(TQ_ERR_INVALID, "ctx and w must be non-NULL");
  tq_status st = tq::check_context_device(ctx);
  if (st != TQ_OK) return st;
  if (ctx->d != tq::kHeadDim) return fail(TQ_ERR_UNSUPPORTED, "d=%d: weight rows are implemented for d = 128", ctx->d);
  if (n_out <= 0 || n_in <= 0 || n_in % ctx->d != 0)
    return fail(TQ_ERR_INVALID, "n_out=%d n_in=%d: both positive, n_in a multiple of d=%d", n_out, n_in, ctx->d);
  if (w->n_seqs != 1 || w->n_kv_heads != n_in / ctx->d || w->block_table)
    return fail(TQ_ERR_INVALID, "w must hold one sequence of n_in / d = %d KV heads, contiguous", n_in / ctx->d);
  if (w->capacity < n_out || w->capacity % 64 != 0)
    return fail(TQ_ERR_INVALID, "capacity=%d must be a multiple of 64 and at least n_out=%d", w->capacity, n_out);
  if (!w->codes_k || !w->norm_k || !aligned16(w->codes_k) || !aligned16(w->norm_k))
    return fail(TQ_ERR_INVALID, "codes_k and norm_k must be non-NULL and 16-byte aligned");
  return TQ_OK;
}

}  // namespace

tq_status tq_weight_quantize(tq_ctx *ctx, const tq_cache *w, const void *w_rows, int32_t n_out, int32_t n_in,
                             void *stream) {
  tq_status st = check_weight_args(ctx, w, n_out, n_in);
  if (st != TQ_OK) return st;
  if (!w_rows || !aligned16(w_rows)) return fail(TQ_ERR_INVALID, "w_rows must be non-NULL and 16-byte aligned");
  tq::DeviceParams p = ctx->dp;
  p.qjl = 0;  // weights keep the MSE codes only
  const long rows = (long)n_out * (n_in / ctx->d);
  const int e = rows <= 1024 ? tq::launch_quantize_rows_k(p, *w, w_rows, nullptr, nullptr, n_out, stream)
                             : tq::launch_quantize_tc(p, *w, w_rows, w_rows, nullptr, nullptr, n_out, true, false,
                                                      stream);
  if (e != 0) return cuda_fail((cudaError_t)e, "tq_weight_quantize launch");
  return TQ_OK;
}

size_t tq_weight_workspace_bytes(const tq_ctx *ctx, int32_t n_tok, int32_t n_in) {
  if (!ctx || n_tok <= 0 || n_in <= 0 || n_in % ctx->d != 0) return 0;
  return tq::weight_workspace_bytes(n_tok, n_in);
}

tq_status tq_weight_gemm(tq_ctx *ctx, const tq_cache *w, int32_t n_out, int32_t n_in, const void *x,
                         int32_t x_dtype, int32_t n_tok, float *y, void *workspace, size_t workspace_bytes,
                         void *stream) {
  tq_status st = check_weight_args(ctx, w, n_out, n_in);
  if (st != TQ_OK) return st;
  if (!x || !y || !workspace) return fail(TQ_ERR_INVALID, "x, y and workspace must be non-NULL");
  if (x_dtype != TQ_BF16 && x_dtype != TQ_F32) return fail(TQ_ERR_INVALID, "x_dtype=%d", x_dtype);
  if (n_tok <= 0 || n_tok > 65520) return fail(TQ_ERR_INVALID, "n_tok=%d outside [1, 65520]", n_tok);
  if (((uintptr_t)x & 3u) || ((uintptr_t)y & 3u) || ((uintptr_t)workspace & 255u))
    return fail(TQ_ERR_INVALID, "misaligned x/y (4 B) or workspace (256 B)");
  const size_t need = tq::weight_workspace_bytes(n_tok, n_in);
  if (workspace_bytes < need) return fail(TQ_ERR_INVALID, "workspace_bytes=%zu < required %zu", workspace_bytes, need);
  const int e = tq::launch_weight_gemm(ctx->dp, *w, n_out, n_in, x, x_dtype, n_tok, y, (char *)workspace, stream);
  if (e != 0) return cuda_fail((cudaError_t)e, "tq_weight_gemm launch");
  return TQ_OK;
}

tq_status tq_check_device_errors(tq_ctx *ctx, void *stream) {
  if (!ctx) return fail(TQ_ERR_INVALID, "ctx is NULL");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned flags = 0;
  e = cudaMemcpy(&flags, ctx->dp.err, sizeof flags, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error flags");
  if (!flags) return TQ_OK;
  e = cudaMemset(ctx->dp.err, 0, sizeof flags);
  if (e != cudaSuccess) return cuda_fail(e, "clear error flags");
  return fail(TQ_ERR_DEVICE, "device error flags 0x%x%s%s%s", flags,
              (flags & tq::kErrTokenRange) ? " [token outside cache]" : "",
              (flags & tq::kErrSeqLen) ? " [seq_len outside range]" : "",
              (flags & tq::kErrWaitExpired) ? " [bounded wait expired]" : "");
}

}  // extern "C"
