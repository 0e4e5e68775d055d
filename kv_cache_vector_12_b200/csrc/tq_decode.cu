// Decode attention over the packed TurboQuant cache, sm_100a: the split
// merge kernel, the choice of the attention kernel's instantiation and the
// launch of both.  The attention kernel itself is in tq_decode_kernel.cuh.
#include <atomic>
#include <cmath>

#include "tq_decode_kernel.cuh"

namespace tq {
namespace {

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

// A bf16 row of DH entries (16-byte aligned): held in registers as
// independent 16-byte loads (DH <= 128, loaded ahead of use) or read on the
// fly (DH = 256).
template <int DH>
struct Bf16Row {
  static constexpr int kHeld = DH <= 128 ? DH / 8 : 1;
  uint4 w[kHeld];
  const uint16_t *row;
  __device__ __forceinline__ void load(const uint16_t *r) {
    row = r;
    if constexpr (DH <= 128) {
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) w[c] = reinterpret_cast<const uint4 *>(r)[c];
    }
  }
  __device__ __forceinline__ uint4 get(int c) const {
    if constexpr (DH <= 128) return w[c];
    else return reinterpret_cast<const uint4 *>(row)[c];
  }
};

// Dot product of a bf16 row with a vector in shared memory, four partial sums.
template <int DH>
__device__ __forceinline__ float dot_bf16_row(const Bf16Row<DH> &w, const float *x) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < DH / 8; ++c) {
    const uint4 v = w.get(c);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 8 * c + 2 * e;
      acc[e] = fmaf(__uint_as_float(u[e] << 16), x[j], acc[e]);
      acc[e] = fmaf(__uint_as_float(u[e] & 0xffff0000u), x[j + 1], acc[e]);
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// PL consecutive floats (PL * 4-byte aligned) as vector loads.
template <int PL>
__device__ __forceinline__ void load_floats(const float *src, float (&v)[PL]) {
  if constexpr (PL == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(src);
    v[0] = x.x, v[1] = x.y;
  } else {
#pragma unroll
    for (int c = 0; c < PL / 4; ++c) {
      const float4 x = reinterpret_cast<const float4 *>(src)[c];
      v[4 * c] = x.x, v[4 * c + 1] = x.y, v[4 * c + 2] = x.z, v[4 * c + 3] = x.w;
    }
  }
}

// ---------------------------------------------------------------------------
// merge: per (sequence, query head) combine the splits (log-sum-exp in log2
// units) and apply Pi^T: o_i = sum_k Pi[vperm(k)][i] o~_k / L.  128 threads;
// thread t owns outputs t (and t + 128 for DH = 256).
// ---------------------------------------------------------------------------
constexpr int kMergeMaxSplits = 1024;

template <int DH>
__global__ void __launch_bounds__(128) merge_kernel(DeviceParams p, int n_q_heads, const int32_t *seq_lens,
                                                    int max_seq_len, int chunk, int n_splits,
                                                    const float *partials, float *out, float *lse) {
  constexpr int PF = DH + 4;                      // floats per split partial: m, l, 2 unused, DH outputs
  constexpr int PL = DH / 32;                     // outputs per lane in the split loads
  constexpr int kOPerWarp = DH == 256 ? 8 : 16;   // splits per warp held in registers
  __shared__ float s_ot[DH];
  __shared__ float s_w[kMergeMaxSplits], s_l[kMergeMaxSplits];
  __shared__ __align__(16) float s_acc[4][DH];
  __shared__ float red[4];
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this thread's rows of Pi^T do not depend on the attention kernel: load
  // them before waiting for that kernel to complete
  Bf16Row<DH> pw0, pw1;
  if (tid < DH) pw0.load(p.pivt + tid * DH);
  if constexpr (DH == 256) pw1.load(p.pivt + (tid + 128) * DH);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel in the stream (an append, the next decode) may launch and
  // load its parameters now; it waits for this grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int s = row / n_q_heads;
  const float *src = partials + (long)row * n_splits * PF;
  // One round of loads: the sequence length, and warp w's outputs of splits
  // w, w + 4, ... (lane j: outputs PL j .. PL j + PL - 1) of every allocated
  // split, requested before any of them is used; splits past the used ones
  // are ignored below (their slots may hold anything).
  float ov[kOPerWarp][PL];
#pragma unroll
  for (int e = 0; e < kOPerWarp; ++e) {
    const int sp = warp + 4 * e;
    if (sp < n_splits) load_floats<PL>(src + sp * PF + 4 + lane * PL, ov[e]);
  }
  // and thread t's (m, l) pair of split t, so that the pairs of the first 128
  // splits do not wait for the sequence length
  float2 ml0 = make_float2(-INFINITY, 0.f);
  if (tid < n_splits) ml0 = *reinterpret_cast<const float2 *>(src + tid * PF);
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
    const float2 ml = *reinterpret_cast<const float2 *>(src + sp * PF);
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
  float acc[PL];
#pragma unroll
  for (int c = 0; c < PL; ++c) acc[c] = 0.f;
#pragma unroll
  for (int e = 0; e < kOPerWarp; ++e) {
    const int sp = warp + 4 * e;
    if (sp < used) {
      const float w = s_w[sp];
#pragma unroll
      for (int c = 0; c < PL; ++c) acc[c] = fmaf(w, ov[e][c], acc[c]);
    }
  }
  // splits beyond 4 * kOPerWarp (long sequences with short splits)
  for (int sp = warp + 4 * kOPerWarp; sp < used; sp += 4) {
    float v[PL];
    load_floats<PL>(src + sp * PF + 4 + lane * PL, v);
    const float w = s_w[sp];
#pragma unroll
    for (int c = 0; c < PL; ++c) acc[c] = fmaf(w, v[c], acc[c]);
  }
#pragma unroll
  for (int c = 0; c < PL; ++c) s_acc[warp][lane * PL + c] = acc[c];
  for (int o = 16; o; o >>= 1) lpart += __shfl_xor_sync(0xffffffffu, lpart, o);
  if (lane == 0) red[warp] = lpart;
  __syncthreads();
  const float ll = (red[0] + red[1]) + (red[2] + red[3]);
  for (int i = tid; i < DH; i += 128) {
    const float oo = (s_acc[0][i] + s_acc[1][i]) + (s_acc[2][i] + s_acc[3][i]);
    s_ot[i] = ll > 0.f ? oo / ll : 0.f;
  }
  __syncthreads();
  // o_i = sum_k Pi^T[i][k] o~_k with Pi^T's columns in the V fragment order
  if (tid < DH) out[(long)row * DH + tid] = dot_bf16_row<DH>(pw0, s_ot);
  if constexpr (DH == 256) out[(long)row * DH + tid + 128] = dot_bf16_row<DH>(pw1, s_ot);
  if (lse && tid == 0) lse[row] = ll > 0.f ? (mm + log2f(ll)) * 0.6931471805599453f : -INFINITY;
}


template <int DH>
DecodeVariant variant_d(int bk, int bv, bool qjl, int nt, int build) {
  switch (bk) {
    case 2: return decode_variant<DH, 2>(bv, qjl, nt, build);
    case 3: return decode_variant<DH, 3>(bv, qjl, nt, build);
    default: return decode_variant<DH, 4>(bv, qjl, nt, build);
  }
}

DecodeVariant variant(int d, int bk, int bv, bool qjl, int nt, int build) {
  if (d == 64) return variant_d<64>(bk, bv, qjl, nt, build);
  if (d == 256) return variant_d<256>(bk, bv, qjl, nt, build);
  return variant_d<128>(bk, bv, qjl, nt, build);
}

int build_of(bool long_splits, bool paged) { return paged ? kPaged : long_splits ? kLong : kShort; }

int dim_index(int d) { return d == 64 ? 0 : d == 128 ? 1 : 2; }

}  // namespace

int decode_ctas_per_sm(int d, int bits_k, int bits_v, int qjl, int group, bool long_splits, bool paged) {
  // cached per variant; atomically, as calls may come from several threads
  // (per device: the attribute and the occupancy query apply to the current one)
  static std::atomic<int> cache[kMaxDevices][3][3][3][2][2][3];
  const int nt = group > 8 ? 2 : 1;
  const int build = build_of(long_splits, paged);
  std::atomic<int> &slot =
      cache[current_device()][dim_index(d)][bits_k - 2][bits_v - 2][qjl ? 1 : 0][nt - 1][build];
  int c = slot.load(std::memory_order_relaxed);
  if (c == 0) {
    const DecodeVariant v = variant(d, bits_k, bits_v, qjl != 0, nt, build);
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

  const DecodeVariant v = variant(p.d, p.bits_k, p.bits_v, p.qjl != 0, group > 8 ? 2 : 1,
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
  const auto merge = p.d == 64 ? merge_kernel<64> : p.d == 256 ? merge_kernel<256> : merge_kernel<128>;
  e = cudaLaunchKernelEx(&mcfg, merge, p, n_q_heads, seq_lens, max_seq_len, split.chunk, split.n_splits,
                         (const float *)partials, out, lse);
  return (int)e;
}

}  // namespace tq
