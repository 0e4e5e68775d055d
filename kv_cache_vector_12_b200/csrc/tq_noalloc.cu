// tq_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) when they
// decode: code running while a stream is being captured into a CUDA graph,
// where an allocation breaks or invalidates the capture; serving engines that
// hand out device memory only from their own pre-carved pool and forbid any
// other allocation; and latency-critical loops that cannot afford
// cudaMalloc's implicit device synchronisation.  Such callers still own their
// inputs and outputs, but they cannot provide the decode workspace.  This
// entry point takes its workspace from one fixed-size array that lives in the
// library's device image instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds TQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  Host
// code cannot use the array's name as a device address; the first call on
// each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it.  All calls in the process share the array:
// two calls whose kernels overlap on the GPU (different streams, or another
// thread) race on it.  The decode kernels write every workspace byte they
// read, so nothing has to start at zero.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "tq_internal.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

namespace {

using tq::kMaxDevices;
std::mutex g_scratch_mutex;
void *g_scratch_address[kMaxDevices];

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(tq_ctx *ctx, const tq_cache *cache, const void *q,
                                                 int32_t q_dtype, int32_t n_q_heads, const int32_t *seq_lens,
                                                 int32_t max_seq_len, float scale, float *out, float *lse,
                                                 void *stream) {
  if (!ctx || !cache) return tq::report_error(TQ_ERR_INVALID, "ctx and cache must be non-NULL");
  // the scratch address below is looked up on the current device: it must be
  // the context's, or the kernels would mix two GPUs' memory
  const tq_status st = tq::check_context_device(ctx);
  if (st != TQ_OK) return st;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::report_error(TQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return tq::report_error(TQ_ERR_UNSUPPORTED, "device %d: at most %d devices are supported", dev, kMaxDevices);

  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_address[dev]) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return tq::report_error(TQ_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev,
                                cudaGetErrorString(e));
      g_scratch_address[dev] = p;
    }
    scratch = g_scratch_address[dev];
  }

  const size_t need = tq_workspace_bytes(ctx, cache->n_seqs, n_q_heads, max_seq_len);
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES)
    return tq::report_error(TQ_ERR_INVALID,
                            "this decode needs %zu bytes of workspace, more than the %d bytes of static scratch "
                            "(use tq_decode_attention with a caller-provided workspace)",
                            need, TQ_NOALLOC_SCRATCH_BYTES);
  return tq_decode_attention(ctx, cache, q, q_dtype, n_q_heads, seq_lens, max_seq_len, scale, out, lse, scratch,
                             (size_t)TQ_NOALLOC_SCRATCH_BYTES, stream);
}
