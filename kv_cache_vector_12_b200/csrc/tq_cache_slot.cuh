// Token slots of the packed cache (device side), for the contiguous and the
// paged layout of tq_cache (include/tq.h): every per-token plane is indexed
// by the same slot, times its bytes per token.
#pragma once

#include "tq_internal.h"

namespace tq {

// Slot of position p of sequence s, KV head h, or -1 when (s, p) lies
// outside the cache or, paged, the block-table entry is out of range.
__device__ __forceinline__ long cache_slot(const tq_cache &c, int s, int h, int p) {
  if (s < 0 || s >= c.n_seqs || p < 0 || p >= c.capacity) return -1;
  if (!c.block_table) return ((long)s * c.n_kv_heads + h) * c.capacity + p;
  const int j = p / c.block_size;
  const int blk = c.block_table[(long)s * (c.capacity / c.block_size) + j];
  if (blk < 0 || blk >= c.n_blocks) return -1;
  return ((long)blk * c.n_kv_heads + h) * c.block_size + (p - j * c.block_size);
}

}  // namespace tq
