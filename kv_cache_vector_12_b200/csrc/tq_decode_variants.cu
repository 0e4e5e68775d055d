// Instantiations of the decode attention kernel for one head dimension and
// one K width, chosen by TQ_DECODE_DH and TQ_DECODE_BK on the compiler's
// command line: the library's build compiles this file once per pair
// (d in {64, 128, 256}, bits_k in {2, 3, 4}) so that the slices compile in
// parallel.  Without the two macros the object is empty.
#include "tq_decode_kernel.cuh"

#if defined(TQ_DECODE_DH) && defined(TQ_DECODE_BK)
namespace tq {

template <int DH, int BK>
DecodeVariant decode_variant(int bits_v, bool qjl, int nt, int build) {
  return variant_k<BK, DH>(bits_v, qjl, nt, build);
}

template DecodeVariant decode_variant<TQ_DECODE_DH, TQ_DECODE_BK>(int, bool, int, int);

}  // namespace tq
#endif
