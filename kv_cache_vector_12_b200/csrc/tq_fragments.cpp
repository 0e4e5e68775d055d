// Coordinate orders inside the decode kernel's tensor-core fragments.
//
// The decode kernel expands the codes a thread loads straight into its MMA
// fragments, so the head dimension appears inside a fragment in an order set
// by the bit layout.  These functions give, for each position of the logical
// (fragment) order, the coordinate of the head vector it holds.  The decode
// kernel computes q_hat (and q_tilde) in the K (and QJL) order from Pi (and
// S) stored with permuted rows; the inverse rotation in merge reads Pi's rows
// in the V order.  Each is a permutation of 0..127.
#include <cstdint>

#include "tq_internal.h"

namespace tq {

// Scores use mma m16n8k32 (int8): k index kappa = 32 s + 16 slot + 4 q + i is
// byte i of the A register of k-step s and slot `slot` held by the threads
// with q = lane % 4.  That register is the byte-permute lookup of selector
// sigma = 2 s + slot of the 32 codes of coordinate group q (coordinates
// 32 q .. 32 q + 31); nibble i of the selector is local code l:
//   3 and 4 bits: selector sigma holds local codes 4 sigma .. 4 sigma + 3;
//   2 bits: sigma = 4 w + 2 par + hh holds codes 16 w + 2 (4 hh + i) + par
//           (even or odd codes of word w, low or high half).
void kperm_of(int bits, uint8_t *perm) {
  for (int kappa = 0; kappa < kHeadDim; ++kappa) {
    const int s = kappa / 32, rem = kappa % 32, slot = rem / 16, q = (rem % 16) / 4, i = rem % 4;
    const int sigma = 2 * s + slot;
    int l;
    if (bits == 2) {
      const int w = sigma / 4, par = (sigma / 2) % 2, hh = sigma % 2;
      l = 16 * w + 2 * (4 * hh + i) + par;
    } else {
      l = 4 * sigma + i;
    }
    perm[kappa] = (uint8_t)(32 * q + l);
  }
}

// QJL signs use the same int8 A layout: byte i of the register of k-step s
// and slot `slot` is bit j + 8 i of word q of the sign bits, j = 2 s + slot,
// i.e. projection index 32 q + j + 8 i.
void jperm_of(uint8_t *perm) {
  for (int kappa = 0; kappa < kHeadDim; ++kappa) {
    const int s = kappa / 32, rem = kappa % 32, slot = rem / 16, q = (rem % 16) / 4, i = rem % 4;
    perm[kappa] = (uint8_t)(32 * q + 2 * s + slot + 8 * i);
  }
}

// Values use mma m16n8k16 (fp16) with the coordinates as M: logical row
// kappa = 16 mt + rho of m-tile mt is held by the threads with
// r = lane / 4 = rho % 8, as the "x" (rho < 8) or "y" (rho >= 8) code of
// selector mt of the thread's 16-coordinate unit r:
//   3 bits: unit r = half r % 2 of group r / 2; selector mt = 2 k + hh holds
//           codes 8 k + 4 h + 2 hh (x) and + 1 (y) of the group (k = 3: the
//           spare column, codes 24 ..);
//   2 bits: unit r = coordinates 16 r ..; mt = 4 yh + 2 par + hh holds codes
//           8 yh + 4 hh + par (x) and + 2 (y);
//   4 bits: unit r = coordinates 16 r ..; selector mt holds codes 2 mt (x)
//           and 2 mt + 1 (y).
void vperm_of(int bits, uint8_t *perm) {
  for (int kappa = 0; kappa < kHeadDim; ++kappa) {
    const int mt = kappa / 16, rho = kappa % 16, r = rho % 8, e = rho / 8;
    int coord;
    if (bits == 3) {
      const int k = mt / 2, hh = mt % 2, h = r & 1, g = r >> 1;
      coord = 32 * g + 8 * k + 4 * h + 2 * hh + e;
    } else if (bits == 2) {
      const int yh = mt / 4, par = (mt / 2) % 2, hh = mt % 2;
      coord = 16 * r + 8 * yh + 4 * hh + par + 2 * e;
    } else {
      coord = 16 * r + 2 * mt + e;
    }
    perm[kappa] = (uint8_t)coord;
  }
}

}  // namespace tq
