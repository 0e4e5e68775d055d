// Coordinate orders inside the decode kernel's tensor-core fragments.
//
// The decode kernel expands the codes a thread loads straight into its MMA
// fragments, so the head dimension appears inside a fragment in an order set
// by the bit layout.  These functions give, for each position of the logical
// (fragment) order, the coordinate of the head vector it holds.  The decode
// kernel computes q_hat (and q_tilde) in the K (and QJL) order from Pi (and
// S) stored with permuted rows; the inverse rotation in merge reads Pi's rows
// in the V order.  Each is a permutation of 0 .. d - 1.
#include <cstdint>

#include "tq_internal.h"

namespace tq {

namespace {
// The lane fields of int8 k index kappa = 32 s + 16 slot + 4 q + i.
struct KIndex {
  int s, slot, q, i;
  explicit KIndex(int kappa) : s(kappa / 32), slot((kappa % 32) / 16), q((kappa % 16) / 4), i(kappa % 4) {}
};
}  // namespace

// Scores use mma m16n8k32 (int8): k index kappa = 32 s + 16 slot + 4 q + i is
// byte i of the A register of k-step s and slot `slot` held by the threads
// with q = lane % 4.  That register is the byte-permute lookup of selector
// sigma of the 32 codes of one coordinate group (coordinates 32 g ..
// 32 g + 31):
//   d = 128: group q, sigma = 2 s + slot;
//   d = 256: group q + 4 (s / 4), sigma = 2 (s % 4) + slot;
//   d = 64:  group q / 2, sigma = 4 (q % 2) + 2 s + slot.
// Nibble i of selector sigma is local code l:
//   3 and 4 bits: l = 4 sigma + i;
//   2 bits: sigma = 4 w + 2 par + hh holds codes 16 w + 2 (4 hh + i) + par
//           (even or odd codes of word w, low or high half).
void kperm_of(int bits, int d, uint8_t *perm) {
  for (int kappa = 0; kappa < d; ++kappa) {
    const KIndex k(kappa);
    const int group = d == 64 ? k.q / 2 : k.q + 4 * (k.s / 4);
    const int sigma = d == 64 ? 4 * (k.q % 2) + 2 * k.s + k.slot : 2 * (k.s % 4) + k.slot;
    int l;
    if (bits == 2) {
      const int w = sigma / 4, par = (sigma / 2) % 2, hh = sigma % 2;
      l = 16 * w + 2 * (4 * hh + k.i) + par;
    } else {
      l = 4 * sigma + k.i;
    }
    perm[kappa] = (uint8_t)(32 * group + l);
  }
}

// QJL signs use the same int8 A layout: byte i of the register of k-step s
// and slot `slot` is bit j + 8 i of sign word wd (32 projections each), with
// (wd, j) = (q + 4 (s / 4), 2 (s % 4) + slot), or (q / 2, 4 (q % 2) + 2 s +
// slot) at d = 64; i.e. projection index 32 wd + j + 8 i.
void jperm_of(int d, uint8_t *perm) {
  for (int kappa = 0; kappa < d; ++kappa) {
    const KIndex k(kappa);
    const int wd = d == 64 ? k.q / 2 : k.q + 4 * (k.s / 4);
    const int j = d == 64 ? 4 * (k.q % 2) + 2 * k.s + k.slot : 2 * (k.s % 4) + k.slot;
    perm[kappa] = (uint8_t)(32 * wd + j + 8 * k.i);
  }
}

// Values use mma m16n8k16 (fp16) with the coordinates as M: logical row
// kappa = 16 mt + rho of m-tile mt is held by the threads with
// r = lane / 4 = rho % 8, as the "x" (rho < 8) or "y" (rho >= 8) code of
// selector mt of the thread's unit r.  For d = 128 and 256 (two halves,
// m-tiles 8 H .. 8 H + 7 for coordinates 128 H ..), per half:
//   3 bits: unit r = half r % 2 of group r / 2; selector mt = 2 k + hh holds
//           codes 8 k + 4 h + 2 hh (x) and + 1 (y) of the group (k = 3: the
//           spare column, codes 24 ..);
//   2 bits: unit r = coordinates 16 r ..; mt = 4 yh + 2 par + hh holds codes
//           8 yh + 4 hh + par (x) and + 2 (y);
//   4 bits: unit r = coordinates 16 r ..; selector mt holds codes 2 mt (x)
//           and 2 mt + 1 (y).
// For d = 64 (four m-tiles, unit r of 8 coordinates):
//   3 bits: byte r % 4 of the words of group r / 4: mt = k holds codes
//           8 k + 2 (r % 4) (x) and + 1 (y);
//   2 bits: bytes 2 h, 2 h + 1 (h = r % 2) of word r / 2: mt = 2 par + hh
//           holds codes 8 h + 4 hh + par (x) and + 2 (y) of the word;
//   4 bits: word r: mt holds codes 2 mt (x) and 2 mt + 1 (y).
void vperm_of(int bits, int d, uint8_t *perm) {
  for (int kappa = 0; kappa < d; ++kappa) {
    const int mt_all = kappa / 16, rho = kappa % 16, r = rho % 8, e = rho / 8;
    int coord;
    if (d == 64) {
      const int mt = mt_all;
      if (bits == 3) {
        coord = 32 * (r / 4) + 8 * mt + 2 * (r % 4) + e;
      } else if (bits == 2) {
        const int par = mt / 2, hh = mt % 2, h = r % 2;
        coord = 16 * (r / 2) + 8 * h + 4 * hh + par + 2 * e;
      } else {
        coord = 8 * r + 2 * mt + e;
      }
    } else {
      const int half = mt_all / 8, mt = mt_all % 8;
      if (bits == 3) {
        const int k = mt / 2, hh = mt % 2, h = r & 1, g = r >> 1;
        coord = 32 * g + 8 * k + 4 * h + 2 * hh + e;
      } else if (bits == 2) {
        const int yh = mt / 4, par = (mt / 2) % 2, hh = mt % 2;
        coord = 16 * r + 8 * yh + 4 * hh + par + 2 * e;
      } else {
        coord = 16 * r + 2 * mt + e;
      }
      coord += 128 * half;
    }
    perm[kappa] = (uint8_t)coord;
  }
}

}  // namespace tq
