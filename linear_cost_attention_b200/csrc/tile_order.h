// Tile order of the minimal basis for the tensor-core path (P = 4, dK = 64 or
// 32).
//
// The basis rows (sorted index tuples, "对称张量分解的核心洞察") are regrouped
// into tiles of 64 features whose structure is fixed, so that one thread per
// token can generate a tile with compile-time register indices.  Indices are
// split into G = dK / 8 octets g = i / 8:
//
//  OUTER  x[i1] * x[8*ga + b] * x[8*gb + c], b, c = 0..7 (64 features):
//         degree 3 with three distinct octets gi < gj < gl (i1 = 8*gi + a;
//         56 octet triples x 8 values of a = 448 tiles), and degree 2 with
//         two distinct octets (i1 absent; 28 tiles).
//  BC     degree 3 with exactly two equal octets: a pair a <= b inside octet
//         g times a full octet g' != g, 36 x 8 = 288 features per ordered
//         (g, g'); two such blocks fill 9 tiles (252 tiles).
//  D      degree 3 inside one octet: the 120 triples a <= b <= c of each
//         octet, concatenated over the 8 octets (15 tiles).
//  MISC   degree 2 inside one octet (36 pairs per octet), degree 1 (dK),
//         degree 0 (1), zero padding.
// dK = 64: 749 tiles (448 OUTER-3, 252 BC, 28 OUTER-2, 15 D, 6 MISC) = 47936
// slots for the 47905 rows.  dK = 32: 103 tiles (32, 54, 6, 8, 3) = 6592 slots
// for the 6545 rows.  The other slots are zero padding.  Per feature, the
// weight is the basis weight 1/sqrt(alpha! dK^(p/2)) of its row.
#pragma once

#include <stdint.h>

#include <vector>

namespace sata {

enum TileType : uint8_t { T_OUTER = 0, T_BC = 1, T_D = 2, T_MISC = 3, T_PAD = 4 };

struct alignas(8) TileDesc {  // 8 bytes, one 64-bit load; read by the generator warps
  uint8_t type, variant, i1, o0, o1, o2, o3, wsel;
};
constexpr uint8_t kNoIndex = 0xff;  // OUTER tile of degree 2: no first index

// Index pairs a <= b and triples a <= b <= c inside one octet, lexicographic.
__host__ __device__ constexpr int pair_a(int p) {
  int n = 0;
  for (int a = 0; a < 8; ++a)
    for (int b = a; b < 8; ++b) {
      if (n == p) return a;
      ++n;
    }
  return 0;
}
__host__ __device__ constexpr int pair_b(int p) {
  int n = 0;
  for (int a = 0; a < 8; ++a)
    for (int b = a; b < 8; ++b) {
      if (n == p) return b;
      ++n;
    }
  return 0;
}
__host__ __device__ constexpr int triple_at(int r, int which) {
  int n = 0;
  for (int a = 0; a < 8; ++a)
    for (int b = a; b < 8; ++b)
      for (int c = b; c < 8; ++c) {
        if (n == r) return which == 0 ? a : which == 1 ? b : c;
        ++n;
      }
  return 0;
}
// Feature order inside OUTER and BC tiles.  Packed word w (features 2w, 2w+1)
// holds two products with the third octet's entries c0 = outer_c(w, 0),
// c1 = outer_c(w, 1), which are (2j, 2j+1) or (2j+1, 2j) for j = (w % 8) / 2:
// the generator multiplies a bf16x2 pair of partial products by one packed
// word of the third octet or by that word with its halves swapped.  OUTER:
// partial products for b = outer_b(w) and b + 1 of the first octet; BC: the
// pairs of chunks 2 (w / 8) and 2 (w / 8) + 1.
__host__ __device__ constexpr int outer_b(int w) { return 2 * (w / 8); }
__host__ __device__ constexpr int outer_c(int w, int half) {
  return 2 * ((w % 8) / 2) + ((w % 2) ^ half);
}
// alpha! of a sorted triple / pair with equal-index runs
__host__ __device__ constexpr int fact3(int a, int b, int c) {
  return (a == b && b == c) ? 6 : (a == b || b == c) ? 2 : 1;
}

struct TileOrder {
  int dK = 0;
  int n_tiles = 0;
  std::vector<TileDesc> tiles;
  std::vector<int32_t> row_of_slot;  // [n_tiles*64] lexicographic basis row, -1 = padding
};

// Builds the tile order for dK = 64 or 32, P = 4, and checks that it covers
// every basis row exactly once.  Returns false if the check fails.
bool build_tile_order(int dK, TileOrder *out);

// Row groups of the tensor-core state kernel (dK = 64 or 32, P = 4).
//
// Every basis monomial of degree <= 3 is a product of three factors taken
// from the rows of K^T plus a row of ones (index dK): x_j x_l x_i, with ones
// standing in for missing indices.  The state kernel's generator thread owns
// kGroupRows rows that share two of their factors (x_j x_l) and differ in the
// third (x_i0 .. x_i3), so per token it loads 2 + kGroupRows factor rows for
// kGroupRows monomials instead of 3 per monomial.  A lane group is one such
// set; an item is 128 lane groups (the 128 TMEM lanes) x kGroupRows rows (the
// item's kGroupRows 128-row state tiles).  Groups, in order: degree 3 over
// three distinct index octets (shared x_j x_l, third factor from the lowest
// octet, uniform across each warp); degree 3 with a pair inside one octet
// (shared pair, third factor from another octet, uniform across runs of 252
// groups); degree 3 inside one octet; degree 2 (shared x_w and ones); degree
// 1; degree 0.  (Groups whose second and third factors are one row for a
// whole warp, with the own factors in whole octets, measured 5 % slower in the
// state kernel at dK = 64 and are not used.)  Unused
// rows of a group are padding (weight 0, no basis row); the tile order's
// empty slots are given to padding rows, so that writing every row's slot
// writes every snapshot column (zeros on the empty ones).
constexpr int kGroupRows = 4;
struct StateGroups {
  int n_items = 0;
  std::vector<uint64_t> lane_idx;  // [item][lane]: j | l<<8 | i0<<16 | i1<<24 | i2<<32 | i3<<40
  std::vector<int32_t> slot;       // [item][f][lane]: tile-order slot (snapshot column) or -1
  std::vector<int32_t> row;        // [item][f][lane]: lexicographic basis row, -1 pad
  std::vector<float> weight;       // [item][f][lane]: basis weight, 0 pad
};

// Builds the row groups for the tile order `to` (same dK) and checks that they
// cover every basis row exactly once.  Returns false if the check fails.
bool build_state_groups(int dK, const TileOrder &to, StateGroups *out);

}  // namespace sata
