// Host construction of the tensor-core tile order (see tile_order.h).
#include <algorithm>
#include <array>
#include <map>

#include "sata_internal.h"
#include "tile_order.h"

namespace sata {
namespace {

// key of a sorted tuple of degree deg (unused slots 0xff)
uint32_t tuple_key(int deg, int i, int j, int l) {
  return (uint32_t)deg | (uint32_t)(i & 0xff) << 8 | (uint32_t)(j & 0xff) << 16 |
         (uint32_t)(l & 0xff) << 24;
}

struct Slot {
  int deg;  // -1 = padding
  int i, j, l;
};

Slot sorted3(int x, int y, int z) {
  int v[3] = {x, y, z};
  std::sort(v, v + 3);
  return {3, v[0], v[1], v[2]};
}
Slot sorted2(int x, int y) { return {2, std::min(x, y), std::max(x, y), -1}; }

}  // namespace

bool build_tile_order(int dK, TileOrder *out) {
  if (dK != 64 && dK != 32) return false;
  const int G = dK / 8;
  HostBasis hb = build_host_basis(dK, 4);
  std::map<uint32_t, int32_t> lex;
  for (int64_t r = 0; r < hb.m; ++r) {
    const int deg = hb.degree[r];
    int ix[3] = {-1, -1, -1};
    for (int s = 0; s < deg; ++s) ix[s] = hb.ix[4 * r + s];
    lex[tuple_key(deg, ix[0], ix[1], ix[2])] = (int32_t)r;
  }
  std::vector<TileDesc> tiles;
  std::vector<Slot> slots;
  auto push = [&](TileDesc td, const std::array<Slot, 64> &s) {
    tiles.push_back(td);
    slots.insert(slots.end(), s.begin(), s.end());
  };
  std::array<Slot, 64> s;
  // OUTER, degree 3: three distinct octets
  for (int gi = 0; gi < G; ++gi)
    for (int gj = gi + 1; gj < G; ++gj)
      for (int gl = gj + 1; gl < G; ++gl)
        for (int a = 0; a < 8; ++a) {
          for (int w = 0; w < 32; ++w) {
            const int b = outer_b(w), c0 = outer_c(w, 0), c1 = outer_c(w, 1);
            s[2 * w] = sorted3(8 * gi + a, 8 * gj + b, 8 * gl + c0);
            s[2 * w + 1] = sorted3(8 * gi + a, 8 * gj + b + 1, 8 * gl + c1);
          }
          push({T_OUTER, 0, (uint8_t)(8 * gi + a), (uint8_t)gj, (uint8_t)gl, 0, 0, 0}, s);
        }
  // BC: pairs of ordered octet pairs (g, g'), g != g'
  std::vector<std::pair<int, int>> og;
  for (int g = 0; g < G; ++g)
    for (int h = 0; h < G; ++h)
      if (h != g) og.push_back({g, h});
  // variant-major: runs of tiles of one variant take one code path in a row
  for (int t = 0; t < 9; ++t)
    for (size_t bp = 0; bp + 1 < og.size(); bp += 2) {
      const auto b0 = og[bp], b1 = og[bp + 1];
      for (int w = 0; w < 32; ++w) {
        // word w: chunks cc, cc + 1 (one pair each) times the third octet
        for (int h = 0; h < 2; ++h) {
          const int cc = 2 * (w / 8) + h, k = 8 * t + cc, blk = k / 36, p = k % 36;
          const int a = pair_a(p), b = pair_b(p);
          const auto gg = blk ? b1 : b0;
          s[2 * w + h] = sorted3(8 * gg.first + a, 8 * gg.first + b, 8 * gg.second + outer_c(w, h));
        }
      }
      push({T_BC, (uint8_t)t, 0, (uint8_t)b0.first, (uint8_t)b0.second, (uint8_t)b1.first,
            (uint8_t)b1.second, 0},
           s);
    }
  // OUTER, degree 2: two distinct octets
  for (int g = 0; g < G; ++g)
    for (int h = g + 1; h < G; ++h) {
      for (int w = 0; w < 32; ++w) {
        s[2 * w] = sorted2(8 * g + outer_b(w), 8 * h + outer_c(w, 0));
        s[2 * w + 1] = sorted2(8 * g + outer_b(w) + 1, 8 * h + outer_c(w, 1));
      }
      push({T_OUTER, 0, kNoIndex, (uint8_t)g, (uint8_t)h, 0, 0, 1}, s);
    }
  // D: triples inside one octet
  const int nD = (120 * G + 63) / 64;
  for (int t = 0; t < nD; ++t) {
    for (int p = 0; p < 64; ++p) {
      const int f = 64 * t + p;
      if (f < 120 * G) {
        const int g = f / 120, r = f % 120;
        s[p] = {3, 8 * g + triple_at(r, 0), 8 * g + triple_at(r, 1), 8 * g + triple_at(r, 2)};
      } else {
        s[p] = {-1, -1, -1, -1};
      }
    }
    push({T_D, (uint8_t)t, 0, 0, 0, 0, 0, 0}, s);
  }
  // MISC: degree-2 pairs inside one octet, degree 1, degree 0, padding
  const int nMisc = 36 * G + dK + 1;
  const int nM = (nMisc + 63) / 64;
  for (int t = 0; t < nM; ++t) {
    for (int p = 0; p < 64; ++p) {
      const int f = 64 * t + p;
      if (f < 36 * G) {
        const int g = f / 36, pr = f % 36;
        s[p] = {2, 8 * g + pair_a(pr), 8 * g + pair_b(pr), -1};
      } else if (f < 36 * G + dK) {
        s[p] = {1, f - 36 * G, -1, -1};
      } else if (f == 36 * G + dK) {
        s[p] = {0, -1, -1, -1};
      } else {
        s[p] = {-1, -1, -1, -1};
      }
    }
    push({T_MISC, (uint8_t)t, 0, 0, 0, 0, 0, 0}, s);
  }
  // coverage check: every basis row exactly once
  std::vector<int> hits(hb.m, 0);
  out->row_of_slot.assign(slots.size(), -1);
  for (size_t k = 0; k < slots.size(); ++k) {
    const Slot &sl = slots[k];
    if (sl.deg < 0) continue;
    auto it = lex.find(tuple_key(sl.deg, sl.i, sl.j, sl.l));
    if (it == lex.end()) return false;
    out->row_of_slot[k] = it->second;
    hits[it->second]++;
  }
  for (int64_t r = 0; r < hb.m; ++r)
    if (hits[r] != 1) return false;
  out->dK = dK;
  out->n_tiles = (int)tiles.size();
  out->tiles = tiles;
  return true;
}

namespace {

// One TMEM lane of a state item: factors j (x_j, the lane's own), l (x_l) and
// per tile f a third factor; valid[f] = false makes row f a padding row (its
// factors are still loaded, so they are chosen to keep the warp's loads
// uniform).
struct LaneGroup {
  int j, l, third[kGroupRows];
  bool valid[kGroupRows];
};

}  // namespace

bool build_state_groups(int dK, const TileOrder &to, StateGroups *out) {
  if ((dK != 64 && dK != 32) || to.dK != dK) return false;
  const int G = dK / 8;
  const int ONES = dK, PAD = -1;
  HostBasis hb = build_host_basis(dK, 4);
  std::map<uint32_t, int32_t> lex;
  for (int64_t r = 0; r < hb.m; ++r) {
    const int deg = hb.degree[r];
    int ix[3] = {-1, -1, -1};
    for (int s = 0; s < deg; ++s) ix[s] = hb.ix[4 * r + s];
    lex[tuple_key(deg, ix[0], ix[1], ix[2])] = (int32_t)r;
  }
  std::vector<int32_t> slot_of_row(hb.m, -1);
  for (size_t k = 0; k < to.row_of_slot.size(); ++k)
    if (to.row_of_slot[k] >= 0) slot_of_row[to.row_of_slot[k]] = (int32_t)k;

  std::vector<LaneGroup> lg;
  auto add = [&](int j, int l, int t0, int t1, int t2, int t3) {
    LaneGroup g{j, l, {t0, t1, t2, t3}, {t0 != PAD, t1 != PAD, t2 != PAD, t3 != PAD}};
    for (int f = 0; f < kGroupRows; ++f)
      if (g.third[f] == PAD) g.third[f] = ONES;
    lg.push_back(g);
  };
  // degree 3, three distinct octets gi < gj < gl: third factor 8 gi + 4 ahi + f
  // (uniform in each warp), shared x_j x_l over the octets gj, gl
  for (int gi = 0; gi < G; ++gi)
    for (int gj = gi + 1; gj < G; ++gj)
      for (int gl = gj + 1; gl < G; ++gl)
        for (int ahi = 0; ahi < 2; ++ahi)
          for (int bh = 0; bh < 2; ++bh)
            for (int lane = 0; lane < 32; ++lane) {
              const int b = 4 * bh + (lane & 3), c = lane >> 2;
              const int t = 8 * gi + 4 * ahi;
              add(8 * gj + b, 8 * gl + c, t, t + 1, t + 2, t + 3);
            }
  // degree 3 with a pair a <= b inside octet g and the third index in octet
  // g' != g: shared pair, third factor 8 g' + 4 h + f (uniform per (g', h))
  for (int g2 = 0; g2 < G; ++g2)
    for (int h = 0; h < 2; ++h)
      for (int g = 0; g < G; ++g) {
        if (g == g2) continue;
        for (int a = 0; a < 8; ++a)
          for (int b = a; b < 8; ++b) {
            const int t = 8 * g2 + 4 * h;
            add(8 * g + a, 8 * g + b, t, t + 1, t + 2, t + 3);
          }
      }
  // degree 3 inside one octet: shared pair a <= b, third c = b..7
  for (int g = 0; g < G; ++g)
    for (int a = 0; a < 8; ++a)
      for (int b = a; b < 8; ++b)
        for (int c0 = b; c0 < 8; c0 += kGroupRows) {
          int t[kGroupRows];
          for (int f = 0; f < kGroupRows; ++f) t[f] = c0 + f < 8 ? 8 * g + c0 + f : PAD;
          add(8 * g + a, 8 * g + b, t[0], t[1], t[2], t[3]);
        }
  // degree 2 (u <= w): shared x_w and ones, third factor u
  for (int w = 0; w < dK; ++w)
    for (int u0 = 0; u0 <= w; u0 += kGroupRows) {
      int t[kGroupRows];
      for (int f = 0; f < kGroupRows; ++f) t[f] = u0 + f <= w ? u0 + f : PAD;
      add(w, ONES, t[0], t[1], t[2], t[3]);
    }
  // degree 1 and degree 0
  for (int u0 = 0; u0 < dK; u0 += kGroupRows) add(ONES, ONES, u0, u0 + 1, u0 + 2, u0 + 3);
  add(ONES, ONES, ONES, PAD, PAD, PAD);
  while (lg.size() % 128) add(ONES, ONES, PAD, PAD, PAD, PAD);

  const int n_items = (int)(lg.size() / 128);
  out->n_items = n_items;
  // tile-order slots that hold no row: given to padding rows (weight 0), so
  // that every snapshot column is written (with zeros there)
  std::vector<int32_t> free_slots;
  for (size_t k = 0; k < to.row_of_slot.size(); ++k)
    if (to.row_of_slot[k] < 0) free_slots.push_back((int32_t)k);
  out->lane_idx.assign((size_t)n_items * 128, 0);
  out->slot.assign((size_t)n_items * kGroupRows * 128, -1);
  out->row.assign((size_t)n_items * kGroupRows * 128, -1);
  out->weight.assign((size_t)n_items * kGroupRows * 128, 0.f);
  std::vector<int> hits(hb.m, 0);
  for (int it = 0; it < n_items; ++it)
    for (int lane = 0; lane < 128; ++lane) {
      const LaneGroup &q = lg[(size_t)it * 128 + lane];
      uint64_t packed = (uint64_t)q.j | (uint64_t)q.l << 8;
      for (int f = 0; f < kGroupRows; ++f) {
        const int t = q.third[f];
        packed |= (uint64_t)t << (16 + 8 * f);
        if (!q.valid[f]) {
          if (!free_slots.empty()) {
            out->slot[((size_t)it * kGroupRows + f) * 128 + lane] = free_slots.back();
            free_slots.pop_back();
          }
          continue;
        }
        int v[3] = {t, q.j, q.l}, idx[3], deg = 0;
        for (int s2 = 0; s2 < 3; ++s2)
          if (v[s2] != ONES) idx[deg++] = v[s2];
        std::sort(idx, idx + deg);
        auto itr = lex.find(tuple_key(deg, deg > 0 ? idx[0] : -1, deg > 1 ? idx[1] : -1,
                                      deg > 2 ? idx[2] : -1));
        if (itr == lex.end()) return false;
        const int32_t r = itr->second;
        const size_t k = ((size_t)it * kGroupRows + f) * 128 + lane;
        out->slot[k] = slot_of_row[r];
        out->row[k] = r;
        out->weight[k] = (float)hb.weight[r];
        if (slot_of_row[r] < 0) return false;
        hits[r]++;
      }
      out->lane_idx[(size_t)it * 128 + lane] = packed;
    }
  for (int64_t r = 0; r < hb.m; ++r)
    if (hits[r] != 1) return false;
  return free_slots.empty();  // every slot of the tile order is written
}

}  // namespace sata
