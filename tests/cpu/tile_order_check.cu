// Host-only check of the tensor-core tile order and of its feature generator
// (the device generator compiled for the host).  Built by
// tests/test_tile_order_cpu.py with nvcc; needs no GPU.
//   1. every basis row appears in exactly one tile slot;
//   2. for random bf16 rows, every generated feature equals the basis weight
//      times the product of its indexed entries, up to bf16 rounding;
//   3. the state kernel's row groups hold every basis row and every tile-order
//      slot once, and each row's shared and third factors are its indices;
// for dK = 64 (8 index octets) and dK = 32 (4 octets).
#include <cmath>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <random>
#include <vector>

#include "../../linear_cost_attention_b200/csrc/sata_internal.h"
#include "../../linear_cost_attention_b200/csrc/tile_gen.cuh"
#include "../../linear_cost_attention_b200/csrc/tile_order.h"

using namespace sata;

// unit_weights: the readout's configuration (unweighted monomials; the
// weights live in the snapshots); then every feature is at most two bf16
// roundings from the exact product, else three (the weight adds one).
template <int G>
int check(int dK, int want_tiles, bool unit_weights) {
  TileOrder to;
  if (!build_tile_order(dK, &to)) {
    printf("FAIL build_tile_order dK=%d\n", dK);
    return 1;
  }
  HostBasis hb = build_host_basis(dK, 4);
  printf("dK %d: tiles %d slots %zu rows %lld\n", dK, to.n_tiles, to.row_of_slot.size(),
         (long long)hb.m);
  if (to.n_tiles != want_tiles) {
    printf("FAIL tile count\n");
    return 1;
  }
  // weights 1/sqrt(alpha! dK^(p/2)) by degree and multiplicity
  const double d = dK;
  tc::GenWeights W;
  W.w3 = (float)(1.0 / std::sqrt(std::pow(d, 1.5)));
  W.w3h = (float)(1.0 / std::sqrt(2.0 * std::pow(d, 1.5)));
  W.w3s = (float)(1.0 / std::sqrt(6.0 * std::pow(d, 1.5)));
  W.w2 = (float)(1.0 / std::sqrt(d));
  W.w2h = (float)(1.0 / std::sqrt(2.0 * d));
  W.w1 = (float)(1.0 / std::sqrt(std::sqrt(d)));
  if (unit_weights) W = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
  const double u = std::ldexp(1.0, -8);  // bf16 unit roundoff
  const double bound = unit_weights ? (1 + u) * (1 + u) - 1 : (1 + u) * (1 + u) * (1 + u) - 1;
  std::mt19937 rng(1234 + dK);
  std::normal_distribution<float> nd(0.f, 1.f);
  double worst = 0;
  long bad = 0;
  for (int trial = 0; trial < 16; ++trial) {
    // a token row in the 128-byte swizzled layout, at row index r (swizzle r % 8);
    // entries past dK are garbage that the generator must not read
    const uint32_t r = trial % 8;
    float x[64];
    uint16_t bits[64];
    for (int i = 0; i < 64; ++i) {
      const float val = i >= dK ? 1e30f : (trial == 15 ? (float)(i % 7) - 3.f : nd(rng));
      __nv_bfloat16 b = __float2bfloat16_rn(val);
      x[i] = __bfloat162float(b);
      memcpy(&bits[i], &b, 2);
    }
    alignas(16) uint8_t row[128];
    for (int i = 0; i < 64; ++i) {
      const int c = i / 8, e = i % 8;
      memcpy(row + (((uint32_t)c ^ r) << 4) + 2 * e, &bits[i], 2);
    }
    for (int t = 0; t < to.n_tiles; ++t) {
      uint32_t out[32];
      tc::gen_tile<G>(to.tiles[t], row, r, W, out);
      for (int p = 0; p < 64; ++p) {
        uint16_t h = (uint16_t)((out[p / 2] >> (16 * (p % 2))) & 0xffff);
        __nv_bfloat16 hbv;
        memcpy(&hbv, &h, 2);
        const float got = __bfloat162float(hbv);
        const int32_t row_id = to.row_of_slot[(size_t)t * 64 + p];
        double ref = 0.0;
        if (row_id >= 0) {
          ref = unit_weights ? 1.0 : hb.weight[row_id];
          for (int s = 0; s < hb.degree[row_id]; ++s) ref *= x[hb.ix[4 * row_id + s]];
        }
        const double err = std::fabs(got - ref);
        const double tol = bound * std::fabs(ref) + 1e-30;
        if (row_id < 0 ? got != 0.f : err > tol) {
          if (bad < 10)
            printf("mismatch dK %d tile %d type %d var %d slot %d row %d got %g ref %g\n", dK, t,
                   to.tiles[t].type, to.tiles[t].variant, p, row_id, got, ref);
          ++bad;
        }
        if (ref != 0) worst = std::fmax(worst, err / std::fabs(ref));
      }
    }
  }
  // the runs the readout's generator loops assume: C(G,3) x 8 OUTER tiles in
  // pairs for the two-tile path, then G (G-1) / 2 BC tiles of each variant
  {
    const int n3 = G * (G - 1) * (G - 2) / 6 * 8, nbc = G * (G - 1) / 2;
    for (int t = 0; t < n3; t += 2)
      if (!tc::outer_pair_ok(to.tiles[t], to.tiles[t + 1])) ++bad;
    for (int v = 0; v < 9; ++v)
      for (int t = n3 + v * nbc; t < n3 + (v + 1) * nbc; ++t)
        if (to.tiles[t].type != T_BC || to.tiles[t].variant != v) ++bad;
  }
  // the readout's two-tile path equals the one-tile path bit for bit
  long pair_bad = 0, pairs = 0;
  for (int trial = 0; trial < 4; ++trial) {
    const uint32_t r = trial % 8;
    alignas(16) uint8_t row[128];
    for (int i = 0; i < 128; i += 2) {
      __nv_bfloat16 b = __float2bfloat16_rn(nd(rng));
      memcpy(row + i, &b, 2);
    }
    for (int t = 0; t + 1 < to.n_tiles; ++t) {
      if (!tc::outer_pair_ok(to.tiles[t], to.tiles[t + 1])) continue;
      ++pairs;
      uint32_t a0[32], a1[32], b0[32], b1[32];
      tc::gen_tile<G>(to.tiles[t], row, r, W, a0);
      tc::gen_tile<G>(to.tiles[t + 1], row, r, W, a1);
      tc::gen_outer_pair(to.tiles[t], row, r, W, b0, b1);
      pair_bad += memcmp(a0, b0, sizeof a0) != 0 || memcmp(a1, b1, sizeof a1) != 0;
    }
  }
  bad += pair_bad;
  printf("dK %d%s: worst relative %.3e (bound %.3e) bad %ld, %ld two-tile checks\n", dK,
         unit_weights ? " unit weights" : "", worst, bound, bad, pairs);
  return bad ? 1 : 0;
}

// The state kernel's row groups: each row's factors (j, l, i_f, with dK
// standing for a ones row) are its index tuple; every basis row and every slot
// of the tile order (padded to an even tile count, as the library does) is
// used exactly once, with the row's weight.
int check_groups(int dK) {
  TileOrder to;
  if (!build_tile_order(dK, &to)) return 1;
  if (to.n_tiles % 2) {
    to.tiles.push_back({T_PAD, 0, 0, 0, 0, 0, 0, 0});
    to.row_of_slot.insert(to.row_of_slot.end(), 64, -1);
    to.n_tiles++;
  }
  StateGroups sg;
  if (!build_state_groups(dK, to, &sg)) {
    printf("FAIL build_state_groups dK=%d\n", dK);
    return 1;
  }
  HostBasis hb = build_host_basis(dK, 4);
  std::vector<int> row_hits(hb.m, 0), slot_hits(to.row_of_slot.size(), 0);
  long bad = 0;
  for (int it = 0; it < sg.n_items; ++it)
    for (int lane = 0; lane < 128; ++lane) {
      const uint64_t ix = sg.lane_idx[(size_t)it * 128 + lane];
      for (int f = 0; f < kGroupRows; ++f) {
        const size_t k = ((size_t)it * kGroupRows + f) * 128 + lane;
        const int r = sg.row[k], slot = sg.slot[k];
        if (slot >= 0) slot_hits[slot]++;
        if (r < 0) {
          if (sg.weight[k] != 0.f || (slot >= 0 && to.row_of_slot[slot] >= 0)) ++bad;
          continue;
        }
        row_hits[r]++;
        int fac[3] = {(int)((ix >> (16 + 8 * f)) & 0xff), (int)(ix & 0xff), (int)((ix >> 8) & 0xff)};
        std::vector<int> got, want;
        for (int q = 0; q < 3; ++q)
          if (fac[q] != dK) got.push_back(fac[q]);
        for (int q = 0; q < hb.degree[r]; ++q) want.push_back(hb.ix[4 * r + q]);
        std::sort(got.begin(), got.end());
        if (got != want || slot < 0 || to.row_of_slot[slot] != r ||
            sg.weight[k] != (float)hb.weight[r])
          ++bad;
      }
    }
  for (int64_t r = 0; r < hb.m; ++r) bad += row_hits[r] != 1;
  for (size_t k = 0; k < slot_hits.size(); ++k) bad += slot_hits[k] != 1;
  return bad ? 1 : 0;
}

int main() {
  int fails = check<8>(64, 749, false) + check<4>(32, 103, false) + check<8>(64, 749, true) +
              check<4>(32, 103, true) + check_groups(64) + check_groups(32);
  if (fails) {
    printf("FAIL\n");
    return 1;
  }
  printf("OK\n");
  return 0;
}
