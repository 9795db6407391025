// Device-side generation of one 64-feature tile of the tile order
// (tile_order.h) for one token, dK = 8 G (G = 8 or 4 index octets).
//
// The token's bf16 row sits in shared memory as a 128-byte row in the
// 128-byte-swizzled layout a TMA load produces: element i is in 16-byte chunk
// i/8, stored at chunk position (i/8) ^ (row % 8); for dK = 32 only chunks
// 0..3 are read.  The 64 outputs are returned as 32 packed bf16x2 words in
// tile order.
//
// Arithmetic (feature = w_alpha * prod x): OUTER and BC tiles form bf16x2
// pairs of partial products u = w * x_i * x_j (OUTER: w x_i rounded to bf16,
// exact for the unit weights the readout uses, times x_j with a packed
// multiply; BC: in fp32) rounded to bf16, and multiply them by the packed
// words of the third octet, halves swapped or not (two roundings); D and MISC
// tiles (21 of 749) load the octets they touch once and form each product in
// fp32, rounding once.
#pragma once

#include <cuda_bf16.h>
#include <string.h>

#include <utility>

#include "tc_common.cuh"
#include "tile_order.h"

#ifndef SATA_HD
#define SATA_HD __host__ __device__ __forceinline__
#endif

namespace sata {
namespace tc {

// Basis weights 1/sqrt(alpha! * dK^(p/2)).
struct GenWeights {
  float w3, w3h;  // degree 3: alpha! = 1, 2
  float w3s;      // degree 3: alpha! = 6
  float w2, w2h;  // degree 2: alpha! = 1, 2
  float w1;       // degree 1
};

SATA_HD float bits_f32(uint32_t b) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(b);
#else
  float f;
  memcpy(&f, &b, 4);
  return f;
#endif
}

SATA_HD float bf16_bits_to_f32(uint32_t bits16) { return bits_f32(bits16 << 16); }

SATA_HD uint4 load_chunk(const uint8_t *row, uint32_t rsw, int c) {
  return *reinterpret_cast<const uint4 *>(row + (((uint32_t)c ^ rsw) << 4));
}

SATA_HD void unpack8(uint4 r, float (&o)[8]) {
  o[0] = bits_f32(r.x << 16);
  o[1] = bits_f32(r.x & 0xffff0000u);
  o[2] = bits_f32(r.y << 16);
  o[3] = bits_f32(r.y & 0xffff0000u);
  o[4] = bits_f32(r.z << 16);
  o[5] = bits_f32(r.z & 0xffff0000u);
  o[6] = bits_f32(r.w << 16);
  o[7] = bits_f32(r.w & 0xffff0000u);
}

SATA_HD float load_elem(const uint8_t *row, uint32_t rsw, int i) {
  const uint16_t b =
      *reinterpret_cast<const uint16_t *>(row + ((((uint32_t)i >> 3) ^ rsw) << 4) + ((i & 7) << 1));
  return bf16_bits_to_f32(b);
}

SATA_HD uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 x, y, z;
  memcpy(&x, &a, 4);
  memcpy(&y, &b, 4);
  z = __hmul2(x, y);
  uint32_t r;
  memcpy(&r, &z, 4);
  return r;
}

SATA_HD uint32_t splat_bf16(float u) {
  __nv_bfloat162 v = __float2bfloat162_rn(u);
  uint32_t r;
  memcpy(&r, &v, 4);
  return r;
}

SATA_HD uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  uint32_t r;
  memcpy(&r, &v, 4);
  return r;
}

// u * (8 values of chunk r) -> out[4*slot .. 4*slot+3]
// 32-bit word holding elements i and i + 1 (i even) of the row.
SATA_HD uint32_t load_pair(const uint8_t *row, uint32_t rsw, int i) {
  return *reinterpret_cast<const uint32_t *>(row + ((((uint32_t)i >> 3) ^ rsw) << 4) +
                                             ((i & 7) << 1));
}

SATA_HD uint32_t swap_halves(uint32_t x) { return (x >> 16) | (x << 16); }

// The 32 words of an OUTER / BC tile from four bf16x2 pairs of partial
// products u[k] (word w uses u[w / 8]) and the third octet's chunk r: word w
// = u[w / 8] * r_j or * swap(r_j), j = (w % 8) / 2 (tile_order.h, outer_c).
SATA_HD void outer_words(const uint32_t (&u)[4], uint4 r, uint32_t (&out)[32]) {
  const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t rs = swap_halves(rw[j]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[8 * k + 2 * j] = bmul2(u[k], rw[j]);
      out[8 * k + 2 * j + 1] = bmul2(u[k], rs);
    }
  }
}

// OUTER: u pairs (s x_b, s x_(b+1)) with s = w x_i1 (w alone for degree 2),
// rounded to bf16, times the third octet's words.
SATA_HD void gen_outer(const TileDesc &td, const uint8_t *row, uint32_t rsw,
                       const GenWeights &W, uint32_t (&out)[32]) {
  const uint4 g = load_chunk(row, rsw, td.o0);
  const uint4 rc = load_chunk(row, rsw, td.o1);
  const uint32_t sp = splat_bf16(
      (td.wsel == 0 ? W.w3 : W.w2) * (td.i1 != kNoIndex ? load_elem(row, rsw, td.i1) : 1.f));
  const uint32_t u[4] = {bmul2(sp, g.x), bmul2(sp, g.y), bmul2(sp, g.z), bmul2(sp, g.w)};
  outer_words(u, rc, out);
}

// Two consecutive degree-3 OUTER tiles that differ only in i1 (i1 even, then
// i1 + 1): the octet chunks and the i1 pair are loaded once.
SATA_HD void gen_outer_pair(const TileDesc &td, const uint8_t *row, uint32_t rsw,
                            const GenWeights &W, uint32_t (&out0)[32], uint32_t (&out1)[32]) {
  const uint4 g = load_chunk(row, rsw, td.o0);
  const uint4 rc = load_chunk(row, rsw, td.o1);
  const uint32_t xi = load_pair(row, rsw, td.i1);
  const uint32_t s0 = splat_bf16(W.w3 * bf16_bits_to_f32(xi & 0xffffu));
  const uint32_t s1 = splat_bf16(W.w3 * bits_f32(xi & 0xffff0000u));
  const uint32_t u0[4] = {bmul2(s0, g.x), bmul2(s0, g.y), bmul2(s0, g.z), bmul2(s0, g.w)};
  const uint32_t u1[4] = {bmul2(s1, g.x), bmul2(s1, g.y), bmul2(s1, g.z), bmul2(s1, g.w)};
  outer_words(u0, rc, out0);
  outer_words(u1, rc, out1);
}

// True when tiles t, t + 1 can take gen_outer_pair.
SATA_HD bool outer_pair_ok(const TileDesc &a, const TileDesc &b) {
  return a.type == T_OUTER && b.type == T_OUTER && a.i1 != kNoIndex && (a.i1 & 1) == 0 &&
         b.i1 == a.i1 + 1 && a.o0 == b.o0 && a.o1 == b.o1 && a.wsel == b.wsel;
}

// ---- BC: tile variant T; chunk cc holds pair k = 8 T + cc (block k / 36 of
// the tile's two octet pairs); chunks 2q, 2q + 1 share the third octet
template <int T, int CC>
SATA_HD float bc_pair_product(const float (&g0)[8], const float (&g1)[8], const GenWeights &W) {
  constexpr int k = 8 * T + CC, blk = k / 36, p = k % 36;
  constexpr int a = pair_a(p), b = pair_b(p);
  const float w = (a == b) ? W.w3h : W.w3;
  return blk == 0 ? w * g0[a] * g0[b] : w * g1[a] * g1[b];
}

template <int T, int Q>
SATA_HD uint32_t bc_u(const float (&g0)[8], const float (&g1)[8], const GenWeights &W) {
  return pack2(bc_pair_product<T, 2 * Q>(g0, g1, W), bc_pair_product<T, 2 * Q + 1>(g0, g1, W));
}

template <int T>
SATA_HD void gen_bc(const TileDesc &td, const uint8_t *row, uint32_t rsw,
                    const GenWeights &W, uint32_t (&out)[32]) {
  constexpr bool need0 = 8 * T < 36, need1 = 8 * T + 7 >= 36;
  float g0[8] = {0, 0, 0, 0, 0, 0, 0, 0}, g1[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint4 r0 = make_uint4(0, 0, 0, 0), r1 = make_uint4(0, 0, 0, 0);
  if (need0) {
    unpack8(load_chunk(row, rsw, td.o0), g0);
    r0 = load_chunk(row, rsw, td.o1);
  }
  if (need1) {
    unpack8(load_chunk(row, rsw, td.o2), g1);
    r1 = load_chunk(row, rsw, td.o3);
  }
  const uint32_t u[4] = {bc_u<T, 0>(g0, g1, W), bc_u<T, 1>(g0, g1, W), bc_u<T, 2>(g0, g1, W),
                         bc_u<T, 3>(g0, g1, W)};
  // the block boundary (pair 36) falls on an even chunk, so both chunks of a
  // word use one third octet; words of chunks in block 1 use r1
  const uint32_t rw0[4] = {r0.x, r0.y, r0.z, r0.w}, rw1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const bool b1 = (8 * T + 2 * q) >= 36;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t rj = b1 ? rw1[j] : rw0[j];
      out[8 * q + 2 * j] = bmul2(u[q], rj);
      out[8 * q + 2 * j + 1] = bmul2(u[q], swap_halves(rj));
    }
  }
}

// ---- D: features 64*T + P of the concatenated in-octet triples; a tile
// touches at most two octets, loaded once (ga = first, gb = second).
template <int G, int T> struct DOctets {
  static constexpr int ga = (64 * T) / 120;
  static constexpr int gb = (64 * T + 63) / 120 < G ? (64 * T + 63) / 120 : G - 1;
};

template <int G, int T, int P>
SATA_HD float d_feature(const float (&xa)[8], const float (&xb)[8], const GenWeights &W) {
  constexpr int f = 64 * T + P;
  if constexpr (f >= 120 * G) {
    return 0.f;
  } else {
    constexpr int g = f / 120, r = f % 120;
    constexpr int a = triple_at(r, 0), b = triple_at(r, 1), c = triple_at(r, 2);
    constexpr int fa = fact3(a, b, c);
    const float w = fa == 1 ? W.w3 : fa == 2 ? W.w3h : W.w3s;
    const float(&x)[8] = (g == DOctets<G, T>::ga) ? xa : xb;
    return w * x[a] * x[b] * x[c];
  }
}

template <int G, int T, int... Q>
SATA_HD void d_variant(const uint8_t *row, uint32_t rsw, const GenWeights &W,
                       uint32_t (&out)[32], std::integer_sequence<int, Q...>) {
  float xa[8], xb[8];
  unpack8(load_chunk(row, rsw, DOctets<G, T>::ga), xa);
  unpack8(load_chunk(row, rsw, DOctets<G, T>::gb), xb);
  ((out[Q] = pack2(d_feature<G, T, 2 * Q>(xa, xb, W), d_feature<G, T, 2 * Q + 1>(xa, xb, W))),
   ...);
}

// ---- MISC: in-octet pairs (degree 2), degree 1, degree 0, padding.  The
// octets a tile needs are loaded once into registers (mask of octets).
template <int G, int T> struct MiscOctets {
  static constexpr int n2 = 36 * G, n1 = 8 * G;
  static constexpr int octet_of(int f) {
    return f < n2 ? f / 36 : (f < n2 + n1 ? (f - n2) / 8 : -1);
  }
  static constexpr unsigned mask() {
    unsigned m = 0;
    for (int p = 0; p < 64; ++p) {
      const int g = octet_of(64 * T + p);
      if (g >= 0) m |= 1u << g;
    }
    return m;
  }
};

template <int G, int T, int P>
SATA_HD float misc_feature(const float (&xo)[8][8], const GenWeights &W) {
  constexpr int f = 64 * T + P;
  constexpr int n2 = 36 * G, n1 = 8 * G;
  if constexpr (f < n2) {
    constexpr int g = f / 36, pr = f % 36;
    constexpr int a = pair_a(pr), b = pair_b(pr);
    return (a == b ? W.w2h : W.w2) * xo[g][a] * xo[g][b];
  } else if constexpr (f < n2 + n1) {
    return W.w1 * xo[(f - n2) / 8][(f - n2) % 8];
  } else if constexpr (f == n2 + n1) {
    return 1.f;
  } else {
    return 0.f;
  }
}

template <int G, int T, int... O>
SATA_HD void misc_load(const uint8_t *row, uint32_t rsw, float (&xo)[8][8],
                       std::integer_sequence<int, O...>) {
  (((MiscOctets<G, T>::mask() >> O) & 1u ? unpack8(load_chunk(row, rsw, O), xo[O]) : void()),
   ...);
}

template <int G, int T, int... Q>
SATA_HD void misc_variant(const uint8_t *row, uint32_t rsw, const GenWeights &W,
                          uint32_t (&out)[32], std::integer_sequence<int, Q...>) {
  float xo[8][8];
  misc_load<G, T>(row, rsw, xo, std::make_integer_sequence<int, G>{});
  ((out[Q] = pack2(misc_feature<G, T, 2 * Q>(xo, W), misc_feature<G, T, 2 * Q + 1>(xo, W))),
   ...);
}

// D and MISC tiles: variant v of the G-octet tile order (the switch keeps
// every tile's indices compile-time constants).
template <int G, int V = 0>
SATA_HD void gen_d(int v, const uint8_t *row, uint32_t rsw, const GenWeights &W,
                   uint32_t (&out)[32]) {
  constexpr int nD = (120 * G + 63) / 64;
  if constexpr (V < nD) {
    if (v == V) {
      d_variant<G, V>(row, rsw, W, out, std::make_integer_sequence<int, 32>{});
      return;
    }
    gen_d<G, V + 1>(v, row, rsw, W, out);
  }
}
template <int G, int V = 0>
SATA_HD void gen_misc(int v, const uint8_t *row, uint32_t rsw, const GenWeights &W,
                      uint32_t (&out)[32]) {
  constexpr int nM = (36 * G + 8 * G + 1 + 63) / 64;
  if constexpr (V < nM) {
    if (v == V) {
      misc_variant<G, V>(row, rsw, W, out, std::make_integer_sequence<int, 32>{});
      return;
    }
    gen_misc<G, V + 1>(v, row, rsw, W, out);
  }
}

// Generates tile td for the token whose swizzled row starts at `row`
// (rsw = row index % 8 of that token inside its 8-row atom); G = dK / 8.
template <int G>
SATA_HD void gen_tile(const TileDesc &td, const uint8_t *row, uint32_t rsw,
                                         const GenWeights &W, uint32_t (&out)[32]) {
  switch (td.type) {
    case T_OUTER:
      gen_outer(td, row, rsw, W, out);
      return;
    case T_BC:
      switch (td.variant) {
        case 0: gen_bc<0>(td, row, rsw, W, out); return;
        case 1: gen_bc<1>(td, row, rsw, W, out); return;
        case 2: gen_bc<2>(td, row, rsw, W, out); return;
        case 3: gen_bc<3>(td, row, rsw, W, out); return;
        case 4: gen_bc<4>(td, row, rsw, W, out); return;
        case 5: gen_bc<5>(td, row, rsw, W, out); return;
        case 6: gen_bc<6>(td, row, rsw, W, out); return;
        case 7: gen_bc<7>(td, row, rsw, W, out); return;
        default: gen_bc<8>(td, row, rsw, W, out); return;
      }
    case T_D:
      gen_d<G>(td.variant, row, rsw, W, out);
      return;
    case T_MISC:
      gen_misc<G>(td.variant, row, rsw, W, out);
      return;
    default:
#pragma unroll
      for (int i = 0; i < 32; ++i) out[i] = 0u;
      return;
  }
}

// Stores the 64 generated features as row `r` of a 128-byte-swizzled tile.
__device__ __forceinline__ void store_tile_row(uint8_t *tile, uint32_t r,
                                               const uint32_t (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4 *>(tile + sw128_offset(r, (uint32_t)c)) =
        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

}  // namespace tc
}  // namespace sata
