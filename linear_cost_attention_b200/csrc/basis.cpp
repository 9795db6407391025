// Host-side minimal symmetric basis for the GPU path.
//
// "对称性感知泰勒近似注意力机制的恒定计算成本工程实现" (blog.hotdry.top), section
// "对称张量分解的核心洞察": an order-p symmetric tensor is fully described by the
// entries of its upper-triangular region, i.e. by the sorted index tuples
// i_1 <= ... <= i_p; there are C(dK+p-1, p) of them and the tables M_p listing
// them are fixed once dK and p are.  Section "硬件优化路径与当前局限" names the
// same ordering i_1 <= i_2 <= ... <= i_p.
//
// Weights: grouping the dK^p ordered monomials of (q.k)^p by their sorted form
// gives p!/alpha! copies of each (multinomial theorem, alpha! = product of the
// factorials of the index multiplicities).  With the Taylor factor
// 1/(p! dK^(p/2)) of (q.k/sqrt(dK))^p/p!, each sorted tuple carries
// 1/(alpha! dK^(p/2)); the library gives each side (query and key) the square
// root, w = 1/sqrt(alpha! dK^(p/2)).
#include <cmath>
#include <cstring>

#include "sata_internal.h"

namespace sata {

int64_t count_basis(int dK, int P) {
  if (dK < 1 || P < 1) return -1;
  // m = sum_{p<P} C(dK+p-1, p), built up term by term: C(n, p) = C(n, p-1)*(n-p+1)/p
  long double total = 0;
  int64_t m = 0;
  for (int p = 0; p < P; ++p) {
    // C(dK+p-1, p) computed exactly in 128-bit-ish steps via the product formula
    unsigned __int128 c = 1;
    for (int r = 1; r <= p; ++r) {
      c = c * (unsigned __int128)(dK + r - 1) / (unsigned __int128)r;
      if (c > (unsigned __int128)INT64_MAX) return -1;
    }
    total += (long double)c;
    if (total > (long double)INT64_MAX) return -1;
    m += (int64_t)c;
  }
  return m;
}

// Next sorted tuple in lexicographic order (in place); false after the last one.
static bool next_sorted_tuple(int *t, int p, int dK) {
  int pos = p - 1;
  while (pos >= 0 && t[pos] == dK - 1) --pos;
  if (pos < 0) return false;
  int val = t[pos] + 1;
  for (int r = pos; r < p; ++r) t[r] = val;  // smallest sorted continuation
  return true;
}

HostBasis build_host_basis(int dK, int P) {
  HostBasis b;
  b.dK = dK;
  b.P = P;
  for (int p = 0; p < P; ++p) {
    int t[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    bool more = true;
    while (more) {
      // alpha! over runs of equal indices
      double fact = 1.0;
      int run = 1;
      for (int r = 1; r <= p; ++r) {
        if (r < p && t[r] == t[r - 1]) {
          ++run;
        } else {
          for (int f = 2; f <= run; ++f) fact *= f;
          run = 1;
        }
      }
      b.degree.push_back((uint8_t)p);
      for (int s = 0; s < 4; ++s) b.ix.push_back((uint8_t)(s < p ? t[s] : dK));
      b.weight.push_back(1.0 / std::sqrt(fact * std::pow((double)dK, 0.5 * p)));
      ++b.m;
      more = (p > 0) && next_sorted_tuple(t, p, dK);
    }
  }
  return b;
}

}  // namespace sata

extern "C" int64_t sata_basis_size(int dK, int P) { return sata::count_basis(dK, P); }

extern "C" int64_t sata_index_table(int dK, int p, int32_t *host_out, int64_t cap_elems) {
  if (dK < 1 || p < 0 || p > 16) return -1;
  int64_t rows = sata::count_basis(dK, p + 1) - (p > 0 ? sata::count_basis(dK, p) : 0);
  if (rows < 1) return -1;
  if (p == 0) return 1;
  if (host_out == nullptr || cap_elems < rows * p) return -1;
  int t[16] = {0};
  int64_t r = 0;
  do {
    for (int s = 0; s < p; ++s) host_out[r * p + s] = t[s];
    ++r;
  } while (sata::next_sorted_tuple(t, p, dK));
  return r;
}
