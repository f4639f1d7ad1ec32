// Random-feature matrix W for FAVOR+ (host side of the C ABI).
//
// "Rethinking Attention with Performers", Abstract and section 제안 방법
// (proposed method): the softmax kernel is estimated with positive
// *orthogonal* random features.  W holds m rows; rows are drawn N(0, I_d),
// orthonormalised in blocks of d, and each is given the length of an
// independent N(0, I_d) vector (a chi(d) norm), so every row keeps the
// N(0, I_d) marginal while rows inside a block are exactly orthogonal.
//
// Random numbers: Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11) and the Box-Muller transform (Box and
// Muller 1958).  The stream convention is documented in favor.h.
#include <cmath>
#include <cstdint>
#include <new>
#include <vector>

#include "favor_internal.h"

namespace favor {
namespace {

constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull;
constexpr uint64_t kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kPhiloxW1 = 0xBB67AE8584CAA73Bull;

struct Block4 {
  uint64_t x[4];
};

inline void mulhilo(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo) {
  unsigned __int128 p = static_cast<unsigned __int128>(a) * b;
  *hi = static_cast<uint64_t>(p >> 64);
  *lo = static_cast<uint64_t>(p);
}

// Ten rounds; the key advances by the Weyl constants before rounds 2..10.
Block4 philox4x64_10(Block4 c, uint64_t k0, uint64_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo(kPhiloxM0, c.x[0], &hi0, &lo0);
    mulhilo(kPhiloxM1, c.x[2], &hi1, &lo1);
    c = Block4{{hi1 ^ c.x[1] ^ k0, lo1, hi0 ^ c.x[3] ^ k1, lo0}};
  }
  return c;
}

inline double to_unit(uint64_t x) {  // (top 52 bits + 1/2) * 2^-52, strictly inside (0, 1)
  return (static_cast<double>(x >> 12) + 0.5) * 0x1p-52;
}

// Normals 0..count-1 of stream `tag` under `seed`.
void normals(uint64_t seed, uint64_t tag, size_t count, double* out) {
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t j = 0; 4 * j < count; ++j) {
    Block4 x = philox4x64_10(Block4{{static_cast<uint64_t>(j), tag, 0, 0}}, seed, 0);
    double z[4];
    for (int p = 0; p < 2; ++p) {
      double r = std::sqrt(-2.0 * std::log(to_unit(x.x[2 * p])));
      double t = two_pi * to_unit(x.x[2 * p + 1]);
      z[2 * p] = r * std::cos(t);
      z[2 * p + 1] = r * std::sin(t);
    }
    for (int i = 0; i < 4 && 4 * j + i < count; ++i) out[4 * j + i] = z[i];
  }
}

// Orthonormalise the rows of the n x n block G in place, first row first.
// Row i loses its components along rows 0..i-1 (coefficients all taken from
// the same vector, then subtracted), twice, and is scaled to unit length.
void gram_schmidt_rows(double* G, int n, std::vector<double>& coef) {
  for (int i = 0; i < n; ++i) {
    double* v = G + static_cast<size_t>(i) * n;
    for (int pass = 0; pass < 2 && i > 0; ++pass) {
      for (int j = 0; j < i; ++j) {
        const double* q = G + static_cast<size_t>(j) * n;
        double s = 0.0;
        for (int k = 0; k < n; ++k) s += q[k] * v[k];
        coef[j] = s;
      }
      for (int j = 0; j < i; ++j) {
        const double* q = G + static_cast<size_t>(j) * n;
        for (int k = 0; k < n; ++k) v[k] -= coef[j] * q[k];
      }
    }
    double s = 0.0;
    for (int k = 0; k < n; ++k) s += v[k] * v[k];
    const double inv = 1.0 / std::sqrt(s);
    for (int k = 0; k < n; ++k) v[k] *= inv;
  }
}

}  // namespace

int make_features(uint64_t seed, int m, int d, int orthogonal, float* W_out) {
  if (!W_out || m < 1 || d < 1) return set_error(FAVOR_ERR_INVALID, "favor_make_features: null W_out or m, d < 1");
  const size_t nblk = (static_cast<size_t>(m) + d - 1) / d;
  const size_t dd = static_cast<size_t>(d) * d;
  try {
    std::vector<double> g(nblk * dd);
    normals(seed, 0, g.size(), g.data());
    if (!orthogonal) {
      for (size_t i = 0; i < static_cast<size_t>(m) * d; ++i) W_out[i] = static_cast<float>(g[i]);
      return FAVOR_OK;
    }
    std::vector<double> coef(d);
    for (size_t b = 0; b < nblk; ++b) gram_schmidt_rows(g.data() + b * dd, d, coef);
    std::vector<double> h(static_cast<size_t>(m) * d);
    normals(seed, 1, h.size(), h.data());
    for (int r = 0; r < m; ++r) {
      double s = 0.0;
      for (int k = 0; k < d; ++k) s += h[static_cast<size_t>(r) * d + k] * h[static_cast<size_t>(r) * d + k];
      const double norm = std::sqrt(s);
      for (int k = 0; k < d; ++k)
        W_out[static_cast<size_t>(r) * d + k] = static_cast<float>(g[static_cast<size_t>(r) * d + k] * norm);
    }
  } catch (const std::bad_alloc&) {
    return set_error(FAVOR_ERR_NOMEM, "favor_make_features: out of host memory");
  }
  return FAVOR_OK;
}

}  // namespace favor
