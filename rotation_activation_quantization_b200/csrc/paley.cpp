// Paley construction I of skew Hadamard matrices of order q + 1 over GF(q), q = p^3 = 3 (mod 4):
// order 28 over GF(27) and order 344 over GF(343).
//
// GF(p^3) = GF(p)[t] / (t^3 + m2 t^2 + m1 t + m0) for an irreducible cubic. An element is the
// digit vector (c0, c1, c2) of c0 + c1 t + c2 t^2, numbered e = c0 + p c1 + p^2 c2. Since
// t^3 = -(m2 t^2 + m1 t + m0), multiplying by t maps (c0, c1, c2) to
// (-m0 c2, c0 - m1 c2, c1 - m2 c2); a product is formed by Horner's rule over the digits of one
// factor. The fields used: GF(27) with t^3 + 2t + 1, GF(343) with t^3 + t + 1.
//
// With chi the quadratic character (+1 on the (q-1)/2 nonzero squares, -1 on the other nonzero
// elements, 0 at 0) and the Jacobsthal matrix Q[e][f] = chi(e - f), the matrix is
// H = I + [[0, 1^T], [-1, Q]]: row 0 is all +1, column 0 is (1, -1, ..., -1), and row/column
// 1 + e belongs to field element e. Because q = 3 (mod 4), -1 is a non-square, Q is skew, and
// H H^T = (q + 1) I with H + H^T = 2 I.
#include <cstdint>
#include <vector>

#include "signrot_internal.h"

namespace signrot {
namespace {

class GfCube {
 public:
  GfCube(int p, int m0, int m1, int m2) : p_(p), m0_(m0), m1_(m1), m2_(m2) {}
  int size() const { return p_ * p_ * p_; }
  int digit(int e, int i) const { return i == 0 ? e % p_ : (i == 1 ? (e / p_) % p_ : e / (p_ * p_)); }
  int make(int c0, int c1, int c2) const { return red(c0) + p_ * red(c1) + p_ * p_ * red(c2); }
  int add(int u, int v) const {
    return make(digit(u, 0) + digit(v, 0), digit(u, 1) + digit(v, 1), digit(u, 2) + digit(v, 2));
  }
  int sub(int u, int v) const {
    return make(digit(u, 0) - digit(v, 0), digit(u, 1) - digit(v, 1), digit(u, 2) - digit(v, 2));
  }
  int times_t(int u) const {
    const int c0 = digit(u, 0), c1 = digit(u, 1), c2 = digit(u, 2);
    return make(-m0_ * c2, c0 - m1_ * c2, c1 - m2_ * c2);
  }
  int scale(int u, int k) const { return make(k * digit(u, 0), k * digit(u, 1), k * digit(u, 2)); }
  int mul(int u, int v) const {
    int r = 0;
    for (int i = 2; i >= 0; --i) r = add(times_t(r), scale(u, digit(v, i)));
    return r;
  }
  std::vector<bool> squares() const {
    std::vector<bool> sq(size(), false);
    for (int y = 1; y < size(); ++y) sq[mul(y, y)] = true;
    return sq;
  }

 private:
  int red(int c) const { return ((c % p_) + p_) % p_; }
  int p_, m0_, m1_, m2_;
};

const GfCube& gf27() {
  static const GfCube f(3, 1, 2, 0);
  return f;
}
const GfCube& gf343() {
  static const GfCube f(7, 1, 1, 0);
  return f;
}

// Row-major order-(q+1) matrix into h.
void paley_matrix(const GfCube& f, int8_t* h) {
  const int q = f.size(), N = q + 1;
  const std::vector<bool> sq = f.squares();
  for (int i = 0; i < N; ++i) {
    for (int j = 0; j < N; ++j) {
      int v;
      if (i == 0) {
        v = 1;
      } else if (j == 0) {
        v = -1;
      } else {
        const int d = f.sub(i - 1, j - 1);
        v = (d == 0 ? 1 : 0) + (d == 0 ? 0 : (sq[d] ? 1 : -1));
      }
      h[i * N + j] = static_cast<int8_t>(v);
    }
  }
}

}  // namespace

void paley_h28(int8_t h[28][28]) { paley_matrix(gf27(), &h[0][0]); }

void paley_h344(int8_t* h) { paley_matrix(gf343(), h); }

GF343Squares gf343_squares() {
  GF343Squares out{};
  const std::vector<bool> sq = gf343().squares();
  for (int e = 0; e < 343; ++e)
    if (sq[e]) out.bits[e >> 5] |= 1u << (e & 31);
  return out;
}

}  // namespace signrot
