// Paley construction I of the order-28 skew Hadamard matrix over GF(27).
//
// GF(27) = GF(3)[t] / (t^3 + 2t + 1). An element is the trit vector (c0, c1, c2) of
// c0 + c1 t + c2 t^2, numbered e = c0 + 3 c1 + 9 c2. Since t^3 = -2t - 1 = t + 2 (mod 3),
// multiplying by t maps (c0, c1, c2) to (2 c2, c0 + c2, c1); a product is formed by Horner's rule
// over the trits of one factor.
//
// With chi the quadratic character (+1 on the 13 nonzero squares, -1 on the other 13 nonzero
// elements, 0 at 0) and the Jacobsthal matrix Q[e][f] = chi(e - f), the matrix is
// H = I + [[0, 1^T], [-1, Q]]: row 0 is all +1, column 0 is (1, -1, ..., -1), and row/column
// 1 + e belongs to field element e. Because 27 = 3 (mod 4), -1 is a non-square, Q is skew, and
// H H^T = 28 I with H + H^T = 2 I.
#include <cstdint>

#include "signrot_internal.h"

namespace signrot {
namespace {

struct Gf27 {
  static int trit(int e, int i) { return i == 0 ? e % 3 : (i == 1 ? (e / 3) % 3 : e / 9); }
  static int make(int c0, int c1, int c2) {
    return ((c0 % 3 + 3) % 3) + 3 * ((c1 % 3 + 3) % 3) + 9 * ((c2 % 3 + 3) % 3);
  }
  static int add(int u, int v) {
    return make(trit(u, 0) + trit(v, 0), trit(u, 1) + trit(v, 1), trit(u, 2) + trit(v, 2));
  }
  static int neg(int u) { return make(-trit(u, 0), -trit(u, 1), -trit(u, 2)); }
  static int times_t(int u) {
    const int c0 = trit(u, 0), c1 = trit(u, 1), c2 = trit(u, 2);
    return make(2 * c2, c0 + c2, c1);
  }
  static int scale(int u, int k) {  // k in {0, 1, 2}
    int r = 0;
    for (int i = 0; i < k; ++i) r = add(r, u);
    return r;
  }
  static int mul(int u, int v) {
    int r = 0;
    for (int i = 2; i >= 0; --i) r = add(times_t(r), scale(u, trit(v, i)));
    return r;
  }
};

}  // namespace

void paley_h28(int8_t h[28][28]) {
  bool square[27] = {};
  for (int y = 1; y < 27; ++y) square[Gf27::mul(y, y)] = true;
  auto chi = [&](int e) { return e == 0 ? 0 : (square[e] ? 1 : -1); };
  for (int i = 0; i < 28; ++i) {
    for (int j = 0; j < 28; ++j) {
      int v;
      if (i == 0) {
        v = 1;
      } else if (j == 0) {
        v = -1;
      } else {
        const int e = i - 1, f = j - 1;
        v = (e == f ? 1 : 0) + chi(Gf27::add(e, Gf27::neg(f)));
      }
      h[i][j] = static_cast<int8_t>(v);
    }
  }
}

}  // namespace signrot
