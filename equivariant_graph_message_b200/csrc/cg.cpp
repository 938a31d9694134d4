// Real-basis Wigner-3j tensors from the Racah closed form.
//
// 1. Complex Clebsch-Gordan coefficients <l1 m1 l2 m2 | l3 m3> (Condon-Shortley
//    phase) from Racah's single-sum formula, in long double.
// 2. The unitary map U from complex harmonics Y_l^m to the real basis used by
//    the library (component-normalised, no Condon-Shortley phase, m = -l..l,
//    l = 1 ~ (y, z, x)):
//      real m > 0 :  ((-1)^m Y^m + Y^-m) / sqrt(2)
//      real m = 0 :  Y^0
//      real m < 0 :  i (Y^-|m| - (-1)^|m| Y^|m|) / sqrt(2)
// 3. Harmonic function values transform with the complex-conjugate
//    representation, for which the (real) CG coefficients are still an
//    intertwiner, so the real tensor that maps real values r1, r2 to r3 is
//      W_ijk = sum U3[k][m3] CG(m1, m2, m3) conj(U1[i][m1]) conj(U2[j][m2]).
//    W is real or purely imaginary (a global phase); the nonzero part is
//    taken, scaled to unit Frobenius norm, and its sign fixed so the first
//    entry with |W| > 1e-9 in row-major (i, j, k) order is positive.
#include <cmath>
#include <complex>
#include <stdexcept>
#include <vector>

#include "plan.h"

namespace e3c {

using ld = long double;
using cplx = std::complex<ld>;

static ld fact(int n) {
  ld r = 1;
  for (int k = 2; k <= n; ++k) r *= k;
  return r;
}

// <j1 m1 j2 m2 | J M>
static ld clebsch_gordan(int j1, int m1, int j2, int m2, int J, int M) {
  if (m1 + m2 != M) return 0;
  if (std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0;
  if (J < std::abs(j1 - j2) || J > j1 + j2) return 0;
  ld pre = std::sqrt((2 * J + 1) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
                     fact(j1 + j2 + J + 1));
  pre *= std::sqrt(fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) * fact(j2 - m2) *
                   fact(j2 + m2));
  int kmin = 0;
  kmin = std::max(kmin, j2 - J - m1);
  kmin = std::max(kmin, j1 - J + m2);
  int kmax = j1 + j2 - J;
  kmax = std::min(kmax, j1 - m1);
  kmax = std::min(kmax, j2 + m2);
  ld sum = 0;
  for (int k = kmin; k <= kmax; ++k) {
    ld den = fact(k) * fact(j1 + j2 - J - k) * fact(j1 - m1 - k) * fact(j2 + m2 - k) *
             fact(J - j2 + m1 + k) * fact(J - j1 - m2 + k);
    sum += ((k % 2) ? -1.0L : 1.0L) / den;
  }
  return pre * sum;
}

// U[(m+l)*(2l+1) + (m'+l)]: real component m from complex component m'.
static std::vector<cplx> real_from_complex(int l) {
  const int d = 2 * l + 1;
  std::vector<cplx> U(static_cast<size_t>(d) * d, cplx(0, 0));
  const ld r2 = 1.0L / std::sqrt(2.0L);
  auto at = [&](int m, int mp) -> cplx& { return U[(m + l) * d + (mp + l)]; };
  at(0, 0) = cplx(1, 0);
  for (int m = 1; m <= l; ++m) {
    ld sgn = (m % 2) ? -1.0L : 1.0L;
    at(m, m) = cplx(sgn * r2, 0);
    at(m, -m) = cplx(r2, 0);
    at(-m, m) = cplx(0, -sgn * r2);
    at(-m, -m) = cplx(0, r2);
  }
  return U;
}

std::vector<double> real_wigner_3j(int l1, int l2, int l3) {
  if (l3 < std::abs(l1 - l2) || l3 > l1 + l2) throw std::invalid_argument("triangle rule");
  const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
  std::vector<cplx> U1 = real_from_complex(l1), U2 = real_from_complex(l2),
                    U3 = real_from_complex(l3);
  std::vector<cplx> W(static_cast<size_t>(d1) * d2 * d3, cplx(0, 0));
  for (int m1 = -l1; m1 <= l1; ++m1)
    for (int m2 = -l2; m2 <= l2; ++m2) {
      int m3 = m1 + m2;
      if (std::abs(m3) > l3) continue;
      ld c = clebsch_gordan(l1, m1, l2, m2, l3, m3);
      if (c == 0) continue;
      for (int i = 0; i < d1; ++i) {
        cplx a = std::conj(U1[i * d1 + (m1 + l1)]);
        if (a == cplx(0, 0)) continue;
        for (int j = 0; j < d2; ++j) {
          cplx b = std::conj(U2[j * d2 + (m2 + l2)]);
          if (b == cplx(0, 0)) continue;
          for (int k = 0; k < d3; ++k) {
            cplx u = U3[k * d3 + (m3 + l3)];
            if (u == cplx(0, 0)) continue;
            W[(i * d2 + j) * d3 + k] += u * c * a * b;
          }
        }
      }
    }
  ld nre = 0, nim = 0;
  for (const auto& w : W) {
    nre += w.real() * w.real();
    nim += w.imag() * w.imag();
  }
  const bool use_re = nre >= nim;
  ld norm = std::sqrt(use_re ? nre : nim);
  std::vector<double> out(W.size());
  for (size_t q = 0; q < W.size(); ++q)
    out[q] = static_cast<double>((use_re ? W[q].real() : W[q].imag()) / norm);
  for (double v : out)
    if (std::fabs(v) > 1e-9) {
      if (v < 0)
        for (double& w : out) w = -w;
      break;
    }
  for (double& v : out)
    if (std::fabs(v) < 1e-15) v = 0.0;
  return out;
}

}  // namespace e3c
