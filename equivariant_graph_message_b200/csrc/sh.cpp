// Real spherical harmonics as polynomials in the components of a unit vector.
//
// The basis (the one the library's CG tables are built for): component
// normalisation (sum_m Y_lm^2 = 2l+1 on the unit sphere), no Condon-Shortley
// phase, z polar axis, components m = -l..l at index l^2 + l + m:
//   Y_l0       = sqrt(2l+1) P_l(z)
//   Y_l(+m)    = N_lm P_l^(m)(z) Re (x + i y)^m      (m > 0)
//   Y_l(-m)    = N_lm P_l^(m)(z) Im (x + i y)^m
//   N_lm       = sqrt(2 (2l+1) (l-m)! / (l+m)!)
// with P_l the Legendre polynomial and P_l^(m) its m-th derivative.  For
// l = 1 this is sqrt(3) (y, z, x).  The spherical harmonics of e3j's edge
// features have parity (-1)^l (page "e3j.core.Convolution", edge irreps).
//
// P_l comes from Bonnet's recursion (n+1) P_{n+1} = (2n+1) z P_n - n P_{n-1};
// the products are expanded exactly in double precision.  The forward kernel
// evaluates these polynomials at r / |r| when it is given edge vectors.
#include <cmath>
#include <map>
#include <tuple>
#include <vector>

#include "plan.h"

namespace e3c {

namespace {

using Poly = std::map<std::tuple<int, int, int>, double>;  // (a, b, c) -> coefficient of x^a y^b z^c

void add(Poly& p, int a, int b, int c, double v) {
  if (v == 0.0) return;
  p[{a, b, c}] += v;
}

Poly mul(const Poly& p, const Poly& q) {
  Poly r;
  for (const auto& [ka, va] : p)
    for (const auto& [kb, vb] : q)
      add(r, std::get<0>(ka) + std::get<0>(kb), std::get<1>(ka) + std::get<1>(kb),
          std::get<2>(ka) + std::get<2>(kb), va * vb);
  return r;
}

// Legendre P_0..P_L as coefficient vectors in z (index = power).
std::vector<std::vector<double>> legendre(int L) {
  std::vector<std::vector<double>> P(L + 1);
  P[0] = {1.0};
  if (L >= 1) P[1] = {0.0, 1.0};
  for (int n = 1; n < L; ++n) {
    std::vector<double> next(n + 2, 0.0);
    for (size_t k = 0; k < P[n].size(); ++k) next[k + 1] += (2.0 * n + 1.0) * P[n][k];
    for (size_t k = 0; k < P[n - 1].size(); ++k) next[k] -= n * P[n - 1][k];
    for (double& v : next) v /= (n + 1.0);
    P[n + 1] = next;
  }
  return P;
}

double factorial(int n) {
  double f = 1.0;
  for (int k = 2; k <= n; ++k) f *= k;
  return f;
}

}  // namespace

std::vector<std::vector<ShMono>> sh_polynomials(int lmax) {
  const auto P = legendre(lmax);
  std::vector<std::vector<ShMono>> out((lmax + 1) * (lmax + 1));
  for (int l = 0; l <= lmax; ++l) {
    for (int m = 0; m <= l; ++m) {
      // m-th derivative of P_l, as a polynomial in z
      std::vector<double> d = P[l];
      for (int k = 0; k < m; ++k) {
        std::vector<double> dd(d.size() > 1 ? d.size() - 1 : 1, 0.0);
        for (size_t q = 1; q < d.size(); ++q) dd[q - 1] = q * d[q];
        d = dd;
      }
      Poly pz;
      for (size_t q = 0; q < d.size(); ++q) add(pz, 0, 0, static_cast<int>(q), d[q]);
      // (x + i y)^m = sum_k C(m,k) x^(m-k) (i y)^k: real part k even, imaginary part k odd
      Poly re, im;
      for (int k = 0; k <= m; ++k) {
        const double c = factorial(m) / (factorial(k) * factorial(m - k));
        const int ik = k % 4;  // i^k = 1, i, -1, -i
        if (ik == 0) add(re, m - k, k, 0, c);
        if (ik == 2) add(re, m - k, k, 0, -c);
        if (ik == 1) add(im, m - k, k, 0, c);
        if (ik == 3) add(im, m - k, k, 0, -c);
      }
      if (m == 0) {
        const double n0 = std::sqrt(2.0 * l + 1.0);
        for (const auto& [k, v] : pz)
          out[l * l + l].push_back({n0 * v, std::get<0>(k), std::get<1>(k), std::get<2>(k)});
        continue;
      }
      const double nlm = std::sqrt(2.0 * (2 * l + 1) * factorial(l - m) / factorial(l + m));
      for (int sgn : {+1, -1}) {
        const Poly prod = mul(pz, sgn > 0 ? re : im);
        auto& dst = out[l * l + l + sgn * m];
        for (const auto& [k, v] : prod)
          if (v != 0.0) dst.push_back({nlm * v, std::get<0>(k), std::get<1>(k), std::get<2>(k)});
      }
    }
  }
  return out;
}

}  // namespace e3c
