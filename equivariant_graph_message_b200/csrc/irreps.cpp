// Irreps parsing and uvu path enumeration.
//
// Paths follow the selection rule of a Clebsch-Gordan product of O(3)
// irreps: (l1, p1) x (l2, (-1)^l2) -> (l3, p3) with |l1 - l2| <= l3 <= l1 + l2
// and p3 = p1 (-1)^l2; the edge features are spherical harmonics of parity
// (-1)^l (e3j.core.Convolution, note on graded-symmetric edge features).
// The requested output irreps act as a filter (e3j "target": a filter on the
// output irreducible blocks); irreps no path produces are dropped.
#include <cctype>
#include <cmath>
#include <set>
#include <utility>

#include "plan.h"

namespace e3c {

bool parse_irreps(const char* text, std::vector<Irrep>& out, std::string& err) {
  out.clear();
  if (!text) {
    err = "irreps string is NULL";
    return false;
  }
  std::string s;
  for (const char* c = text; *c; ++c)
    if (!std::isspace(static_cast<unsigned char>(*c))) s.push_back(*c);
  size_t pos = 0;
  while (pos <= s.size()) {
    size_t end = s.find('+', pos);
    if (end == std::string::npos) end = s.size();
    std::string term = s.substr(pos, end - pos);
    if (term.empty()) {
      err = "empty term in irreps '" + std::string(text) + "'";
      return false;
    }
    long mul = 1;
    size_t x = term.find('x');
    std::string rest = term;
    if (x != std::string::npos) {
      std::string m = term.substr(0, x);
      if (m.empty() || m.size() > 7) {
        err = "bad multiplicity in '" + term + "'";
        return false;
      }
      for (char ch : m)
        if (!std::isdigit(static_cast<unsigned char>(ch))) {
          err = "bad multiplicity in '" + term + "'";
          return false;
        }
      mul = std::stol(m);
      rest = term.substr(x + 1);
    }
    if (rest.size() < 2 || rest.size() > 4) {
      err = "bad irrep '" + term + "'";
      return false;
    }
    char par = rest.back();
    std::string ls = rest.substr(0, rest.size() - 1);
    for (char ch : ls)
      if (!std::isdigit(static_cast<unsigned char>(ch))) {
        err = "bad degree in '" + term + "'";
        return false;
      }
    if (par != 'e' && par != 'o') {
      err = "bad parity in '" + term + "'";
      return false;
    }
    if (mul < 1) {
      err = "multiplicity must be >= 1 in '" + term + "'";
      return false;
    }
    out.push_back(Irrep{static_cast<int>(mul), std::stoi(ls), par == 'e' ? 1 : -1});
    pos = end + 1;
    if (end == s.size()) break;
  }
  if (out.empty()) {
    err = "no irreps in '" + std::string(text) + "'";
    return false;
  }
  return true;
}

static constexpr int kMaxL = 6;

int build_paths(Plan& pl, std::string& err) {
  if (pl.node.empty()) {
    err = "no node irreps";
    return E3CONV_ERR_IRREPS;
  }
  pl.C = pl.node[0].mul;
  for (const auto& ir : pl.node) {
    if (ir.mul != pl.C) {
      err = "all node irreps must have the same multiplicity (the channel count C)";
      return E3CONV_ERR_IRREPS;
    }
    if (ir.l > kMaxL) {
      err = "node irrep degree above 6";
      return E3CONV_ERR_UNSUPPORTED;
    }
  }
  std::set<std::pair<int, int>> seen;
  for (const auto& ir : pl.filt) {
    if (ir.mul != pl.C) {
      err = "output multiplicities must equal C (channelwise product)";
      return E3CONV_ERR_IRREPS;
    }
    if (!seen.insert({ir.l, ir.p}).second) {
      err = "output irrep listed twice";
      return E3CONV_ERR_IRREPS;
    }
    if (ir.l > kMaxL) {
      err = "output irrep degree above 6";
      return E3CONV_ERR_UNSUPPORTED;
    }
  }
  pl.nx = 0;
  for (const auto& ir : pl.node) pl.nx += ir.dim();
  pl.ny = (pl.lmax + 1) * (pl.lmax + 1);

  struct Raw {
    int n1, l1, p1, x_off, l2, l3, p3;
  };
  std::vector<Raw> raw;
  std::set<std::pair<int, int>> produced;
  int x_off = 0;
  for (size_t n1 = 0; n1 < pl.node.size(); ++n1) {
    const Irrep& a = pl.node[n1];
    for (int l2 = 0; l2 <= pl.lmax; ++l2) {
      int p2 = (l2 % 2 == 0) ? 1 : -1;
      for (const auto& o : pl.filt) {
        if (std::abs(a.l - l2) <= o.l && o.l <= a.l + l2 && o.p == a.p * p2) {
          raw.push_back(Raw{static_cast<int>(n1), a.l, a.p, x_off, l2, o.l, o.p});
          produced.insert({o.l, o.p});
        }
      }
    }
    x_off += a.dim();
  }
  pl.outputs.clear();
  int off = 0;
  for (const auto& o : pl.filt) {
    if (produced.count({o.l, o.p})) {
      pl.outputs.push_back(Output{o.l, o.p, off});
      off += 2 * o.l + 1;
    }
  }
  pl.nout = off;
  pl.paths.clear();
  const double scale_none = 1.0;
  for (const auto& r : raw) {
    Path p;
    p.n1 = r.n1;
    p.l1 = r.l1;
    p.p1 = r.p1;
    p.x_off = r.x_off;
    p.l2 = r.l2;
    p.y_off = r.l2 * r.l2;
    p.l3 = r.l3;
    p.p3 = r.p3;
    p.o = -1;
    for (size_t k = 0; k < pl.outputs.size(); ++k)
      if (pl.outputs[k].l == r.l3 && pl.outputs[k].p == r.p3) {
        p.o = static_cast<int>(k);
        p.out_off = pl.outputs[k].off;
      }
    std::vector<double> w = real_wigner_3j(r.l1, r.l2, r.l3);
    double scale = pl.norm == E3CONV_NORM_SQRT_DIM_OUT ? std::sqrt(2.0 * r.l3 + 1.0) : scale_none;
    const int d1 = 2 * r.l1 + 1, d2 = 2 * r.l2 + 1, d3 = 2 * r.l3 + 1;
    p.cg.resize(w.size());
    for (size_t q = 0; q < w.size(); ++q) p.cg[q] = scale * w[q];
    for (int i = 0; i < d1; ++i)
      for (int j = 0; j < d2; ++j)
        for (int k = 0; k < d3; ++k) {
          double c = p.cg[(i * d2 + j) * d3 + k];
          if (std::fabs(c) > 1e-12) p.nnz.push_back(Nnz{i, j, k, c});
        }
    pl.paths.push_back(std::move(p));
  }
  return E3CONV_OK;
}

}  // namespace e3c
