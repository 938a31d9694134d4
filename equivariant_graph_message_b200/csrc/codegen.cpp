// CUDA source generator for the fused forward kernel of one plan.
//
// The kernel evaluates, for receiver b and channel u,
//   out[b, o+k, u] = inv_avg * sum_{e in row b} sum_{p -> o}
//                    s[e,p,u] * sum_{(i,j,k,c) in nnz(p)} c * Y[e, y_p + j] * x[a_e, x_p + i, u]
// with every path's nonzero CG coefficients unrolled as float32 immediates
// (the per-edge gather, tensor product, scalar mix, segmented sum over the
// receiver's CSR row and 1/N scale of e3j.core.Convolution, fused).
//
// Lane mapping: each lane owns V consecutive channels u0..u0+V-1 and keeps
// its nout*V partial sums in registers while it walks the receiver's row
// sequentially, so the segmented reduction needs no atomics and no
// cross-lane traffic.  Channels are independent in the channelwise product.
//
// Two variants:
//  * direct:  an "item" (receiver, channel tile) per team of TL lanes; each
//             lane loads its x / s slices with vector loads (<= 16 bytes).
//  * staged:  persistent warps, one 32*V-channel receiver row per warp at a
//             time (receivers w, w+W, w+2W, ...).  Lane 0 copies the next
//             edges' s row, sender x row and Y row into a per-warp ring of
//             shared-memory stages with 1-D bulk async copies (no multicast)
//             completed on mbarriers; the warp computes the current edge from
//             shared memory.  Waits are bounded: on timeout the kernel sets
//             bit 4 of the status word, drains its copies (bounded) and exits.
//
// Per path the cheaper of two equivalent evaluation orders is emitted:
//   scale-input  (2l1+1 <= 2l3+1): z_i = s_p x_i, then acc_k += (c Y_j) z_i
//   scale-output (otherwise):      t_k = sum (c Y_j) x_i, then acc_k += s_p t_k
// The products c*Y_j do not depend on the channel and are shared by the V
// channels of a lane.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <functional>
#include <map>
#include <set>
#include <sstream>

#include "plan.h"

namespace e3c {

namespace {

int align_up(int v, int a) { return (v + a - 1) / a * a; }

}  // namespace

// A group of lanes forming and applying the per-edge A entries of some paths
// (the staged variant's contract-first form): a whole team, or one warp of a
// team whose row's paths are split over its warps.
struct CoopGroupInfo {
  std::vector<int> paths;       // paths computed, canonical order
  std::vector<AEntry> ent;      // their A entries, build order within each path
  std::vector<int> acc;         // output component -> accumulator index (-1: not computed)
  int nacc = 0;                 // accumulators (output components) of the group
  int amode = 0;                // A layout (Shape::amode)
  int a_bytes = 0;              // shared memory of the group's A entries
};

std::vector<std::vector<int>> path_split_outputs(const Plan& pl, int warps);
std::vector<CoopGroupInfo> coop_groups(const Plan& pl, const Shape& sh);

std::vector<AEntry> build_a_entries(const Plan& pl) {
  std::vector<AEntry> out;
  for (size_t p = 0; p < pl.paths.size(); ++p) {
    const Path& P = pl.paths[p];
    std::map<std::pair<int, int>, size_t> where;  // (k, i) -> entry
    std::vector<AEntry> mine;
    for (const auto& n : P.nnz) {
      auto key = std::make_pair(n.k, n.i);
      auto it = where.find(key);
      if (it == where.end()) {
        where[key] = mine.size();
        mine.push_back(AEntry{static_cast<int>(p), n.i, n.k, {}});
        it = where.find(key);
      }
      mine[it->second].terms.push_back({P.y_off + n.j, n.c});  // index into the full Y row
    }
    std::sort(mine.begin(), mine.end(), [](const AEntry& a, const AEntry& b) {
      return a.k != b.k ? a.k < b.k : a.i < b.i;
    });
    out.insert(out.end(), mine.begin(), mine.end());
  }
  return out;
}

Shape choose_shape(const Plan& pl, int dtype) {
  Shape s;
  const int elem = dtype == E3CONV_F16 ? 2 : 4;
  const int vmax = 16 / elem;
  s.s_bytes = static_cast<int>(pl.paths.size()) * pl.C * elem;
  s.x_bytes = pl.nx * pl.C * elem;
  s.y_bytes = pl.req_vec ? 16 : pl.ny * elem;
  s.vec = pl.req_vec != 0;
  const bool bytes_ok = s.s_bytes % 16 == 0 && s.x_bytes % 16 == 0 && s.y_bytes % 16 == 0;

  // Tensor-core variant: float16 inputs, 128 channels (the MMA's M), at most
  // 16 node components (one K step) and at most 256 path outputs (N).
  const bool want_tc = pl.req_tc == 1 && !pl.tc_fallback;  // opt-in (E3CONV_OPT_TENSOR_CORES)
  if (want_tc && pl.req_stages != 0 && dtype == E3CONV_F16 && pl.C == 128 && pl.nx <= 16 &&
      bytes_ok) {
    int ncols = 0;
    for (const auto& P : pl.paths) ncols += 2 * P.l3 + 1;
    ncols = align_up(ncols, 16);
    if (ncols <= 256) {
      s.tc = true;
      s.V = 1;
      s.team = 4;
      s.TL = 32;
      s.tiles = 1;
      s.ipw = 1;
      s.ncols = ncols;
      s.tmem_cols = 512;
      s.tstride = align_up(ncols, 32);              // a team's T columns start on a 32-column boundary
      s.tbufs = std::min(3, 512 / s.tstride);       // teams per block: T columns fit in 512, registers in 64K
      if (pl.tc_team_cap > 0) s.tbufs = std::min(s.tbufs, pl.tc_team_cap);
      s.block = 128 * s.tbufs;                      // four warps per team
      int S = pl.req_stages > 0 ? std::max(pl.req_stages, 2) : 4;
      s.x_off = 0;                                  // 16 rows x 128 channels x 2 B, two 128B-swizzled halves
      s.s_off = 4096;
      s.y_off = s.s_off + align_up(s.s_bytes, 128);
      s.stage_bytes = align_up(s.y_off + s.y_bytes, 1024);
      s.b_bytes = 32 * ncols;                       // 16 x ncols f16, K-major core matrices
      s.b_stride = s.b_bytes + 128;                 // + scratch for the builders' padding lanes
      auto layout = [&](int stages) {
        s.stages = stages;
        s.b_off = stages * s.stage_bytes;
        s.yf_off = s.b_off + 2 * s.b_stride;
        s.hdr_off = s.yf_off + 4 * 4 * align_up(pl.ny, 4);
        s.bar_off = align_up(s.hdr_off + 16 * stages, 8);
        s.warp_smem = align_up(s.bar_off + 8 * (stages + 1), 1024);  // one team
        s.tslot_off = s.tbufs * s.warp_smem;
        s.smem_request = std::max(s.tslot_off + 16, 116 * 1024);    // one block per SM
      };
      layout(S);
      while (s.smem_request > 227 * 1024 && s.stages > 2) layout(s.stages - 1);
      while (s.smem_request > 227 * 1024 && s.tbufs > 1) {
        s.tbufs -= 1;
        s.block = 128 * s.tbufs;
        layout(s.stages);
      }
      if (s.smem_request <= 227 * 1024) return s;
      s = Shape{};
      s.s_bytes = static_cast<int>(pl.paths.size()) * pl.C * elem;
      s.x_bytes = pl.nx * pl.C * elem;
      s.y_bytes = pl.req_vec ? 16 : pl.ny * elem;
      s.vec = pl.req_vec != 0;
    }
  }

  // Staged variant: a team of `team` warps covers the C channels of one
  // receiver row, V channels per lane.  Preferred: one channel pair per lane
  // (V = 2, team = C / 64), which keeps registers low and warps many.
  int V = 0, team = 0, psplit = 1;
  const int one_warp_V = pl.C / 32;  // channels per lane when one warp covers C
  if (pl.req_stages != 0 && bytes_ok && pl.C % 32 == 0) {
    if (pl.req_psplit >= 2 && pl.req_coop != 0 && pl.req_V <= 0 && one_warp_V <= vmax &&
        (one_warp_V == 1 || one_warp_V % 2 == 0) &&
        pl.req_psplit <= static_cast<int>(pl.outputs.size())) {
      V = one_warp_V;  // every warp of the team covers C; the row's paths are split over them
      team = psplit = pl.req_psplit;
    } else if (pl.req_V > 0) {
      if (pl.C % (32 * pl.req_V) == 0 && pl.req_V <= vmax) {
        V = pl.req_V;
        team = pl.C / (32 * V);
      }
    } else if (pl.C / 32 <= vmax && pl.nout * (pl.C / 32) <= 128 && pl.C / 32 != 3) {
      V = pl.C / 32;  // one warp per receiver row (measured fastest)
      team = 1;
    } else if (pl.C % 64 == 0) {
      V = 2;          // channel pairs, teams of C/64 warps share the row
      team = pl.C / 64;
    } else {
      V = 1;
      team = pl.C / 32;
    }
    if (team > 8) V = team = 0;
  }
  if (V > 0) {
    s.V = V;
    s.team = team;
    s.TL = 32;
    s.tiles = 1;
    s.ipw = 1;
    // The ring: NS stages in regions of s rows, sender rows and Y rows (a group of G
    // consecutive stages takes G consecutive edges' s rows and Y rows in one copy each).
    s.group = pl.req_group > 0 ? pl.req_group : 1;
    int S = pl.req_stages > 0 ? pl.req_stages : 2 * s.group;
    S = (std::max(S, s.group) + s.group - 1) / s.group * s.group;
    s.x_slot = align_up(s.x_bytes, 128);
    s.s_off = 0;
    s.x_off = align_up(S * s.s_bytes, 128);
    s.y_off = s.x_off + S * s.x_slot;
    s.stage_bytes = align_up(s.y_off + S * s.y_bytes, 128);  // the whole ring
    s.coop = pl.req_coop != 0 && (V == 1 || V % 2 == 0);
    s.psplit = s.coop ? psplit : 1;
    // A layout: float slots in round order (a lane broadcasts each entry to a pair), or
    // broadcast pairs in round order (the default where a lane holds one channel pair), or
    // broadcast pairs in apply order read two per 16-byte load
    s.amode = 0;  // measured fastest for every workload (large_f32 4.05 vs 4.83 ms with pairs)
    if (s.coop && V % 2 == 0 && pl.req_alayout >= 0) s.amode = pl.req_alayout;
    s.dup_a = s.amode == 1 || s.amode == 2;
    s.na = s.coop ? static_cast<int>(build_a_entries(pl).size()) : 0;
    int a_bytes = 0;
    if (s.coop)
      for (const auto& g : coop_groups(pl, s)) a_bytes += g.a_bytes;
    const int y_bytes = s.coop ? s.psplit * align_up(4 * pl.ny, 16) : 0;
    s.stages = S;
    s.a_off = s.stage_bytes;
    s.yf_off = s.a_off + a_bytes;
    s.bar_off = align_up(s.yf_off + y_bytes, 8);
    s.hdr_off = s.bar_off + 8 * (S / s.group);
    s.warp_smem = align_up(s.hdr_off + 16 * S, 128);
    const int team_threads = 32 * team;
    int block = pl.req_block > 0 ? pl.req_block : (pl.auto_block > 0 ? pl.auto_block : 4 * team_threads);
    if (block % team_threads != 0 || block / team_threads > 15 ||
        (block / team_threads) * s.warp_smem > 227 * 1024) {
      if (pl.req_block > 0) {
        s.stages = 0;  // the requested block does not fit the staged variant
      } else {
        int teams = std::max(1, std::min(15, 227 * 1024 / s.warp_smem));
        block = teams * team_threads;
        if (block > 1024) block = (1024 / team_threads) * team_threads;
      }
    }
    if (s.stages > 0 && s.warp_smem > 227 * 1024) s.stages = 0;
    s.block = block;
    if (s.stages > 0) return s;
    s = Shape{};
    s.s_bytes = static_cast<int>(pl.paths.size()) * pl.C * elem;
    s.x_bytes = pl.nx * pl.C * elem;
    s.y_bytes = pl.req_vec ? 16 : pl.ny * elem;
    s.vec = pl.req_vec != 0;
  }

  // Direct variant.
  V = 1;
  if (pl.req_V > 0) {
    V = pl.req_V;
  } else {
    for (int v : {8, 4, 2, 1}) {
      if (v <= vmax && pl.C % v == 0 && (pl.nout * v <= 128 || v == 1)) {
        V = v;
        break;
      }
    }
  }
  s.V = V;
  const int lanes = pl.C / V;
  if (lanes >= 32) {
    s.TL = 32;
    s.tiles = (pl.C + 32 * V - 1) / (32 * V);
    s.ipw = 1;
  } else {
    s.TL = lanes;
    s.tiles = 1;
    s.ipw = 32 / lanes;
  }
  s.block = pl.req_block > 0 ? pl.req_block : 128;
  // software-pipelined row walk when two register sets of one edge's inputs stay small
  const int per_edge = (pl.nx + static_cast<int>(pl.paths.size())) * V + pl.ny;
  s.dpipe = pl.req_dpipe == 1 || (pl.req_dpipe == -1 && per_edge <= 64);
  return s;
}

static std::string flt(double c) {
  char buf[64];
  std::snprintf(buf, sizeof buf, "%.9ef", static_cast<double>(static_cast<float>(c)));
  return buf;
}

namespace {

struct Emitter {
  std::ostringstream o;
  int ind = 0;
  void line(const std::string& s) {
    for (int k = 0; k < ind; ++k) o << "  ";
    o << s << "\n";
  }
};

std::string S(long long v) { return std::to_string(v); }

// Loads V consecutive elements at `ptr` into float variables name_0 .. name_{V-1};
// `pre` is "ldg" (read-only global) or "lds" (shared).
void emit_vec_load(Emitter& em, int dtype, int V, const std::string& pre, const std::string& ptr,
                   const std::string& name) {
  if (dtype == E3CONV_F32) {
    if (V == 4) {
      em.line("{ const float4 t_ = " + pre + "_f4(" + ptr + "); " + name + "_0 = t_.x; " + name +
              "_1 = t_.y; " + name + "_2 = t_.z; " + name + "_3 = t_.w; }");
    } else if (V == 2) {
      em.line("{ const float2 t_ = " + pre + "_f2(" + ptr + "); " + name + "_0 = t_.x; " + name +
              "_1 = t_.y; }");
    } else {
      em.line(name + "_0 = " + pre + "_f1(" + ptr + ");");
    }
  } else {
    if (V == 8) {
      em.line("{ const uint4 t_ = " + pre + "_u4(" + ptr + ");");
      const char* w[4] = {"t_.x", "t_.y", "t_.z", "t_.w"};
      for (int q = 0; q < 4; ++q)
        em.line("  " + name + "_" + S(2 * q) + " = lo_h2f(" + w[q] + "); " + name + "_" +
                S(2 * q + 1) + " = hi_h2f(" + w[q] + ");");
      em.line("}");
    } else if (V == 4) {
      em.line("{ const uint2 t_ = " + pre + "_u2(" + ptr + "); " + name + "_0 = lo_h2f(t_.x); " +
              name + "_1 = hi_h2f(t_.x); " + name + "_2 = lo_h2f(t_.y); " + name +
              "_3 = hi_h2f(t_.y); }");
    } else if (V == 2) {
      em.line("{ const unsigned int t_ = " + pre + "_u1(" + ptr + "); " + name +
              "_0 = lo_h2f(t_); " + name + "_1 = hi_h2f(t_); }");
    } else {
      em.line(name + "_0 = " + pre + "_h1(" + ptr + ");");
    }
  }
}

void emit_prelude(Emitter& em) {
  em.line("__device__ __forceinline__ float h2f(unsigned short h) { float f; asm(\"cvt.f32.f16 %0, %1;\" : \"=f\"(f) : \"h\"(h)); return f; }");
  em.line("__device__ __forceinline__ float lo_h2f(unsigned int w) { return h2f(static_cast<unsigned short>(w & 0xffffu)); }");
  em.line("__device__ __forceinline__ float hi_h2f(unsigned int w) { return h2f(static_cast<unsigned short>(w >> 16)); }");
  for (const char* pre : {"ldg", "lds"}) {
    const bool g = pre[2] == 'g';
    auto rd = [&](const std::string& type, const std::string& p) {
      return g ? "__ldg(reinterpret_cast<const " + type + "*>(" + p + "))"
               : "*reinterpret_cast<const " + type + "*>(" + p + ")";
    };
    const std::string P(pre);
    em.line("__device__ __forceinline__ float " + P + "_f1(const float* p) { return " + rd("float", "p") + "; }");
    em.line("__device__ __forceinline__ float2 " + P + "_f2(const float* p) { return " + rd("float2", "p") + "; }");
    em.line("__device__ __forceinline__ float4 " + P + "_f4(const float* p) { return " + rd("float4", "p") + "; }");
    em.line("__device__ __forceinline__ float " + P + "_h1(const unsigned short* p) { return h2f(" + rd("unsigned short", "p") + "); }");
    em.line("__device__ __forceinline__ unsigned int " + P + "_u1(const unsigned short* p) { return " + rd("unsigned int", "p") + "; }");
    em.line("__device__ __forceinline__ uint2 " + P + "_u2(const unsigned short* p) { return " + rd("uint2", "p") + "; }");
    em.line("__device__ __forceinline__ uint4 " + P + "_u4(const unsigned short* p) { return " + rd("uint4", "p") + "; }");
  }
}

// Packed float32x2 helpers: a register pair (lo, hi), broadcast, fma / mul / add.
void emit_pair_ops(Emitter& em) {
  em.line("__device__ __forceinline__ unsigned long long pk(float lo, float hi) { unsigned long long r; asm(\"mov.b64 %0, {%1, %2};\" : \"=l\"(r) : \"f\"(lo), \"f\"(hi)); return r; }");
  em.line("__device__ __forceinline__ unsigned long long bc(float a) { return pk(a, a); }");
  em.line("__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) { unsigned long long d; asm(\"fma.rn.f32x2 %0, %1, %2, %3;\" : \"=l\"(d) : \"l\"(a), \"l\"(b), \"l\"(c)); return d; }");
  em.line("__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) { unsigned long long d; asm(\"mul.rn.f32x2 %0, %1, %2;\" : \"=l\"(d) : \"l\"(a), \"l\"(b)); return d; }");
  em.line("__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) { unsigned long long d; asm(\"add.rn.f32x2 %0, %1, %2;\" : \"=l\"(d) : \"l\"(a), \"l\"(b)); return d; }");
}

// Declares and loads y0..y{ny-1} from `yr` (global or shared).
void emit_y_load(Emitter& em, const Plan& pl, int dtype, const std::string& pre,
                 const std::string& yr) {
  const bool f16 = dtype == E3CONV_F16;
  std::string decl = "float";
  for (int j = 0; j < pl.ny; ++j) decl += std::string(j ? "," : "") + " y" + S(j);
  em.line(decl + ";");
  if (!f16 && pl.ny % 4 == 0) {
    for (int j = 0; j < pl.ny; j += 4)
      em.line("{ const float4 t_ = " + pre + "_f4(" + yr + " + " + S(j) + "); y" + S(j) +
              " = t_.x; y" + S(j + 1) + " = t_.y; y" + S(j + 2) + " = t_.z; y" + S(j + 3) +
              " = t_.w; }");
  } else if (f16 && pl.ny % 8 == 0) {
    for (int j = 0; j < pl.ny; j += 8) {
      em.line("{ const uint4 t_ = " + pre + "_u4(" + yr + " + " + S(j) + ");");
      const char* w[4] = {"t_.x", "t_.y", "t_.z", "t_.w"};
      for (int q = 0; q < 4; ++q)
        em.line("  y" + S(j + 2 * q) + " = lo_h2f(" + w[q] + "); y" + S(j + 2 * q + 1) +
                " = hi_h2f(" + w[q] + ");");
      em.line("}");
    }
  } else if (f16 && pl.ny % 2 == 0) {
    for (int j = 0; j < pl.ny; j += 2)
      em.line("{ const unsigned int t_ = " + pre + "_u1(" + yr + " + " + S(j) + "); y" + S(j) +
              " = lo_h2f(t_); y" + S(j + 1) + " = hi_h2f(t_); }");
  } else {
    for (int j = 0; j < pl.ny; ++j)
      em.line("y" + S(j) + " = " + pre + (f16 ? "_h1" : "_f1") + "(" + yr + " + " + S(j) + ");");
  }
}

// Declares y0..y{ny-1} = the real harmonics of the unit vector of (vx, vy, vz)
// (a zero vector gives Y_0 = 1 and 0 for l > 0), from the plan's polynomials.
void emit_sh_eval(Emitter& em, const Plan& pl, const std::string& vx, const std::string& vy,
                  const std::string& vz) {
  const auto polys = sh_polynomials(pl.lmax);
  std::string decl = "float";
  for (int j = 0; j < pl.ny; ++j) decl += std::string(j ? "," : "") + " y" + S(j);
  em.line(decl + ";");
  em.line("{");
  em.ind++;
  em.line("const float r2_ = fmaf(" + vx + ", " + vx + ", fmaf(" + vy + ", " + vy + ", " + vz +
          " * " + vz + "));");
  em.line("const float inv_ = r2_ > 0.f ? 1.f / sqrtf(r2_) : 0.f;");
  em.line("const float ux_ = " + vx + " * inv_, uy_ = " + vy + " * inv_, uz_ = " + vz + " * inv_;");
  const char* base[3] = {"ux_", "uy_", "uz_"};
  const char* nm[3] = {"px", "py", "pz"};
  for (int d = 0; d < 3; ++d)
    for (int a = 1; a <= pl.lmax; ++a)
      em.line(std::string("const float ") + nm[d] + S(a) + "_ = " +
              (a == 1 ? std::string(base[d]) : std::string(nm[d]) + S(a - 1) + "_ * " + base[d]) + ";");
  std::map<std::tuple<int, int, int>, std::string> mono;
  auto monomial = [&](int a, int b, int c) -> std::string {
    auto key = std::make_tuple(a, b, c);
    auto it = mono.find(key);
    if (it != mono.end()) return it->second;
    std::vector<std::string> f;
    if (a) f.push_back("px" + S(a) + "_");
    if (b) f.push_back("py" + S(b) + "_");
    if (c) f.push_back("pz" + S(c) + "_");
    std::string name;
    if (f.size() == 1) {
      name = f[0];
    } else {
      name = "m" + S(a) + S(b) + S(c) + "_";
      std::string e = f[0];
      for (size_t k = 1; k < f.size(); ++k) e += " * " + f[k];
      em.line("const float " + name + " = " + e + ";");
    }
    mono[key] = name;
    return name;
  };
  for (int j = 0; j < pl.ny; ++j) {
    std::string expr;
    double constant = 0.0;
    for (const auto& m : polys[j]) {
      if (m.px + m.py + m.pz == 0) {
        constant += m.coef;
        continue;
      }
      const std::string mm = monomial(m.px, m.py, m.pz);
      expr = expr.empty() ? flt(m.coef) + " * " + mm : "fmaf(" + flt(m.coef) + ", " + mm + ", " + expr + ")";
    }
    if (constant != 0.0) expr = expr.empty() ? flt(constant) : expr + " + " + flt(constant);
    if (expr.empty()) expr = "0.f";
    em.line("y" + S(j) + " = " + expr + ";");
  }
  std::string zero = "y0 = 1.f;";
  for (int j = 1; j < pl.ny; ++j) zero += " y" + S(j) + " = 0.f;";
  em.line("if (!(r2_ > 0.f)) { " + zero + " }");
  em.ind--;
  em.line("}");
}

// Fills the float32 Y row `yf` (shared memory) of the edge staged at `ysrc`
// with `nl` lanes (index `ln`): each converts components ln, ln + nl, ... of the
// staged harmonics, or, from edge vectors, every lane evaluates the harmonics
// and stores those components.
void emit_yf_fill(Emitter& em, const Plan& pl, int dtype, const Shape& sh, const std::string& ysrc,
                  const std::string& ln, int nl, const std::string& yf) {
  if (!sh.vec) {
    const bool f16 = dtype == E3CONV_F16;
    const std::string Ty = f16 ? "unsigned short" : "float";
    em.line("for (int j_ = " + ln + "; j_ < " + S(pl.ny) + "; j_ += " + S(nl) + ") " + yf +
            "[j_] = " + (f16 ? "h2f" : "") + "(reinterpret_cast<const " + Ty + "*>(" + ysrc +
            ")[j_]);");
    return;
  }
  em.line("{");
  em.ind++;
  em.line("const float4 v_ = *reinterpret_cast<const float4*>(" + ysrc + ");");
  emit_sh_eval(em, pl, "v_.x", "v_.y", "v_.z");
  std::string sel = "y" + S(pl.ny - 1);
  for (int j = pl.ny - 2; j >= 0; --j) sel = "(j_ == " + S(j) + " ? y" + S(j) + " : " + sel + ")";
  em.line("for (int j_ = " + ln + "; j_ < " + S(pl.ny) + "; j_ += " + S(nl) + ") " + yf + "[j_] = " +
          sel + ";");
  em.ind--;
  em.line("}");
}

// The per-edge contribution: x slices at xr + comp*C, s slices at sr + p*C
// (both already offset by the lane's first channel), Y in y0..; adds into a*.
void emit_edge_body(Emitter& em, const Plan& pl, int dtype, int V, const std::string& pre,
                    const std::string& xr, const std::string& sr) {
  size_t p = 0;
  while (p < pl.paths.size()) {
    const int n1 = pl.paths[p].n1;
    size_t q = p;
    while (q < pl.paths.size() && pl.paths[q].n1 == n1) ++q;
    const Path& first = pl.paths[p];
    const int d1 = 2 * first.l1 + 1;
    em.line("{  // node irrep " + S(n1) + " (l=" + S(first.l1) + ")");
    em.ind++;
    for (int i = 0; i < d1; ++i) {
      std::string decl = "float";
      for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " x" + S(i) + "_" + S(v);
      em.line(decl + ";");
      if (pre == "reg") {  // values already in registers cx<comp>_<v> (software pipeline)
        for (int v = 0; v < V; ++v)
          em.line("x" + S(i) + "_" + S(v) + " = cx" + S(first.x_off + i) + "_" + S(v) + ";");
      } else {
        emit_vec_load(em, dtype, V, pre, xr + " + " + S((first.x_off + i) * pl.C), "x" + S(i));
      }
    }
    for (size_t r = p; r < q; ++r) {
      const Path& P = pl.paths[r];
      const int d3 = 2 * P.l3 + 1;
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3) + ", " +
              S(P.nnz.size()) + " coefficients");
      em.ind++;
      {
        std::string decl = "float";
        for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " s_" + S(v);
        em.line(decl + ";");
        if (pre == "reg") {
          for (int v = 0; v < V; ++v) em.line("s_" + S(v) + " = cs" + S(r) + "_" + S(v) + ";");
        } else {
          emit_vec_load(em, dtype, V, pre, sr + " + " + S(static_cast<long long>(r) * pl.C), "s");
        }
      }
      std::map<std::pair<float, int>, std::string> cy;
      auto cyname = [&](const Nnz& n) -> std::string {
        auto key = std::make_pair(static_cast<float>(n.c), n.j);
        auto it = cy.find(key);
        if (it != cy.end()) return it->second;
        std::string nm = "c" + S(cy.size());
        em.line("const float " + nm + " = " + flt(n.c) + " * y" + S(P.y_off + n.j) + ";");
        cy[key] = nm;
        return nm;
      };
      std::vector<Nnz> nz = P.nnz;
      std::stable_sort(nz.begin(), nz.end(), [](const Nnz& a, const Nnz& b) { return a.k < b.k; });
      for (const auto& n : nz) cyname(n);
      if (d1 <= d3) {  // scale-input
        std::vector<bool> used(d1, false);
        for (const auto& n : nz) used[n.i] = true;
        for (int i = 0; i < d1; ++i) {
          if (!used[i]) continue;
          for (int v = 0; v < V; ++v)
            em.line("const float z" + S(i) + "_" + S(v) + " = s_" + S(v) + " * x" + S(i) + "_" +
                    S(v) + ";");
        }
        for (const auto& n : nz) {
          const std::string c = cyname(n);
          for (int v = 0; v < V; ++v) {
            std::string acc = "a" + S(P.out_off + n.k) + "_" + S(v);
            em.line(acc + " = fmaf(" + c + ", z" + S(n.i) + "_" + S(v) + ", " + acc + ");");
          }
        }
      } else {  // scale-output
        for (int k = 0; k < d3; ++k) {
          std::vector<Nnz> row;
          for (const auto& n : nz)
            if (n.k == k) row.push_back(n);
          if (row.empty()) continue;
          for (int v = 0; v < V; ++v) {
            std::string t = "t" + S(k) + "_" + S(v);
            em.line("float " + t + " = " + cyname(row[0]) + " * x" + S(row[0].i) + "_" + S(v) + ";");
            for (size_t m = 1; m < row.size(); ++m)
              em.line(t + " = fmaf(" + cyname(row[m]) + ", x" + S(row[m].i) + "_" + S(v) + ", " +
                      t + ");");
            std::string acc = "a" + S(P.out_off + k) + "_" + S(v);
            em.line(acc + " = fmaf(s_" + S(v) + ", " + t + ", " + acc + ");");
          }
        }
      }
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
    p = q;
  }
}

void emit_acc_decl(Emitter& em, const Plan& pl, int V) {
  for (int c = 0; c < pl.nout; ++c) {
    std::string l = "float";
    for (int v = 0; v < V; ++v)
      l += std::string(v ? "," : "") + " a" + S(c) + "_" + S(v) + " = 0.f";
    em.line(l + ";");
  }
}

// Stores acc * scale (or zeros) at orow + comp*C (+ lane offset already applied);
// with `add` the scaled sums are added to what the row already holds (a
// previous chunk of the same row, written by the same lane).
void emit_store(Emitter& em, const Plan& pl, int V, const std::string& orow, bool zero,
                bool reset, bool add = false) {
  for (int c = 0; c < pl.nout; ++c) {
    auto a = [&](int v) {
      return zero ? std::string("0.f") : "a" + S(c) + "_" + S(v) + " * inv_avg";
    };
    const std::string dst = orow + " + " + S(c * pl.C);
    if (V % 4 == 0) {
      for (int v = 0; v < V; v += 4) {
        const std::string d = "reinterpret_cast<float4*>(" + dst + " + " + S(v) + ")";
        if (add)
          em.line("{ const float4 o_ = *" + d + "; *" + d + " = make_float4(o_.x + " + a(v) +
                  ", o_.y + " + a(v + 1) + ", o_.z + " + a(v + 2) + ", o_.w + " + a(v + 3) + "); }");
        else
          em.line("*" + d + " = make_float4(" + a(v) + ", " + a(v + 1) + ", " + a(v + 2) + ", " +
                  a(v + 3) + ");");
      }
    } else if (V == 2) {
      const std::string d = "reinterpret_cast<float2*>(" + dst + ")";
      if (add)
        em.line("{ const float2 o_ = *" + d + "; *" + d + " = make_float2(o_.x + " + a(0) +
                ", o_.y + " + a(1) + "); }");
      else
        em.line("*" + d + " = make_float2(" + a(0) + ", " + a(1) + ");");
    } else {
      em.line("*(" + dst + ") " + (add ? "+= " : "= ") + a(0) + ";");
    }
    if (reset)
      for (int v = 0; v < V; ++v) em.line("a" + S(c) + "_" + S(v) + " = 0.f;");
  }
}

// Row flush of the scalar accumulators: store (first chunk of the row) or add.
void emit_flush(Emitter& em, const Plan& pl, int V, const std::string& orow,
                const std::string& add_cond, bool reset) {
  em.line("if (" + add_cond + ") {");
  em.ind++;
  emit_store(em, pl, V, orow, false, reset, true);
  em.ind--;
  em.line("} else {");
  em.ind++;
  emit_store(em, pl, V, orow, false, reset, false);
  em.ind--;
  em.line("}");
}

void emit_signature(Emitter& em, const std::string& T, int block, int minb, bool vec) {
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(block) +
          (minb > 0 ? ", " + S(minb) : std::string()) + ") e3conv_fwd(");
  em.line("    const " + T + "* __restrict__ x, const " + (vec ? std::string("float") : T) +
          "* __restrict__ Y, const " + T + "* __restrict__ s,");
  em.line("    const int* __restrict__ senders, const int* __restrict__ row_ptr,");
  em.line("    int num_nodes, int row_begin, int row_end, float* __restrict__ out, float inv_avg,");
  em.line("    unsigned int* __restrict__ status)");
}

// Edge range of the rows [row_begin, row_end): the edge buffers hold edges
// e_base .. e_end-1 of row_ptr's numbering at local index e - e_base.
void emit_edge_range(Emitter& em) {
  em.line("const int e_base = __ldg(row_ptr + row_begin), e_end = __ldg(row_ptr + row_end);");
}

// A receiver row is summed in chunks of E3_ROW_CHUNK edges: each chunk in its
// own float32 accumulators, the scaled chunk sums added into the output row.
// Only rows longer than one chunk take the extra read-add-write.
void emit_chunk_define(Emitter& em) { em.line("#define E3_ROW_CHUNK 128"); }

// Loads edge `ee`'s sender row (all nx components), harmonics and scalars (all
// paths) into registers <p>x<comp>_<v>, <p>y<j>, <p>s<path>_<v> and the flag <p>ok.
void emit_direct_edge_load(Emitter& em, const Plan& pl, int dtype, const Shape& sh,
                           const std::string& T, const std::string& ee, const std::string& p) {
  const int V = sh.V;
  em.line("{");
  em.ind++;
  em.line("const long long le_ = " + ee + " - e_base;");
  em.line("const int a_ = senders[le_];");
  em.line(p + "ok = (unsigned int)a_ < (unsigned int)num_nodes;");
  em.line("if (!" + p + "ok) atomicOr(status, 2u);");
  if (sh.vec) {
    em.line("const float4 v_ = __ldg(reinterpret_cast<const float4*>(Y) + le_);");
    emit_sh_eval(em, pl, "v_.x", "v_.y", "v_.z");
  } else {
    em.line("const " + T + "* yr_ = Y + le_ * " + S(pl.ny) + ";");
    emit_y_load(em, pl, dtype, "ldg", "yr_");
  }
  for (int j = 0; j < pl.ny; ++j) em.line(p + "y" + S(j) + " = y" + S(j) + ";");
  em.line("const " + T + "* xr_ = x + (long long)(" + p + "ok ? a_ : 0) * " + S(pl.nx * pl.C) + " + u0;");
  for (int i = 0; i < pl.nx; ++i) {
    std::string decl = "float";
    for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " t" + S(i) + "_" + S(v);
    em.line(decl + ";");
    emit_vec_load(em, dtype, V, "ldg", "xr_ + " + S(i * pl.C), "t" + S(i));
    for (int v = 0; v < V; ++v) em.line(p + "x" + S(i) + "_" + S(v) + " = t" + S(i) + "_" + S(v) + ";");
  }
  em.line("const " + T + "* sr_ = s + le_ * " + S(static_cast<long long>(pl.paths.size()) * pl.C) + " + u0;");
  for (size_t r = 0; r < pl.paths.size(); ++r) {
    std::string decl = "float";
    for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " q" + S(r) + "_" + S(v);
    em.line(decl + ";");
    emit_vec_load(em, dtype, V, "ldg", "sr_ + " + S(static_cast<long long>(r) * pl.C), "q" + S(r));
    for (int v = 0; v < V; ++v) em.line(p + "s" + S(r) + "_" + S(v) + " = q" + S(r) + "_" + S(v) + ";");
  }
  em.ind--;
  em.line("}");
}

// The direct variant's row walk, software-pipelined: edge e+1's loads are issued
// before edge e's products, into a second register set.
void emit_direct_pipelined(Emitter& em, const Plan& pl, int dtype, const Shape& sh,
                           const std::string& T) {
  const int V = sh.V;
  for (const char* p : {"c", "n"}) {
    const std::string P(p);
    std::string d = "float";
    bool first = true;
    for (int i = 0; i < pl.nx; ++i)
      for (int v = 0; v < V; ++v) { d += std::string(first ? " " : ", ") + P + "x" + S(i) + "_" + S(v); first = false; }
    for (size_t r = 0; r < pl.paths.size(); ++r)
      for (int v = 0; v < V; ++v) d += ", " + P + "s" + S(r) + "_" + S(v);
    for (int j = 0; j < pl.ny; ++j) d += ", " + P + "y" + S(j);
    em.line(d + ";");
    em.line("bool " + P + "ok = false;");
  }
  em.line("if (e0 < e1)");
  emit_direct_edge_load(em, pl, dtype, sh, T, "e0", "c");
  em.line("#pragma unroll 1");
  em.line("for (int e = e0; e < e1; ++e) {");
  em.ind++;
  em.line("if (e > e0 && (e - e0) % E3_ROW_CHUNK == 0) {  // chunk of a long row done");
  em.ind++;
  emit_flush(em, pl, V, "orow", "e - e0 > E3_ROW_CHUNK", true);
  em.ind--;
  em.line("}");
  em.line("if (e + 1 < e1)");
  emit_direct_edge_load(em, pl, dtype, sh, T, "e + 1", "n");
  em.line("if (cok) {");
  em.ind++;
  for (int j = 0; j < pl.ny; ++j) em.line("const float y" + S(j) + " = cy" + S(j) + ";");
  emit_edge_body(em, pl, dtype, V, "reg", "", "");
  em.ind--;
  em.line("}");
  // the next edge becomes the current one
  for (int i = 0; i < pl.nx; ++i)
    for (int v = 0; v < V; ++v) em.line("cx" + S(i) + "_" + S(v) + " = nx" + S(i) + "_" + S(v) + ";");
  for (size_t r = 0; r < pl.paths.size(); ++r)
    for (int v = 0; v < V; ++v) em.line("cs" + S(r) + "_" + S(v) + " = ns" + S(r) + "_" + S(v) + ";");
  for (int j = 0; j < pl.ny; ++j) em.line("cy" + S(j) + " = ny" + S(j) + ";");
  em.line("cok = nok;");
  em.ind--;
  em.line("}");
}

std::string direct_source(const Plan& pl, int dtype, const Shape& sh) {
  Emitter em;
  const int V = sh.V;
  const bool f16 = dtype == E3CONV_F16;
  const std::string T = f16 ? "unsigned short" : "float";
  em.line("// generated by libe3conv: fused equivariant convolution forward (direct loads)");
  em.line("// C=" + S(pl.C) + " nx=" + S(pl.nx) + " ny=" + S(pl.ny) + " nout=" + S(pl.nout) +
          " paths=" + S(pl.paths.size()) + " dtype=" + (f16 ? "f16" : "f32") + " V=" + S(V) +
          " TL=" + S(sh.TL) + " tiles=" + S(sh.tiles) + " ipw=" + S(sh.ipw) +
          " pipelined=" + S(sh.dpipe ? 1 : 0));
  emit_prelude(em);
  emit_chunk_define(em);
  emit_signature(em, T, sh.block, 0, sh.vec);
  em.line("{");
  em.ind++;
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const long long gwarp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;");
  em.line("const int sub = lane / " + S(sh.TL) + ";");
  em.line("const int within = lane - sub * " + S(sh.TL) + ";");
  em.line("if (sub >= " + S(sh.ipw) + ") return;");
  em.line("const long long item = gwarp * " + S(sh.ipw) + " + sub;");
  em.line("const long long b = row_begin + item / " + S(sh.tiles) + ";");
  em.line("const int tile = (int)(item - (b - row_begin) * " + S(sh.tiles) + ");");
  em.line("if (b >= row_end) return;");
  em.line("const int u0 = tile * " + S(sh.TL * V) + " + within * " + S(V) + ";");
  em.line("if (u0 >= " + S(pl.C) + ") return;");
  emit_edge_range(em);
  emit_acc_decl(em, pl, V);
  em.line("int e0 = row_ptr[b];");
  em.line("int e1 = row_ptr[b + 1];");
  em.line("if (e0 < e_base || e1 < e0 || e1 > e_end) { atomicOr(status, 1u); e1 = e0; }");
  em.line("float* orow = out + (b - row_begin) * " + S(pl.nout * pl.C) + " + u0;");
  if (sh.dpipe) {
    emit_direct_pipelined(em, pl, dtype, sh, T);
    emit_flush(em, pl, V, "orow", "e1 - e0 > E3_ROW_CHUNK", false);
    em.ind--;
    em.line("}");
    return em.o.str();
  }
  em.line("#pragma unroll 1");
  em.line("for (int e = e0; e < e1; ++e) {");
  em.ind++;
  em.line("if (e > e0 && (e - e0) % E3_ROW_CHUNK == 0) {  // chunk of a long row done");
  em.ind++;
  emit_flush(em, pl, V, "orow", "e - e0 > E3_ROW_CHUNK", true);
  em.ind--;
  em.line("}");
  em.line("const long long le = e - e_base;  // local edge index");
  em.line("const int a = senders[le];");
  em.line("if ((unsigned int)a >= (unsigned int)num_nodes) { atomicOr(status, 2u); continue; }");
  if (sh.vec) {
    em.line("const float4 v_ = __ldg(reinterpret_cast<const float4*>(Y) + le);");
    emit_sh_eval(em, pl, "v_.x", "v_.y", "v_.z");
  } else {
    em.line("const " + T + "* yr = Y + le * " + S(pl.ny) + ";");
    emit_y_load(em, pl, dtype, "ldg", "yr");
  }
  em.line("const " + T + "* xr = x + (long long)a * " + S(pl.nx * pl.C) + " + u0;");
  em.line("const " + T + "* sr = s + le * " +
          S(static_cast<long long>(pl.paths.size()) * pl.C) + " + u0;");
  emit_edge_body(em, pl, dtype, V, "ldg", "xr", "sr");
  em.ind--;
  em.line("}");
  emit_flush(em, pl, V, "orow", "e1 - e0 > E3_ROW_CHUNK", false);
  em.ind--;
  em.line("}");
  return em.o.str();
}


// ---------------------------------------------------------------------------
// Cooperative contraction body (staged variant).
//
// Phase 1: lanes 0..ny-1 convert the edge's Y row to float32 in shared
// memory; then every lane forms its share of the A entries (entries sorted by
// term count and dealt to lanes in rounds of 32, so a round runs the same
// number of terms in every lane) from a coefficient table in global memory,
// and writes them to the warp's A area.
// Phase 2: every lane applies A to its V channels: packed float32x2 FMAs on
// channel pairs (V even) or scalar FMAs (V == 1).

struct Lanes {
  int V;
  bool pairs() const { return V % 2 == 0; }
  int groups() const { return pairs() ? V / 2 : 1; }
  std::string type() const { return pairs() ? "unsigned long long" : "float"; }
  std::string fma(const std::string& a, const std::string& b, const std::string& c) const {
    return pairs() ? "fma2(" + a + ", " + b + ", " + c + ")" : "fmaf(" + a + ", " + b + ", " + c + ")";
  }
  std::string mul(const std::string& a, const std::string& b) const {
    return pairs() ? "mul2(" + a + ", " + b + ")" : "(" + a + " * " + b + ")";
  }
  std::string bc(const std::string& a) const { return pairs() ? "bc(" + a + ")" : a; }
};

// Loads the lane's V channels at `ptr` (shared) into groups name_0..name_{G-1}.
void emit_group_load(Emitter& em, int dtype, const Lanes& L, const std::string& ptr,
                     const std::string& name) {
  const bool f16 = dtype == E3CONV_F16;
  std::string decl = L.type();
  for (int g = 0; g < L.groups(); ++g) decl += std::string(g ? "," : "") + " " + name + "_" + S(g);
  em.line(decl + ";");
  if (!L.pairs()) {
    em.line(name + "_0 = " + (f16 ? "lds_h1(" : "lds_f1(") + ptr + ");");
    return;
  }
  if (!f16) {
    for (int g = 0; g < L.groups(); g += 2) {
      if (g + 1 < L.groups())
        em.line("{ const ulonglong2 t_ = *reinterpret_cast<const ulonglong2*>(" + ptr + " + " +
                S(2 * g) + "); " + name + "_" + S(g) + " = t_.x; " + name + "_" + S(g + 1) +
                " = t_.y; }");
      else
        em.line(name + "_" + S(g) + " = *reinterpret_cast<const unsigned long long*>(" + ptr +
                " + " + S(2 * g) + ");");
    }
  } else {
    for (int g = 0; g < L.groups(); g += 2) {
      if (g + 1 < L.groups())
        em.line("{ const uint2 t_ = lds_u2(" + ptr + " + " + S(2 * g) + "); " + name + "_" + S(g) +
                " = pk(lo_h2f(t_.x), hi_h2f(t_.x)); " + name + "_" + S(g + 1) +
                " = pk(lo_h2f(t_.y), hi_h2f(t_.y)); }");
      else
        em.line("{ const unsigned int t_ = lds_u1(" + ptr + " + " + S(2 * g) + "); " + name + "_" +
                S(g) + " = pk(lo_h2f(t_), hi_h2f(t_)); }");
    }
  }
}

// One group of lanes that forms the A entries of some paths and applies them:
// the whole team (channel split: the team's lanes share one A area) or one warp
// of the team (path split: each warp owns a set of output irreps, the paths
// into them and their A entries).
struct CoopGroup {
  std::vector<int> paths;       // paths computed, canonical order
  std::vector<AEntry> ent;      // their A entries, build order within each path
  int RW = 32;                  // lanes forming the entries
  std::string lane;             // lane index among them ("tl" or "lane")
  std::string sfx;              // suffix of the generated table
  std::vector<int> acc;         // output component -> accumulator index (-1: not computed)
  int a_off = 0, yf_off = 0;    // the group's A entries and float32 Y (bytes from tbase)
  int amode = 0;                // A layout (Shape::amode)
};

struct CoopTables {
  std::string source;      // __device__ table of phase 1
  int rounds = 0;
  std::vector<int> terms;  // terms per round
  std::vector<int> slot;   // entry -> position in the group's A area
};

// Phase 1 deals the entries to the group's RW lanes in rounds, longest first.
// Without pairs, entry number q of that order goes to A[q] (every round writes
// RW consecutive slots: no bank conflicts) and phase 2 reads A at slot[n].
// With pairs, the slots follow phase 2's order (path by path, each path padded
// to an even count) so that phase 2 loads two entries per 16-byte load; the
// slot of each dealt entry travels in the high bits of its first term's index.
CoopTables coop_tables(const CoopGroup& G) {
  const std::vector<AEntry>& ent = G.ent;
  const int RW = G.RW;
  CoopTables T;
  std::vector<int> order(ent.size());
  for (size_t n = 0; n < ent.size(); ++n) order[n] = static_cast<int>(n);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return ent[a].terms.size() > ent[b].terms.size();
  });
  T.slot.assign(ent.size(), -1);
  if (G.amode == 2 || G.amode == 3) {
    // apply order, each path's run padded to the load width (2 pairs or 4 floats per 16 bytes)
    const int w = G.amode == 2 ? 2 : 4;
    int pos = 0;
    for (int p : G.paths) {
      for (size_t n = 0; n < ent.size(); ++n)
        if (ent[n].path == p) T.slot[n] = pos++;
      pos = (pos + w - 1) / w * w;
    }
  } else {
    for (size_t q = 0; q < order.size(); ++q) T.slot[order[q]] = static_cast<int>(q);
  }
  T.rounds = static_cast<int>((ent.size() + RW - 1) / RW);
  std::ostringstream c, lay;
  c << "__device__ const int2 e3_atab" << G.sfx << "[] = {\n";
  lay << "// A layout" << G.sfx << " (entry: path i k slot):";
  for (size_t q = 0; q < order.size(); ++q)
    lay << " " << ent[order[q]].path << ":" << ent[order[q]].i << ":" << ent[order[q]].k << ":"
        << T.slot[order[q]];
  lay << "\n";
  for (int r = 0; r < T.rounds; ++r) {
    int tr = 0;
    for (int l = 0; l < RW; ++l) {
      size_t q = static_cast<size_t>(r) * RW + l;
      if (q < order.size()) tr = std::max<int>(tr, static_cast<int>(ent[order[q]].terms.size()));
    }
    T.terms.push_back(tr);
    for (int t = 0; t < tr; ++t) {
      for (int l = 0; l < RW; ++l) {
        size_t q = static_cast<size_t>(r) * RW + l;
        double cv = 0.0;
        int j = 0;
        if (q < order.size() && t < static_cast<int>(ent[order[q]].terms.size())) {
          j = ent[order[q]].terms[t].first;
          cv = ent[order[q]].terms[t].second;
        }
        if (G.amode >= 2 && t == 0 && q < order.size()) j |= T.slot[order[q]] << 8;
        const float cf = static_cast<float>(cv);
        unsigned int bits;
        std::memcpy(&bits, &cf, sizeof bits);
        c << "{" << static_cast<int>(bits) << ", " << j << "},";
      }
      c << "\n";
    }
  }
  c << "};\n";
  lay << "// A rounds" << G.sfx << " (lanes " << RW << ", mode " << G.amode << "):";
  for (int tr : T.terms) lay << " " << tr;
  lay << "\n";
  T.source = lay.str() + c.str();
  return T;
}

// Phase 1 + phase 2 of one group for the edge staged at `stg` (Y already in
// float32 at the group's yf, made visible to the group by the caller).
void emit_coop_edge(Emitter& em, const Plan& pl, int dtype, const Shape& sh, const CoopGroup& G,
                    const CoopTables& T, const std::string& group_sync) {
  const bool f16 = dtype == E3CONV_F16;
  const std::string Ty = f16 ? "unsigned short" : "float";
  const Lanes L{sh.V};
  const int RW = G.RW;
  const std::string& ln = G.lane;
  if (G.amode == 1 || G.amode == 2)
    em.line("unsigned long long* Aw = reinterpret_cast<unsigned long long*>(tbase + " + S(G.a_off) + ");");
  else
    em.line("float* Aw = reinterpret_cast<float*>(tbase + " + S(G.a_off) + ");");
  em.line("const float* yf = reinterpret_cast<const float*>(tbase + " + S(G.yf_off) + ");");
  int base = 0;
  const int na = static_cast<int>(G.ent.size());
  for (int r = 0; r < T.rounds; ++r) {
    em.line("{  // round terms: " + S(T.terms[r]));
    em.ind++;
    for (int t = 0; t < T.terms[r]; ++t)
      em.line("const int2 k" + S(t) + " = __ldg(&e3_atab" + G.sfx + "[" + S(base + t * RW) + " + " +
              ln + "]);");
    const std::string j0 = G.amode >= 2 ? "(k0.y & 255)" : "k0.y";
    std::string v = "__int_as_float(k0.x) * yf[" + j0 + "]";
    for (int t = 1; t < T.terms[r]; ++t)
      v = "fmaf(__int_as_float(k" + S(t) + ".x), yf[k" + S(t) + ".y], " + v + ")";
    const std::string dst = G.amode >= 2 ? "Aw[k0.y >> 8]" : "Aw[" + S(r * RW) + " + " + ln + "]";
    if (G.amode == 1 || G.amode == 2) v = "bc(" + v + ")";
    if ((r + 1) * RW <= na)
      em.line(dst + " = " + v + ";");
    else
      em.line("if (" + ln + " < " + S(na - r * RW) + ") " + dst + " = " + v + ";");
    em.ind--;
    em.line("}");
    base += T.terms[r] * RW;
  }
  em.line(group_sync + ";");
  em.line("const " + Ty + "* xs = reinterpret_cast<const " + Ty + "*>(stg_x) + u0;");
  em.line("const " + Ty + "* ss = reinterpret_cast<const " + Ty + "*>(stg_s) + u0;");
  // entry index of (path, i, k)
  std::map<std::tuple<int, int, int>, int> idx;
  for (size_t n = 0; n < G.ent.size(); ++n)
    idx[{G.ent[n].path, G.ent[n].i, G.ent[n].k}] = static_cast<int>(n);
  const int NG = L.groups();
  auto accv = [&](int comp, int g) {
    return "q" + S(G.acc[comp]) + "_" + S(g);
  };
  size_t p = 0;
  while (p < G.paths.size()) {
    const int n1 = pl.paths[G.paths[p]].n1;
    size_t q = p;
    while (q < G.paths.size() && pl.paths[G.paths[q]].n1 == n1) ++q;
    const Path& first = pl.paths[G.paths[p]];
    const int d1 = 2 * first.l1 + 1;
    em.line("{  // node irrep " + S(n1) + " (l=" + S(first.l1) + ")");
    em.ind++;
    for (int i = 0; i < d1; ++i)
      emit_group_load(em, dtype, L, "xs + " + S((first.x_off + i) * pl.C), "x" + S(i));
    for (size_t rr = p; rr < q; ++rr) {
      const int r = G.paths[rr];
      const Path& P = pl.paths[r];
      const int d3 = 2 * P.l3 + 1;
      std::vector<const AEntry*> pe;
      for (const auto& e : G.ent)
        if (e.path == r) pe.push_back(&e);
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3) + ", " +
              S(pe.size()) + " entries");
      em.ind++;
      emit_group_load(em, dtype, L, "ss + " + S(static_cast<long long>(r) * pl.C), "s");
      auto aval = [&](const AEntry* e) {
        return "A" + S(idx[{e->path, e->i, e->k}]);
      };
      if (G.amode == 2) {
        // entries in slot order, two per 16-byte load
        std::vector<const AEntry*> bys(pe);
        std::sort(bys.begin(), bys.end(), [&](const AEntry* a, const AEntry* b) {
          return T.slot[idx[{a->path, a->i, a->k}]] < T.slot[idx[{b->path, b->i, b->k}]];
        });
        for (size_t m = 0; m < bys.size(); m += 2) {
          const int s0 = T.slot[idx[{bys[m]->path, bys[m]->i, bys[m]->k}]];
          if (m + 1 < bys.size())
            em.line("unsigned long long " + aval(bys[m]) + ", " + aval(bys[m + 1]) +
                    "; { const ulonglong2 t_ = *reinterpret_cast<const ulonglong2*>(Aw + " + S(s0) +
                    "); " + aval(bys[m]) + " = t_.x; " + aval(bys[m + 1]) + " = t_.y; }");
          else
            em.line("const unsigned long long " + aval(bys[m]) + " = Aw[" + S(s0) + "];");
        }
      } else if (G.amode == 3) {
        // float entries in slot order, four per 16-byte load, broadcast to pairs
        std::vector<const AEntry*> bys(pe);
        std::sort(bys.begin(), bys.end(), [&](const AEntry* a, const AEntry* b) {
          return T.slot[idx[{a->path, a->i, a->k}]] < T.slot[idx[{b->path, b->i, b->k}]];
        });
        const char* comp[4] = {"x", "y", "z", "w"};
        for (size_t m = 0; m < bys.size(); m += 4) {
          const int s0 = T.slot[idx[{bys[m]->path, bys[m]->i, bys[m]->k}]];
          std::string decl = "const float4 a4_" + S(s0) + " = *reinterpret_cast<const float4*>(Aw + " + S(s0) + ");";
          em.line(decl);
          for (size_t u = 0; u < 4 && m + u < bys.size(); ++u)
            em.line("const " + L.type() + " " + aval(bys[m + u]) + " = " +
                    L.bc("a4_" + S(s0) + "." + comp[u]) + ";");
        }
      } else {
        for (const AEntry* e : pe) {
          const std::string ld = "Aw[" + S(T.slot[idx[{e->path, e->i, e->k}]]) + "]";
          em.line("const " + L.type() + " " + aval(e) + " = " + (G.amode >= 1 ? ld : L.bc(ld)) + ";");
        }
      }
      if (d1 <= d3) {  // scale-input
        std::vector<bool> used(d1, false);
        for (const AEntry* e : pe) used[e->i] = true;
        for (int i = 0; i < d1; ++i) {
          if (!used[i]) continue;
          for (int g = 0; g < NG; ++g)
            em.line("const " + L.type() + " z" + S(i) + "_" + S(g) + " = " +
                    L.mul("s_" + S(g), "x" + S(i) + "_" + S(g)) + ";");
        }
        // i outer, k inner: consecutive FMAs update different accumulators
        std::vector<const AEntry*> byi(pe);
        std::stable_sort(byi.begin(), byi.end(), [](const AEntry* a, const AEntry* b) {
          return a->i != b->i ? a->i < b->i : a->k < b->k;
        });
        for (const AEntry* e : byi)
          for (int g = 0; g < NG; ++g) {
            const std::string acc = accv(P.out_off + e->k, g);
            em.line(acc + " = " + L.fma(aval(e), "z" + S(e->i) + "_" + S(g), acc) + ";");
          }
      } else {  // scale-output: t_k = sum_i A[i,k] x_i (i outer, k inner), then acc_k += s t_k
        std::vector<const AEntry*> byi(pe);
        std::stable_sort(byi.begin(), byi.end(), [](const AEntry* a, const AEntry* b) {
          return a->i != b->i ? a->i < b->i : a->k < b->k;
        });
        std::vector<bool> started(d3, false);
        for (const AEntry* e : byi)
          for (int g = 0; g < NG; ++g) {
            std::string tv = "t" + S(e->k) + "_" + S(g);
            std::string xv = "x" + S(e->i) + "_" + S(g);
            if (!started[e->k])
              em.line(L.type() + " " + tv + " = " + L.mul(aval(e), xv) + ";");
            else
              em.line(tv + " = " + L.fma(aval(e), xv, tv) + ";");
            if (g == NG - 1) started[e->k] = true;
          }
        for (int k = 0; k < d3; ++k) {
          if (!started[k]) continue;
          for (int g = 0; g < NG; ++g) {
            const std::string acc = accv(P.out_off + k, g);
            em.line(acc + " = " + L.fma("s_" + S(g), "t" + S(k) + "_" + S(g), acc) + ";");
          }
        }
      }
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
    p = q;
  }
}

void emit_group_acc_decl(Emitter& em, int nacc, const Lanes& L) {
  for (int c = 0; c < nacc; ++c) {
    std::string l = L.type();
    for (int g = 0; g < L.groups(); ++g)
      l += std::string(g ? "," : "") + " q" + S(c) + "_" + S(g) + (L.pairs() ? " = 0ull" : " = 0.f");
    em.line(l + ";");
  }
}

// Stores the packed accumulators (times 1/N) of the group's output components at
// orow + comp*C and resets them; with `add` the values are added to what the row
// already holds.
void emit_group_store(Emitter& em, const Plan& pl, const Lanes& L, const std::string& orow,
                      const std::vector<int>& acc, bool add = false) {
  for (int c = 0; c < pl.nout; ++c) {
    if (acc[c] < 0) continue;
    const std::string q = "q" + S(acc[c]);
    const std::string dst = orow + " + " + S(c * pl.C);
    if (!L.pairs()) {
      em.line("*(" + dst + ") " + (add ? "+= " : "= ") + q + "_0 * inv_avg;");
      em.line(q + "_0 = 0.f;");
      continue;
    }
    auto val = [&](int g, const std::string& old) {
      const std::string m = "mul2(" + q + "_" + S(g) + ", inv2)";
      return add ? "add2(" + old + ", " + m + ")" : m;
    };
    for (int g = 0; g < L.groups(); g += 2) {
      if (g + 1 < L.groups()) {
        const std::string d = "reinterpret_cast<ulonglong2*>(" + dst + " + " + S(2 * g) + ")";
        if (add)
          em.line("{ const ulonglong2 o_ = *" + d + "; *" + d + " = make_ulonglong2(" +
                  val(g, "o_.x") + ", " + val(g + 1, "o_.y") + "); }");
        else
          em.line("*" + d + " = make_ulonglong2(" + val(g, "") + ", " + val(g + 1, "") + ");");
      } else {
        const std::string d = "reinterpret_cast<unsigned long long*>(" + dst + " + " + S(2 * g) + ")";
        em.line("*" + d + " = " + val(g, "*" + d) + ";");
      }
    }
    for (int g = 0; g < L.groups(); ++g) em.line(q + "_" + S(g) + " = 0ull;");
  }
}

}  // namespace

// Output irreps of each warp of a path-split team: longest-processing-time
// assignment of the output irreps, weighted by their per-channel FMA count
// (A entries + min(2l1+1, 2l3+1) of every path into them).
std::vector<std::vector<int>> path_split_outputs(const Plan& pl, int warps) {
  std::vector<double> cost(pl.outputs.size(), 0.0);
  const std::vector<AEntry> ent = build_a_entries(pl);
  for (const auto& e : ent) cost[pl.paths[e.path].o] += 1.0;
  for (const auto& P : pl.paths) cost[P.o] += std::min(2 * P.l1 + 1, 2 * P.l3 + 1);
  std::vector<int> order(pl.outputs.size());
  for (size_t k = 0; k < order.size(); ++k) order[k] = static_cast<int>(k);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<std::vector<int>> out(warps);
  std::vector<double> load(warps, 0.0);
  for (int o : order) {
    int w = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
    out[w].push_back(o);
    load[w] += cost[o];
  }
  for (auto& v : out) std::sort(v.begin(), v.end());
  return out;
}

// The coop groups of a staged shape: one for the whole team, or one per warp
// of a path-split team (in that case A and yf areas follow one another).
std::vector<CoopGroupInfo> coop_groups(const Plan& pl, const Shape& sh) {
  std::vector<CoopGroupInfo> gs;
  const std::vector<AEntry> all = build_a_entries(pl);
  const int amode = sh.amode;
  if (sh.psplit <= 1) {
    CoopGroupInfo g;
    for (size_t p = 0; p < pl.paths.size(); ++p) g.paths.push_back(static_cast<int>(p));
    g.ent = all;
    g.acc.resize(pl.nout);
    for (int c = 0; c < pl.nout; ++c) g.acc[c] = c;
    g.amode = amode;
    gs.push_back(g);
  } else {
    for (const auto& outs : path_split_outputs(pl, sh.psplit)) {
      CoopGroupInfo g;
      g.acc.assign(pl.nout, -1);
      int n = 0;
      for (int o : outs)
        for (int k = 0; k < 2 * pl.outputs[o].l + 1; ++k) g.acc[pl.outputs[o].off + k] = n++;
      for (size_t p = 0; p < pl.paths.size(); ++p)
        if (std::find(outs.begin(), outs.end(), pl.paths[p].o) != outs.end())
          g.paths.push_back(static_cast<int>(p));
      for (const auto& e : all)
        if (std::find(g.paths.begin(), g.paths.end(), e.path) != g.paths.end()) g.ent.push_back(e);
      g.amode = amode;
      gs.push_back(g);
    }
  }
  for (auto& g : gs) {
    int slots = 0;
    if (g.amode == 2 || g.amode == 3) {
      const int w = g.amode == 2 ? 2 : 4;
      for (int p : g.paths) {
        int n = 0;
        for (const auto& e : g.ent) n += e.path == p;
        slots += (n + w - 1) / w * w;
      }
    } else {
      slots = static_cast<int>(g.ent.size());
    }
    g.a_bytes = align_up((g.amode == 1 || g.amode == 2 ? 8 : 4) * slots, 16);
    g.nacc = 0;
    for (int a : g.acc) g.nacc = std::max(g.nacc, a + 1);
  }
  return gs;
}

namespace {

// The flush of every group's accumulators into the row at `orow`.
void emit_groups_store(Emitter& em, const Plan& pl, const Lanes& L,
                       const std::vector<CoopGroup>& groups, bool split, bool add) {
  if (!split) {
    emit_group_store(em, pl, L, "orow", groups[0].acc, add);
    return;
  }
  for (size_t w = 0; w < groups.size(); ++w) {
    em.line(std::string(w ? "} else " : "") + (w + 1 < groups.size() ? "if (tw == " + S(w) + ") " : "") + "{");
    em.ind++;
    emit_group_store(em, pl, L, "orow", groups[w].acc, add);
    em.ind--;
  }
  em.line("}");
}

std::string staged_source(const Plan& pl, int dtype, const Shape& sh) {
  Emitter em;
  const int V = sh.V;
  const int NS = sh.stages;
  const bool f16 = dtype == E3CONV_F16;
  const std::string T = f16 ? "unsigned short" : "float";
  const int TW = sh.team;                  // warps per team
  const int teams = sh.block / (32 * TW);  // teams per block
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  const long long o_row = static_cast<long long>(pl.nout) * pl.C;
  em.line("// generated by libe3conv: fused equivariant convolution forward (staged ring)");
  em.line("// C=" + S(pl.C) + " nx=" + S(pl.nx) + " ny=" + S(pl.ny) + " nout=" + S(pl.nout) +
          " paths=" + S(pl.paths.size()) + " dtype=" + (f16 ? "f16" : "f32") + " V=" + S(V) +
          " team=" + S(TW) + " teams/block=" + S(teams) + " stages=" + S(NS) +
          " ring_bytes=" + S(sh.stage_bytes) + " copy_group=" + S(sh.group) +
          " contract_first=" + S(sh.coop ? 1 : 0) +
          " path_split=" + S(sh.coop ? sh.psplit : 1) + " a_layout=" + S(sh.amode));
  emit_prelude(em);
  std::vector<CoopGroup> groups;
  std::vector<CoopTables> tabs;
  const Lanes L{V};
  const bool split = sh.coop && sh.psplit > 1;  // a row's paths split over the team's warps
  const int yf_bytes = align_up(4 * pl.ny, 16);
  emit_pair_ops(em);
  emit_chunk_define(em);
  int nacc = pl.nout;
  if (sh.coop) {
    const std::vector<CoopGroupInfo> infos = coop_groups(pl, sh);
    int a_off = sh.a_off;
    nacc = 0;
    for (size_t w = 0; w < infos.size(); ++w) {
      CoopGroup G;
      G.paths = infos[w].paths;
      G.ent = infos[w].ent;
      G.acc = infos[w].acc;
      G.amode = infos[w].amode;
      G.RW = split ? 32 : 32 * TW;
      G.lane = split ? "lane" : "tl";
      G.sfx = split ? "_w" + S(w) : "";
      G.yf_off = sh.yf_off + (split ? static_cast<int>(w) * yf_bytes : 0);
      G.a_off = a_off;
      a_off += infos[w].a_bytes;
      nacc = std::max(nacc, infos[w].nacc);
      groups.push_back(G);
      tabs.push_back(coop_tables(G));
      em.o << tabs.back().source;
    }
  }
  em.line("#define E3_SPIN_LIMIT (1u << 22)");
  em.line("__device__ __forceinline__ unsigned int smem_u32(const void* p) { return static_cast<unsigned int>(__cvta_generic_to_shared(p)); }");
  em.line("__device__ __forceinline__ void bar_init(unsigned long long* b) { asm volatile(\"mbarrier.init.shared::cta.b64 [%0], 1;\" :: \"r\"(smem_u32(b)) : \"memory\"); }");
  em.line("__device__ __forceinline__ void bar_expect(unsigned long long* b, unsigned int bytes) { asm volatile(\"mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\" :: \"r\"(smem_u32(b)), \"r\"(bytes) : \"memory\"); }");
  em.line("__device__ __forceinline__ bool bar_try(unsigned long long* b, unsigned int parity) {");
  em.line("  unsigned int ok; asm volatile(\"{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }\" : \"=r\"(ok) : \"r\"(smem_u32(b)), \"r\"(parity) : \"memory\"); return ok != 0; }");
  em.line("__device__ __forceinline__ bool bar_wait(unsigned long long* b, unsigned int parity) {");
  em.line("  for (unsigned int it = 0; it < E3_SPIN_LIMIT; ++it) if (bar_try(b, parity)) return true; return false; }");
  em.line("__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned int bytes, unsigned long long* b, unsigned long long policy) {");
  em.line("  asm volatile(\"cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\" :: \"r\"(smem_u32(dst)), \"l\"(src), \"r\"(bytes), \"r\"(smem_u32(b)), \"l\"(policy) : \"memory\"); }");
  em.line("__device__ __forceinline__ unsigned long long policy_evict_first() { unsigned long long p; asm volatile(\"createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\" : \"=l\"(p)); return p; }");
  em.line("__device__ __forceinline__ unsigned long long policy_evict_last() { unsigned long long p; asm volatile(\"createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\" : \"=l\"(p)); return p; }");
  em.line("__device__ __forceinline__ void fence_async_smem() { asm volatile(\"fence.proxy.async.shared::cta;\" ::: \"memory\"); }");
  emit_signature(em, T, sh.block, 1, sh.vec);
  em.line("{");
  em.ind++;
  em.line("extern __shared__ __align__(128) unsigned char smem[];");
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const int warp = threadIdx.x >> 5;");
  em.line("const int team = warp / " + S(TW) + ";       // team in this block");
  em.line("const int tw = warp - team * " + S(TW) + ";  // warp in team");
  em.line("const int tl = tw * 32 + lane;               // lane in team");
  if (TW > 1) {
    em.line("const unsigned int bar_id = 1u + (unsigned int)team;");
    em.line("auto team_sync = [&]() { asm volatile(\"bar.sync %0, " + S(32 * TW) + ";\" :: \"r\"(bar_id) : \"memory\"); };");
    em.line("auto team_all = [&](bool ok) { unsigned int r; asm volatile(\"{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, " + S(32 * TW) + ", p; selp.u32 %0, 1, 0, q; }\" : \"=r\"(r) : \"r\"((unsigned int)ok), \"r\"(bar_id) : \"memory\"); return r != 0u; };");
  } else {
    em.line("auto team_sync = [&]() { __syncwarp(); };");
    em.line("auto team_all = [&](bool ok) { return __all_sync(0xffffffffu, ok) != 0; };");
  }
  em.line("unsigned char* tbase = smem + team * " + S(sh.warp_smem) + ";");
  em.line("unsigned long long* bars = reinterpret_cast<unsigned long long*>(tbase + " + S(sh.bar_off) + ");");
  em.line("int* hdr = reinterpret_cast<int*>(tbase + " + S(sh.hdr_off) + ");  // per stage: sender, receiver, last");
  em.line("const bool issuer = tw == 0 && lane == 0;  // the lane that issues the team's copies");
  em.line("if (issuer) {");
  em.line("  for (int k = 0; k < " + S(NS / sh.group) + "; ++k) bar_init(bars + k);");
  em.line("  asm volatile(\"fence.mbarrier_init.release.cluster;\" ::: \"memory\");");
  em.line("}");
  em.line("team_sync();");
  em.line("const unsigned long long pol_stream = policy_evict_first();");
  em.line("const unsigned long long pol_keep = policy_evict_last();");
  em.line("const long long W = (long long)gridDim.x * " + S(teams) + ";  // teams in the grid");
  em.line(std::string("const int u0 = ") + (split ? "lane" : "tl") + " * " + S(V) +
          ";  // first channel of this lane");
  emit_edge_range(em);
  em.line("long long pb = row_begin + (long long)blockIdx.x * " + S(teams) + " + team - W;  // producer receiver");
  em.line("int pe = 0, pe1 = 0, pr0 = 0;  // producer edge cursor within row pb, which starts at pr0");
  em.line("int pwin = -1, psw = 0;   // sender window base (edge index) and this lane's sender");
  em.line("bool pdone = false;");
  em.line("unsigned int ppos = 0, cpos = 0;");
  if (sh.coop) {
    emit_group_acc_decl(em, nacc, L);
    if (L.pairs()) em.line("const unsigned long long inv2 = bc(inv_avg);");
  } else {
    emit_acc_decl(em, pl, V);
  }
  // Every warp of the team walks the same rows (same decisions); only the
  // issuer lane writes the stage headers and issues the bulk copies.  The ring
  // has NS stages in NG = NS / G groups; one produce() fills a group with up to
  // G consecutive edges of one row: one bulk copy of their s rows, one of their
  // Y rows (both contiguous in memory and in the ring), one per sender row, and
  // one mbarrier per group.  Unused stages of a group are marked empty (-3).
  const int G = sh.group, NG = NS / G;
  const std::string s_at = "tbase + " + S(sh.s_off) + " + ";    // + stage * s_bytes
  em.line("auto produce = [&]() {");
  em.ind++;
  em.line("while (!pdone && pe >= pe1) {");
  em.line("  pb += W;");
  em.line("  if (pb >= row_end) { pdone = true; break; }");
  em.line("  int r0 = row_ptr[pb], r1 = row_ptr[pb + 1];");
  em.line("  if (r0 < e_base || r1 < r0 || r1 > e_end) { if (issuer) atomicOr(status, 1u); r1 = r0; }");
  em.line("  pe = r0; pe1 = r1; pr0 = r0; pwin = -1;");
  em.line(std::string("  if (r0 == r1") + (split ? " && tw == 0" : "") + ") {  // empty row: zeros");
  em.line("    float* zrow = out + (pb - row_begin) * " + S(o_row) + " + u0;");
  em.ind += 2;
  emit_store(em, pl, V, "zrow", true, false);
  em.ind -= 2;
  em.line("  }");
  em.line("}");
  em.line("if (pdone) return;");
  em.line("const int n = min(" + S(G) + ", pe1 - pe);  // edges in this group");
  em.line("if (pwin < 0 || pe + n > pwin + 32) {");
  em.line("  pwin = pe;");
  em.line("  psw = (pe + lane < pe1) ? senders[pe + lane - e_base] : 0;");
  em.line("}");
  em.line("const unsigned int g0 = (ppos % " + S(NG) + ") * " + S(G) + ";  // first stage of the group");
  em.line("unsigned int xbytes = 0;");
  for (int k = 0; k < G; ++k) {
    em.line("const int a" + S(k) + " = __shfl_sync(0xffffffffu, psw, min(pe + " + S(k) + " - pwin, 31));");
    em.line("const bool v" + S(k) + " = " + S(k) + " < n && (unsigned int)a" + S(k) +
            " < (unsigned int)num_nodes;");
    em.line("if (v" + S(k) + ") xbytes += " + S(sh.x_bytes) + "u;");
  }
  em.line("if (issuer) {");
  em.ind++;
  for (int k = 0; k < G; ++k) {
    em.line("{");
    em.line("  const unsigned int st = g0 + " + S(k) + ";");
    em.line("  const int ek = pe + " + S(k) + ";");
    em.line("  hdr[4 * st] = " + S(k) + " < n ? (v" + S(k) + " ? a" + S(k) + " : -1) : -3;");
    em.line("  hdr[4 * st + 1] = (int)(pb - row_begin);");
    em.line("  // 1: last edge of the row, 2: last edge of a chunk, 4: an earlier chunk was flushed");
    em.line("  hdr[4 * st + 2] = (ek + 1 == pe1 ? 1 : ((ek + 1 - pr0) % E3_ROW_CHUNK == 0 ? 2 : 0)) |");
    em.line("                    (ek - pr0 >= E3_ROW_CHUNK ? 4 : 0);");
    em.line("}");
  }
  em.line("fence_async_smem();");
  em.line("unsigned long long* bar = bars + ppos % " + S(NG) + ";");
  em.line("bar_expect(bar, (unsigned int)n * " + S(sh.s_bytes + sh.y_bytes) + "u + xbytes);");
  em.line("bulk_g2s(" + s_at + "g0 * " + S(sh.s_bytes) + ", s + (long long)(pe - e_base) * " +
          S(s_row) + ", (unsigned int)n * " + S(sh.s_bytes) + "u, bar, pol_stream);");
  em.line("bulk_g2s(tbase + " + S(sh.y_off) + " + g0 * " + S(sh.y_bytes) + ", Y + (long long)(pe - e_base) * " +
          S(sh.vec ? 4 : pl.ny) + ", (unsigned int)n * " + S(sh.y_bytes) + "u, bar, pol_stream);");
  for (int k = 0; k < G; ++k)
    em.line("if (v" + S(k) + ") bulk_g2s(tbase + " + S(sh.x_off) + " + (g0 + " + S(k) + ") * " +
            S(sh.x_slot) + ", x + (long long)a" + S(k) + " * " +
            S(static_cast<long long>(pl.nx) * pl.C) + ", " + S(sh.x_bytes) + "u, bar, pol_keep);");
  em.ind--;
  em.line("}");
  em.line("pe += n;");
  em.line("++ppos;");
  em.ind--;
  em.line("};");
  em.line("for (int k = 0; k < " + S(NG) + "; ++k) produce();");
  em.line("team_sync();");
  em.line("#pragma unroll 1");
  em.line("while (cpos != ppos) {");
  em.ind++;
  em.line("const unsigned int g0 = (cpos % " + S(NG) + ") * " + S(G) + ";");
  em.line("if (!team_all(bar_wait(bars + cpos % " + S(NG) + ", (cpos / " + S(NG) + ") & 1u))) {");
  em.line("  // bounded wait ran out: flag it, let the issuer drain its copies (bounded), stop");
  em.line("  if (issuer) {");
  em.line("    atomicOr(status, 4u);");
  em.line("    for (unsigned int q = cpos; q != ppos; ++q) bar_wait(bars + q % " + S(NG) + ", (q / " + S(NG) + ") & 1u);");
  em.line("  }");
  em.line("  return;");
  em.line("}");
  em.line("#pragma unroll 1");
  em.line("for (int k = 0; k < " + S(G) + "; ++k) {");
  em.ind++;
  em.line("const unsigned int st = g0 + k;");
  em.line("const int a = hdr[4 * st];");
  em.line("if (a == -3) break;  // the group's unused stages");
  em.line("const unsigned char* stg_s = tbase + " + S(sh.s_off) + " + st * " + S(sh.s_bytes) + ";");
  em.line("const unsigned char* stg_x = tbase + " + S(sh.x_off) + " + st * " + S(sh.x_slot) + ";");
  em.line("const unsigned char* stg_y = tbase + " + S(sh.y_off) + " + st * " + S(sh.y_bytes) + ";");
  em.line("const long long b = hdr[4 * st + 1];");
  em.line("const int flags = hdr[4 * st + 2];");
  em.line("if (a >= 0) {");
  em.ind++;
  if (sh.coop) {
    if (split) {
      // every warp converts the edge's Y row into its own float32 copy
      em.line("{");
      em.ind++;
      em.line("float* yfw = reinterpret_cast<float*>(tbase + " + S(sh.yf_off) + " + tw * " +
              S(yf_bytes) + ");");
      emit_yf_fill(em, pl, dtype, sh, "stg_y", "lane", 32, "yfw");
      em.ind--;
      em.line("}");
      em.line("__syncwarp();");
      for (size_t w = 0; w < groups.size(); ++w) {
        em.line(std::string(w ? "} else " : "") + (w + 1 < groups.size() ? "if (tw == " + S(w) + ") " : "") +
                "{  // warp " + S(w) + " of the team: " + S(groups[w].paths.size()) + " paths");
        em.ind++;
        emit_coop_edge(em, pl, dtype, sh, groups[w], tabs[w], "__syncwarp()");
        em.ind--;
      }
      em.line("}");
    } else {
      em.line("{");
      em.ind++;
      em.line("float* yfw = reinterpret_cast<float*>(tbase + " + S(sh.yf_off) + ");");
      emit_yf_fill(em, pl, dtype, sh, "stg_y", "tl", 32 * TW, "yfw");
      em.ind--;
      em.line("}");
      em.line("team_sync();");
      emit_coop_edge(em, pl, dtype, sh, groups[0], tabs[0], "team_sync()");
    }
  } else {
    if (sh.vec) {
      em.line("const float4 v_ = *reinterpret_cast<const float4*>(stg_y);");
      emit_sh_eval(em, pl, "v_.x", "v_.y", "v_.z");
    } else {
      em.line("const " + T + "* ys = reinterpret_cast<const " + T + "*>(stg_y);");
      emit_y_load(em, pl, dtype, "lds", "ys");
    }
    em.line("const " + T + "* xs = reinterpret_cast<const " + T + "*>(stg_x) + u0;");
    em.line("const " + T + "* ss = reinterpret_cast<const " + T + "*>(stg_s) + u0;");
    emit_edge_body(em, pl, dtype, V, "lds", "xs", "ss");
  }
  em.ind--;
  em.line("} else if (issuer) {");
  em.line("  atomicOr(status, 2u);");
  em.line("}");
  em.line("if (flags & 3) {  // row (or a chunk of a long row) complete");
  em.ind++;
  em.line("float* orow = out + b * " + S(o_row) + " + u0;");
  em.line("if (flags & 4) {");
  em.ind++;
  if (sh.coop)
    emit_groups_store(em, pl, L, groups, split, true);
  else
    emit_store(em, pl, V, "orow", false, true, true);
  em.ind--;
  em.line("} else {");
  em.ind++;
  if (sh.coop)
    emit_groups_store(em, pl, L, groups, split, false);
  else
    emit_store(em, pl, V, "orow", false, true);
  em.ind--;
  em.line("}");
  em.ind--;
  em.line("}");
  em.line("team_sync();  // stage and A area free for reuse");
  em.ind--;
  em.line("}");
  em.line("++cpos;");
  em.line("produce();");
  em.ind--;
  em.line("}");
  em.ind--;
  em.line("}");
  return em.o.str();
}


// ---------------------------------------------------------------------------
// Tensor-core variant (float16 inputs, C = 128).
//
// Per edge e of receiver b (one block = 4 warps = 128 threads, thread u owns
// channel u):
//   T[u, n] = sum_i x[a, i, u] * B[i, n],   n = (p, k),  B[i,(p,k)] = A_p[i,k]
// with A_p[i,k] = sum_j CG_p[i,j,k] Y_j formed per edge by the block (each
// entry split into float16 hi + lo parts, so hi + lo carries ~22 bits), and
//   m[b, o(p)+k, u] += s[e, p, u] * T[u, (p,k)]   (float32 FMA per channel).
// T is produced by two tcgen05.mma (kind::f16, M = 128, N = ncols, K = 16:
// A operand = the sender's x rows staged by a 2-D TMA copy with 128-byte
// swizzle, MN-major; B operand = A_hi / A_lo in shared memory, K-major, no
// swizzle) into tensor memory and read back with tcgen05.ld.
// Copies (2-D TMA for x, 1-D bulk for s and Y) go through the same ring of
// stages as the staged variant; all waits are bounded.

struct BTable {
  std::string source;
  int rounds = 0;
  std::vector<int> terms;
};

// Entries dealt to the 128 threads in rounds, longest first; per entry the
// byte offset of its element in the K-major B tile.
BTable tc_tables(const Plan& pl, const std::vector<AEntry>& ent, const std::vector<int>& colbase,
                 int RW) {
  BTable T;
  std::vector<int> order(ent.size());
  for (size_t n = 0; n < ent.size(); ++n) order[n] = static_cast<int>(n);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return ent[a].terms.size() > ent[b].terms.size();
  });
  T.rounds = static_cast<int>((ent.size() + RW - 1) / RW);
  std::ostringstream c, d;
  c << "__device__ const int2 e3_btab[] = {\n";
  d << "__device__ const int e3_boff[] = {\n";
  for (int r = 0; r < T.rounds; ++r) {
    int tr = 0;
    for (int l = 0; l < RW; ++l) {
      size_t q = static_cast<size_t>(r) * RW + l;
      if (q < order.size()) tr = std::max<int>(tr, static_cast<int>(ent[order[q]].terms.size()));
    }
    T.terms.push_back(tr);
    for (int t = 0; t < tr; ++t) {
      for (int l = 0; l < RW; ++l) {
        size_t q = static_cast<size_t>(r) * RW + l;
        double cv = 0.0;
        int j = 0;
        if (q < order.size() && t < static_cast<int>(ent[order[q]].terms.size())) {
          j = ent[order[q]].terms[t].first;
          cv = ent[order[q]].terms[t].second;
        }
        const float cf = static_cast<float>(cv);
        unsigned int bits;
        std::memcpy(&bits, &cf, sizeof bits);
        c << "{" << static_cast<int>(bits) << ", " << j << "},";
      }
      c << "\n";
    }
    for (int l = 0; l < RW; ++l) {
      size_t q = static_cast<size_t>(r) * RW + l;
      int off = -1;
      if (q < order.size()) {
        const AEntry& e = ent[order[q]];
        const int i = pl.paths[e.path].x_off + e.i;       // K index: node component
        const int n = colbase[e.path] + e.k;               // N index: path output column
        off = (n / 8) * 256 + (i / 8) * 128 + (n % 8) * 16 + (i % 8) * 2;
      }
      d << off << ",";
    }
    d << "\n";
  }
  c << "};\n";
  d << "};\n";
  T.source = c.str() + d.str();
  return T;
}

// Tensor-core forward, teams of four warps.  A team (128 threads, one warp per
// tensor-memory lane quarter, thread tl <-> channel tl) owns receiver rows
// g, g+W, g+2W, ... (g = its index in the grid, W = teams in the grid) and a
// private ring of S stages, A tile and T columns.  Per edge:
//   1. wait for the edge's stage (x tile by 4-D TMA, s and Y rows by bulk copy);
//   2. build A = sum_j CG Y_j as float16 hi/lo K-major tiles (128 threads,
//      branch-free, coefficient table in registers);
//   3. one team barrier (bar.red.and.pred: also agrees on bounded-wait timeouts);
//   4. a thread of warp 1 issues T = x^T A_hi + x^T A_lo (tcgen05.mma, M = 128
//      channels) and commits to the team's mbarrier while warp 0 refills the
//      ring slot the barrier has just freed;
//   5. every thread loads its channel's s, waits for the commit, reads T from
//      tensor memory in 32-column chunks and accumulates s * T in registers.
// Several teams per SM overlap one another's latency.
std::string tc_source(const Plan& pl, const Shape& sh) {
  Emitter em;
  const int NS = sh.stages;
  const int TEAMS = sh.tbufs;
  const int TBYTES = sh.warp_smem;            // shared memory of one team
  const int BS = sh.b_stride;
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  const long long o_row = static_cast<long long>(pl.nout) * pl.C;
  std::vector<int> colbase(pl.paths.size());
  int ncols_raw = 0;
  for (size_t p = 0; p < pl.paths.size(); ++p) {
    colbase[p] = ncols_raw;
    ncols_raw += 2 * pl.paths[p].l3 + 1;
  }
  std::vector<AEntry> ent = build_a_entries(pl);
  BTable tab = tc_tables(pl, ent, colbase, 128);
  // T is read in pieces of at most 16 columns, each load issued one piece ahead of the FMAs that
  // use the piece before it (two pieces of registers live, as one 32-column piece would be)
  std::vector<std::pair<int, int>> chunks;  // (start column, width), start a multiple of width
  for (int pos = 0; pos < ncols_raw;) {
    int w = 16;
    while (w > 1 && (pos % w != 0 || pos + w > ncols_raw)) w /= 2;
    chunks.push_back({pos, w});
    pos += w;
  }
  em.line("// generated by libe3conv: fused equivariant convolution forward (tensor cores, teams)");
  em.line("// C=" + S(pl.C) + " nx=" + S(pl.nx) + " ny=" + S(pl.ny) + " nout=" + S(pl.nout) +
          " paths=" + S(pl.paths.size()) + " dtype=f16 ncols=" + S(sh.ncols) + " teams=" + S(TEAMS) +
          " tstride=" + S(sh.tstride) + " stages=" + S(NS) + " stage_bytes=" + S(sh.stage_bytes) +
          " team_bytes=" + S(TBYTES) + " entries=" + S(ent.size()) + " producer_threads=128");
  em.o << tab.source;
  em.line("__device__ __forceinline__ float h2f(unsigned short h) { float f; asm(\"cvt.f32.f16 %0, %1;\" : \"=f\"(f) : \"h\"(h)); return f; }");
  em.line("__device__ __forceinline__ unsigned short f2h(float f) { unsigned short h; asm(\"cvt.rn.f16.f32 %0, %1;\" : \"=h\"(h) : \"f\"(f)); return h; }");
  em.line("#define E3_SPIN_LIMIT (1u << 22)");
  emit_chunk_define(em);
  em.line("struct __align__(64) E3TensorMap { unsigned long long v[16]; };");
  em.line("__device__ __forceinline__ unsigned int smem_u32(const void* p) { return static_cast<unsigned int>(__cvta_generic_to_shared(p)); }");
  em.line("__device__ __forceinline__ void bar_init(unsigned long long* b, unsigned int count) { asm volatile(\"mbarrier.init.shared::cta.b64 [%0], %1;\" :: \"r\"(smem_u32(b)), \"r\"(count) : \"memory\"); }");
  em.line("__device__ __forceinline__ void bar_arrive(unsigned long long* b) { asm volatile(\"mbarrier.arrive.shared::cta.b64 _, [%0];\" :: \"r\"(smem_u32(b)) : \"memory\"); }");
  em.line("__device__ __forceinline__ void bar_expect(unsigned long long* b, unsigned int bytes) { asm volatile(\"mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\" :: \"r\"(smem_u32(b)), \"r\"(bytes) : \"memory\"); }");
  em.line("__device__ __forceinline__ bool bar_try(unsigned long long* b, unsigned int parity) {");
  em.line("  unsigned int ok; asm volatile(\"{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }\" : \"=r\"(ok) : \"r\"(smem_u32(b)), \"r\"(parity) : \"memory\"); return ok != 0; }");
  em.line("__device__ __forceinline__ bool bar_wait(unsigned long long* b, unsigned int parity) {");
  em.line("  for (unsigned int it = 0; it < E3_SPIN_LIMIT; ++it) if (bar_try(b, parity)) return true; return false; }");
  em.line("__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned int bytes, unsigned long long* b, unsigned long long policy) {");
  em.line("  asm volatile(\"cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\" :: \"r\"(smem_u32(dst)), \"l\"(src), \"r\"(bytes), \"r\"(smem_u32(b)), \"l\"(policy) : \"memory\"); }");
  em.line("// the sender's tile: box {64 channels, 16 rows, 2 halves} of node `node` (rows >= nx zero-filled)");
  em.line("__device__ __forceinline__ void tma_x_g2s(void* dst, const E3TensorMap* map, int node, unsigned long long* b, unsigned long long policy) {");
  em.line("  asm volatile(\"cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %2, %2, %3}], [%4], %5;\" :: \"r\"(smem_u32(dst)), \"l\"(map), \"r\"(0), \"r\"(node), \"r\"(smem_u32(b)), \"l\"(policy) : \"memory\"); }");
  em.line("__device__ __forceinline__ unsigned long long policy_evict_first() { unsigned long long p; asm volatile(\"createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\" : \"=l\"(p)); return p; }");
  em.line("__device__ __forceinline__ unsigned long long policy_evict_last() { unsigned long long p; asm volatile(\"createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\" : \"=l\"(p)); return p; }");
  em.line("__device__ __forceinline__ void fence_async_smem() { asm volatile(\"fence.proxy.async.shared::cta;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void tc_before() { asm volatile(\"tcgen05.fence::before_thread_sync;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void tc_after() { asm volatile(\"tcgen05.fence::after_thread_sync;\" ::: \"memory\"); }");
  em.line("// barrier of the team's 128 threads that also ANDs a predicate over them");
  em.line("__device__ __forceinline__ bool team_all(bool ok, unsigned int id) { unsigned int r; asm volatile(\"{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, 128, p; selp.u32 %0, 1, 0, q; }\" : \"=r\"(r) : \"r\"((unsigned int)ok), \"r\"(id) : \"memory\"); return r != 0u; }");
  for (int n = 1; n <= 32; n *= 2) {
    std::string regs, outs;
    for (int r = 0; r < n; ++r) {
      regs += std::string(r ? "," : "") + "%" + S(r);
      outs += std::string(r ? ", " : "") + "\"=r\"(r[" + S(r) + "])";
    }
    em.line("#define TMEM_LD" + S(n) + "(addr, r) asm volatile(\"tcgen05.ld.sync.aligned.32x32b.x" + S(n) +
            ".b32 {" + regs + "}, [%" + S(n) + "];\" : " + outs + " : \"r\"(addr))");
  }
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(sh.block) + ", 1) e3conv_fwd(");
  em.line(std::string("    const unsigned short* __restrict__ x, const ") +
          (sh.vec ? "float" : "unsigned short") + "* __restrict__ Y,");
  em.line("    const unsigned short* __restrict__ s, const int* __restrict__ senders,");
  em.line("    const int* __restrict__ row_ptr, int num_nodes, int row_begin, int row_end, float* __restrict__ out,");
  em.line("    float inv_avg, unsigned int* __restrict__ status, const __grid_constant__ E3TensorMap xmap)");
  em.line("{");
  em.ind++;
  em.line("extern __shared__ __align__(1024) unsigned char smem[];");
  em.line("const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;");
  em.line("const int team = warp >> 2, tw = warp & 3, tl = tid & 127;  // tl = channel = tensor-memory lane");
  em.line("const unsigned int bar_id = 1u + (unsigned int)team;");
  em.line("unsigned char* tbase = smem + team * " + S(TBYTES) + ";");
  em.line("unsigned char* Bhi = tbase + " + S(sh.b_off) + ";  // A_hi; A_lo at +" + S(BS) + "; bytes " + S(sh.b_bytes) + ".. of each are scratch");
  em.line("unsigned char* Blo = Bhi + " + S(BS) + ";");
  em.line("float* yfw = reinterpret_cast<float*>(tbase + " + S(sh.yf_off) + ") + tw * " + S(align_up(pl.ny, 4)) + ";");
  em.line("int* hdr = reinterpret_cast<int*>(tbase + " + S(sh.hdr_off) + ");  // per stage: sender (-1 invalid, -2 end), receiver, last");
  em.line("unsigned long long* sfull = reinterpret_cast<unsigned long long*>(tbase + " + S(sh.bar_off) + ");");
  em.line("unsigned long long* tdone = sfull + " + S(NS) + ";");
  em.line("unsigned int* tslot = reinterpret_cast<unsigned int*>(smem + " + S(sh.tslot_off) + ");");
  em.line("for (int q = tl; q < " + S(2 * BS / 16) + "; q += 128) reinterpret_cast<uint4*>(Bhi)[q] = make_uint4(0u, 0u, 0u, 0u);");
  em.line("if (tl == 0) {");
  em.line("  for (int k = 0; k < " + S(NS) + "; ++k) bar_init(sfull + k, 1u);");
  em.line("  bar_init(tdone, 1u);");
  em.line("  asm volatile(\"fence.mbarrier_init.release.cluster;\" ::: \"memory\");");
  em.line("}");
  em.line("if (warp == 0) {");
  em.line("  asm volatile(\"tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], " + S(sh.tmem_cols) + ";\" :: \"r\"(smem_u32(tslot)) : \"memory\");");
  em.line("  asm volatile(\"tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\" ::: \"memory\");");
  em.line("}");
  em.line("fence_async_smem();");
  em.line("tc_before();");
  em.line("__syncthreads();");
  em.line("tc_after();");
  em.line("const unsigned int tmem = *tslot;");
  em.line("const unsigned int tcol = tmem + ((unsigned int)(32 * tw) << 16) + (unsigned int)(team * " + S(sh.tstride) + ");");
  em.line("const unsigned int tmma = tmem + (unsigned int)(team * " + S(sh.tstride) + ");");
  em.line("const unsigned int idesc = (1u << 4) | (1u << 15) | ((unsigned int)(" + S(sh.ncols) + " >> 3) << 17) | ((unsigned int)(128 >> 4) << 24);");
  em.line("const long long W = (long long)gridDim.x * " + S(TEAMS) + ";");
  // A-tile table in registers
  {
    int base = 0;
    for (int r = 0; r < tab.rounds; ++r) {
      for (int t2 = 0; t2 < tab.terms[r]; ++t2)
        em.line("const int2 k" + S(r) + "_" + S(t2) + " = __ldg(&e3_btab[" + S(base + t2 * 128) + " + tl]);");
      em.line("const int off" + S(r) + " = __ldg(&e3_boff[" + S(r * 128) + " + tl]) >= 0 ? __ldg(&e3_boff[" + S(r * 128) + " + tl]) : " + S(sh.b_bytes) + ";  // padding lanes write the scratch bytes");
      base += tab.terms[r] * 128;
    }
  }
  // row walk (warp tw == 0 of the team; lane 0 issues the copies)
  em.line("// row walk of warp 0 of the team, loads one row ahead: the open row [pe, pe1) of receiver");
  em.line("// pb with sender windows psw (edges pwin..) and psw2 (the next 32); the next row nb [n0, n1)");
  em.line("// with its first windows in flight; row_ptr of the row after (mb) in flight");
  emit_edge_range(em);
  em.line("long long pb = -1, nb = row_begin + (long long)blockIdx.x * " + S(TEAMS) + " + team, mb = nb + W;");
  em.line("int pr0 = 0;  // first edge of the open row");
  em.line("int pe = 0, pe1 = 0, pwin = 0, psw = 0, psw2 = 0, n0 = 0, n1 = 0, nsw = 0, nsw2 = 0, m0 = 0, m1 = 0;");
  em.line("unsigned int qi = 0;  // positions issued");
  em.line("bool walk_done = false;");
  em.line("unsigned long long pol_stream = 0, pol_keep = 0;");
  em.line("if (tw == 0) {");
  em.line("  pol_stream = policy_evict_first();");
  em.line("  pol_keep = policy_evict_last();");
  em.line("  if (nb < row_end) {");
  em.line("    n0 = row_ptr[nb]; n1 = row_ptr[nb + 1];");
  em.line("    if (n0 < e_base || n1 < n0 || n1 > e_end) { if (lane == 0) atomicOr(status, 1u); n1 = n0; }");
  em.line("    nsw = (n0 + lane < n1) ? senders[n0 + lane - e_base] : 0;");
  em.line("    nsw2 = (n0 + 32 + lane < n1) ? senders[n0 + 32 + lane - e_base] : 0;");
  em.line("  }");
  em.line("  if (mb < row_end) { m0 = row_ptr[mb]; m1 = row_ptr[mb + 1]; }");
  em.line("}");
  em.line("// issue position qi into stage qi % S (warp 0 of the team only)");
  em.line("auto issue = [&]() {");
  em.ind++;
  em.line("const unsigned int st = qi % " + S(NS) + ";");
  em.line("while (pe >= pe1) {  // open the next row");
  em.line("  pb = nb;");
  em.line("  if (pb >= row_end) { walk_done = true; break; }");
  em.line("  pe = n0; pe1 = n1; pr0 = n0; pwin = n0; psw = nsw; psw2 = nsw2;");
  em.line("  if (pe == pe1) {");
  em.line("    float* zrow = out + (pb - row_begin) * " + S(o_row) + ";");
  em.line("    for (int k = lane; k < " + S(o_row) + "; k += 32) zrow[k] = 0.f;");
  em.line("  }");
  em.line("  nb = mb; n0 = m0; n1 = m1;");
  em.line("  if (nb < row_end) {");
  em.line("    if (n0 < e_base || n1 < n0 || n1 > e_end) { if (lane == 0) atomicOr(status, 1u); n1 = n0; }");
  em.line("    nsw = (n0 + lane < n1) ? senders[n0 + lane - e_base] : 0;");
  em.line("    nsw2 = (n0 + 32 + lane < n1) ? senders[n0 + 32 + lane - e_base] : 0;");
  em.line("  }");
  em.line("  mb = nb + W;");
  em.line("  if (mb < row_end) { m0 = row_ptr[mb]; m1 = row_ptr[mb + 1]; }");
  em.line("}");
  em.line("if (walk_done) {");
  em.line("  if (lane == 0) { hdr[4 * st] = -2; bar_arrive(sfull + st); }  // end marker");
  em.line("  ++qi;");
  em.line("  return;");
  em.line("}");
  em.line("if (pe >= pwin + 32) {  // next window of the row");
  em.line("  pwin += 32; psw = psw2;");
  em.line("  psw2 = (pwin + 32 + lane < pe1) ? senders[pwin + 32 + lane - e_base] : 0;");
  em.line("}");
  em.line("const int a = __shfl_sync(0xffffffffu, psw, pe - pwin);");
  em.line("const bool valid = (unsigned int)a < (unsigned int)num_nodes;");
  em.line("if (lane == 0) {");
  em.line("  unsigned char* stg = tbase + st * " + S(sh.stage_bytes) + ";");
  em.line("  hdr[4 * st] = valid ? a : -1;");
  em.line("  hdr[4 * st + 1] = (int)(pb - row_begin);");
  em.line("  // 1: last edge of the row, 2: last edge of a chunk, 4: an earlier chunk was flushed");
  em.line("  hdr[4 * st + 2] = (pe + 1 == pe1 ? 1 : ((pe + 1 - pr0) % E3_ROW_CHUNK == 0 ? 2 : 0)) |");
  em.line("                    (pe - pr0 >= E3_ROW_CHUNK ? 4 : 0);");
  em.line("  bar_expect(sfull + st, " + S(sh.s_bytes + sh.y_bytes) + "u + (valid ? 4096u : 0u));");
  em.line("  bulk_g2s(stg + " + S(sh.s_off) + ", s + (long long)(pe - e_base) * " + S(s_row) + ", " + S(sh.s_bytes) + "u, sfull + st, pol_stream);");
  em.line("  bulk_g2s(stg + " + S(sh.y_off) + ", Y + (long long)(pe - e_base) * " + S(sh.vec ? 4 : pl.ny) + ", " + S(sh.y_bytes) + "u, sfull + st, pol_stream);");
  em.line("  if (valid) tma_x_g2s(stg, &xmap, a, sfull + st, pol_keep);");
  em.line("}");
  em.line("__syncwarp();");
  em.line("++pe;");
  em.line("++qi;");
  em.ind--;
  em.line("};");
  em.line("if (tw == 0)");
  em.line("  for (int k = 0; k < " + S(NS - 1) + " && !walk_done; ++k) issue();");
  {
    std::string decl = "float";
    for (int c = 0; c < pl.nout; ++c) decl += std::string(c ? "," : "") + " a" + S(c) + " = 0.f";
    em.line(decl + ";");
  }
  em.line("unsigned int q = 0, v = 0;");
  em.line("bool ok = true;");
  em.line("#pragma unroll 1");
  em.line("while (true) {");
  em.ind++;
  em.line("const unsigned int st = q % " + S(NS) + ";");
  em.line("const unsigned char* stg = tbase + st * " + S(sh.stage_bytes) + ";");
  em.line("const bool landed = bar_wait(sfull + st, (q / " + S(NS) + ") & 1u);");
  em.line("if (landed && hdr[4 * st] >= 0) {  // A tile of this edge (the MMA of the previous edge has completed)");
  em.ind++;
  if (sh.vec) {
    emit_yf_fill(em, pl, E3CONV_F16, sh, "stg + " + S(sh.y_off), "lane", 32, "yfw");
  } else {
    em.line("const unsigned short* ys = reinterpret_cast<const unsigned short*>(stg + " + S(sh.y_off) + ");");
    em.line("for (int j = lane; j < " + S(pl.ny) + "; j += 32) yfw[j] = h2f(ys[j]);");
  }
  em.line("__syncwarp();");
  em.line("// all loads and products first, then the float16 splits and the stores");
  for (int r = 0; r < tab.rounds; ++r) {
    std::string val = "__int_as_float(k" + S(r) + "_0.x) * yfw[k" + S(r) + "_0.y]";
    for (int t2 = 1; t2 < tab.terms[r]; ++t2)
      val = "fmaf(__int_as_float(k" + S(r) + "_" + S(t2) + ".x), yfw[k" + S(r) + "_" + S(t2) + ".y], " + val + ")";
    em.line("const float v" + S(r) + " = " + val + ";");
  }
  for (int r = 0; r < tab.rounds; ++r)
    em.line("const unsigned short h" + S(r) + " = f2h(v" + S(r) + "), l" + S(r) + " = f2h(v" + S(r) + " - h2f(h" + S(r) + "));");
  for (int r = 0; r < tab.rounds; ++r) {
    em.line("*reinterpret_cast<unsigned short*>(Bhi + off" + S(r) + ") = h" + S(r) + ";");
    em.line("*reinterpret_cast<unsigned short*>(Blo + off" + S(r) + ") = l" + S(r) + ";");
  }
  em.line("fence_async_smem();");
  em.ind--;
  em.line("}");
  em.line("tc_before();");
  em.line("ok = team_all(ok && landed, bar_id);  // A tile written, T of the previous edge read, all waits in time");
  em.line("if (!ok) break;");
  em.line("tc_after();");
  em.line("const int a = hdr[4 * st];");
  em.line("if (a == -2) break;");
  em.line("const long long b = hdr[4 * st + 1];");
  em.line("const int flags = hdr[4 * st + 2];");
  em.line("if (a >= 0 && tl == 32) {  // warp 1 issues the MMAs while warp 0 refills the ring");
  em.line("  const unsigned long long adesc = (unsigned long long)((smem_u32(stg) & 0x3FFFF) >> 4) | (128ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);");
  em.line("  const unsigned long long hdesc = (unsigned long long)((smem_u32(Bhi) & 0x3FFFF) >> 4) | (8ull << 16) | (16ull << 32) | (1ull << 46);");
  em.line("  const unsigned long long ldesc = (unsigned long long)((smem_u32(Blo) & 0x3FFFF) >> 4) | (8ull << 16) | (16ull << 32) | (1ull << 46);");
  em.line("  asm volatile(\"{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }\" :: \"r\"(tmma), \"l\"(adesc), \"l\"(hdesc), \"r\"(idesc), \"r\"(0u) : \"memory\");");
  em.line("  asm volatile(\"{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }\" :: \"r\"(tmma), \"l\"(adesc), \"l\"(ldesc), \"r\"(idesc), \"r\"(1u) : \"memory\");");
  em.line("  asm volatile(\"tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\" :: \"r\"(smem_u32(tdone)) : \"memory\");");
  em.line("}");
  em.line("// the slot of the previous edge is free: every thread of the team has passed the barrier");
  em.line("if (tw == 0 && !walk_done) issue();");
  em.line("if (a >= 0) {");
  em.ind++;
  em.line("const unsigned short* sv = reinterpret_cast<const unsigned short*>(stg + " + S(sh.s_off) + ") + tl;");
  for (size_t p = 0; p < pl.paths.size(); ++p)
    em.line("const float s" + S(p) + " = h2f(sv[" + S(static_cast<long long>(p) * pl.C) + "]);");
  em.line("ok = bar_wait(tdone, v & 1u);");
  em.line("tc_after();");
  // the wait names the registers of the piece it completes, so that no use moves above it
  auto wait_piece = [&](size_t k) {
    std::string ops;
    for (int r = 0; r < chunks[k].second; ++r)
      ops += std::string(r ? ", " : "") + "\"+r\"(r" + S(k) + "_[" + S(r) + "])";
    em.line("asm volatile(\"tcgen05.wait::ld.sync.aligned;\" : " + ops + " :: \"memory\");");
  };
  auto load_piece = [&](size_t k) {
    em.line("unsigned int r" + S(k) + "_[" + S(chunks[k].second) + "];");
    em.line("TMEM_LD" + S(chunks[k].second) + "(tcol + " + S(chunks[k].first) + "u, r" + S(k) + "_);");
  };
  load_piece(0);
  wait_piece(0);
  for (size_t k = 0; k < chunks.size(); ++k) {
    if (k + 1 < chunks.size()) load_piece(k + 1);
    for (int col = chunks[k].first; col < chunks[k].first + chunks[k].second; ++col) {
      size_t p = 0;
      while (!(col >= colbase[p] && col < colbase[p] + 2 * pl.paths[p].l3 + 1)) ++p;
      const std::string acc = "a" + S(pl.paths[p].out_off + col - colbase[p]);
      em.line(acc + " = fmaf(s" + S(p) + ", __uint_as_float(r" + S(k) + "_[" + S(col - chunks[k].first) + "]), " + acc + ");");
    }
    if (k + 1 < chunks.size()) wait_piece(k + 1);
  }
  em.line("++v;");
  em.ind--;
  em.line("} else if (tl == 0) {");
  em.line("  atomicOr(status, 2u);");
  em.line("}");
  em.line("if (flags & 3) {  // row (or a chunk of a long row) complete");
  em.line("  float* orow = out + b * " + S(o_row) + " + tl;");
  em.line("  if (flags & 4) {");
  for (int c = 0; c < pl.nout; ++c) em.line("    orow[" + S(static_cast<long long>(c) * pl.C) + "] += a" + S(c) + " * inv_avg; a" + S(c) + " = 0.f;");
  em.line("  } else {");
  for (int c = 0; c < pl.nout; ++c) em.line("    orow[" + S(static_cast<long long>(c) * pl.C) + "] = a" + S(c) + " * inv_avg; a" + S(c) + " = 0.f;");
  em.line("  }");
  em.line("}");
  em.line("++q;");
  em.ind--;
  em.line("}");
  em.line("if (!ok && tl == 0) atomicOr(status, 4u);");
  em.line("// drain (bounded): the team's copies still in flight and its last MMA complete");
  em.line("if (tl == 0) {");
  em.line("  for (unsigned int k = q; k < qi; ++k) bar_wait(sfull + k % " + S(NS) + ", (k / " + S(NS) + ") & 1u);");
  em.line("  if (v > 0u) bar_wait(tdone, (v - 1u) & 1u);");
  em.line("}");
  em.line("tc_before();");
  em.line("__syncthreads();");
  em.line("tc_after();");
  em.line("if (warp == 0) asm volatile(\"tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, " + S(sh.tmem_cols) + ";\" :: \"r\"(tmem) : \"memory\");");
  em.ind--;
  em.line("}");
  return em.o.str();
}

}  // namespace

// ---------------------------------------------------------------------------
// Backward kernels (gradients of sum(g * out) for an upstream gradient g of the
// forward's output).  The forward is linear in each of x, Y and s, so every
// gradient is the forward's four-factor product with one factor removed:
//   gs[e, p, u]       = inv_avg sum_{i,j,k} CG_p[i,j,k] x[a,i,u] Y[e,j] g[b,o_p+k,u]
//   gY[e, j]          = inv_avg sum_p sum_u sum_{i,k} CG_p[i,j,k] s[e,p,u] x[a,i,u] g[b,o_p+k,u]
//   gx[a, i, u]       = inv_avg sum_{e: senders[e] = a} sum_p sum_{j,k} CG_p[i,j,k] s[e,p,u] Y[e,j] g[b,o_p+k,u]
// (a = sender, b = receiver of edge e).  Two kernels, every CG nonzero
// unrolled as a constant:
//  * edges (receiver order, like the forward): an item of TL lanes per
//    receiver row holds the row's g in registers (V channels per lane), and
//    for each edge writes gs and the channel-reduced gY (butterfly over the
//    item's lanes; TL is a power of two, lanes past C contribute zeros);
//  * nodes (sender order): an item per sender walks the sender's edges
//    through the sender CSR (sender_row_ptr, sender_perm) and keeps gx in
//    registers; one store per sender.

BwdShape choose_backward_shape(const Plan& pl, int dtype) {
  BwdShape b;
  const int vmax = dtype == E3CONV_F16 ? 8 : 4;
  int V = 1;
  while (V < vmax && pl.C > 32 * V) V *= 2;
  if (pl.C > 32 * V || pl.C % V != 0) {
    // one item must cover every channel (the gY reduction stays inside a warp)
    b.ok = false;
    return b;
  }
  b.V = V;
  int TL = 1;
  while (TL * V < pl.C) TL *= 2;
  b.TL = TL;
  b.ipw = 32 / TL;
  b.block = 128;
  b.ok = true;
  // staged edges kernel: one receiver per warp, channel pairs per lane, 16-byte rows
  const int elem = dtype == E3CONV_F16 ? 2 : 4;
  b.s_bytes = static_cast<int>(pl.paths.size()) * pl.C * elem;
  b.x_bytes = pl.nx * pl.C * elem;
  b.y_bytes = (pl.ny * elem + 15) / 16 * 16;
  b.stage_bytes = b.s_bytes + b.x_bytes + b.y_bytes;
  b.smem = (b.block / 32) * 2 * b.stage_bytes;
  b.staged = TL == 32 && V % 2 == 0 && b.s_bytes % 16 == 0 && b.x_bytes % 16 == 0 &&
             (pl.ny * elem) % 4 == 0 && b.smem <= 112 * 1024;
  b.g_bytes = pl.nout * pl.C * 4;
  b.nstage_bytes = b.s_bytes + b.g_bytes + b.y_bytes;
  b.nsmem = (b.block / 32) * 2 * b.nstage_bytes;
  b.nstaged = TL == 32 && V % 2 == 0 && b.s_bytes % 16 == 0 && b.g_bytes % 16 == 0 &&
              (pl.ny * elem) % 4 == 0 && b.nsmem <= 220 * 1024;
  // a grad_out row of more than 64 registers per lane: the edges kernel (and the staged nodes
  // kernel) run as two launches, each over half of the output irreps (balanced by their (i, k)
  // terms), so each holds half of the row and stages only its paths' scalars (and, for grad_x,
  // only its outputs' gradient rows)
  b.eparts = 1;
  b.out_part.assign(pl.outputs.size(), 0);
  for (int t = 0; t < 4; ++t) {
    b.esmem[t] = b.smem;
    b.nsmem_p[t] = b.nsmem;
  }
  // parts: as requested (E3CONV_OPT_BACKWARD_PARTS), else one while a lane's row takes at most
  // 64 registers and one per 44 beyond (measured on large_f16: 2 / 3 / 4 launches 69.8 / 63.5 /
  // 66.9 ms; one launch is fastest for mace and large_f32)
  int want = pl.req_bparts > 0 ? pl.req_bparts : pl.nout * V <= 64 ? 1 : (pl.nout * V + 43) / 44;
  want = std::min<int>({want, 4, static_cast<int>(pl.outputs.size())});
  if (b.staged && want > 1 && (pl.C * elem) % 16 == 0) {
    std::vector<std::pair<long long, int>> work;  // (terms, output irrep)
    for (size_t o = 0; o < pl.outputs.size(); ++o) {
      long long w = 0;
      for (const auto& P : pl.paths)
        if (P.o == static_cast<int>(o)) {
          std::set<std::pair<int, int>> ik;
          for (const auto& n : P.nnz) ik.insert({n.i, n.k});
          w += static_cast<long long>(ik.size());
        }
      work.push_back({w, static_cast<int>(o)});
    }
    std::sort(work.begin(), work.end(), std::greater<std::pair<long long, int>>());
    std::vector<long long> load(want, 0);
    for (const auto& wo : work) {
      const int t = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
      b.out_part[wo.second] = t;
      load[t] += wo.first;
    }
    if (*std::min_element(load.begin(), load.end()) > 0) {
      b.eparts = want;
      for (int t = 0; t < want; ++t) {
        int np = 0, nc = 0;
        for (const auto& P : pl.paths) np += b.out_part[P.o] == t;
        for (size_t o = 0; o < pl.outputs.size(); ++o)
          if (b.out_part[o] == t) nc += 2 * pl.outputs[o].l + 1;
        b.esmem[t] = (b.block / 32) * 2 * (np * pl.C * elem + b.x_bytes + b.y_bytes);
        b.nsmem_p[t] = (b.block / 32) * 2 * (np * pl.C * elem + nc * pl.C * 4 + b.y_bytes);
      }
    }
  }
  return b;
}

namespace {

// Declares g loads: g{c}_{v} for the given output components at grow + c*C.
void emit_g_load(Emitter& em, const Plan& pl, int V, const std::string& grow, int c0, int c1,
                 const std::string& active) {
  for (int c = c0; c < c1; ++c) {
    std::string decl = "float";
    for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " g" + S(c) + "_" + S(v) + " = 0.f";
    em.line(decl + ";");
    em.line("if (" + active + ") {");
    em.ind++;
    emit_vec_load(em, E3CONV_F32, V, "ldg", grow + " + " + S(c * pl.C), "g" + S(c));
    em.ind--;
    em.line("}");
  }
}

std::string bwd_prelude(Emitter& em, const Plan& pl, int dtype, const BwdShape& b) {
  const bool f16 = dtype == E3CONV_F16;
  em.line(std::string("// generated by libe3conv: backward of the equivariant convolution (") +
          "C=" + S(pl.C) + " nx=" + S(pl.nx) + " ny=" + S(pl.ny) + " nout=" + S(pl.nout) +
          " paths=" + S(pl.paths.size()) + " dtype=" + (f16 ? "f16" : "f32") + " V=" + S(b.V) +
          " TL=" + S(b.TL) + " ipw=" + S(b.ipw) + ")");
  emit_prelude(em);
  return f16 ? "unsigned short" : "float";
}

std::string bwd_edges_source(const Plan& pl, int dtype, const BwdShape& b) {
  Emitter em;
  const std::string T = bwd_prelude(em, pl, dtype, b);
  const int V = b.V;
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(b.block) + ") e3conv_bwd_edges(");
  em.line("    const " + T + "* __restrict__ x, const " + T + "* __restrict__ Y, const " + T +
          "* __restrict__ s,");
  em.line("    const int* __restrict__ senders, const int* __restrict__ row_ptr, int num_nodes,");
  em.line("    const float* __restrict__ g, float* __restrict__ gY, float* __restrict__ gs,");
  em.line("    float inv_avg, unsigned int* __restrict__ status)");
  em.line("{");
  em.ind++;
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const long long gwarp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;");
  em.line("const int sub = lane / " + S(b.TL) + ";");
  em.line("const int within = lane - sub * " + S(b.TL) + ";");
  em.line("const unsigned int item_mask = " + std::string(b.TL == 32 ? "0xffffffffu" :
          "((1u << " + S(b.TL) + ") - 1u) << (sub * " + S(b.TL) + ")") + ";");
  em.line("const long long bb = gwarp * " + S(b.ipw) + " + sub;");
  em.line("if (bb >= num_nodes) return;  // the whole item (lanes of one receiver) leaves");
  em.line("const int u0 = within * " + S(V) + ";");
  em.line("const bool active = u0 < " + S(pl.C) + ";");
  em.line("const int e_base = __ldg(row_ptr), e_end = __ldg(row_ptr + num_nodes);");
  em.line("int e0 = row_ptr[bb], e1 = row_ptr[bb + 1];");
  em.line("if (e0 < e_base || e1 < e0 || e1 > e_end) { if (within == 0) atomicOr(status, 1u); e1 = e0; }");
  em.line("if (e0 == e1) return;");
  emit_g_load(em, pl, V, "g + bb * " + S(static_cast<long long>(pl.nout) * pl.C) + " + u0", 0,
              pl.nout, "active");
  em.line("#pragma unroll 1");
  em.line("for (int e = e0; e < e1; ++e) {");
  em.ind++;
  em.line("const long long le = e - e_base;");
  em.line("const int a = senders[le];");
  em.line("const bool valid = (unsigned int)a < (unsigned int)num_nodes;");
  em.line("if (!valid && within == 0) atomicOr(status, 2u);");
  em.line("const " + T + "* yr = Y + le * " + S(pl.ny) + ";");
  emit_y_load(em, pl, dtype, "ldg", "yr");
  std::string dy = "float";
  for (int j = 0; j < pl.ny; ++j) dy += std::string(j ? "," : "") + " dy" + S(j) + " = 0.f";
  em.line(dy + ";");
  em.line("const bool go = valid && active;");
  em.line("const " + T + "* xr = x + (long long)(valid ? a : 0) * " + S(pl.nx * pl.C) + " + u0;");
  em.line("const " + T + "* sr = s + le * " + S(s_row) + " + u0;");
  em.line("float* gsr = gs + le * " + S(s_row) + " + u0;");
  size_t p = 0;
  while (p < pl.paths.size()) {
    const int n1 = pl.paths[p].n1;
    size_t q = p;
    while (q < pl.paths.size() && pl.paths[q].n1 == n1) ++q;
    const Path& first = pl.paths[p];
    const int d1 = 2 * first.l1 + 1;
    em.line("{  // node irrep " + S(n1) + " (l=" + S(first.l1) + ")");
    em.ind++;
    for (int i = 0; i < d1; ++i) {
      std::string decl = "float";
      for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " x" + S(i) + "_" + S(v) + " = 0.f";
      em.line(decl + ";");
      em.line("if (go) {");
      em.ind++;
      emit_vec_load(em, dtype, V, "ldg", "xr + " + S((first.x_off + i) * pl.C), "x" + S(i));
      em.ind--;
      em.line("}");
    }
    for (size_t r = p; r < q; ++r) {
      const Path& P = pl.paths[r];
      const int d3 = 2 * P.l3 + 1;
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3));
      em.ind++;
      {
        std::string decl = "float";
        for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " s_" + S(v) + " = 0.f";
        em.line(decl + ";");
        em.line("if (go) {");
        em.ind++;
        emit_vec_load(em, dtype, V, "ldg", "sr + " + S(static_cast<long long>(r) * pl.C), "s");
        em.ind--;
        em.line("}");
      }
      // t_k = sum (c Y_j) x_i   (for gs);  dY_j += c (s x_i) g_k   (summed over channels)
      for (int k = 0; k < d3; ++k)
        for (int v = 0; v < V; ++v) em.line("float t" + S(k) + "_" + S(v) + " = 0.f;");
      for (int i = 0; i < d1; ++i)
        for (int v = 0; v < V; ++v)
          em.line("const float z" + S(i) + "_" + S(v) + " = s_" + S(v) + " * x" + S(i) + "_" + S(v) + ";");
      for (const auto& n : P.nnz) {
        const std::string c = flt(n.c);
        const std::string yj = "y" + S(P.y_off + n.j);
        for (int v = 0; v < V; ++v) {
          const std::string xv = "x" + S(n.i) + "_" + S(v), zv = "z" + S(n.i) + "_" + S(v);
          const std::string gv = "g" + S(P.out_off + n.k) + "_" + S(v);
          em.line("t" + S(n.k) + "_" + S(v) + " = fmaf(" + c + " * " + yj + ", " + xv + ", t" +
                  S(n.k) + "_" + S(v) + ");");
          em.line("dy" + S(P.y_off + n.j) + " = fmaf(" + c + ", " + zv + " * " + gv + ", dy" +
                  S(P.y_off + n.j) + ");");
        }
      }
      // gs[e, p, u0..u0+V) = inv_avg sum_k g_k t_k
      std::vector<std::string> dsv(V);
      for (int v = 0; v < V; ++v) {
        std::string acc = "0.f";
        for (int k = 0; k < d3; ++k)
          acc = "fmaf(g" + S(P.out_off + k) + "_" + S(v) + ", t" + S(k) + "_" + S(v) + ", " + acc + ")";
        dsv[v] = "inv_avg * " + acc;
      }
      em.line("if (active) {");
      em.ind++;
      const std::string dst = "gsr + " + S(static_cast<long long>(r) * pl.C);
      if (V % 4 == 0) {
        for (int v = 0; v < V; v += 4)
          em.line("*reinterpret_cast<float4*>(" + dst + " + " + S(v) + ") = make_float4(" + dsv[v] +
                  ", " + dsv[v + 1] + ", " + dsv[v + 2] + ", " + dsv[v + 3] + ");");
      } else if (V == 2) {
        em.line("*reinterpret_cast<float2*>(" + dst + ") = make_float2(" + dsv[0] + ", " + dsv[1] + ");");
      } else {
        em.line("*(" + dst + ") = " + dsv[0] + ";");
      }
      em.ind--;
      em.line("}");
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
    p = q;
  }
  // channel reduction of dY over the item's lanes (butterfly inside the item's aligned group
  // of TL lanes; items of one warp walk rows of different lengths, so the mask names only
  // the item's own lanes), then one lane stores
  for (int off = b.TL / 2; off >= 1; off /= 2)
    for (int j = 0; j < pl.ny; ++j)
      em.line("dy" + S(j) + " += __shfl_xor_sync(item_mask, dy" + S(j) + ", " + S(off) + ");");
  em.line("if (within == 0) {");
  em.ind++;
  for (int j = 0; j < pl.ny; ++j)
    em.line("gY[le * " + S(pl.ny) + " + " + S(j) + "] = inv_avg * dy" + S(j) + ";");
  em.ind--;
  em.line("}");
  em.ind--;
  em.line("}");
  em.ind--;
  em.line("}");
  return em.o.str();
}

// Edges kernel, staged: a warp per receiver row (32 lanes x V channels = C), its g row in
// registers as channel pairs; a two-stage per-warp ring in shared memory receives each edge's
// s row, sender row x and Y row by 16-byte cp.async copies (the Y row by 4-byte copies),
// issued one edge ahead.  Per edge and path, with A_ik = sum_j c_ijk Y_j formed per lane:
//   t_k = sum_i A_ik x_i                       (channel pairs, fma.rn.f32x2)
//   gs[e, p, c] = (1/N) sum_k g_k t_k
//   W_ik = sum_{lane's channels} (s x_i) g_k,   dY_j += sum_{(i,k)} c_ijk W_ik
// then dY is summed over the warp's lanes and lane 0 stores it.
std::string bwd_edges_staged_source(const Plan& pl, int dtype, const BwdShape& b, int part) {
  Emitter em;
  // this launch's output irreps and paths: the part's outputs, or all of them
  std::vector<bool> own_out(pl.outputs.size(), true), own_path(pl.paths.size(), true);
  if (b.eparts > 1)
    for (size_t o = 0; o < pl.outputs.size(); ++o) own_out[o] = b.out_part[o] == part;
  std::vector<int> slot(pl.paths.size(), -1);  // the path's s segment in the ring
  int nslots = 0;
  for (size_t r = 0; r < pl.paths.size(); ++r) {
    own_path[r] = own_out[pl.paths[r].o];
    if (own_path[r]) slot[r] = nslots++;
  }
  const bool accumulate = b.eparts > 1 && part > 0;  // adds to the grad_Y an earlier part stored
  const std::string T = bwd_prelude(em, pl, dtype, b);
  emit_pair_ops(em);
  em.line("__device__ __forceinline__ void upk(unsigned long long w, float& lo, float& hi) { asm(\"mov.b64 {%0, %1}, %2;\" : \"=f\"(lo), \"=f\"(hi) : \"l\"(w)); }");
  em.line("__device__ __forceinline__ void cp16(void* dst, const void* src) { asm volatile(\"cp.async.cg.shared.global [%0], [%1], 16;\" :: \"r\"(static_cast<unsigned int>(__cvta_generic_to_shared(dst))), \"l\"(src) : \"memory\"); }");
  em.line("__device__ __forceinline__ void cp4(void* dst, const void* src) { asm volatile(\"cp.async.ca.shared.global [%0], [%1], 4;\" :: \"r\"(static_cast<unsigned int>(__cvta_generic_to_shared(dst))), \"l\"(src) : \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_commit() { asm volatile(\"cp.async.commit_group;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_wait1() { asm volatile(\"cp.async.wait_group 1;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_wait0() { asm volatile(\"cp.async.wait_group 0;\" ::: \"memory\"); }");
  const bool f16 = dtype == E3CONV_F16;
  const int V = b.V, NG = V / 2, elem = f16 ? 2 : 4;
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  const int s_bytes = nslots * pl.C * elem;             // the part's scalars in the ring
  const int SB = s_bytes + b.x_bytes + b.y_bytes;
  em.line("// part " + S(part) + " of " + S(b.eparts) + ": " + S(nslots) + " of " + S(pl.paths.size()) +
          " paths" + (accumulate ? ", grad_Y added to the earlier part's" : ""));
  // a split launch holds less: as many blocks per SM as shared memory allows (at most three)
  const int minb = b.eparts > 1 ? std::max(1, std::min(3, (220 * 1024) / std::max(1, b.esmem[part]))) : 1;
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(b.block) +
          (minb > 1 ? ", " + S(minb) : std::string()) + ") e3conv_bwd_edges(");
  em.line("    const " + T + "* __restrict__ x, const " + T + "* __restrict__ Y, const " + T +
          "* __restrict__ s,");
  em.line("    const int* __restrict__ senders, const int* __restrict__ row_ptr, int num_nodes,");
  em.line("    const float* __restrict__ g, float* __restrict__ gY, float* __restrict__ gs,");
  em.line("    float inv_avg, unsigned int* __restrict__ status)");
  em.line("{");
  em.ind++;
  em.line("extern __shared__ __align__(16) unsigned char smem_[];");
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const long long bb = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;");
  em.line("if (bb >= num_nodes) return;  // the whole warp (one receiver) leaves");
  em.line("unsigned char* ring = smem_ + (threadIdx.x >> 5) * " + S(2 * SB) + ";");
  em.line("const int u0 = lane * " + S(V) + ";");
  em.line("const int e_base = __ldg(row_ptr), e_end = __ldg(row_ptr + num_nodes);");
  em.line("int e0 = row_ptr[bb], e1 = row_ptr[bb + 1];");
  em.line("if (e0 < e_base || e1 < e0 || e1 > e_end) { if (lane == 0) atomicOr(status, 1u); e1 = e0; }");
  em.line("if (e0 == e1) return;");
  // g row as pairs (the part's output components)
  std::vector<bool> own_k(pl.nout, false);
  for (size_t o = 0; o < pl.outputs.size(); ++o)
    if (own_out[o])
      for (int k = 0; k < 2 * pl.outputs[o].l + 1; ++k) own_k[pl.outputs[o].off + k] = true;
  for (int k = 0; k < pl.nout; ++k) {
    if (!own_k[k]) continue;
    const std::string src = "g + bb * " + S(static_cast<long long>(pl.nout) * pl.C) + " + " +
                            S(static_cast<long long>(k) * pl.C) + " + u0";
    if (NG == 2) {
      em.line("unsigned long long g" + S(k) + "_0, g" + S(k) + "_1; { const float4 t_ = ldg_f4(" + src +
              "); g" + S(k) + "_0 = pk(t_.x, t_.y); g" + S(k) + "_1 = pk(t_.z, t_.w); }");
    } else {
      for (int q = 0; q < NG; ++q)
        em.line("unsigned long long g" + S(k) + "_" + S(q) + "; { const float2 t_ = ldg_f2(" + src +
                " + " + S(2 * q) + "); g" + S(k) + "_" + S(q) + " = pk(t_.x, t_.y); }");
    }
  }
  // copy issue of edge e into stage st (every lane; the s and x rows in 16-byte pieces)
  em.line("auto issue = [&](int e, int st) {");
  em.ind++;
  em.line("const long long le = e - e_base;");
  em.line("const int a = senders[le];");
  em.line("const bool valid = (unsigned int)a < (unsigned int)num_nodes;");
  em.line("if (!valid && lane == 0) atomicOr(status, 2u);");
  em.line("unsigned char* dst = ring + st * " + S(SB) + ";");
  em.line("const unsigned char* ssrc = reinterpret_cast<const unsigned char*>(s + le * " + S(s_row) + ");");
  if (nslots == static_cast<int>(pl.paths.size())) {
    em.line("#pragma unroll");
    em.line("for (int q = lane; q < " + S(s_bytes / 16) + "; q += 32) cp16(dst + 16 * q, ssrc + 16 * q);");
  } else {
    // the part's paths: one contiguous C-channel segment each
    const int seg = pl.C * elem / 16;
    for (size_t r = 0; r < pl.paths.size(); ++r)
      if (own_path[r])
        em.line("for (int q = lane; q < " + S(seg) + "; q += 32) cp16(dst + " + S(slot[r] * pl.C * elem) +
                " + 16 * q, ssrc + " + S(static_cast<long long>(r) * pl.C * elem) + " + 16 * q);");
  }
  em.line("if (valid) {");
  em.line("  const unsigned char* xsrc = reinterpret_cast<const unsigned char*>(x + (long long)a * " +
          S(static_cast<long long>(pl.nx) * pl.C) + ");");
  em.line("  #pragma unroll");
  em.line("  for (int q = lane; q < " + S(b.x_bytes / 16) + "; q += 32) cp16(dst + " + S(s_bytes) +
          " + 16 * q, xsrc + 16 * q);");
  em.line("} else {");
  em.line("  #pragma unroll");
  em.line("  for (int q = lane; q < " + S(b.x_bytes / 16) + "; q += 32) *reinterpret_cast<uint4*>(dst + " +
          S(s_bytes) + " + 16 * q) = make_uint4(0u, 0u, 0u, 0u);");
  em.line("}");
  em.line("const unsigned char* ysrc = reinterpret_cast<const unsigned char*>(Y + le * " + S(pl.ny) + ");");
  em.line("for (int q = lane; q < " + S(pl.ny * elem / 4) + "; q += 32) cp4(dst + " +
          S(s_bytes + b.x_bytes) + " + 4 * q, ysrc + 4 * q);");
  em.line("cp_commit();");
  em.ind--;
  em.line("};");
  em.line("const unsigned long long inv2 = bc(inv_avg);");
  em.line("issue(e0, 0);");
  em.line("#pragma unroll 1");
  em.line("for (int e = e0; e < e1; ++e) {");
  em.ind++;
  em.line("const int st = (e - e0) & 1;");
  em.line("if (e + 1 < e1) issue(e + 1, st ^ 1); else cp_commit();");
  em.line("cp_wait1();");
  em.line("__syncwarp();");
  em.line("const long long le = e - e_base;");
  em.line("const unsigned char* cur = ring + st * " + S(SB) + ";");
  em.line("const " + T + "* ys = reinterpret_cast<const " + T + "*>(cur + " + S(s_bytes + b.x_bytes) + ");");
  emit_y_load(em, pl, dtype, "lds", "ys");
  em.line("const " + T + "* xs = reinterpret_cast<const " + T + "*>(cur + " + S(s_bytes) + ") + u0;");
  em.line("const " + T + "* ss = reinterpret_cast<const " + T + "*>(cur) + u0;");
  em.line("float* gsr = gs + le * " + S(s_row) + " + u0;");
  {
    std::string dy = "float";
    for (int j = 0; j < pl.ny; ++j) dy += std::string(j ? "," : "") + " dy" + S(j) + " = 0.f";
    em.line(dy + ";");
  }
  // loads V channels of a shared row into NG pairs name_0 .. name_{NG-1}
  auto load_pairs = [&](const std::string& ptr, const std::string& name) {
    if (f16) {
      if (NG == 2) {
        em.line("unsigned long long " + name + "_0, " + name + "_1; { const uint2 t_ = lds_u2(" + ptr +
                "); " + name + "_0 = pk(lo_h2f(t_.x), hi_h2f(t_.x)); " + name +
                "_1 = pk(lo_h2f(t_.y), hi_h2f(t_.y)); }");
      } else {
        for (int q = 0; q < NG; ++q)
          em.line("unsigned long long " + name + "_" + S(q) + "; { const unsigned int t_ = lds_u1(" + ptr +
                  " + " + S(2 * q) + "); " + name + "_" + S(q) + " = pk(lo_h2f(t_), hi_h2f(t_)); }");
      }
    } else {
      if (NG == 2) {
        em.line("unsigned long long " + name + "_0, " + name + "_1; { const float4 t_ = lds_f4(" + ptr +
                "); " + name + "_0 = pk(t_.x, t_.y); " + name + "_1 = pk(t_.z, t_.w); }");
      } else {
        for (int q = 0; q < NG; ++q)
          em.line("unsigned long long " + name + "_" + S(q) + "; { const float2 t_ = lds_f2(" + ptr +
                  " + " + S(2 * q) + "); " + name + "_" + S(q) + " = pk(t_.x, t_.y); }");
      }
    }
  };
  size_t p = 0;
  while (p < pl.paths.size()) {
    const int n1 = pl.paths[p].n1;
    size_t q = p;
    while (q < pl.paths.size() && pl.paths[q].n1 == n1) ++q;
    const Path& first = pl.paths[p];
    const int d1 = 2 * first.l1 + 1;
    em.line("{  // node irrep " + S(n1) + " (l=" + S(first.l1) + ")");
    em.ind++;
    for (size_t r = p; r < q; ++r) {
      if (!own_path[r]) continue;
      const Path& P = pl.paths[r];
      const int d3 = 2 * P.l3 + 1;
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3));
      em.ind++;
      load_pairs("ss + " + S(static_cast<long long>(slot[r]) * pl.C), "s");
      // distinct (i, k) of the path with their (j, c) terms
      std::map<std::pair<int, int>, std::vector<std::pair<int, double>>> ik;
      for (const auto& n : P.nnz) ik[{n.i, n.k}].push_back({n.j, n.c});
      std::vector<bool> zi(d1, false), tk(d3, false);
      for (const auto& kv : ik) {
        zi[kv.first.first] = true;
        tk[kv.first.second] = true;
      }
      {
        std::string decl;
        for (int k = 0; k < d3; ++k)
          if (tk[k])
            for (int g = 0; g < NG; ++g)
              decl += (decl.empty() ? "" : ", ") + std::string("t") + S(k) + "_" + S(g) + " = 0ull";
        if (!decl.empty()) em.line("unsigned long long " + decl + ";");
      }
      // (i, k) in i-major order: z_i = s x_i is formed just before its first use, so one z_i
      // is live at a time
      std::vector<bool> started(d3, false);
      int zopen = -1;
      for (const auto& kv : ik) {
        const int i = kv.first.first, k = kv.first.second;
        if (i != zopen) {
          if (zopen >= 0) {
            em.ind--;
            em.line("}");
          }
          em.line("{  // x" + S(i) + " (from the ring) and z" + S(i) + " = s x" + S(i));
          em.ind++;
          load_pairs("xs + " + S((first.x_off + i) * pl.C), "x" + S(i));
          for (int g = 0; g < NG; ++g)
            em.line("const unsigned long long z" + S(i) + "_" + S(g) + " = mul2(s_" + S(g) + ", x" + S(i) +
                    "_" + S(g) + ");");
          zopen = i;
        }
        std::string expr;
        for (const auto& jc : kv.second) {
          const std::string yj = "y" + S(P.y_off + jc.first);
          expr = expr.empty() ? flt(jc.second) + " * " + yj
                              : "fmaf(" + flt(jc.second) + ", " + yj + ", " + expr + ")";
        }
        em.line("{  // (i, k) = (" + S(i) + ", " + S(k) + ")");
        em.ind++;
        em.line("const unsigned long long A_ = bc(" + expr + ");");
        for (int g = 0; g < NG; ++g) {
          const std::string tv = "t" + S(k) + "_" + S(g), xv = "x" + S(i) + "_" + S(g);
          em.line(tv + " = " + (started[k] ? "fma2(A_, " + xv + ", " + tv + ")" : "mul2(A_, " + xv + ")") + ";");
        }
        started[k] = true;
        std::string w = "mul2(z" + S(i) + "_0, g" + S(P.out_off + k) + "_0)";
        for (int g = 1; g < NG; ++g)
          w = "fma2(z" + S(i) + "_" + S(g) + ", g" + S(P.out_off + k) + "_" + S(g) + ", " + w + ")";
        em.line("float wl_, wh_; upk(" + w + ", wl_, wh_);");
        em.line("const float W_ = wl_ + wh_;");
        for (const auto& jc : kv.second) {
          const std::string dj = "dy" + S(P.y_off + jc.first);
          em.line(dj + " = fmaf(" + flt(jc.second) + ", W_, " + dj + ");");
        }
        em.ind--;
        em.line("}");
      }
      if (zopen >= 0) {
        em.ind--;
        em.line("}");
      }
      // gs[e, p, u0 ..] = inv_avg sum_k g_k t_k
      em.line("{");
      em.ind++;
      for (int g = 0; g < NG; ++g) {
        std::string a_;
        for (int k = 0; k < d3; ++k) {
          if (!tk[k]) continue;
          const std::string gk = "g" + S(P.out_off + k) + "_" + S(g), tv = "t" + S(k) + "_" + S(g);
          a_ = a_.empty() ? "mul2(" + gk + ", " + tv + ")" : "fma2(" + gk + ", " + tv + ", " + a_ + ")";
        }
        em.line("const unsigned long long o" + S(g) + "_ = " + (a_.empty() ? "0ull" : "mul2(inv2, " + a_ + ")") + ";");
      }
      const std::string dst = "gsr + " + S(static_cast<long long>(r) * pl.C);
      if (NG == 2) {
        em.line("float a0_, a1_, a2_, a3_; upk(o0_, a0_, a1_); upk(o1_, a2_, a3_);");
        em.line("*reinterpret_cast<float4*>(" + dst + ") = make_float4(a0_, a1_, a2_, a3_);");
      } else {
        for (int g = 0; g < NG; ++g)
          em.line("{ float a_, b_; upk(o" + S(g) + "_, a_, b_); *reinterpret_cast<float2*>(" + dst + " + " +
                  S(2 * g) + ") = make_float2(a_, b_); }");
      }
      em.ind--;
      em.line("}");
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
    p = q;
  }
  for (int off = 16; off >= 1; off /= 2)
    for (int j = 0; j < pl.ny; ++j)
      em.line("dy" + S(j) + " += __shfl_xor_sync(0xffffffffu, dy" + S(j) + ", " + S(off) + ");");
  em.line("if (lane == 0) {");
  em.ind++;
  for (int j = 0; j < pl.ny; ++j)
    em.line("gY[le * " + S(pl.ny) + " + " + S(j) + "] = " +
            (accumulate ? "gY[le * " + S(pl.ny) + " + " + S(j) + "] + " : std::string()) + "inv_avg * dy" +
            S(j) + ";");
  em.ind--;
  em.line("}");
  em.line("__syncwarp();  // every lane has read this stage before the next edge's copies reuse it");
  em.ind--;
  em.line("}");
  em.line("cp_wait0();");
  em.ind--;
  em.line("}");
  return em.o.str();
}

// Nodes kernel, staged: a warp per sender (32 lanes x V channels = C) walks the sender's
// edges in sender order; a two-stage per-warp ring receives each edge's s row, its
// receiver's gradient row g (float32) and its Y row by cp.async, one edge ahead.  Per edge
// and path, with A_ik = sum_j c_ijk Y_j formed per lane and u_k = s g_k (channel pairs):
//   h_i += sum_k A_ik u_k,   grad_x[a] = (1/N) h.
std::string bwd_nodes_staged_source(const Plan& pl, int dtype, const BwdShape& b, int part) {
  Emitter em;
  // this launch's output irreps (their gradient rows and paths), as in the edges kernel
  std::vector<bool> own_out(pl.outputs.size(), true);
  if (b.eparts > 1)
    for (size_t o = 0; o < pl.outputs.size(); ++o) own_out[o] = b.out_part[o] == part;
  std::vector<int> slot(pl.paths.size(), -1), gpos(pl.outputs.size(), -1);
  int nslots = 0, ncomp = 0;
  for (size_t r = 0; r < pl.paths.size(); ++r)
    if (own_out[pl.paths[r].o]) slot[r] = nslots++;
  for (size_t o = 0; o < pl.outputs.size(); ++o)
    if (own_out[o]) {
      gpos[o] = ncomp;
      ncomp += 2 * pl.outputs[o].l + 1;
    }
  const bool accumulate = b.eparts > 1 && part > 0;
  const std::string T = bwd_prelude(em, pl, dtype, b);
  emit_pair_ops(em);
  em.line("__device__ __forceinline__ void upk(unsigned long long w, float& lo, float& hi) { asm(\"mov.b64 {%0, %1}, %2;\" : \"=f\"(lo), \"=f\"(hi) : \"l\"(w)); }");
  em.line("__device__ __forceinline__ void cp16(void* dst, const void* src) { asm volatile(\"cp.async.cg.shared.global [%0], [%1], 16;\" :: \"r\"(static_cast<unsigned int>(__cvta_generic_to_shared(dst))), \"l\"(src) : \"memory\"); }");
  em.line("__device__ __forceinline__ void cp4(void* dst, const void* src) { asm volatile(\"cp.async.ca.shared.global [%0], [%1], 4;\" :: \"r\"(static_cast<unsigned int>(__cvta_generic_to_shared(dst))), \"l\"(src) : \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_commit() { asm volatile(\"cp.async.commit_group;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_wait1() { asm volatile(\"cp.async.wait_group 1;\" ::: \"memory\"); }");
  em.line("__device__ __forceinline__ void cp_wait0() { asm volatile(\"cp.async.wait_group 0;\" ::: \"memory\"); }");
  const bool f16 = dtype == E3CONV_F16;
  const int V = b.V, NG = V / 2, elem = f16 ? 2 : 4;
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  const long long g_row = static_cast<long long>(pl.nout) * pl.C;
  const int s_bytes = nslots * pl.C * elem, g_bytes = ncomp * pl.C * 4;
  const int SB = s_bytes + g_bytes + b.y_bytes;
  const int g_off = s_bytes, y_off = s_bytes + g_bytes;
  em.line("// part " + S(part) + " of " + S(b.eparts) + ": " + S(nslots) + " of " + S(pl.paths.size()) +
          " paths" + (accumulate ? ", grad_x added to the earlier part's" : ""));
  const int minb = std::max(1, std::min(3, (220 * 1024) / std::max(1, (b.block / 32) * 2 * SB)));
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(b.block) +
          (minb > 1 ? ", " + S(minb) : std::string()) + ") e3conv_bwd_nodes(");
  em.line("    const " + T + "* __restrict__ Y, const " + T + "* __restrict__ s,");
  em.line("    const int* __restrict__ receivers, const int* __restrict__ row_ptr,");
  em.line("    const int* __restrict__ sender_row_ptr, const int* __restrict__ sender_perm,");
  em.line("    int num_nodes, const float* __restrict__ g, float* __restrict__ gx, float inv_avg,");
  em.line("    unsigned int* __restrict__ status)");
  em.line("{");
  em.ind++;
  em.line("extern __shared__ __align__(16) unsigned char smem_[];");
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const long long a = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;");
  em.line("if (a >= num_nodes) return;  // the whole warp (one sender) leaves");
  em.line("unsigned char* ring = smem_ + (threadIdx.x >> 5) * " + S(2 * SB) + ";");
  em.line("const int u0 = lane * " + S(V) + ";");
  em.line("const int e_base = __ldg(row_ptr), e_end = __ldg(row_ptr + num_nodes);");
  em.line("const int ne = e_end - e_base;");
  for (int i = 0; i < pl.nx; ++i) {
    std::string l = "unsigned long long";
    for (int g = 0; g < NG; ++g) l += std::string(g ? "," : "") + " h" + S(i) + "_" + S(g) + " = 0ull";
    em.line(l + ";");
  }
  em.line("int t0 = sender_row_ptr[a], t1 = sender_row_ptr[a + 1];");
  em.line("if (t0 < 0 || t1 < t0 || t1 > ne) { if (lane == 0) atomicOr(status, 1u); t1 = t0; }");
  em.line("auto issue = [&](int t, int st) {");
  em.ind++;
  em.line("int le = sender_perm[t];");
  em.line("bool valid = (unsigned int)le < (unsigned int)ne;");
  em.line("const int bb = valid ? receivers[le] : 0;");
  em.line("valid = valid && (unsigned int)bb < (unsigned int)num_nodes;");
  em.line("if (!valid && lane == 0) atomicOr(status, 2u);");
  em.line("unsigned char* dst = ring + st * " + S(SB) + ";");
  em.line("if (valid) {");
  em.ind++;
  em.line("const unsigned char* ssrc = reinterpret_cast<const unsigned char*>(s + (long long)le * " + S(s_row) + ");");
  em.line("const unsigned char* gsrc = reinterpret_cast<const unsigned char*>(g + (long long)bb * " + S(g_row) + ");");
  em.line("const unsigned char* ysrc = reinterpret_cast<const unsigned char*>(Y + (long long)le * " + S(pl.ny) + ");");
  for (size_t r = 0; r < pl.paths.size(); ++r)      // the part's paths' scalars
    if (slot[r] >= 0)
      em.line("for (int q = lane; q < " + S(pl.C * elem / 16) + "; q += 32) cp16(dst + " +
              S(slot[r] * pl.C * elem) + " + 16 * q, ssrc + " + S(static_cast<long long>(r) * pl.C * elem) +
              " + 16 * q);");
  for (size_t o = 0; o < pl.outputs.size(); ++o)     // the part's gradient components
    if (gpos[o] >= 0)
      em.line("for (int q = lane; q < " + S((2 * pl.outputs[o].l + 1) * pl.C * 4 / 16) + "; q += 32) cp16(dst + " +
              S(g_off + gpos[o] * pl.C * 4) + " + 16 * q, gsrc + " +
              S(static_cast<long long>(pl.outputs[o].off) * pl.C * 4) + " + 16 * q);");
  em.line("for (int q = lane; q < " + S(pl.ny * elem / 4) + "; q += 32) cp4(dst + " + S(y_off) + " + 4 * q, ysrc + 4 * q);");
  em.ind--;
  em.line("} else {  // a bad index contributes nothing: a zero row of scalars and harmonics");
  em.ind++;
  em.line("#pragma unroll");
  em.line("for (int q = lane; q < " + S(s_bytes / 16) + "; q += 32) *reinterpret_cast<uint4*>(dst + 16 * q) = make_uint4(0u, 0u, 0u, 0u);");
  em.line("#pragma unroll");
  em.line("for (int q = lane; q < " + S(g_bytes / 16) + "; q += 32) *reinterpret_cast<uint4*>(dst + " + S(g_off) + " + 16 * q) = make_uint4(0u, 0u, 0u, 0u);");
  em.line("for (int q = lane; q < " + S(b.y_bytes / 4) + "; q += 32) *reinterpret_cast<unsigned int*>(dst + " + S(y_off) + " + 4 * q) = 0u;");
  em.ind--;
  em.line("}");
  em.line("cp_commit();");
  em.ind--;
  em.line("};");
  em.line("if (t0 < t1) issue(t0, 0);");
  em.line("#pragma unroll 1");
  em.line("for (int t = t0; t < t1; ++t) {");
  em.ind++;
  em.line("const int st = (t - t0) & 1;");
  em.line("if (t + 1 < t1) issue(t + 1, st ^ 1); else cp_commit();");
  em.line("cp_wait1();");
  em.line("__syncwarp();");
  em.line("const unsigned char* cur = ring + st * " + S(SB) + ";");
  em.line("const " + T + "* ys = reinterpret_cast<const " + T + "*>(cur + " + S(y_off) + ");");
  emit_y_load(em, pl, dtype, "lds", "ys");
  em.line("const " + T + "* ss = reinterpret_cast<const " + T + "*>(cur) + u0;");
  em.line("const float* gs_ = reinterpret_cast<const float*>(cur + " + S(g_off) + ") + u0;");
  auto load_s = [&](const std::string& ptr) {
    if (f16) {
      if (NG == 2)
        em.line("unsigned long long s_0, s_1; { const uint2 t_ = lds_u2(" + ptr + "); s_0 = pk(lo_h2f(t_.x), hi_h2f(t_.x)); s_1 = pk(lo_h2f(t_.y), hi_h2f(t_.y)); }");
      else
        for (int q = 0; q < NG; ++q)
          em.line("unsigned long long s_" + S(q) + "; { const unsigned int t_ = lds_u1(" + ptr + " + " + S(2 * q) + "); s_" + S(q) + " = pk(lo_h2f(t_), hi_h2f(t_)); }");
    } else {
      if (NG == 2)
        em.line("unsigned long long s_0, s_1; { const float4 t_ = lds_f4(" + ptr + "); s_0 = pk(t_.x, t_.y); s_1 = pk(t_.z, t_.w); }");
      else
        for (int q = 0; q < NG; ++q)
          em.line("unsigned long long s_" + S(q) + "; { const float2 t_ = lds_f2(" + ptr + " + " + S(2 * q) + "); s_" + S(q) + " = pk(t_.x, t_.y); }");
    }
  };
  for (size_t o = 0; o < pl.outputs.size(); ++o) {
    if (!own_out[o]) continue;
    const int d3 = 2 * pl.outputs[o].l + 1, off = gpos[o];  // off: the component in the ring
    bool any = false;
    for (const auto& P : pl.paths) any = any || P.o == static_cast<int>(o);
    if (!any) continue;
    em.line("{  // output irrep " + S(o));
    em.ind++;
    for (int k = 0; k < d3; ++k) {
      if (NG == 2)
        em.line("unsigned long long g" + S(k) + "_0, g" + S(k) + "_1; { const float4 t_ = lds_f4(gs_ + " +
                S((off + k) * pl.C) + "); g" + S(k) + "_0 = pk(t_.x, t_.y); g" + S(k) + "_1 = pk(t_.z, t_.w); }");
      else
        for (int q = 0; q < NG; ++q)
          em.line("unsigned long long g" + S(k) + "_" + S(q) + "; { const float2 t_ = lds_f2(gs_ + " +
                  S((off + k) * pl.C + 2 * q) + "); g" + S(k) + "_" + S(q) + " = pk(t_.x, t_.y); }");
    }
    for (size_t r = 0; r < pl.paths.size(); ++r) {
      const Path& P = pl.paths[r];
      if (P.o != static_cast<int>(o)) continue;
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3));
      em.ind++;
      load_s("ss + " + S(static_cast<long long>(slot[r]) * pl.C));
      std::map<std::pair<int, int>, std::vector<std::pair<int, double>>> ki;  // k-major
      for (const auto& n : P.nnz) ki[{n.k, n.i}].push_back({n.j, n.c});
      int uopen = -1;
      for (const auto& kv : ki) {
        const int k = kv.first.first, i = kv.first.second;
        if (k != uopen) {
          if (uopen >= 0) {
            em.ind--;
            em.line("}");
          }
          em.line("{  // u" + S(k) + " = s g" + S(k));
          em.ind++;
          for (int g = 0; g < NG; ++g)
            em.line("const unsigned long long u" + S(k) + "_" + S(g) + " = mul2(s_" + S(g) + ", g" + S(k) + "_" + S(g) + ");");
          uopen = k;
        }
        std::string expr;
        for (const auto& jc : kv.second) {
          const std::string yj = "y" + S(P.y_off + jc.first);
          expr = expr.empty() ? flt(jc.second) + " * " + yj
                              : "fmaf(" + flt(jc.second) + ", " + yj + ", " + expr + ")";
        }
        em.line("{ const unsigned long long A_ = bc(" + expr + ");");
        for (int g = 0; g < NG; ++g) {
          const std::string hv = "h" + S(P.x_off + i) + "_" + S(g);
          em.line("  " + hv + " = fma2(A_, u" + S(k) + "_" + S(g) + ", " + hv + ");");
        }
        em.line("}");
      }
      if (uopen >= 0) {
        em.ind--;
        em.line("}");
      }
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
  }
  em.line("__syncwarp();  // every lane has read this stage before the next edge's copies reuse it");
  em.ind--;
  em.line("}");
  em.line("cp_wait0();");
  em.line("const unsigned long long inv2 = bc(inv_avg);");
  em.line("float* xo = gx + a * " + S(static_cast<long long>(pl.nx) * pl.C) + " + u0;");
  for (int i = 0; i < pl.nx; ++i) {
    const std::string dst = "xo + " + S(i * pl.C);
    if (NG == 2) {
      em.line("{ float a0_, a1_, a2_, a3_; upk(mul2(inv2, h" + S(i) + "_0), a0_, a1_); upk(mul2(inv2, h" + S(i) +
              "_1), a2_, a3_);");
      if (accumulate)
        em.line("  const float4 p_ = *reinterpret_cast<const float4*>(" + dst + "); a0_ += p_.x; a1_ += p_.y; a2_ += p_.z; a3_ += p_.w;");
      em.line("  *reinterpret_cast<float4*>(" + dst + ") = make_float4(a0_, a1_, a2_, a3_); }");
    } else {
      for (int g = 0; g < NG; ++g) {
        em.line("{ float a_, b_; upk(mul2(inv2, h" + S(i) + "_" + S(g) + "), a_, b_);");
        if (accumulate)
          em.line("  const float2 p_ = *reinterpret_cast<const float2*>(" + dst + " + " + S(2 * g) + "); a_ += p_.x; b_ += p_.y;");
        em.line("  *reinterpret_cast<float2*>(" + dst + " + " + S(2 * g) + ") = make_float2(a_, b_); }");
      }
    }
  }
  em.ind--;
  em.line("}");
  return em.o.str();
}

std::string bwd_nodes_source(const Plan& pl, int dtype, const BwdShape& b) {
  Emitter em;
  const std::string T = bwd_prelude(em, pl, dtype, b);
  const int V = b.V;
  const long long s_row = static_cast<long long>(pl.paths.size()) * pl.C;
  em.line("extern \"C\" __global__ void __launch_bounds__(" + S(b.block) + ") e3conv_bwd_nodes(");
  em.line("    const " + T + "* __restrict__ Y, const " + T + "* __restrict__ s,");
  em.line("    const int* __restrict__ receivers, const int* __restrict__ row_ptr,");
  em.line("    const int* __restrict__ sender_row_ptr, const int* __restrict__ sender_perm,");
  em.line("    int num_nodes, const float* __restrict__ g, float* __restrict__ gx, float inv_avg,");
  em.line("    unsigned int* __restrict__ status)");
  em.line("{");
  em.ind++;
  em.line("const int lane = threadIdx.x & 31;");
  em.line("const long long gwarp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;");
  em.line("const int sub = lane / " + S(b.TL) + ";");
  em.line("const int within = lane - sub * " + S(b.TL) + ";");
  em.line("const long long a = gwarp * " + S(b.ipw) + " + sub;");
  em.line("if (a >= num_nodes) return;");
  em.line("const int u0 = within * " + S(V) + ";");
  em.line("if (u0 >= " + S(pl.C) + ") return;");
  em.line("const int e_base = __ldg(row_ptr), e_end = __ldg(row_ptr + num_nodes);");
  em.line("const int ne = e_end - e_base;");
  for (int i = 0; i < pl.nx; ++i) {
    std::string l = "float";
    for (int v = 0; v < V; ++v) l += std::string(v ? "," : "") + " h" + S(i) + "_" + S(v) + " = 0.f";
    em.line(l + ";");
  }
  em.line("int t0 = sender_row_ptr[a], t1 = sender_row_ptr[a + 1];");
  em.line("if (t0 < 0 || t1 < t0 || t1 > ne) { if (within == 0) atomicOr(status, 1u); t1 = t0; }");
  em.line("#pragma unroll 1");
  em.line("for (int t = t0; t < t1; ++t) {");
  em.ind++;
  em.line("const int le = sender_perm[t];");
  em.line("if ((unsigned int)le >= (unsigned int)ne) { if (within == 0) atomicOr(status, 2u); continue; }");
  em.line("const int bb = receivers[le];");
  em.line("if ((unsigned int)bb >= (unsigned int)num_nodes) { if (within == 0) atomicOr(status, 2u); continue; }");
  em.line("const " + T + "* yr = Y + (long long)le * " + S(pl.ny) + ";");
  emit_y_load(em, pl, dtype, "ldg", "yr");
  em.line("const " + T + "* sr = s + (long long)le * " + S(s_row) + " + u0;");
  em.line("const float* gr = g + (long long)bb * " + S(static_cast<long long>(pl.nout) * pl.C) + " + u0;");
  // paths grouped by output irrep: g of the irrep loaded once
  for (size_t o = 0; o < pl.outputs.size(); ++o) {
    const int d3 = 2 * pl.outputs[o].l + 1, off = pl.outputs[o].off;
    em.line("{  // output irrep " + S(o));
    em.ind++;
    emit_g_load(em, pl, V, "gr", off, off + d3, "true");
    for (size_t r = 0; r < pl.paths.size(); ++r) {
      const Path& P = pl.paths[r];
      if (P.o != static_cast<int>(o)) continue;
      em.line("{  // path " + S(r) + ": " + S(P.l1) + " x " + S(P.l2) + " -> " + S(P.l3));
      em.ind++;
      {
        std::string decl = "float";
        for (int v = 0; v < V; ++v) decl += std::string(v ? "," : "") + " s_" + S(v);
        em.line(decl + ";");
        emit_vec_load(em, dtype, V, "ldg", "sr + " + S(static_cast<long long>(r) * pl.C), "s");
      }
      for (int k = 0; k < d3; ++k)
        for (int v = 0; v < V; ++v)
          em.line("const float w" + S(k) + "_" + S(v) + " = s_" + S(v) + " * g" + S(off + k) + "_" + S(v) + ";");
      for (const auto& n : P.nnz)
        for (int v = 0; v < V; ++v) {
          const std::string h = "h" + S(P.x_off + n.i) + "_" + S(v);
          em.line(h + " = fmaf(" + flt(n.c) + " * y" + S(P.y_off + n.j) + ", w" + S(n.k) + "_" +
                  S(v) + ", " + h + ");");
        }
      em.ind--;
      em.line("}");
    }
    em.ind--;
    em.line("}");
  }
  em.ind--;
  em.line("}");
  em.line("float* xo = gx + a * " + S(static_cast<long long>(pl.nx) * pl.C) + " + u0;");
  for (int i = 0; i < pl.nx; ++i) {
    const std::string dst = "xo + " + S(i * pl.C);
    auto h = [&](int v) { return "inv_avg * h" + S(i) + "_" + S(v); };
    if (V % 4 == 0) {
      for (int v = 0; v < V; v += 4)
        em.line("*reinterpret_cast<float4*>(" + dst + " + " + S(v) + ") = make_float4(" + h(v) + ", " +
                h(v + 1) + ", " + h(v + 2) + ", " + h(v + 3) + ");");
    } else if (V == 2) {
      em.line("*reinterpret_cast<float2*>(" + dst + ") = make_float2(" + h(0) + ", " + h(1) + ");");
    } else {
      em.line("*(" + dst + ") = " + h(0) + ";");
    }
  }
  em.ind--;
  em.line("}");
  return em.o.str();
}

}  // namespace

std::string generate_backward_source(const Plan& pl, int dtype, const BwdShape& b, bool nodes) {
  if (nodes) return b.nstaged ? bwd_nodes_staged_source(pl, dtype, b, 0) : bwd_nodes_source(pl, dtype, b);
  return b.staged ? bwd_edges_staged_source(pl, dtype, b, 0) : bwd_edges_source(pl, dtype, b);
}

std::string generate_backward_edges_part(const Plan& pl, int dtype, const BwdShape& b, int part) {
  return bwd_edges_staged_source(pl, dtype, b, part);
}

std::string generate_backward_nodes_part(const Plan& pl, int dtype, const BwdShape& b, int part) {
  return bwd_nodes_staged_source(pl, dtype, b, part);
}

// Standalone harmonics: one thread per edge evaluates the plan's polynomials of
// v / |v| (emit_sh_eval, as the forward does with edge vectors) and stores the row in
// the input dtype; 16-byte stores where the row length allows.
std::string generate_sh_source(const Plan& pl, int dtype) {
  Emitter em;
  const bool f16 = dtype == E3CONV_F16;
  const std::string T = f16 ? "unsigned short" : "float";
  em.line("// generated by libe3conv: real spherical harmonics of edge vectors");
  em.line("// lmax=" + S(pl.lmax) + " ny=" + S(pl.ny) + " dtype=" + (f16 ? "f16" : "f32"));
  em.line("__device__ __forceinline__ unsigned short f2h(float f) { unsigned short h; "
          "asm(\"cvt.rn.f16.f32 %0, %1;\" : \"=h\"(h) : \"f\"(f)); return h; }");
  em.line("__device__ __forceinline__ unsigned int pkh(float a, float b) { "
          "return static_cast<unsigned int>(f2h(a)) | (static_cast<unsigned int>(f2h(b)) << 16); }");
  em.line("extern \"C\" __global__ void __launch_bounds__(256) e3conv_edge_sh(const float4* "
          "__restrict__ vec, long long num_edges, " + T + "* __restrict__ out) {");
  em.ind++;
  em.line("for (long long e = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; e < num_edges;"
          " e += static_cast<long long>(gridDim.x) * 256) {");
  em.ind++;
  em.line("const float4 v_ = __ldg(vec + e);");
  emit_sh_eval(em, pl, "v_.x", "v_.y", "v_.z");
  em.line(T + "* o_ = out + e * " + S(pl.ny) + ";");
  auto y = [](int j) { return "y" + S(j); };
  if (!f16 && pl.ny % 4 == 0) {
    for (int j = 0; j < pl.ny; j += 4)
      em.line("reinterpret_cast<float4*>(o_)[" + S(j / 4) + "] = make_float4(" + y(j) + ", " +
              y(j + 1) + ", " + y(j + 2) + ", " + y(j + 3) + ");");
  } else if (f16 && pl.ny % 8 == 0) {
    for (int j = 0; j < pl.ny; j += 8)
      em.line("reinterpret_cast<uint4*>(o_)[" + S(j / 8) + "] = make_uint4(pkh(" + y(j) + ", " +
              y(j + 1) + "), pkh(" + y(j + 2) + ", " + y(j + 3) + "), pkh(" + y(j + 4) + ", " +
              y(j + 5) + "), pkh(" + y(j + 6) + ", " + y(j + 7) + "));");
  } else {
    for (int j = 0; j < pl.ny; ++j)
      em.line("o_[" + S(j) + "] = " + (f16 ? "f2h(" + y(j) + ")" : y(j)) + ";");
  }
  em.ind--;
  em.line("}");
  em.ind--;
  em.line("}");
  return em.o.str();
}

std::string generate_forward_source(const Plan& pl, int dtype, const Shape& sh) {
  if (sh.tc) return tc_source(pl, sh);
  return sh.stages > 0 ? staged_source(pl, dtype, sh) : direct_source(pl, dtype, sh);
}

}  // namespace e3c
