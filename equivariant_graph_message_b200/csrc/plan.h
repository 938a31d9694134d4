// Internal plan structures of libe3conv (host side).
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/e3conv.h"

namespace e3c {

struct Irrep {
  int mul, l, p;  // p = +1 even, -1 odd
  int dim() const { return 2 * l + 1; }
};

// One nonzero CG coefficient of a path: out[k] += c * x[i] * Y[j].
struct Nnz {
  int i, j, k;
  double c;
};

struct Path {
  int n1, l1, p1, x_off;  // node irrep index, degree, parity, first component
  int l2, y_off;          // harmonic degree, first component (l2^2)
  int o, l3, p3, out_off; // output irrep index, degree, parity, first component
  std::vector<double> cg; // dense [2l1+1][2l2+1][2l3+1], normalisation included
  std::vector<Nnz> nnz;   // entries with |c| > 1e-12
};

struct Output {
  int l, p, off;
};

// Launch shape of the generated forward kernel.
struct Shape {
  int V = 1;       // channels per lane
  int TL = 32;     // lanes per (receiver, channel tile) item
  int tiles = 1;   // channel tiles per receiver
  int ipw = 1;     // items per warp
  int block = 128; // threads per block
  bool dpipe = false;  // direct variant: the next edge's inputs loaded during this edge's products
  // Staged (persistent, shared-memory ring) variant; stages == 0: direct loads.
  int stages = 0;
  int s_bytes = 0, x_bytes = 0, y_bytes = 0;  // row sizes staged per edge
  int s_off = 0, x_off = 0, y_off = 0;        // offsets inside one stage
  int stage_bytes = 0;                        // tensor cores: one stage; staged: the whole ring
  int group = 1;                              // staged: edges per ring group (one s / Y copy each)
  int x_slot = 0;                             // staged: bytes between sender rows of the ring
  int team = 1;                               // warps that share one receiver row (32*V*team = C)
  int warp_smem = 0;                          // shared memory of one team (ring, A, barriers)
  int bar_off = 0, hdr_off = 0;               // offsets inside a team's region
  // Cooperative contraction (staged variant): per edge the warp first forms
  // A_p[i,k] = sum_j CG_p[i,j,k] Y_j in shared memory, then every lane applies
  // it to its channels with packed float32x2 FMAs.
  bool coop = false;
  bool dup_a = false;                         // A stored as (a, a) pairs (amode >= 1)
  int amode = 0;                              // A layout: 0 float slots, round order; 1 pairs, round
                                              // order; 2 pairs, apply order (two per 16-byte load)
  int psplit = 1;                             // > 1: the team's warps split a row's paths (each covers C)
  int na = 0;                                 // number of A entries (all paths)
  int a_off = 0, yf_off = 0;                  // A entries and float32 Y inside a team's region
  // Tensor-core variant (float16 inputs, C = 128): per edge, T = x^T (A_hi + A_lo)
  // with tcgen05.mma (M = 128 channels, K = 16 node components, N = ncols path
  // outputs) into tensor memory, then T is scaled by s per channel.
  bool tc = false;
  int ncols = 0;                              // sum over paths of 2l3+1, padded to 16
  int tmem_cols = 0;                          // tensor-memory columns allocated (power of 2)
  int tbufs = 0, tstride = 0;                 // teams per block (one T each), columns between their T
  int b_stride = 0;                           // bytes from A_hi to A_lo (tile + scratch)
  int b_off = 0, b_bytes = 0;                 // A_hi at b_off (b_bytes used by the MMA), A_lo at b_off + b_stride
  int tslot_off = 0;                          // tensor-memory address slot
  // Edge input: false = the harmonics Y [E][ny] in the input dtype; true = the
  // edge vectors r_ab as float32 [E][4] (x, y, z, unused), Y computed in the kernel.
  bool vec = false;
  int smem_request = 0;                       // dynamic shared memory requested per block
};

// One term coef * x^px y^py z^pz of a real spherical harmonic on the unit sphere.
struct ShMono {
  double coef;
  int px, py, pz;
};

// One entry A_p[i,k] of the per-edge contraction of CG with Y.
struct AEntry {
  int path, i, k;
  std::vector<std::pair<int, double>> terms;  // (index into the edge's Y row, CG coefficient)
};

// Launch shape of the backward kernels: V channels per lane, TL lanes (a power
// of two) per item, one item per node covering all C channels.
struct BwdShape {
  bool ok = false;
  int V = 1, TL = 32, ipw = 1, block = 128;
  // edges kernel with a per-warp shared-memory ring: the next edge's scalars, sender row
  // and harmonics are copied (cp.async) while this edge's products run; packed float32x2
  // arithmetic over channel pairs
  bool staged = false;
  int s_bytes = 0, x_bytes = 0, y_bytes = 0, stage_bytes = 0;  // one stage: s, x, Y rows
  int smem = 0;                                                // dynamic shared memory per block
  // nodes kernel (grad_x, sender order) with the same kind of ring: s, g (float32) and Y rows
  bool nstaged = false;
  int g_bytes = 0, nstage_bytes = 0, nsmem = 0;
  // edges kernel split over output irreps: eparts launches, out_part[o] = the launch of
  // output irrep o, esmem[p] = its dynamic shared memory per block
  int eparts = 1;
  std::vector<int> out_part;
  int esmem[4] = {0, 0, 0, 0};
  int nsmem_p[4] = {0, 0, 0, 0};  // the staged nodes kernel's launches, likewise
};

struct BwdVariant {
  bool compiled = false;
  BwdShape shape;
  // module 2 p + k: part p (of the split over the output irreps; part 0 when not split) of the
  // edges (k = 0) or nodes (k = 1) kernel
  std::string source[8];
  std::vector<char> cubin[8];
  std::string log[8];
  CUmodule module[8] = {};
  CUfunction fn[8] = {};
  int regs[8] = {-1, -1, -1, -1, -1, -1, -1, -1}, local_bytes[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
};

struct ShVariant {  // standalone harmonics kernel (compiled on first use)
  bool compiled = false;
  std::string source;
  std::vector<char> cubin;
  std::string log;
  CUmodule module = nullptr;
  CUfunction fn = nullptr;
  int regs = -1, local_bytes = -1;
};

struct Variant {
  bool compiled = false;
  Shape shape;
  std::string source;
  std::vector<char> cubin;
  std::string log;
  int regs = -1, local_bytes = -1;  // registers per thread; local memory per thread (stack frame)
  CUmodule module = nullptr;
  CUfunction fn = nullptr;
  int grid_blocks = 0;  // persistent grid of the staged variant (blocks per SM x SMs)
};

// Radial MLP of a plan (e3conv_set_radial_mlp): host copies of the packed
// weights and their device copies (owned by the plan).
struct RadialPlan {
  bool set = false;
  int nb = 0, hidden = 0, layers = 0, nout = 0, chunks = 0;
  double r_max = 0.0;
  int scale_exp_0 = 0, scale_exp_h = 0, scale_exp_o = 0;  // weights scaled by 2^s before the split
  std::vector<unsigned char> w0, wh, wo;  // packed hi / lo float16 operands
  void* d_w0 = nullptr;
  void* d_wh = nullptr;
  void* d_wo = nullptr;
};

// Irreps linear layer (e3conv_linear_*): per output irrep block, where its rows
// come from and which packed weights mix them.
constexpr int kLinMaxBlocks = 16;
struct LinBlock {
  int dim;          // 2l+1
  int in_off;       // first input element of the matching input irrep (-1: none)
  int out_off;      // first output element of the irrep
  int first_tile;   // first 128-row tile of the irrep (set per launch)
  long long w_off;  // matched weight block (prepare) / its byte offset (launch); -1: zeros
  float scale;      // scale / sqrt(mul_in) / 2^s
};

struct LinearPlan {
  std::vector<Irrep> in, out;
  int K = 0, N = 0;                 // mul_in, mul_out
  int dim_in = 0, dim_out = 0;      // floats per node row
  double scale = 1.0;
  int num_weight_blocks = 0;        // matched irreps, in output order
  std::vector<LinBlock> blocks;     // one per output irrep
  std::vector<unsigned char> packed;
  int scale_exp = 0;
  bool weights_set = false;
  bool allow_tma = true;            // the tensor-map kernel where the shape allows it
  int device = -1;
  void* d_w = nullptr;
  unsigned* status = nullptr;
  // arguments of the last tensor-map launch, reused while x, y and the node count repeat (a
  // layer is used from one host thread at a time)
  mutable std::vector<unsigned char> tma_args;
  mutable const void* tma_x = nullptr;
  mutable const void* tma_y = nullptr;
  mutable const void* tma_w = nullptr;
  mutable long long tma_nodes = -1;
};

struct Plan {
  int C = 0, nx = 0, ny = 0, nout = 0, lmax = 0;
  std::vector<Irrep> node, filt;
  std::vector<Path> paths;
  std::vector<Output> outputs;
  double avg = 1.0;
  int norm = 0;
  int dtype = E3CONV_F32;
  int req_V = 0, req_block = 0, req_stages = -1;  // -1: automatic
  int auto_block = 0;                              // block chosen after a first compile (0: none)
  int req_coop = -1;                               // -1: automatic, 0: off, 1: on
  int req_tc = -1;                                 // -1: automatic, 0: off, 1: on
  int req_dpipe = -1;                              // -1: automatic, 0/1: direct-variant pipelining
  int req_group = -1;                              // -1: automatic, else edges per ring group (1..4)
  int req_alayout = -1;                            // -1: automatic, else Shape::amode (channel pairs only)
  int req_vec = 0;                                 // 1: edges given as vectors, Y computed in the kernel
  int req_psplit = -1;                             // -1: automatic, 0/1: off, k: split a row's paths over k warps
  int req_bparts = -1;                             // -1: automatic, else launches of each backward kernel (1..4)
  int tc_team_cap = 0;                             // > 0: at most this many tensor-core teams per block
  bool tc_fallback = false;                        // tensor cores requested but the kernel spills: float32 variant
  int device = -1;                 // -1: host-only plan
  CUcontext ctx = nullptr;
  unsigned int* status = nullptr;  // device status word
  Variant var[2];
  BwdVariant bwd[2];               // backward kernels per input dtype (compiled on first use)
  ShVariant shk[2];                // standalone harmonics kernel per input dtype
  std::string trace[2];            // the forward's compile attempts (shape, registers, local bytes)
  RadialPlan radial;
};

// irreps.cpp
bool parse_irreps(const char* text, std::vector<Irrep>& out, std::string& err);
int build_paths(Plan& plan, std::string& err);

// cg.cpp
std::vector<double> real_wigner_3j(int l1, int l2, int l3);

// sh.cpp: component j = l^2 + l + m of the real harmonics, as polynomial terms
std::vector<std::vector<ShMono>> sh_polynomials(int lmax);

// radial.cu
int radial_prepare(RadialPlan& rp, int nb, double r_max, int hidden, int layers, const float* w0,
                   const float* const* wh, const float* wo, int nout, std::string& err);
size_t radial_smem_bytes(const RadialPlan& rp);
int radial_launch(const RadialPlan& rp, const void* dev_w0, const void* dev_wh, const void* dev_wo,
                  const float* vec, long long num_edges, void* s, int out_f16, unsigned* status,
                  int grid, cudaStream_t st, std::string& err, const CUtensorMap* smap);

// linear.cu
int linear_prepare(LinearPlan& lp, const std::vector<Irrep>& in, const std::vector<Irrep>& out,
                   double scale, std::string& err);
int linear_pack(LinearPlan& lp, const float* w, std::string& err);
size_t linear_smem_bytes(const LinearPlan& lp);
// cuTensorMapEncodeTiled, resolved by the caller through the runtime (nullptr: no tensor maps)
using TensorMapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                       const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                       const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                       CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
int linear_launch(const LinearPlan& lp, const void* dev_w, const float* x, long long nodes, float* y,
                  unsigned* status, int grid, cudaStream_t st, TensorMapEncodeFn encode,
                  std::string& err);
// whether linear_launch runs the tensor-map kernel for this layer (given an encoder)
bool linear_uses_tma(const LinearPlan& lp);

// codegen.cpp
std::vector<AEntry> build_a_entries(const Plan& plan);
Shape choose_shape(const Plan& plan, int dtype);
std::string generate_forward_source(const Plan& plan, int dtype, const Shape& shape);
BwdShape choose_backward_shape(const Plan& plan, int dtype);
std::string generate_backward_source(const Plan& plan, int dtype, const BwdShape& shape, bool nodes);
std::string generate_sh_source(const Plan& plan, int dtype);
std::string generate_backward_edges_part(const Plan& plan, int dtype, const BwdShape& shape, int part);
std::string generate_backward_nodes_part(const Plan& plan, int dtype, const BwdShape& shape, int part);

}  // namespace e3c

struct e3conv_plan_s {
  e3c::Plan p;
};

struct e3conv_linear_s {
  e3c::LinearPlan p;
};
