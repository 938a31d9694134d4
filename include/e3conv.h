/*
 * e3conv — equivariant message-passing convolution on one NVIDIA B200 (sm_100a).
 *
 * C ABI of libe3conv.so.  Plain pointers and sizes only; every device buffer
 * is owned and allocated by the caller.
 *
 * The operation (page "e3j.core.Convolution", class docstring and the
 * "__call__" parameter list):
 *
 *     m_b = (1/N) sum_{a -> b} (x_a (x)_CG Y_ab) . s_ab
 *
 *   x_a   node features of the sender a, irreps `irreps_node`, all with one
 *         multiplicity C (the channels);
 *   Y_ab  edge features, the real spherical harmonics of the edge (no channel
 *         axis; broadcast over channels, "__call__" notes);
 *   (x)_CG the channelwise ("uvu") Clebsch-Gordan tensor product: channel u
 *         of x times Y gives channel u of every produced irrep (cuEquivariance
 *         notes, "Dense polynomial": channelwise products, weights first);
 *   . s_ab  every path p and channel u is scaled by its own edge scalar
 *         s_ab[p, u] (e3j "__call__": edge_scalars (num_edges, num_scalars, C));
 *         paths that produce the same output irrep are summed;
 *   1/N   avg_num_neighbors (e3j parameters), N > 0.
 *
 * Layout (trailing channels, e3j "layout: TRAILING_CHANNELS is faster"):
 *   node_features [num_nodes][nx][C]     nx = sum over node irreps of 2l+1
 *   edge_sh       [num_edges][ny]        ny = (lmax+1)^2, l-major, m = -l..l
 *   edge_scalars  [num_edges][P][C]      P paths in the canonical order below
 *   out           [num_nodes][nout][C]   float32, nout = sum over produced
 *                                        output irreps of 2l+1
 * Edges must be sorted by receiver (e3j "__call__" note: fused kernels need
 * edges sorted by the endpoint of the graph ordering; RECEIVER ordering is
 * the one used here): the edges of receiver b are
 * receiver_row_ptr[b] .. receiver_row_ptr[b+1]-1, in any order.
 *
 * Canonical path order: node irrep (in the order given) -> spherical-harmonic
 * degree l2 (ascending) -> output irrep (in the order of `irreps_out`).  A
 * path (l1,p1) x (l2,(-1)^l2) -> (l3,p3) exists iff |l1-l2| <= l3 <= l1+l2
 * and p3 = p1 (-1)^l2.  `irreps_out` is a filter: output irreps no path
 * produces are dropped from `out` (e3j "target ... enforces a filter").
 *
 * Spherical-harmonic basis: real, component-normalised (sum_m Y_lm^2 = 2l+1),
 * no Condon-Shortley phase, z polar axis, components m = -l..l; l = 1 is
 * sqrt(3) (y, z, x).  The CG tensors are the real Wigner-3j tensors of this
 * basis with unit Frobenius norm, sign fixed so that the first nonzero entry
 * in row-major (i, j, k) order is positive, times sqrt(2 l3 + 1) for
 * E3CONV_NORM_SQRT_DIM_OUT (the e3j default normalisation) or times 1 for
 * E3CONV_NORM_NONE.
 *
 * Errors: every int-returning call returns E3CONV_OK (0) or an E3CONV_ERR_*
 * code; nothing is thrown across the ABI.  e3conv_last_error() gives a
 * message for the last failing call of the calling thread.  Device kernels
 * never trap: out-of-range indices they read are skipped and recorded in a
 * status word that e3conv_check() / e3conv_csr_check() report.
 *
 * Streams: every device call is stream-ordered on the given stream (NULL is
 * the legacy default stream), does not synchronise the host and does not
 * allocate device memory.  e3conv_stream has the same type as cudaStream_t.
 */
#ifndef E3CONV_H
#define E3CONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define E3CONV_VERSION 1

#if defined(__GNUC__)
#define E3CONV_API __attribute__((visibility("default")))
#else
#define E3CONV_API
#endif

typedef struct e3conv_plan_s* e3conv_plan;
typedef struct e3conv_linear_s* e3conv_linear;
typedef struct CUstream_st* e3conv_stream;

/* error codes */
#define E3CONV_OK 0
#define E3CONV_ERR_INVALID_ARG 1   /* null pointer, negative size, misaligned buffer ... */
#define E3CONV_ERR_IRREPS 2        /* irreps string malformed or inconsistent */
#define E3CONV_ERR_UNSUPPORTED 3   /* valid request this library does not implement */
#define E3CONV_ERR_CUDA 4          /* a CUDA runtime / driver call failed */
#define E3CONV_ERR_NOMEM 5         /* host or device allocation failed (plan creation only) */
#define E3CONV_ERR_COMPILE 6       /* NVRTC failed to compile the generated kernel */
#define E3CONV_ERR_NO_DEVICE 7     /* plan has no device module (created without a GPU) */
#define E3CONV_ERR_BAD_INDEX 8     /* a kernel met an out-of-range index (see checks) */
#define E3CONV_ERR_WORKSPACE 9     /* workspace missing or too small */

/* input element types */
#define E3CONV_F32 0
#define E3CONV_F16 1

/* CG normalisations */
#define E3CONV_NORM_SQRT_DIM_OUT 0
#define E3CONV_NORM_NONE 1

/* ---------------------------------------------------------------------------
 * Plans
 */

/* Builds a plan: parses the irreps, enumerates the paths, generates the real
 * CG tables in float64 on the host and compiles the forward kernel for
 * sm_100a with NVRTC (all CG coefficients unrolled as constants).  If a CUDA
 * device is current, the kernel module is loaded on it and a 4-byte status
 * word is allocated there; without a device the plan is host-only (queries
 * work, e3conv_forward returns E3CONV_ERR_NO_DEVICE).
 *   irreps_node: e.g. "128x0e+128x1o"; every multiplicity equal (C >= 1).
 *   irreps_sh:   "1x0e+1x1o+...+1xLp", consecutive l from 0, parity (-1)^l.
 *   irreps_out:  filter, e.g. "128x0e+128x1o+128x2e"; multiplicities = C;
 *                no irrep twice.
 *   avg_num_neighbors: N > 0 (finite).
 *   normalization: E3CONV_NORM_SQRT_DIM_OUT or E3CONV_NORM_NONE.
 * The input dtype starts as E3CONV_F32.  Degrees up to l = 6 are accepted.
 * On success *plan owns its host tables, module and status word; release it
 * with e3conv_destroy.  On failure *plan is set to NULL. */
E3CONV_API int e3conv_create(e3conv_plan* plan, const char* irreps_node, const char* irreps_sh,
                  const char* irreps_out, double avg_num_neighbors, int normalization);

/* Frees everything the plan owns.  NULL is accepted.  The caller must make
 * sure no forward launched with this plan is still running. */
E3CONV_API void e3conv_destroy(e3conv_plan plan);

/* Selects the element type of node_features, edge_sh and edge_scalars
 * (E3CONV_F32 or E3CONV_F16; accumulation and output stay float32).
 * Compiles and loads that kernel variant on first use (host-side, blocking). */
E3CONV_API int e3conv_set_input_dtype(e3conv_plan plan, int dtype);

/* Overrides the launch shape of the forward kernel: channels_per_lane in
 * {0 (automatic), 1, 2, 4, 8} (must divide C and fit one 16-byte load),
 * block_threads in {0 (automatic), 32, 64, ..., 1024}, and stages: -1
 * (automatic), 0 (direct global loads) or 2..8 (persistent warps with a
 * shared-memory ring of that many edges, used when one warp covers all C
 * channels and every staged row is a multiple of 16 bytes; otherwise the
 * direct variant is used).  Recompiles the current dtype's kernel
 * (host-side, blocking). */
E3CONV_API int e3conv_set_launch_config(e3conv_plan plan, int channels_per_lane, int block_threads,
                                        int stages);

/* Options of the forward kernel (host-side; each recompiles the current
 * dtype's kernel):
 *   Each option takes -1 (automatic) and the values listed with it.
 *   E3CONV_OPT_CONTRACT_FIRST: -1 automatic (default), 0 or 1.  With 1 the
 *   staged variant first contracts every path's CG tensor with the edge's Y
 *   into A_p[i,k] = sum_j CG_p[i,j,k] Y_j (channel-independent, shared by the
 *   warp in shared memory) and then applies A_p to each channel with packed
 *   float32x2 FMAs; with 0 every lane forms the products CG*Y_j itself.
 *   Same arithmetic up to rounding order. */
#define E3CONV_OPT_CONTRACT_FIRST 1
/*   E3CONV_OPT_TENSOR_CORES: 0 (default; -1 means the same) or 1.  With float16
 *   inputs, C = 128, at most 16 node components and at most 256 path outputs,
 *   the forward forms per edge T = x^T A on the tensor cores (tcgen05.mma,
 *   M = 128 channels, K = node components, N = path outputs; A = sum_j CG Y_j
 *   split into float16 hi + lo parts, float32 accumulation in tensor memory)
 *   and then scales T by the edge scalars with float32 FMAs.  It launches one
 *   block per SM (three teams of four warps, or two where three would spill
 *   registers; all 512 tensor-memory columns);
 *   a requested ring depth is used from 2 up, one that does not fit shared
 *   memory is lowered (e3conv_kernel_info reports the depth used).
 *   Requesting it for a shape outside those limits, or one whose kernel would
 *   still use local memory with two teams, keeps the float32 staged variant. */
#define E3CONV_OPT_TENSOR_CORES 2
/*   E3CONV_OPT_PATH_SPLIT: -1 automatic (default), 0 or 1 off, k = 2..8.  With
 *   k the staged contract-first variant gives each receiver row to a team of
 *   k warps that each cover all C channels (one warp must cover C: C/32
 *   channels per lane, 1 or even) and split the row's output irreps among
 *   themselves (balanced on FMA count): each warp forms only its paths' CG x Y
 *   contractions and keeps only its outputs' sums in registers, so more warps
 *   fit on an SM.  Same arithmetic per output element as without it.  Ignored
 *   (the usual shape) where it does not apply. */
#define E3CONV_OPT_PATH_SPLIT 3
/*   E3CONV_OPT_EDGE_VECTORS: 0 (default) or 1.  With 1 the forward's edge_sh
 *   argument holds the edge vectors r_ab = p_b - p_a as float32 [E][4]
 *   (x, y, z, ignored: 16-byte rows) in every input dtype, and the kernel
 *   evaluates the real spherical harmonics of r_ab / |r_ab| itself (the basis
 *   above, l <= the plan's lmax; a zero vector gives Y_0 = 1, the rest 0),
 *   in float32, instead of reading ny harmonics per edge. */
#define E3CONV_OPT_EDGE_VECTORS 4
/*   E3CONV_OPT_A_LAYOUT: -1 automatic (default), 0 .. 3: the shared-memory
 *   layout of the contract-first A entries where a lane holds channel pairs:
 *   0 float entries in the order they are formed (a lane duplicates each into
 *   a pair), 1 the entries stored as (a, a) pairs in that order, 2 (a, a)
 *   pairs in the order they are applied, read two per 16-byte load, 3 float
 *   entries in the order they are applied, read four per 16-byte load.
 *   Automatic: 0.  Same arithmetic. */
#define E3CONV_OPT_A_LAYOUT 5
/*   E3CONV_OPT_COPY_GROUP: -1 automatic (default: 1) or 1..4: the staged
 *   variant's ring takes up to this many consecutive edges of a row per group,
 *   with one bulk copy of their edge scalars, one of their harmonics and one
 *   mbarrier per group (sender rows stay one copy each).  The ring depth is
 *   rounded up to a multiple of the group.  Same arithmetic. */
#define E3CONV_OPT_COPY_GROUP 6
/*   E3CONV_OPT_DIRECT_PIPELINE: -1 automatic (default), 0 or 1: the direct
 *   variant (small channel counts) loads the next edge's sender row,
 *   harmonics and scalars into a second set of registers while the current
 *   edge's products run.  Automatic: on when one edge's inputs take at most 64
 *   values per lane.  Same arithmetic. */
#define E3CONV_OPT_DIRECT_PIPELINE 7
/*   E3CONV_OPT_BACKWARD_PARTS: -1 automatic (default) or 1..4: the staged
 *   backward kernels run as this many launches each, every launch over a
 *   share of the output irreps (balanced by their terms) that holds only its
 *   outputs' gradient rows and stages only its paths' scalars; the later
 *   launches add to the earlier ones' grad_Y and grad_x.  Automatic: one
 *   while a lane's gradient row takes at most 64 registers, else one per 44
 *   of them.  Affects e3conv_backward only. */
#define E3CONV_OPT_BACKWARD_PARTS 8
E3CONV_API int e3conv_set_option(e3conv_plan plan, int option, int value);

/* The current value of an option (as set; -1 where automatic). */
E3CONV_API int e3conv_get_option(e3conv_plan plan, int option, int* value);

/* The plan's real spherical harmonics of vec[3] / |vec| (host, double; the
 * polynomials the kernels evaluate with E3CONV_OPT_EDGE_VECTORS), written to
 * out[ny]; a zero vector gives 1, 0, 0, ... */
E3CONV_API int e3conv_spherical_harmonics(e3conv_plan plan, const double* vec, double* out);

/* edge_sh[e] = Y(edge_vectors[e]) for e < num_edges (device): the polynomials
 * of e3conv_spherical_harmonics, evaluated in float32 and stored in the plan's
 * input dtype as the forward's edge_sh operand, [num_edges][ny].
 * edge_vectors float32 [num_edges][4] (x, y, z, ignored).  Both buffers
 * 16-byte aligned.  The first call compiles the kernel (NVRTC) and loads it;
 * every call is one launch on `stream` with no allocation and no host
 * synchronisation.  num_edges == 0 launches nothing (NULL buffers allowed). */
E3CONV_API int e3conv_edge_harmonics(e3conv_plan plan, const float* edge_vectors, int64_t num_edges,
                                     void* edge_sh, e3conv_stream stream);

/* Sizes: C channels, nx node components, ny edge components, nout output
 * components, num_paths P.  Any pointer may be NULL. */
E3CONV_API int e3conv_query(e3conv_plan plan, int* C, int* nx, int* ny, int* nout, int* num_paths);

/* Path p (0 <= p < P): (l1, p1) x l2 -> (l3, p3), with x_off the first node
 * component of the input irrep and out_off the first output component of
 * the output irrep.  Parities are +1 (even) or -1 (odd).  NULL outputs are
 * skipped. */
E3CONV_API int e3conv_path(e3conv_plan plan, int p, int* l1, int* p1, int* l2, int* l3, int* p3,
                int* x_off, int* out_off);

/* Number of produced output irreps, and irrep k's (l, parity, offset). */
E3CONV_API int e3conv_num_outputs(e3conv_plan plan, int* count);
E3CONV_API int e3conv_output_irrep(e3conv_plan plan, int k, int* l, int* p, int* offset);

/* Dense CG tensor of path p, including the normalisation factor, written to
 * dense_out[(2l1+1)*(2l2+1)*(2l3+1)] in row-major (i, j, k) order (host). */
E3CONV_API int e3conv_cg(e3conv_plan plan, int p, double* dense_out);

/* Launch shape and resources of the forward kernel for `dtype`:
 * channels per lane, lanes per receiver tile, block threads, ring stages
 * (0: direct variant), whether the CG x Y contraction is formed first
 * (E3CONV_OPT_CONTRACT_FIRST), whether the tensor-core variant is used
 * (E3CONV_OPT_TENSOR_CORES), registers per thread and local-memory (spill)
 * bytes per thread.  Any pointer may be NULL. */
E3CONV_API int e3conv_kernel_info(e3conv_plan plan, int dtype, int* channels_per_lane,
                                  int* lanes_per_tile, int* block_threads, int* stages,
                                  int* contract_first, int* tensor_cores, int* registers,
                                  int* local_bytes);

/* Copies the generated CUDA source for `dtype` (NUL-terminated) into buf if
 * buf_len is large enough; *needed receives the required size in bytes. */
E3CONV_API int e3conv_kernel_source(e3conv_plan plan, int dtype, char* buf, size_t buf_len, size_t* needed);

/* The forward's compile record for `dtype`, as e3conv_kernel_source: one line
 * per compile attempt of the launch-shape search (block, channels per lane,
 * team, stages, registers, local bytes per thread; "loaded:" lines give what
 * the loaded function reports), then the NVRTC log of the kept compile. */
E3CONV_API int e3conv_kernel_log(e3conv_plan plan, int dtype, char* buf, size_t buf_len, size_t* needed);

/* ---------------------------------------------------------------------------
 * Forward (the fused gather -> CG product -> scalar mix -> segmented sum ->
 * 1/N scale -> store of e3j's four plain steps; one kernel launch)
 *
 * node_features: device, [num_nodes][nx][C] of the plan's dtype.
 * edge_sh:       device, [E][ny], receiver-sorted (with E3CONV_OPT_EDGE_VECTORS:
 *                the edge vectors, float32 [E][4]).
 * edge_scalars:  device, [E][P][C], receiver-sorted.
 * senders:       device int32 [E], receiver-sorted, in [0, num_nodes).
 * receiver_row_ptr: device int32 [num_nodes+1], nondecreasing, row_ptr[0] = 0
 *                (e3conv_build_csr makes it).
 * out:           device float32 [num_nodes][nout][C]; fully overwritten
 *                (rows of receivers without edges become 0).
 * The edge count is E = receiver_row_ptr[num_nodes]; it stays on the device
 * (the kernel reads it; the host never does), so the edge buffers must hold
 * at least that many rows.  Edge buffers may be NULL only when E = 0.
 * Feature buffers must be 16-byte aligned.  0 <= num_nodes < 2^31, E < 2^31.
 * With num_nodes == 0 nothing is launched.
 * Out-of-range senders are skipped, and row ranges that decrease or leave
 * [row_ptr[0], row_ptr[num_nodes]] are treated as empty; both set the plan's
 * status word (e3conv_check).  The staged and tensor-core variants' bounded
 * waits on their shared-memory rings, if they ever time out, also set the
 * status word and end the kernel early.
 * Each receiver row is summed in float32, in chunks of 128 edges whose scaled
 * sums are added in the output row (rows of up to 128 edges: one chunk).
 * Launches exactly one kernel on `stream`; no host synchronisation, no
 * allocation.  Concurrent forwards with one plan share its status word. */
E3CONV_API int e3conv_forward(e3conv_plan plan, const void* node_features, const void* edge_sh,
                              const void* edge_scalars, const int32_t* senders,
                              const int32_t* receiver_row_ptr, int64_t num_nodes, float* out,
                              e3conv_stream stream);

/* The forward over the receiver rows row_begin .. row_end-1 only: the rows a
 * rank owns when receivers are partitioned into contiguous CSR row ranges
 * (one output row per receiver, so no reduction across ranks follows).
 *   node_features: [num_nodes][nx][C], the table the senders index: every
 *                  node a sender may name (on a rank: its own rows plus the
 *                  rows received from the others).
 *   receiver_row_ptr: device int32; entries row_begin .. row_end are read,
 *                  nondecreasing; the edges of row b are row_ptr[b] ..
 *                  row_ptr[b+1]-1 in row_ptr's numbering.
 *   edge_sh, edge_scalars, senders: the edges of these rows only, edge e of
 *                  row_ptr's numbering at index e - receiver_row_ptr[row_begin].
 *   out:           [row_end - row_begin][nout][C], row b at b - row_begin.
 * 0 <= row_begin <= row_end < 2^31 (the row count need not equal num_nodes);
 * nothing is launched for an empty range.  e3conv_forward is this call with
 * row_begin = 0 and row_end = num_nodes.  A row's result does not depend on
 * the range it is computed in: the same rows give bitwise the same output.
 * Everything else as e3conv_forward. */
E3CONV_API int e3conv_forward_rows(e3conv_plan plan, const void* node_features, int64_t num_nodes,
                                   const void* edge_sh, const void* edge_scalars,
                                   const int32_t* senders, const int32_t* receiver_row_ptr,
                                   int64_t row_begin, int64_t row_end, float* out,
                                   e3conv_stream stream);

/* ---------------------------------------------------------------------------
 * Radial scalars: the edge scalars s_ab as an MLP of radial-basis encodings of
 * the edge length (e3j "Convolution" docstring: the scalars are an MLP of RBF
 * encodings; gate_points_2102 page, "Scope": bessel bases, cosine cutoff, and
 * its number_of_basis / radial_layers / radial_neurons parameters):
 *   h_0[n] = sqrt(2/r) sin((n+1) pi d / r) / d * (1 + cos(pi d / r)) / 2,
 *            n < num_basis, d = |r_ab| < r (0 for d >= r; d = 0: the limit)
 *   h_l    = SiLU(h_{l-1} W_{l-1}),  l = 1 .. layers   (SiLU(v) = v / (1 + e^-v))
 *   s_ab   = h_layers W_layers, reshaped [P][C]          (no biases)
 * Every layer's product runs on the tensor cores (tcgen05, float16 hi + lo
 * splits of both operands: float32 accuracy; layer 0 with the bases zero-padded
 * to K = 16); the bases, the cutoff and SiLU on the CUDA cores.
 */

/* Sets the plan's radial MLP from HOST float32 weights (row-major, input
 * index first, as in h W):
 *   w0       [num_basis][hidden]
 *   w_hidden [layers-1][hidden][hidden] (NULL when layers == 1)
 *   w_out    [hidden][P*C], output column p*C + u = path p, channel u.
 * 1 <= num_basis <= 16, hidden in {32, 64}, 1 <= layers <= 4, r_max > 0 (shared
 * memory: up to three hidden-to-hidden layers at width 64).
 * Packs the weights and copies them to device memory the plan owns (this
 * call allocates; the radial calls below do not).  Replaces an earlier MLP. */
E3CONV_API int e3conv_set_radial_mlp(e3conv_plan plan, int num_basis, double r_max, int hidden,
                                     int layers, const float* w0, const float* w_hidden,
                                     const float* w_out);

/* edge_scalars[e] = s(r_e) for e < num_edges (device): edge_vectors float32
 * [num_edges][4] (x, y, z, ignored), edge_scalars [num_edges][P][C] in the
 * plan's input dtype.  Both 16-byte aligned.  One kernel launch on `stream`
 * (a persistent grid of one CTA per SM); no allocation, no host
 * synchronisation.  A timed-out pipeline wait sets the status word
 * (e3conv_check reports E3CONV_ERR_CUDA). */
E3CONV_API int e3conv_radial_scalars(e3conv_plan plan, const float* edge_vectors, int64_t num_edges,
                                     void* edge_scalars, e3conv_stream stream);

/* ---------------------------------------------------------------------------
 * Irreps linear layer (cuEquivariance-JAX notes, "Flax NNX layers":
 * IrrepsLinear mixes the channels of matching irreps with
 * scale / sqrt(mul_in) normalisation; unmatched outputs are zero), the layer
 * that follows the convolution on its output:
 *   y[n, o, k, v] = scale / sqrt(mul_in) * sum_u x[n, o, k, u] W_o[u, v]
 * for each output irrep o = (l, p) also among the input irreps; 0 for the
 * others.  Both feature arrays use the convolution's layout: per node, each
 * irrep block is [2l+1][mul] (components outer, channels inner).  A GEMM per
 * matched irrep on the tensor cores (tcgen05, float16 hi + lo splits of both
 * operands: float32 accuracy).
 */

/* irreps_in / irreps_out: regrouped (each (l, parity) once), one multiplicity
 * each: mul_in in {32, 64, 128}, mul_out a multiple of 16 in [16, 256], at
 * most 16 output irreps.  scale finite.  Allocates a 4-byte device status word
 * when a device is present. */
E3CONV_API int e3conv_linear_create(e3conv_linear* linear, const char* irreps_in,
                                    const char* irreps_out, double scale);
E3CONV_API void e3conv_linear_destroy(e3conv_linear linear);

/* Floats per node row of x and y, matched irreps (weight blocks), mul_in, mul_out. */
E3CONV_API int e3conv_linear_query(e3conv_linear linear, int* dim_in, int* dim_out,
                                   int* num_weight_blocks, int* mul_in, int* mul_out);

/* *uses_tma = 1 when e3conv_linear_forward runs the tensor-map kernel for
 * this layer (mul_out a multiple of 32, at most 8 output irreps, 2l+1 <= 128,
 * and two input stages fit in shared memory: every shape but mul_in = 128
 * with mul_out > 128): whole-node tiles moved by 3-D TMA boxes in and out,
 * warp roles pipelined over a ring of input stages (each split in place into
 * the float16 operand) and two tensor-memory accumulators.  0: the row-per-thread kernel (thread t loads and stores row
 * t of a 128-row tile).  Both give the same results up to float32 rounding. */
E3CONV_API int e3conv_linear_uses_tma(e3conv_linear linear, int* uses_tma);
/* enable = 0: always the row-per-thread kernel; 1 (the default): the
 * tensor-map kernel wherever the shape allows it. */
E3CONV_API int e3conv_linear_set_tma(e3conv_linear linear, int enable);

/* HOST float32 weights [num_weight_blocks][mul_in][mul_out], one block per
 * matched output irrep in output order.  Packs and copies them to device
 * memory the layer owns (this call allocates). */
E3CONV_API int e3conv_linear_set_weights(e3conv_linear linear, const float* w);

/* y [num_nodes][dim_out] from x [num_nodes][dim_in] (device float32, 16-byte
 * aligned).  One kernel launch on `stream`; no device allocation, no host
 * synchronisation.  The tensor-map kernel's arguments (its tensor maps of x and
 * y) are kept in the layer's host memory and reused while x, y, num_nodes and
 * the weights repeat; a layer is to be called from one host thread at a time. */
E3CONV_API int e3conv_linear_forward(e3conv_linear linear, const float* x, int64_t num_nodes,
                                     float* y, e3conv_stream stream);

/* Synchronises `stream`, reads and clears the layer's status word:
 * E3CONV_ERR_CUDA if a pipeline wait timed out. */
E3CONV_API int e3conv_linear_check(e3conv_linear linear, e3conv_stream stream);

/* Partition of the receiver rows into `parts` contiguous CSR row ranges for
 * as many ranks (host only; row_ptr is HOST memory here, int32
 * [num_nodes+1], nondecreasing).  Rank r owns rows bounds[r] .. bounds[r+1]-1
 * (bounds: int64 [parts+1], bounds[0] = 0, bounds[parts] = num_nodes,
 * nondecreasing, so every row belongs to exactly one range).  The ranges are
 * balanced on edges plus one per row: boundary r is the row b whose prefix
 * cost (row_ptr[b] - row_ptr[0]) + b is nearest to r/parts of the total (of
 * the first row reaching it and the row before), so every boundary's prefix
 * cost is within one row's cost (its edges + 1) of its share.
 * Returns E3CONV_ERR_INVALID_ARG for NULL pointers, parts < 1 or a row_ptr
 * that decreases. */
E3CONV_API int e3conv_partition_rows(const int32_t* row_ptr, int64_t num_nodes, int parts,
                                     int64_t* bounds);

/* ---------------------------------------------------------------------------
 * Backward: gradients of sum(grad_out * out) for an upstream gradient grad_out
 * of the forward's output.  The forward is linear in each of x, Y and s, so
 * each gradient is the forward's product with one factor removed:
 *   grad_scalars[e, p, u] = (1/N) sum_{i,j,k} CG_p[i,j,k] x[a,i,u] Y[e,j] grad_out[b, o_p+k, u]
 *   grad_sh[e, j]         = (1/N) sum_{p,u,i,k} CG_p[i,j,k] s[e,p,u] x[a,i,u] grad_out[b, o_p+k, u]
 *   grad_x[a, i, u]       = (1/N) sum_{e: senders[e] = a} sum_{p,j,k} CG_p[i,j,k] s[e,p,u] Y[e,j]
 *                                                              grad_out[b, o_p+k, u]
 * with a = senders[e], b = receivers[e] (p over the paths that involve the
 * component).  grad_sh and grad_scalars come from one kernel in receiver order
 * (each receiver's grad_out row read once, edges in CSR order, no atomics);
 * grad_x from one kernel in sender order (e3j "graph_ordering" notes: the
 * SENDER-ordered gather), which needs the edges sorted by sender: sender_row_ptr
 * [num_nodes+1] and sender_perm [E] (sender_perm[t] = the t-th edge of the
 * receiver-sorted arrays in sender order), which e3conv_build_csr makes from
 * `senders`.  Every CG nonzero is unrolled as a constant; float32 accumulation.
 *
 *   node_features, edge_sh, edge_scalars, senders, receiver_row_ptr: as for
 *                  e3conv_forward (harmonics as input: not with
 *                  E3CONV_OPT_EDGE_VECTORS).
 *   receivers:     device int32 [E], receiver of each (receiver-sorted) edge;
 *                  needed for grad_x only.
 *   grad_out:      device float32 [num_nodes][nout][C].
 *   grad_x:        device float32 [num_nodes][nx][C], fully overwritten, or NULL.
 *   grad_sh:       device float32 [E][ny], or NULL.
 *   grad_scalars:  device float32 [E][P][C], or NULL (NULL exactly when
 *                  grad_sh is NULL).
 * C <= 128 (float32 inputs) or <= 256 (float16).  Out-of-range indices are
 * skipped and set the status word (e3conv_check).  Up to two kernel launches
 * on `stream`; no host synchronisation, no allocation.  The first call for a
 * dtype generates and compiles the two kernels (host-side, blocking); call
 * e3conv_prepare_backward to do that ahead of time. */
E3CONV_API int e3conv_backward(e3conv_plan plan, const void* node_features, const void* edge_sh,
                               const void* edge_scalars, const int32_t* senders,
                               const int32_t* receivers, const int32_t* receiver_row_ptr,
                               const int32_t* sender_row_ptr, const int32_t* sender_perm,
                               int64_t num_nodes, const float* grad_out, float* grad_x,
                               float* grad_sh, float* grad_scalars, e3conv_stream stream);

/* Generates, compiles and loads the backward kernels of the plan's current
 * dtype (host-side, blocking). */
E3CONV_API int e3conv_prepare_backward(e3conv_plan plan);

/* Generated CUDA source of a backward kernel (which = 0: edges, 1: nodes;
 * where the kernels are split over the output irreps, 2: the second edges
 * launch and 3: the second nodes launch; E3CONV_ERR_INVALID_ARG where they are
 * not), as e3conv_kernel_source. */
E3CONV_API int e3conv_backward_source(e3conv_plan plan, int which, char* buf, size_t buf_len,
                                      size_t* needed);

/* Synchronises `stream`, reads and clears the plan's status word.  Returns
 * E3CONV_OK, E3CONV_ERR_BAD_INDEX if a forward since the last check met an
 * out-of-range sender or row range, or E3CONV_ERR_CUDA if a pipeline wait
 * timed out. */
E3CONV_API int e3conv_check(e3conv_plan plan, e3conv_stream stream);

/* ---------------------------------------------------------------------------
 * Receiver-sorted CSR indexing (e3j "graph_ordering": RECEIVER, edges sorted
 * by receiver so aggregation is a segmented reduction without atomics).
 */

/* Workspace bytes e3conv_build_csr needs for these sizes. */
E3CONV_API int e3conv_csr_workspace_size(int64_t num_edges, int64_t num_nodes, size_t* bytes);

/* From receivers[e] (device int32, any order) computes, on the device:
 *   row_ptr[b] = #{e : receivers[e] < b}, b = 0..num_nodes  (int32 [num_nodes+1])
 *   perm[t]    = the t-th edge in (receiver, original index) order, i.e. a
 *                stable counting sort of the edges by receiver (int32 [num_edges]).
 * Bit-exact and deterministic.  Receivers outside [0, num_nodes) are placed
 * after all valid edges in perm, are not counted in row_ptr, and set the
 * workspace status word (e3conv_csr_check).  `workspace` is device memory
 * of at least e3conv_csr_workspace_size bytes, 256-byte aligned; its
 * contents need not be initialised and it must not be used by another call
 * until this one has finished on `stream`.  No host synchronisation. */
E3CONV_API int e3conv_build_csr(const int32_t* receivers, int64_t num_edges, int64_t num_nodes,
                     int32_t* row_ptr, int32_t* perm, void* workspace, size_t workspace_bytes,
                     e3conv_stream stream);

/* Allocation-free variant of e3conv_build_csr (no counterpart on the pages
 * this library follows; it exists for callers that cannot allocate device
 * memory: code that runs where a framework's allocator owns all device
 * memory, plugins handed a fixed memory budget, or latency-critical paths
 * that must not call cudaMalloc because it can synchronise the device).
 * Same arguments, results and kernels as e3conv_build_csr, but the scratch
 * is a fixed 32 MiB array of device memory inside this library (every GPU
 * that loads the library holds it until the process exits), so the caller
 * passes only inputs and outputs.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - Sizes whose workspace (e3conv_csr_workspace_size) exceeds 32 MiB are
 *     rejected with E3CONV_ERR_WORKSPACE before anything is launched (about
 *     two million edges fit).
 *   - Every call looks up the array's device address on the current device
 *     with cudaGetSymbolAddress (the first call on a device also loads the
 *     library's device code there); make the first call on a device before
 *     any stream capture.
 *   - All calls share the one array, which keeps the last call's contents:
 *     every call clears what must start at zero itself, but two calls whose
 *     work overlaps on the GPU (different streams, or different host threads,
 *     on one device) race on the array and give wrong results.  Order them.
 *   - Receivers outside [0, num_nodes) are sorted after all valid edges and
 *     not counted, so row_ptr[num_nodes] < num_edges reveals them (there is
 *     no workspace status word to read). */
E3CONV_API int e3conv_build_csr_noalloc(const int32_t* receivers, int64_t num_edges,
                                        int64_t num_nodes, int32_t* row_ptr, int32_t* perm,
                                        e3conv_stream stream);

/* Number of kernels one e3conv_build_csr call with these sizes launches
 * (it also issues two cudaMemsetAsync calls).  Host only. */
E3CONV_API int e3conv_csr_kernel_count(int64_t num_edges, int64_t num_nodes, int* count);

/* Synchronises `stream` and reports the status word of the last
 * e3conv_build_csr that used `workspace`: E3CONV_OK or E3CONV_ERR_BAD_INDEX. */
E3CONV_API int e3conv_csr_check(const void* workspace, e3conv_stream stream);

/* dst[t] = src[perm[t]] for rows of row_bytes bytes, t < num_rows (device).
 * Puts edge features / scalars into CSR order.  Rows whose perm entry is
 * outside [0, num_src_rows) are zero-filled and set *status (device int32,
 * may be NULL) to a nonzero value.  row_bytes must be a multiple of 4 and
 * src / dst 16-byte aligned. */
E3CONV_API int e3conv_permute_rows(const void* src, int64_t num_src_rows, const int32_t* perm,
                        int64_t num_rows, int64_t row_bytes, void* dst, int32_t* status,
                        e3conv_stream stream);

/* ---------------------------------------------------------------------------
 * Errors and version
 */
E3CONV_API const char* e3conv_strerror(int code);
E3CONV_API const char* e3conv_last_error(void);
E3CONV_API int e3conv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* E3CONV_H */
