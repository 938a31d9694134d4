// Radial scalars s_ab on the tensor cores: bessel basis x cosine cutoff of the
// edge length, SiLU MLP, output layer of P*C scalars per edge.
//
// What it computes (e3j.core.Convolution, class docstring: the edge scalars
// are an MLP of radial-basis encodings; gate_points_2102 page, "Scope":
// bessel radial bases and a cosine cutoff, and its Network parameters
// number_of_basis, radial_layers, radial_neurons), for edge e of length d:
//   h_0[n] = sqrt(2/r) sin((n+1) pi d / r) / d * (1 + cos(pi d / r)) / 2   (d < r; 0 beyond;
//            evaluated as sinpi / cospi of (n+1) d / r and d / r
//            d = 0 takes the limit (n+1) pi / r)
//   h_1    = SiLU(h_0 W_0)                      (num_basis -> hidden, tensor cores, K padded to 16)
//   h_l+1  = SiLU(h_l W_l),  l = 1 .. L-1       (hidden -> hidden, tensor cores)
//   s      = h_L W_L                            (hidden -> P*C, tensor cores)
// with SiLU(v) = v / (1 + exp(-v)), no biases.
//
// Tensor-core layers: D = A B^T in tensor memory (float32) with both operands
// K-major float16 in shared memory (core matrices of 8 rows x 16 bytes, no
// swizzle).  Both operands are split into float16 hi + lo parts,
// D = A_hi B_hi + A_hi B_lo + A_lo B_hi (the lo x lo term is below float32
// rounding), which keeps the products at float32 accuracy; the weights are
// scaled by a power of two before the split (undone exactly on the way out)
// so that their lo parts stay normal float16 numbers.  Every layer puts the
// tile's 128 edges on the MMA's M side: A = activations [128 x K], B = weights
// [N x K]; the output layer runs in chunks of N = 128 columns.
//
// One persistent CTA per SM over tiles of 128 edges, in warp roles that hand
// work over through mbarriers:
//   warps 4-11  (two threads per edge row, each half of the row's hidden
//               columns) compute the bases, read the hidden accumulator, apply
//               SiLU and write the activation operands (two buffers where
//               shared memory allows: the next tile's hidden layers run while
//               the output layer still reads this tile's);
//   warp 12     issues layer 0's and the hidden layers' MMAs;
//   warp 13     issues the output layer's MMAs, chunk by chunk, into three
//               tensor-memory accumulators;
//   warp 14     requests the output-weight chunks into a ring of 2-4 buffers,
//               each as soon as its buffer is free;
//   warps 0-3   (thread t <-> edge row t <-> tensor-memory lane t) read each
//               output chunk out of its accumulator into a ring of swizzled
//               [128 rows x 128 bytes] staging boxes, each stored by a 2-D TMA
//               tensor store as soon as it is written (rows past the last edge
//               and columns past P*C are clipped by the TMA; rows whose byte
//               length is not a multiple of 16 are stored element by element).
// The stores stream at the SM's store rate while the next tile's bases and
// hidden layers run; what is left between chunks is the output MMAs' wait for
// a free accumulator.
// All waits are bounded: on timeout a CTA sets bit 4 of the status word,
// drains what it issued (bounded) and stops.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "plan.h"
#include "tc_common.cuh"

namespace e3c {

namespace {

using namespace tc;
using namespace tc_host;

constexpr int kTile = 128;           // edges per tile (MMA M)
constexpr int kMaxBasis = 16;        // radial bases = the K of layer 0's MMA (zero-padded)
constexpr int kChunk = 128;          // output columns per output-layer chunk (MMA N)
constexpr int kStageBytes = kTile * kChunk * 4;  // staging ring: four boxes of 128 rows x 128 bytes
constexpr int kMaxWBufs = 4;         // output-weight chunk buffers in shared memory (at most)
constexpr int kOutBufs = 3;          // output-layer accumulators in tensor memory
constexpr int kOutCol = 128;         // tensor-memory column of the output accumulators (>= hidden)
constexpr int kTmemCols = 512;       // hidden D [0, H) and three output accumulators of 128
constexpr int kRadThreads = 480;     // 4 drain warps, 8 compute warps, 2 MMA warps, 1 loader
constexpr int kRadBars = 24;         // mbarriers (and the tensor-memory slot after them)

struct RadialArgs {
  const float* vec;        // [E][4] edge vectors (x, y, z, unused)
  long long num_edges;
  const unsigned char* w0; // layer 0: hi then lo, [H x kMaxBasis] K-major each
  const unsigned char* wh; // hidden layers 1..L-1: per layer hi then lo, [H x H] K-major each
  const unsigned char* wo; // output layer: per chunk hi then lo, [kChunk x H] K-major each
  float w_scale_inv_0;     // 2^-s of layer 0's weight scale
  float w_scale_inv_h;     // 2^-s of the hidden weights' scale
  float w_scale_inv_o;     // 2^-s of the output weights' scale
  float pi_r, inv_r, norm; // pi / r_max, 1 / r_max and sqrt(2 / r_max)
  int nb, layers;          // basis size, hidden layers L (>= 1)
  int nout, chunks;        // P*C outputs, chunks of kChunk (the last padded with zero weights)
  int wbufs, abufs;        // output-weight chunk buffers, activation buffers
  int stage_bytes;         // staging ring of the drain (its boxes for the output dtype)
  float r_max;
  void* s;                 // [E][nout] float32 or float16
  int out_f16;
  int tma;                 // 1: TMA tensor stores through the map; 0: element stores
  unsigned* status;
};

// Shared memory of one CTA (bytes): the staging ring, layer 0's and the hidden layers' weights,
// the basis values and the activations (hi, lo each; one or two activation
// buffers), the output-weight chunk ring (hi, lo each), barriers and the
// tensor-memory slot.
template <int H>
struct Smem {
  static constexpr int kW0 = H * kMaxBasis * 2;          // one [H x 16] float16 operand
  static constexpr int kBas = kTile * kMaxBasis * 2;     // one [128 x 16] float16 operand
  static constexpr int kAct = kTile * H * 2;     // one K-major [128 x H] float16 operand
  static constexpr int kWhid = H * H * 2;        // one [H x H] float16 operand
  static constexpr int kWout = kChunk * H * 2;   // one [kChunk x H] float16 operand
};

inline size_t radial_smem_for(int H, int layers, int abufs, int wbufs, int stage_bytes) {
  const size_t h = static_cast<size_t>(H);
  return stage_bytes + 2 * h * kMaxBasis * 2 + (layers - 1) * 2 * h * h * 2 + 2 * kTile * kMaxBasis * 2 +
         abufs * 2 * kTile * h * 2 + wbufs * 2 * kChunk * h * 2 + kRadBars * 8;
}

template <int H>
__global__ void __launch_bounds__(kRadThreads, 1) k_radial(RadialArgs a, const __grid_constant__ CUtensorMap smap) {
  extern __shared__ __align__(1024) unsigned char sm[];
  using L = Smem<H>;
  constexpr int HH = H / 2;  // hidden columns of one compute thread
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int A = a.abufs, W = a.wbufs;
  unsigned char* stage = sm;                                          // 1024-byte aligned (swizzle)
  unsigned char* w0s = stage + a.stage_bytes;                         // layer 0 (hi, lo)
  unsigned char* whs = w0s + 2 * L::kW0;                              // (layers-1) x (hi, lo)
  unsigned char* bas = whs + (a.layers - 1) * 2 * L::kWhid;           // basis values (hi, lo)
  unsigned char* acts = bas + 2 * L::kBas;                            // A x (hi, lo)
  unsigned char* wos = acts + A * 2 * L::kAct;                        // W x (hi, lo)
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(wos + W * 2 * L::kWout);
  unsigned long long* bar_wh = bars;         // layer 0's and the hidden layers' weights landed
  unsigned long long* bas_full = bars + 1;   // basis operand written (8 compute warps)
  unsigned long long* act_full = bars + 2;   // a hidden layer's input written (8 compute warps)
  unsigned long long* hid_read = bars + 3;   // hidden accumulator read (8 compute warps)
  unsigned long long* hid_done = bars + 4;   // layer-0 / hidden-layer MMAs done
  unsigned long long* out_full = bars + 5;   // [2] the output layer's input written (8 warps)
  unsigned long long* act_free = bars + 7;   // [2] a tile's output MMAs done with its buffer
  unsigned long long* mma_done = bars + 9;   // [3] output chunk in an accumulator
  unsigned long long* tm_empty = bars + 12;  // [3] accumulator read (4 drain warps)
  unsigned long long* bar_w = bars + 15;     // [4] output-weight chunk landed
  unsigned long long* w_free = bars + 19;    // [4] MMAs done with an output-weight chunk
  unsigned* tslot = reinterpret_cast<unsigned*>(bars + 23);
  auto act = [&](long long k) { return acts + static_cast<int>(k % A) * 2 * L::kAct; };
  if (tid == 0) {
    mbar_init(bar_wh, 1);
    mbar_init(bas_full, 8);
    mbar_init(act_full, 8);
    mbar_init(hid_read, 8);
    mbar_init(hid_done, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(out_full + q, 8);
      mbar_init(act_free + q, 1);
    }
    for (int b = 0; b < kOutBufs; ++b) {
      mbar_init(mma_done + b, 1);
      mbar_init(tm_empty + b, 4);
    }
    for (int q = 0; q < kMaxWBufs; ++q) {
      mbar_init(bar_w + q, 1);
      mbar_init(w_free + q, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)), "n"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const unsigned tmem = *tslot;
  const unsigned t_hid = tmem;  // columns [0, H): hidden-layer accumulator
  auto t_out = [&](int b) { return tmem + static_cast<unsigned>(kOutCol + kChunk * b); };
  const long long tiles = (a.num_edges + kTile - 1) / kTile;
  const long long my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const long long total = my_tiles * a.chunks;  // this CTA's output chunks, tile by tile
  // a named barrier of `count` threads that also ANDs a predicate over them
  auto team_and = [](int id, int count, bool p) {
    unsigned r;
    asm volatile(
        "{ .reg .pred q, o; setp.ne.u32 q, %1, 0; bar.red.and.pred o, %2, %3, q; selp.u32 %0, 1, 0, o; }"
        : "=r"(r)
        : "r"(static_cast<unsigned>(p)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
  };
  bool ok = true;

  if (warp == 12) {  // ---- layer 0's and the hidden layers' MMAs
    if (lane == 0) {
      const unsigned hb = static_cast<unsigned>((a.layers - 1) * 2 * L::kWhid);
      mbar_expect(bar_wh, 2 * L::kW0 + hb);
      bulk_g2s(w0s, a.w0, 2 * L::kW0, bar_wh);
      if (hb) bulk_g2s(whs, a.wh, hb, bar_wh);
      ok = mbar_wait(bar_wh, 0);
      int nhid = 0, nact = 0;  // MMA groups issued, hidden-layer inputs consumed
      const unsigned idh = idesc_f16(kTile, H);
      for (long long k = 0; k < my_tiles && ok; ++k) {
        ok = mbar_wait(bas_full, k & 1);
        if (ok && nhid > 0) ok = mbar_wait(hid_read, (nhid - 1) & 1);
        if (!ok) break;
        tc_after();
        mma_f16(t_hid, kmajor_desc(bas), kmajor_desc(w0s), idh, 0);
        mma_f16(t_hid, kmajor_desc(bas), kmajor_desc(w0s + L::kW0), idh, 1);
        mma_f16(t_hid, kmajor_desc(bas + L::kBas), kmajor_desc(w0s), idh, 1);
        mma_commit(hid_done);
        ++nhid;
        for (int l = 1; l < a.layers && ok; ++l) {
          ok = mbar_wait(act_full, nact & 1) && mbar_wait(hid_read, (nhid - 1) & 1);
          if (!ok) break;
          ++nact;
          tc_after();
          const unsigned char* whi = whs + (l - 1) * 2 * L::kWhid;
          const unsigned long long d_ahi = kmajor_desc(act(k)), d_alo = kmajor_desc(act(k) + L::kAct);
          const unsigned long long d_whi = kmajor_desc(whi), d_wlo = kmajor_desc(whi + L::kWhid);
#pragma unroll
          for (int ks = 0; ks < H / 16; ++ks) {
            const unsigned long long ao = static_cast<unsigned long long>(ks * kTile * 32) >> 4;
            const unsigned long long bo = static_cast<unsigned long long>(ks * H * 32) >> 4;
            mma_f16(t_hid, d_ahi + ao, d_whi + bo, idh, ks > 0);
            mma_f16(t_hid, d_ahi + ao, d_wlo + bo, idh, 1);
            mma_f16(t_hid, d_alo + ao, d_whi + bo, idh, 1);
          }
          mma_commit(hid_done);
          ++nhid;
        }
      }
      if (nhid > 0) mbar_wait(hid_done, (nhid - 1) & 1);  // nothing in flight at exit
      if (!ok) {
        mbar_wait(bar_wh, 0);
        atomicOr(a.status, 4u);
      }
    }
  } else if (warp == 13) {  // ---- the output layer's MMAs and weight chunks
    if (lane == 0) {
      long long g = 0;  // chunks issued (their weights come from the loader warp)
      const unsigned ido = idesc_f16(kTile, kChunk);
      for (long long k = 0; k < my_tiles && ok; ++k) {
        ok = mbar_wait(out_full + (k % A), (k / A) & 1);
        if (!ok) break;
        tc_after();
        const unsigned long long d_hhi = kmajor_desc(act(k)), d_hlo = kmajor_desc(act(k) + L::kAct);
        for (int c = 0; c < a.chunks && ok; ++c, ++g) {
          const int wb = static_cast<int>(g % W), b = static_cast<int>(g % kOutBufs);
          ok = mbar_wait(bar_w + wb, (g / W) & 1);
          if (ok && g >= kOutBufs) ok = mbar_wait(tm_empty + b, ((g / kOutBufs) - 1) & 1);
          if (!ok) break;
          tc_after();
          const unsigned long long d_whi = kmajor_desc(wos + wb * 2 * L::kWout);
          const unsigned long long d_wlo = kmajor_desc(wos + wb * 2 * L::kWout + L::kWout);
#pragma unroll
          for (int ks = 0; ks < H / 16; ++ks) {
            const unsigned long long ho = static_cast<unsigned long long>(ks * kTile * 32) >> 4;
            const unsigned long long wo = static_cast<unsigned long long>(ks * kChunk * 32) >> 4;
            mma_f16(t_out(b), d_hhi + ho, d_whi + wo, ido, ks > 0);
            mma_f16(t_out(b), d_hhi + ho, d_wlo + wo, ido, 1);
            mma_f16(t_out(b), d_hlo + ho, d_whi + wo, ido, 1);
          }
          mma_commit(mma_done + b);
          mma_commit(w_free + wb);
        }
        if (!ok) break;
        mma_commit(act_free + (k % A));
      }
      // nothing in flight at exit: the last commits have arrived
      for (long long q = (g > W ? g - W : 0); q < g; ++q) mbar_wait(w_free + q % W, (q / W) & 1);
      if (g > 0) mbar_wait(mma_done + (g - 1) % kOutBufs, ((g - 1) / kOutBufs) & 1);
      if (ok && my_tiles > 0) mbar_wait(act_free + (my_tiles - 1) % A, ((my_tiles - 1) / A) & 1);
      if (!ok) atomicOr(a.status, 4u);
    }
  } else if (warp == 14) {  // ---- output-weight chunks into the ring
    // lane 0 requests chunk q's weights as soon as the MMAs of chunk q - W have released its
    // buffer, independently of the MMA warp's own waits
    if (lane == 0) {
      long long q = 0;
      for (; q < total && ok; ++q) {
        const int wb = static_cast<int>(q % W);
        if (q >= W) ok = mbar_wait(w_free + wb, static_cast<unsigned>(((q / W) - 1) & 1));
        if (!ok) break;
        mbar_expect(bar_w + wb, 2 * L::kWout);
        bulk_g2s(wos + wb * 2 * L::kWout, a.wo + static_cast<size_t>(q % a.chunks) * 2 * L::kWout,
                 2 * L::kWout, bar_w + wb);
      }
      // no copy outlives the block: the last requested chunks have landed (bounded)
      for (long long p = (q > W ? q - W : 0); p < q; ++p) mbar_wait(bar_w + p % W, (p / W) & 1);
      if (!ok) atomicOr(a.status, 4u);
    }
  } else if (warp >= 4) {  // ---- warps 4-11: bases, SiLU, activation operands
    const int st = tid - 128, row = st & (kTile - 1), half = st >> 7;
    // warps w and w + 4 read tensor-memory lanes 32 (w % 4) .. + 31: this thread's row
    const unsigned lane_off = static_cast<unsigned>(32 * (warp & 3)) << 16;
    const float pi_r = a.pi_r, norm = a.norm;
    int nhid = 0;  // hidden accumulators read
    float h[HH];
    auto read_hidden = [&](float scale_inv) {  // SiLU(D) of this thread's half of the row
      ok = team_and(2, 256, mbar_wait(hid_done, nhid & 1));
      if (!ok) return;
      tc_after();
      float v[32];
      tmem_ld32(t_hid + lane_off + half * HH, v);
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(hid_read);
      ++nhid;
#pragma unroll
      for (int q = 0; q < HH; ++q) h[q] = silu(v[q] * scale_inv);
    };
    for (long long k = 0; k < my_tiles && ok; ++k) {
      const long long tile = blockIdx.x + k * gridDim.x;
      const long long e = tile * kTile + row;
      // layer 0's input: bessel basis x cosine cutoff on the CUDA cores (the previous tile's
      // layer-0 MMAs have read the basis operand: this thread waited for them)
      if (half == 0) {
        float d = 0.f;
        const bool valid = e < a.num_edges;
        if (valid) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(a.vec) + e);
          d = sqrtf(fmaf(v.x, v.x, fmaf(v.y, v.y, v.z * v.z)));
        }
        const bool inside = valid && d < a.r_max;
        const float t = d * a.inv_r;                // d / r in [0, 1) inside
        const float u = 0.5f * (1.0f + cospif(t));  // cos(pi d / r)
        float b[kMaxBasis];
#pragma unroll
        for (int n = 0; n < kMaxBasis; ++n) {
          b[n] = (!inside || n >= a.nb) ? 0.f
                                        : (d > 0.f ? norm * sinpif((n + 1) * t) / d : norm * (n + 1) * pi_r) * u;
        }
        store_split_row<kMaxBasis>(bas, bas + L::kBas, row, b, kTile);
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bas_full);
      read_hidden(a.w_scale_inv_0);
      if (!ok) break;
      // this tile's activation buffer: free once the output MMAs of tile k - A are done
      if (k >= A) ok = team_and(2, 256, mbar_wait(act_free + (k % A), ((k / A) - 1) & 1));
      if (!ok) break;
      unsigned char* ab = act(k);
      for (int l = 1; l < a.layers && ok; ++l) {
        store_split_part<HH>(ab, ab + L::kAct, row, h, kTile, half * HH);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(act_full);
        read_hidden(a.w_scale_inv_h);
      }
      if (!ok) break;
      store_split_part<HH>(ab, ab + L::kAct, row, h, kTile, half * HH);  // the output layer's input
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full + (k % A));
    }
    if (!ok && st == 0) atomicOr(a.status, 4u);
  } else {  // ---- warps 0-3: output chunks out of tensor memory (thread t <-> row t <-> lane t)
    const unsigned lane_off = static_cast<unsigned>(32 * warp) << 16;
    const int row = tid;
    const float f = a.w_scale_inv_o;
    const int boxes = a.out_f16 ? kChunk / 64 : kChunk / 32;  // 128-byte column boxes per chunk
    const int bcols = a.out_f16 ? 64 : 32;
    for (long long g = 0; g < total && ok; ++g) {
      const long long tile = blockIdx.x + (g / a.chunks) * gridDim.x;
      const int c = static_cast<int>(g % a.chunks), b = static_cast<int>(g % kOutBufs);
      const long long e = tile * kTile + row;
      const int col0 = c * kChunk;
      ok = team_and(1, 128, mbar_wait(mma_done + b, (g / kOutBufs) & 1));
      if (!ok) break;
      tc_after();
      if (a.tma) {
        // staging: a ring of `boxes` slots of [128 rows x 128 bytes], row r at r * 128, its
        // 16-byte piece q at (q ^ (r & 7)) * 16; box q of this chunk reuses slot q of the
        // previous one (thread 0 waits until that store has read it) and is stored as soon as
        // it is written, so the stores stream while the next boxes are staged
        // staging and storing box q of this chunk in slot q (a ring across chunks)
        auto stage_box = [&](int q, auto&& write) {
          unsigned char* slot = stage + q * (kTile * 128);
          if (tid == 0) {
            if (boxes == 4)
              bulk_wait_read_but<3>();
            else
              bulk_wait_read_but<1>();
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");  // slot q is free
          write(slot + row * 128);
          if (q == boxes - 1) {  // the accumulator is read: free it for the chunk after next
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tm_empty + b);
          }
          fence_async_smem();
          asm volatile("bar.sync 1, 128;" ::: "memory");  // box q is staged
          if (tid == 0) {
            if (col0 + q * bcols < a.nout)
              tma_store_2d(&smap, slot, col0 + q * bcols, static_cast<int>(tile * kTile));
            bulk_commit();  // one group per box (empty past the last column)
          }
        };
        if (a.out_f16) {
          // float16, two boxes of 64 columns: four loads of 32 columns, each issued one ahead
          unsigned r0[32], r1[32];
          auto writeh = [&](unsigned char* dst, int hh, const unsigned* r) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4*>(dst + (((hh * 4 + i) ^ (row & 7)) * 16)) = make_uint4(
                  pack_half2(__uint_as_float(r[8 * i]) * f, __uint_as_float(r[8 * i + 1]) * f),
                  pack_half2(__uint_as_float(r[8 * i + 2]) * f, __uint_as_float(r[8 * i + 3]) * f),
                  pack_half2(__uint_as_float(r[8 * i + 4]) * f, __uint_as_float(r[8 * i + 5]) * f),
                  pack_half2(__uint_as_float(r[8 * i + 6]) * f, __uint_as_float(r[8 * i + 7]) * f));
          };
          tmem_ld32_async(t_out(b) + lane_off, r0);
          tmem_wait32(r0);
          tmem_ld32_async(t_out(b) + lane_off + 32, r1);
          stage_box(0, [&](unsigned char* dst) {
            writeh(dst, 0, r0);
            tmem_wait32(r1);
            tmem_ld32_async(t_out(b) + lane_off + 64, r0);
            writeh(dst, 1, r1);
          });
          tmem_wait32(r0);
          tmem_ld32_async(t_out(b) + lane_off + 96, r1);
          stage_box(1, [&](unsigned char* dst) {
            writeh(dst, 0, r0);
            tmem_wait32(r1);
            writeh(dst, 1, r1);
          });
        } else {
          // float32, four boxes: each box's tensor-memory load is issued one box ahead, so its
          // latency overlaps the staging and the barriers of the box before it
          unsigned r0[32], r1[32];
          auto write32 = [&](unsigned* r) {
            return [&, r](unsigned char* dst) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                *reinterpret_cast<float4*>(dst + ((i ^ (row & 7)) * 16)) =
                    make_float4(__uint_as_float(r[4 * i]) * f, __uint_as_float(r[4 * i + 1]) * f,
                                __uint_as_float(r[4 * i + 2]) * f, __uint_as_float(r[4 * i + 3]) * f);
            };
          };
          tmem_ld32_async(t_out(b) + lane_off, r0);
          tmem_wait32(r0);
          tmem_ld32_async(t_out(b) + lane_off + 32, r1);
          stage_box(0, write32(r0));
          tmem_wait32(r1);
          tmem_ld32_async(t_out(b) + lane_off + 64, r0);
          stage_box(1, write32(r1));
          tmem_wait32(r0);
          tmem_ld32_async(t_out(b) + lane_off + 96, r1);
          stage_box(2, write32(r0));
          tmem_wait32(r1);
          stage_box(3, write32(r1));
        }
      } else {  // rows whose byte length is not a multiple of 16: element stores
        const int cols = min(kChunk, a.nout - col0);
        for (int j0 = 0; j0 < kChunk; j0 += 32) {
          float v[32];
          tmem_ld32(t_out(b) + lane_off + j0, v);
          if (e < a.num_edges) {
            const long long base = e * a.nout + col0 + j0;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              if (j0 + q >= cols) continue;
              if (a.out_f16)
                static_cast<__half*>(a.s)[base + q] = __float2half_rn(v[q] * f);
              else
                static_cast<float*>(a.s)[base + q] = v[q] * f;
            }
          }
        }
        tc_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tm_empty + b);
      }
    }
    if (tid == 0) bulk_wait_all();  // every store has landed
    if (!ok && tid == 0) atomicOr(a.status, 4u);
  }
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTmemCols)
                 : "memory");
}

}  // namespace

int radial_prepare(RadialPlan& rp, int nb, double r_max, int hidden, int layers, const float* w0,
                   const float* const* wh, const float* wo, int nout, std::string& err) {
  if (hidden != 64 && hidden != 32) {
    err = "radial hidden width must be 32 or 64";
    return E3CONV_ERR_UNSUPPORTED;
  }
  if (nb < 1 || nb > kMaxBasis || layers < 1 || layers > 4 || !(r_max > 0) || nout < 1) {
    err = "radial MLP: 1 <= num_basis <= 16, 1 <= layers <= 4, r_max > 0";
    return E3CONV_ERR_INVALID_ARG;
  }
  rp = RadialPlan{};
  rp.nb = nb;
  rp.hidden = hidden;
  rp.layers = layers;
  rp.r_max = r_max;
  rp.nout = nout;
  rp.chunks = (nout + kChunk - 1) / kChunk;
  // layer 0: W_0^T as the MMA's B operand, [hidden x 16] K-major, bases beyond nb zero
  const int s0 = weight_scale_exp(w0, static_cast<size_t>(nb) * hidden);
  rp.scale_exp_0 = s0;
  const float f0 = std::ldexp(1.0f, s0);
  rp.w0.assign(static_cast<size_t>(2) * hidden * kMaxBasis * 2, 0);
  pack_kmajor(rp.w0, 0, hidden, kMaxBasis, [&](int r, int k) {
    return k < nb ? w0[static_cast<size_t>(k) * hidden + r] * f0 : 0.f;
  });
  // hidden weights: one scale for all hidden layers
  int sh = 30;
  for (int l = 1; l < layers; ++l)
    sh = std::min(sh, weight_scale_exp(wh[l - 1], static_cast<size_t>(hidden) * hidden));
  if (layers == 1) sh = 0;
  rp.scale_exp_h = sh;
  const float fh = std::ldexp(1.0f, sh);
  rp.wh.assign(static_cast<size_t>(layers - 1) * 2 * hidden * hidden * 2, 0);
  for (int l = 1; l < layers; ++l)
    pack_kmajor(rp.wh, static_cast<size_t>(l - 1) * 2 * hidden * hidden * 2, hidden, hidden,
                [&](int r, int k) { return wh[l - 1][static_cast<size_t>(k) * hidden + r] * fh; });
  const int so = weight_scale_exp(wo, static_cast<size_t>(hidden) * nout);
  rp.scale_exp_o = so;
  const float fo = std::ldexp(1.0f, so);
  const size_t chunk_bytes = static_cast<size_t>(kChunk) * hidden * 2;
  rp.wo.assign(static_cast<size_t>(rp.chunks) * 2 * chunk_bytes, 0);
  for (int c = 0; c < rp.chunks; ++c)
    pack_kmajor(rp.wo, static_cast<size_t>(c) * 2 * chunk_bytes, kChunk, hidden, [&](int r, int k) {
      const int col = c * kChunk + r;
      return col < nout ? wo[static_cast<size_t>(k) * nout + col] * fo : 0.f;
    });
  return E3CONV_OK;
}

// activation and output-weight buffers: two and as many chunk buffers (2-4) as fit, else one
// activation buffer and two chunk buffers
// staging for the output dtype (float16 scalars need half of it), then two activation buffers
// and as many chunk buffers (2-4) as fit, else one activation buffer and two chunk buffers
static void radial_buffers(const RadialPlan& rp, int out_f16, int& abufs, int& wbufs, int& stage) {
  constexpr size_t kMax = 227 * 1024;
  stage = out_f16 ? kStageBytes / 2 : kStageBytes;
  abufs = 2;
  for (wbufs = kMaxWBufs; wbufs > 2; --wbufs)
    if (radial_smem_for(rp.hidden, rp.layers, abufs, wbufs, stage) <= kMax) return;
  if (radial_smem_for(rp.hidden, rp.layers, abufs, wbufs, stage) > kMax) abufs = 1;
}

size_t radial_smem_bytes(const RadialPlan& rp) {  // the float32 scalars' (the larger) need
  int abufs = 0, wbufs = 0, stage = 0;
  radial_buffers(rp, 0, abufs, wbufs, stage);
  return radial_smem_for(rp.hidden, rp.layers, abufs, wbufs, stage);
}

int radial_launch(const RadialPlan& rp, const void* dev_w0, const void* dev_wh, const void* dev_wo,
                  const float* vec, long long num_edges, void* s, int out_f16, unsigned* status,
                  int grid, cudaStream_t st, std::string& err, const CUtensorMap* smap) {
  if (num_edges == 0) return E3CONV_OK;
  RadialArgs a;
  CUtensorMap map;
  std::memset(&map, 0, sizeof map);
  a.tma = smap != nullptr;
  if (smap) map = *smap;
  a.vec = vec;
  a.num_edges = num_edges;
  a.w0 = static_cast<const unsigned char*>(dev_w0);
  a.w_scale_inv_0 = std::ldexp(1.0f, -rp.scale_exp_0);
  a.wh = static_cast<const unsigned char*>(dev_wh);
  a.wo = static_cast<const unsigned char*>(dev_wo);
  a.w_scale_inv_h = std::ldexp(1.0f, -rp.scale_exp_h);
  a.w_scale_inv_o = std::ldexp(1.0f, -rp.scale_exp_o);
  a.pi_r = static_cast<float>(3.14159265358979323846 / rp.r_max);
  a.inv_r = static_cast<float>(1.0 / rp.r_max);
  a.norm = static_cast<float>(std::sqrt(2.0 / rp.r_max));
  a.nb = rp.nb;
  a.layers = rp.layers;
  a.nout = rp.nout;
  a.chunks = rp.chunks;
  a.r_max = static_cast<float>(rp.r_max);
  a.s = s;
  a.out_f16 = out_f16;
  a.status = status;
  radial_buffers(rp, out_f16, a.abufs, a.wbufs, a.stage_bytes);
  const size_t smem = radial_smem_for(rp.hidden, rp.layers, a.abufs, a.wbufs, a.stage_bytes);
  const long long tiles = (num_edges + kTile - 1) / kTile;
  auto launch = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    int per_sm = 0;
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kRadThreads, smem);
    if (e != cudaSuccess || per_sm < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    // tensor memory: all 512 columns per CTA, so one CTA per SM
    per_sm = 1;
    const unsigned blocks = static_cast<unsigned>(std::min<long long>(tiles, static_cast<long long>(grid) * per_sm));
    kernel<<<blocks, kRadThreads, smem, st>>>(a, map);
    return cudaSuccess;
  };
  cudaError_t e = rp.hidden == 32 ? launch(k_radial<32>) : launch(k_radial<64>);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    err = "radial kernel launch failed";
    return E3CONV_ERR_CUDA;
  }
  return E3CONV_OK;
}

}  // namespace e3c
