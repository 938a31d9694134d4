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
// Tensor-core layers: one CTA of 256 threads per tile of 128 edges: threads t
// and t + 128 share edge row t (tensor-memory lane t) and each reads, applies
// SiLU to, and stores half of the row's columns.  A = the tile's activations
// [128 edges x hidden], B = the weights [N outputs x hidden] (both K-major,
// float16, core matrices of 8 rows x 16 bytes, no swizzle), D = A B^T in
// tensor memory (float32).  Both operands are split into float16 hi + lo
// parts, D = A_hi B_hi + A_hi B_lo + A_lo B_hi (the lo x lo term is below
// float32 rounding), which keeps the products at float32 accuracy; the
// weights are scaled by a power of two before the split (undone exactly on
// the way out) so that their lo parts stay normal float16 numbers.
// The output layer runs in chunks of 128 columns (one N = 128 MMA per K step
// and split term): their weights are double-buffered in shared memory (bulk
// copies of prepacked chunks), their products alternate between two
// tensor-memory buffers, so the MMAs of chunk c overlap the stores of chunk
// c-1.  Stores: the threads write the chunk's [128 edges x 128 columns] tile
// into shared memory in the TMA's 128-byte swizzle (thread t, row t: its
// 16-byte pieces land in distinct banks), and one thread stores it with 2-D
// TMA tensor stores of 128 rows x 128 bytes (rows past the last edge and
// columns past P*C are clipped by the TMA); rows whose byte length is not a
// multiple of 16 are stored element by element instead.  All
// waits are bounded: on timeout a CTA sets bit 4 of the status word, drains
// what it issued (bounded) and stops.
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
constexpr int kWBufs = 2;            // output-weight chunk buffers in shared memory
constexpr int kStageBytes = kTile * kChunk * 4;  // one chunk's output tile (float32)
constexpr int kOutCol = 128;         // tensor-memory column of the output buffers (>= hidden)
constexpr int kTmemCols = 512;       // hidden D [0, H) and two output buffers of kChunk

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
  float r_max;
  void* s;                 // [E][nout] float32 or float16
  int out_f16;
  int tma;                 // 1: TMA tensor stores through the map; 0: element stores
  unsigned* status;
};

// Shared memory of one CTA (bytes): layer 0's and the hidden layers' weights,
// the basis values and the activations (hi, lo each), two output-weight chunks
// (hi, lo each), the staged output rows, barriers and the tensor-memory slot.
template <int H>
struct Smem {
  static constexpr int kW0 = H * kMaxBasis * 2;          // one [H x 16] float16 operand
  static constexpr int kBas = kTile * kMaxBasis * 2;     // one [128 x 16] float16 operand
  static constexpr int kAct = kTile * H * 2;     // one K-major [128 x H] float16 operand
  static constexpr int kWhid = H * H * 2;        // one [H x H] float16 operand
  static constexpr int kWout = kChunk * H * 2;   // one [kChunk x H] float16 operand

};

template <int H>
__global__ void __launch_bounds__(256, 1) k_radial(RadialArgs a, const __grid_constant__ CUtensorMap smap) {
  extern __shared__ __align__(1024) unsigned char sm[];
  using L = Smem<H>;
  constexpr int HH = H / 2;                       // hidden columns of one thread
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row = tid & (kTile - 1), half = tid >> 7;  // edge row, which half of its columns
  unsigned char* w0s = sm;                                            // layer 0 (hi, lo)
  unsigned char* whs = w0s + 2 * L::kW0;                              // (layers-1) x (hi, lo)
  unsigned char* bas = whs + (a.layers - 1) * 2 * L::kWhid;           // basis values (hi, lo)
  unsigned char* act = bas + 2 * L::kBas;                             // hi, lo
  unsigned char* wos = act + 2 * L::kAct;                             // 2 buffers x (hi, lo)
  unsigned char* stage = wos + kWBufs * 2 * L::kWout;  // 1024-byte aligned (128-byte swizzle)
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(stage + kStageBytes);
  unsigned long long* bar_w = bars;                 // [kWBufs] output-weight chunk landed
  unsigned long long* bar_mma = bars + kWBufs;      // [2] output MMAs of a chunk done
  unsigned long long* bar_hid = bars + kWBufs + 2;  // hidden-layer MMAs done
  unsigned long long* bar_wh = bars + kWBufs + 3;   // hidden weights landed
  unsigned* tslot = reinterpret_cast<unsigned*>(bars + kWBufs + 4);

  if (tid == 0) {
    for (int k = 0; k < kWBufs + 4; ++k) mbar_init(bars + k, 1);
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
  const unsigned t_hid = tmem;                 // columns [0, H): hidden-layer D
  // output-layer D: two buffers of kChunk columns at kOutCol and kOutCol + kChunk
  // warps w and w + 4 both read tensor-memory lanes 32 (w % 4) .. + 31
  const unsigned lane_off = static_cast<unsigned>(32 * (warp & 3)) << 16;
  bool ok = true;
  // phase bits (bit b: buffer b) of the weight-chunk and output-MMA barriers
  unsigned ph_w = 0, ph_mma = 0, ph_hid = 0;
  // copies and MMAs thread 0 issued and has not yet seen complete (bit b: buffer b; drained on
  // a timeout)
  unsigned pend_w = 0, pend_mma = 0;
  bool pend_hid = false, pend_wh = false;
  if (tid == 0) {  // layer 0's and the hidden layers' weights, once per CTA
    const unsigned hb = static_cast<unsigned>((a.layers - 1) * 2 * L::kWhid);
    mbar_expect(bar_wh, 2 * L::kW0 + hb);
    bulk_g2s(w0s, a.w0, 2 * L::kW0, bar_wh);
    if (hb) bulk_g2s(whs, a.wh, hb, bar_wh);
    pend_wh = true;
  }
  ok = __syncthreads_and(mbar_wait(bar_wh, 0));
  pend_wh = !ok;
  const float pi_r = a.pi_r;
  const float norm = a.norm;
  const long long tiles = (a.num_edges + kTile - 1) / kTile;
  for (long long tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
    const long long e = tile * kTile + row;
    const bool valid = e < a.num_edges;
    // prefetch the first output-weight chunks of this tile (every buffer is free: the
    // previous tile waited for all of its output MMAs)
    if (tid == 0) {
      for (int c = 0; c < kWBufs && c < a.chunks; ++c) {
        mbar_expect(bar_w + c, 2 * L::kWout);
        bulk_g2s(wos + c * 2 * L::kWout, a.wo + static_cast<size_t>(c) * 2 * L::kWout,
                 2 * L::kWout, bar_w + c);
        pend_w |= 1u << c;
      }
    }
    // layer 0: basis x cutoff on the CUDA cores, SiLU(h0 W0) with h0 W0 on the tensor cores
    float h[HH];  // this thread's half of the row's hidden values: columns half * HH ..
    if (half == 0) {
      float d = 0.f;
      if (valid) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(a.vec) + e);
        d = sqrtf(fmaf(v.x, v.x, fmaf(v.y, v.y, v.z * v.z)));
      }
      const bool inside = valid && d < a.r_max;
      const float t = d * a.inv_r;                        // d / r in [0, 1) inside
      const float u = 0.5f * (1.0f + cospif(t));          // cos(pi d / r)
      float b[kMaxBasis];
#pragma unroll
      for (int n = 0; n < kMaxBasis; ++n) {
        b[n] = (!inside || n >= a.nb)
                   ? 0.f
                   : (d > 0.f ? norm * sinpif((n + 1) * t) / d : norm * (n + 1) * pi_r) * u;
      }
      store_split_row<kMaxBasis>(bas, bas + L::kBas, row, b, kTile);
      fence_async_smem();
    }
    {
      tc_before();
      __syncthreads();
      tc_after();
      if (tid == 0) {
        const unsigned id0 = idesc_f16(kTile, H);
        mma_f16(t_hid, kmajor_desc(bas), kmajor_desc(w0s), id0, 0);
        mma_f16(t_hid, kmajor_desc(bas), kmajor_desc(w0s + L::kW0), id0, 1);
        mma_f16(t_hid, kmajor_desc(bas + L::kBas), kmajor_desc(w0s), id0, 1);
        mma_commit(bar_hid);
        pend_hid = true;
      }
      ok = __syncthreads_and(mbar_wait(bar_hid, ph_hid));
      tc_after();
      if (!ok) break;
      ph_hid ^= 1u;
      pend_hid = false;
      {
        float v[32];
        tmem_ld32(t_hid + lane_off + half * HH, v);
#pragma unroll
        for (int q = 0; q < HH; ++q) h[q] = silu(v[q] * a.w_scale_inv_0);
      }
      tc_before();
      __syncthreads();  // every thread has read D before the next layer's MMAs overwrite it
      tc_after();
    }
    // hidden layers 1 .. L-1 on the tensor cores
    for (int l = 1; l < a.layers && ok; ++l) {
      store_split_part<HH>(act, act + L::kAct, row, h, kTile, half * HH);
      fence_async_smem();
      tc_before();
      __syncthreads();
      tc_after();
      if (tid == 0) {
        const unsigned char* whi = whs + (l - 1) * 2 * L::kWhid;
        const unsigned id = idesc_f16(kTile, H);
        const unsigned long long d_ahi = kmajor_desc(act), d_alo = kmajor_desc(act + L::kAct);
        const unsigned long long d_whi = kmajor_desc(whi), d_wlo = kmajor_desc(whi + L::kWhid);
#pragma unroll
        for (int ks = 0; ks < H / 16; ++ks) {
          const unsigned long long ao = static_cast<unsigned long long>(ks * kTile * 32) >> 4;
          const unsigned long long bo = static_cast<unsigned long long>(ks * H * 32) >> 4;
          mma_f16(t_hid, d_ahi + ao, d_whi + bo, id, ks > 0);
          mma_f16(t_hid, d_ahi + ao, d_wlo + bo, id, 1);
          mma_f16(t_hid, d_alo + ao, d_whi + bo, id, 1);
        }
        mma_commit(bar_hid);
        pend_hid = true;
      }
      ok = __syncthreads_and(mbar_wait(bar_hid, ph_hid));
      tc_after();
      if (!ok) break;
      ph_hid ^= 1u;
      pend_hid = false;
      {
        float v[32];
        tmem_ld32(t_hid + lane_off + half * HH, v);
#pragma unroll
        for (int q = 0; q < HH; ++q) h[q] = silu(v[q] * a.w_scale_inv_h);
      }
      tc_before();
      __syncthreads();  // every thread has read D before the next layer's MMAs overwrite it
      tc_after();
    }
    if (!ok) break;
    // output layer: chunks of 128 columns
    store_split_part<HH>(act, act + L::kAct, row, h, kTile, half * HH);
    fence_async_smem();
    tc_before();
    __syncthreads();
    tc_after();
    const unsigned id = idesc_f16(kTile, kChunk);
    // descriptors: the activations' hi / lo operands and the weight buffers; K step ks adds
    // its byte offset / 16 to the start-address field
    const unsigned long long d_ahi = kmajor_desc(act), d_alo = kmajor_desc(act + L::kAct);
    for (int c = 0; c <= a.chunks && ok; ++c) {
      if (c < a.chunks) {
        const int wb = c % kWBufs, buf = c & 1;
        ok = __syncthreads_and(mbar_wait(bar_w + wb, (ph_w >> wb) & 1u));
        if (!ok) break;
        ph_w ^= 1u << wb;
        pend_w &= ~(1u << wb);
        if (tid == 0) {
          const unsigned long long d_whi = kmajor_desc(wos + wb * 2 * L::kWout);
          const unsigned long long d_wlo = kmajor_desc(wos + wb * 2 * L::kWout + L::kWout);
          const unsigned td = tmem + static_cast<unsigned>(kOutCol + kChunk * buf);
#pragma unroll
          for (int ks = 0; ks < H / 16; ++ks) {
            const unsigned long long ao = static_cast<unsigned long long>(ks * kTile * 32) >> 4;
            const unsigned long long bo = static_cast<unsigned long long>(ks * kChunk * 32) >> 4;
            mma_f16(td, d_ahi + ao, d_whi + bo, id, ks > 0);
            mma_f16(td, d_ahi + ao, d_wlo + bo, id, 1);
            mma_f16(td, d_alo + ao, d_whi + bo, id, 1);
          }
          mma_commit(bar_mma + buf);
          pend_mma |= 1u << buf;
        }
      }
      if (c >= 1) {  // chunk c-1: its weight buffer takes chunk c+1, then its stores
        const int pb = (c - 1) & 1, pw = (c - 1) % kWBufs;
        // the previous chunk's TMA stores have read the staging tile (thread 0 issued them);
        // the barrier below publishes that to every thread
        if (tid == 0) bulk_wait_read();
        ok = __syncthreads_and(mbar_wait(bar_mma + pb, (ph_mma >> pb) & 1u));
        tc_after();
        if (!ok) break;
        ph_mma ^= 1u << pb;
        pend_mma &= ~(1u << pb);
        if (tid == 0 && c - 1 + kWBufs < a.chunks) {
          mbar_expect(bar_w + pw, 2 * L::kWout);
          bulk_g2s(wos + pw * 2 * L::kWout,
                   a.wo + static_cast<size_t>(c - 1 + kWBufs) * 2 * L::kWout, 2 * L::kWout,
                   bar_w + pw);
          pend_w |= 1u << pw;
        }
        const int col0 = (c - 1) * kChunk;
        const int cols = min(kChunk, a.nout - col0);
        const float f = a.w_scale_inv_o;
        if (a.tma) {
          // staging tile: per 128-byte column box (32 floats or 64 halves), row r at r * 128,
          // its 16-byte piece q at (q ^ (r & 7)) * 16
#pragma unroll 1
          for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            float v[32];
            tmem_ld32(tmem + static_cast<unsigned>(kOutCol + kChunk * pb + j0) + lane_off, v);
            if (a.out_f16) {
              unsigned char* box = stage + (j0 / 64) * (kTile * 128) + row * 128;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int piece = (j0 % 64) / 8 + q;
                *reinterpret_cast<uint4*>(box + ((piece ^ (row & 7)) * 16)) =
                    make_uint4(pack_half2(v[8 * q] * f, v[8 * q + 1] * f),
                               pack_half2(v[8 * q + 2] * f, v[8 * q + 3] * f),
                               pack_half2(v[8 * q + 4] * f, v[8 * q + 5] * f),
                               pack_half2(v[8 * q + 6] * f, v[8 * q + 7] * f));
              }
            } else {
              unsigned char* box = stage + (j0 / 32) * (kTile * 128) + row * 128;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(box + ((q ^ (row & 7)) * 16)) =
                    make_float4(v[4 * q] * f, v[4 * q + 1] * f, v[4 * q + 2] * f, v[4 * q + 3] * f);
            }
          }
          fence_async_smem();
          __syncthreads();  // the whole tile is staged
          if (tid == 0) {
            const int boxes = a.out_f16 ? kChunk / 64 : kChunk / 32;
            const int bcols = a.out_f16 ? 64 : 32;
            for (int q = 0; q < boxes; ++q)
              if (col0 + q * bcols < a.nout)
                tma_store_2d(&smap, stage + q * (kTile * 128), col0 + q * bcols,
                             static_cast<int>(tile * kTile));
            bulk_commit();
          }
        } else {
#pragma unroll 1
          for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 32) {
            float v[32];
            tmem_ld32(tmem + static_cast<unsigned>(kOutCol + kChunk * pb + j0) + lane_off, v);
            if (valid) {
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
        }
        tc_before();
        __syncthreads();  // chunk c-1's columns read by every thread before they are reused
        tc_after();
      }
    }
  }
  bulk_wait_all();  // every row store of this thread has landed
  if (!ok && tid == 0) {
    atomicOr(a.status, 4u);
    // drain (bounded): copies and MMAs issued but not seen complete
    for (int b = 0; b < kWBufs; ++b)
      if ((pend_w >> b) & 1u) mbar_wait(bar_w + b, (ph_w >> b) & 1u);
    for (int b = 0; b < 2; ++b)
      if ((pend_mma >> b) & 1u) mbar_wait(bar_mma + b, (ph_mma >> b) & 1u);
    if (pend_hid) mbar_wait(bar_hid, ph_hid);
    if (pend_wh) mbar_wait(bar_wh, 0);
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

size_t radial_smem_bytes(const RadialPlan& rp) {
  const size_t H = rp.hidden;
  return 2 * H * kMaxBasis * 2 + (rp.layers - 1) * 2 * H * H * 2 + 2 * kTile * kMaxBasis * 2 +
         2 * kTile * H * 2 + kWBufs * 2 * kChunk * H * 2 + kStageBytes + (kWBufs + 4) * 8 + 16;
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
  const size_t smem = radial_smem_bytes(rp);
  const long long tiles = (num_edges + kTile - 1) / kTile;
  auto launch = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    int per_sm = 0;
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, smem);
    if (e != cudaSuccess || per_sm < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    // tensor memory: all 512 columns per CTA, so one CTA per SM
    per_sm = 1;
    const unsigned blocks = static_cast<unsigned>(std::min<long long>(tiles, static_cast<long long>(grid) * per_sm));
    kernel<<<blocks, 256, smem, st>>>(a, map);
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
