// Irreps linear layer on the tensor cores: channel mixing within matching
// irreps (cuEquivariance-JAX notes, "Flax NNX layers": IrrepsLinear mixes the
// channels of matching irreps with scale / sqrt(mul_in) normalisation;
// unmatched outputs are zero):
//   y[n, o, k, v] = scale / sqrt(mul_in(o)) * sum_u x[n, o, k, u] W_o[u, v]
// for every output irrep o that also appears among the input irreps, and 0
// for the others.  Features use the convolution's trailing-channel layout:
// per node, each irrep block is [2l+1][mul] (components outer, channels
// inner).
//
// Per matched irrep the rows (n, k) form a GEMM [N (2l+1) x mul_in] x
// [mul_in x mul_out].  One CTA of 128 threads per contiguous range of
// 128-row tiles: thread t loads row t of the tile (mul_in float32 values),
// splits it into float16 hi + lo parts in shared memory (A, K-major), the
// weights W_o^T (B, K-major, prepacked hi / lo, scaled by a power of two)
// are bulk-copied in when the irrep changes, D = A_hi B_hi + A_hi B_lo +
// A_lo B_hi accumulates in tensor memory (float32), and thread t stores its
// row of D.  The next tile's rows are loaded while the MMAs run.  All waits
// are bounded (timeout: status bit 4, drain, stop).
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <algorithm>
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

constexpr int kTile = 128;

struct LinArgs {
  const float* x;
  float* y;
  const unsigned char* w;   // packed hi / lo operands of the matched irreps
  long long nodes;
  int dim_in, dim_out, n_out;  // row lengths; mul_out (MMA N)
  int nblocks;                 // output irrep blocks
  int tiles_total;
  unsigned tmem_cols;          // tensor-memory columns of a CTA: the power of two >= mul_out
  unsigned* status;
  LinBlock blk[kLinMaxBlocks];
};

template <int K>
__global__ void __launch_bounds__(128, 1) k_linear(LinArgs a) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int N = a.n_out;
  unsigned char* bw = sm;                                   // hi then lo, [N x K] each
  unsigned char* act = sm + 2 * N * K * 2;                  // hi then lo, [128 x K] each
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(act + 2 * kTile * K * 2);
  unsigned long long* bar_w = bars;
  unsigned long long* bar_mma = bars + 1;
  unsigned* tslot = reinterpret_cast<unsigned*>(bars + 2);
  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)), "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const unsigned tmem = *tslot;
  const unsigned lane_off = static_cast<unsigned>(32 * warp) << 16;
  // contiguous tile range of this CTA
  const long long per = (a.tiles_total + gridDim.x - 1) / gridDim.x;
  const long long t0 = blockIdx.x * per;
  const long long t1 = (t0 + per < a.tiles_total) ? t0 + per : static_cast<long long>(a.tiles_total);
  bool ok = true;
  unsigned ph_w = 0, ph_mma = 0;
  bool pend_w = false, pend_mma = false;
  int cur = -1;  // block whose weights are in shared memory
  // where tile t's row of this thread lives
  auto locate = [&](long long t, int& b, const float*& src, float*& dst) {
    b = 0;
    while (b + 1 < a.nblocks && t >= a.blk[b + 1].first_tile) ++b;
    const LinBlock& B = a.blk[b];
    const long long r = (t - B.first_tile) * kTile + tid;
    src = nullptr;
    dst = nullptr;
    if (r < a.nodes * B.dim) {
      const long long n = r / B.dim, k = r - n * B.dim;
      dst = a.y + n * a.dim_out + B.out_off + k * N;
      if (B.w_off >= 0) src = a.x + n * a.dim_in + B.in_off + k * K;
    }
  };
  float R[K];
  auto load = [&](const float* src) {
#pragma unroll
    for (int q = 0; q < K; q += 4) {
      const float4 v = src ? __ldg(reinterpret_cast<const float4*>(src + q)) : make_float4(0.f, 0.f, 0.f, 0.f);
      R[q] = v.x;
      R[q + 1] = v.y;
      R[q + 2] = v.z;
      R[q + 3] = v.w;
    }
  };
  int b;
  const float* src;
  float* dst;
  if (t0 < t1) {
    locate(t0, b, src, dst);
    load(src);
  }
  for (long long t = t0; t < t1 && ok; ++t) {
    locate(t, b, src, dst);
    const LinBlock& B = a.blk[b];
    if (B.w_off < 0) {  // output irrep without a matching input irrep: zeros
      if (dst)
        for (int q = 0; q < N; q += 4) *reinterpret_cast<float4*>(dst + q) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t + 1 < t1) {
        int b2;
        const float* s2;
        float* d2;
        locate(t + 1, b2, s2, d2);
        load(s2);
      }
      continue;
    }
    if (b != cur) {  // this irrep's weights
      __syncthreads();
      if (tid == 0) {
        const unsigned bytes = static_cast<unsigned>(2 * N * K * 2);
        mbar_expect(bar_w, bytes);
        bulk_g2s(bw, a.w + B.w_off, bytes, bar_w);
        pend_w = true;
      }
      ok = __syncthreads_and(mbar_wait(bar_w, ph_w));
      if (!ok) break;
      ph_w ^= 1u;
      pend_w = false;
      cur = b;
    }
    store_split_row<K>(act, act + kTile * K * 2, tid, R, kTile);
    fence_async_smem();
    tc_before();
    __syncthreads();
    tc_after();
    if (tid == 0) {
      const unsigned id = idesc_f16(kTile, N);
      const unsigned char* whi = bw;
      const unsigned char* wlo = bw + N * K * 2;
      for (int ks = 0; ks < K / 16; ++ks) {
        const int ao = ks * kTile * 32, bo = ks * N * 32;
        mma_f16(tmem, kmajor_desc(act + ao), kmajor_desc(whi + bo), id, ks > 0);
        mma_f16(tmem, kmajor_desc(act + ao), kmajor_desc(wlo + bo), id, 1);
        mma_f16(tmem, kmajor_desc(act + kTile * K * 2 + ao), kmajor_desc(whi + bo), id, 1);
      }
      mma_commit(bar_mma);
      pend_mma = true;
    }
    if (t + 1 < t1) {  // the next tile's row, while the MMAs run
      int b2;
      const float* s2;
      float* d2;
      locate(t + 1, b2, s2, d2);
      load(s2);
    }
    ok = __syncthreads_and(mbar_wait(bar_mma, ph_mma));
    tc_after();
    if (!ok) break;
    ph_mma ^= 1u;
    pend_mma = false;
    for (int j0 = 0; j0 < N; j0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_off + j0, v);
      if (dst) {
        const int cols = min(32, N - j0);
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          if (q < cols)
            *reinterpret_cast<float4*>(dst + j0 + q) =
                make_float4(v[q] * B.scale, v[q + 1] * B.scale, v[q + 2] * B.scale, v[q + 3] * B.scale);
      }
    }
    tc_before();
    __syncthreads();  // every row read out of tensor memory before the next MMAs
    tc_after();
  }
  if (!ok && tid == 0) {
    atomicOr(a.status, 4u);
    if (pend_w) mbar_wait(bar_w, ph_w);
    if (pend_mma) mbar_wait(bar_mma, ph_mma);
  }
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(a.tmem_cols)
                 : "memory");
}


// ---- tensor-map variant: node-aligned tiles moved by TMA, warp roles, pipelined
//
// A tile of irrep block b holds nn = floor(128 / (2l+1)) whole nodes: rows (n, k) in order,
// nn (2l+1) <= 128 of the MMA's 128 rows.  Its input rows are one 3-D box per 32 channels
// ({32 channels, 2l+1, nn} of the [nodes][2l+1][mul_in] view, 128-byte swizzle) into a stage
// of a ring; its output one 3-D box per 32 output channels, stored from a swizzled staging
// tile.  Nodes past the end are zero-filled on load and clipped on store.  Roles:
//   warp 12       issues the loads of a stage once the MMAs have released it;
//   warps 4-11    (256 threads: row r, half h of its channels) read the landed float32 rows,
//                 then overwrite the same stage with their float16 hi / lo operand (the
//                 128 x mul_in float32 tile and its two float16 parts take the same bytes);
//   warp 13       fetches the irrep's weights when it changes, issues the MMAs of a stage into
//                 one of two tensor-memory accumulators and releases the stage;
//   warps 0-3     (thread t <-> row t <-> tensor-memory lane t) read an accumulator out into
//                 the staging tiles and store them; they also write the zero tiles.

constexpr int kChunkBytes = kTile * 128;  // 128 rows x 32 float32: one box of a stage
constexpr int kTmaMaxBlocks = 8;
constexpr int kTmaMaxStages = 6;
constexpr int kTmaThreads = 448;

struct LinTmaBlock {
  int dim, nn, first_tile, out_off;
  long long w_off;  // byte offset of the packed weights; -1: zeros
  float scale;
};

struct LinTmaArgs {
  CUtensorMap in_map[kTmaMaxBlocks];   // {mul_in, 2l+1, nodes} of x at the matched input irrep
  CUtensorMap out_map[kTmaMaxBlocks];  // {mul_out, 2l+1, nodes} of y at the output irrep
  LinTmaBlock blk[kTmaMaxBlocks];
  float* y;
  const unsigned char* w;
  long long nodes;
  int dim_out, n_out, nblocks, tiles_total, stages;
  unsigned tmem_half;  // tensor-memory columns of one accumulator buffer (power of two >= mul_out)
  unsigned* status;
};

struct LinTmaLayout {
  size_t stage, stg, bw, bars, total;  // offsets from the 1024-byte aligned base; total size
};

__host__ __device__ inline LinTmaLayout lin_tma_layout(int K, int N, int stages) {
  LinTmaLayout L;
  L.stage = static_cast<size_t>(K / 32) * kChunkBytes;  // = 128 x K x (2 + 2) operand bytes
  L.stg = static_cast<size_t>(stages) * L.stage;
  L.bw = L.stg + 2 * static_cast<size_t>(kChunkBytes);
  L.bars = L.bw + 2 * static_cast<size_t>(N) * K * 2;
  L.total = L.bars + 8 * 32 + 1024;  // barriers, and room to align the base
  return L;
}

template <int K>
__global__ void __launch_bounds__(kTmaThreads, 1) k_linear_tma(const __grid_constant__ LinTmaArgs a) {
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* sm = sm_raw + ((1024 - (smem_u32(sm_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = a.n_out, RS = a.stages;
  const LinTmaLayout L = lin_tma_layout(K, N, RS);
  unsigned char* stg = sm + L.stg;
  unsigned char* bw = sm + L.bw;
  unsigned long long* bars = reinterpret_cast<unsigned long long*>(sm + L.bars);
  unsigned long long* st_full = bars;                       // [RS] loads landed
  unsigned long long* st_empty = bars + kTmaMaxStages;      // [RS] MMAs done with the stage
  unsigned long long* op_full = bars + 2 * kTmaMaxStages;   // [RS] operand written
  unsigned long long* mma_done = bars + 3 * kTmaMaxStages;  // [2]
  unsigned long long* tm_empty = mma_done + 2;              // [2]
  unsigned long long* bar_w = mma_done + 4;
  unsigned* tslot = reinterpret_cast<unsigned*>(mma_done + 5);
  auto stage = [&](int s) { return sm + static_cast<size_t>(s) * L.stage; };
  if (tid == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(st_full + s, 1);
      mbar_init(st_empty + s, 1);
      mbar_init(op_full + s, 8);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(mma_done + q, 1);
      mbar_init(tm_empty + q, 4);
    }
    mbar_init(bar_w, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tslot)), "r"(2 * a.tmem_half)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const unsigned tmem = *tslot;
  const long long per = (a.tiles_total + gridDim.x - 1) / gridDim.x;
  const long long t0 = blockIdx.x * per;
  const long long t1 = (t0 + per < a.tiles_total) ? t0 + per : static_cast<long long>(a.tiles_total);
  auto block_of = [&](long long t) {
    int b = 0;
    while (b + 1 < a.nblocks && t >= a.blk[b + 1].first_tile) ++b;
    return b;
  };
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

  if (warp == 12) {  // ---- loads
    if (lane == 0) {
      int j = 0;
      for (long long t = t0; t < t1 && ok; ++t) {
        const int b = block_of(t);
        const LinTmaBlock& B = a.blk[b];
        if (B.w_off < 0) continue;
        const int s = j % RS;
        if (j >= RS) ok = mbar_wait(st_empty + s, ((j / RS) - 1) & 1);
        if (!ok) break;
        const int node0 = static_cast<int>((t - B.first_tile) * B.nn);
        mbar_expect(st_full + s, static_cast<unsigned>((K / 32) * 128 * B.dim * B.nn));
        for (int c = 0; c < K / 32; ++c)
          tma_load_3d(stage(s) + c * kChunkBytes, &a.in_map[b], st_full + s, 32 * c, 0, node0);
        ++j;
      }
      // no load outlives the block: wait for the last ones to land
      for (int q = (j > RS ? j - RS : 0); q < j; ++q) mbar_wait(st_full + q % RS, (q / RS) & 1);
      if (!ok) atomicOr(a.status, 4u);
    }
  } else if (warp == 13) {  // ---- weights and MMAs
    if (lane == 0) {
      int j = 0, cur = -1;
      unsigned ph_w = 0;
      const unsigned id = idesc_f16(kTile, N);
      for (long long t = t0; t < t1 && ok; ++t) {
        const int b = block_of(t);
        const LinTmaBlock& B = a.blk[b];
        if (B.w_off < 0) continue;
        if (b != cur) {  // every MMA on the previous weights has completed before they are replaced
          if (j > 0) ok = mbar_wait(mma_done + ((j - 1) & 1), ((j - 1) >> 1) & 1);
          if (!ok) break;
          const unsigned bytes = static_cast<unsigned>(2 * N * K * 2);
          mbar_expect(bar_w, bytes);
          bulk_g2s(bw, a.w + B.w_off, bytes, bar_w);
          ok = mbar_wait(bar_w, ph_w);
          if (!ok) break;
          ph_w ^= 1u;
          cur = b;
        }
        const int s = j % RS;
        ok = mbar_wait(op_full + s, (j / RS) & 1);
        if (ok && j >= 2) ok = mbar_wait(tm_empty + (j & 1), ((j - 2) >> 1) & 1);
        if (!ok) break;
        tc_after();
        const unsigned d = tmem + (j & 1) * a.tmem_half;
        const unsigned char* whi = bw;
        const unsigned char* wlo = bw + N * K * 2;
        const unsigned char* ahi = stage(s);
        const unsigned char* alo = ahi + kTile * K * 2;
        for (int ks = 0; ks < K / 16; ++ks) {
          const int ao = ks * kTile * 32, bo = ks * N * 32;
          mma_f16(d, kmajor_desc(ahi + ao), kmajor_desc(whi + bo), id, ks > 0);
          mma_f16(d, kmajor_desc(ahi + ao), kmajor_desc(wlo + bo), id, 1);
          mma_f16(d, kmajor_desc(alo + ao), kmajor_desc(whi + bo), id, 1);
        }
        mma_commit(mma_done + (j & 1));
        mma_commit(st_empty + s);
        ++j;
      }
      // nothing in flight at exit: every commit of the last tiles has arrived
      if (j > 0) mbar_wait(mma_done + ((j - 1) & 1), ((j - 1) >> 1) & 1);
      for (int q = (j > RS ? j - RS : 0); q < j; ++q) mbar_wait(st_empty + q % RS, (q / RS) & 1);
      if (!ok) atomicOr(a.status, 4u);
    }
  } else if (warp >= 4) {  // ---- warps 4-11: float32 rows -> float16 hi / lo operand, in place
    constexpr int KH = K / 2;  // channels of one thread
    const int st = tid - 128, r = st & (kTile - 1), h = st >> 7;
    int j = 0;
    float R[KH];
    for (long long t = t0; t < t1 && ok; ++t) {
      const int b = block_of(t);
      const LinTmaBlock& B = a.blk[b];
      if (B.w_off < 0) continue;
      const int s = j % RS;
      ok = team_and(2, 256, mbar_wait(st_full + s, (j / RS) & 1));
      if (!ok) break;
      unsigned char* base = stage(s);
      const bool live = r < B.dim * B.nn;
      // channels [h KH, (h + 1) KH) of row r: 16-byte pieces (h KH + 4 i) / 4 of the row's
      // 32-channel boxes, each at piece ^ (r & 7) within its 128-byte row
#pragma unroll
      for (int i = 0; i < KH / 4; ++i) {
        const int q = h * (KH / 4) + i;  // piece of the row
        const float4 v = live ? *reinterpret_cast<const float4*>(base + (q >> 3) * kChunkBytes + r * 128 +
                                                                 (((q & 7) ^ (r & 7)) << 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        R[4 * i] = v.x;
        R[4 * i + 1] = v.y;
        R[4 * i + 2] = v.z;
        R[4 * i + 3] = v.w;
      }
      asm volatile("bar.sync 2, 256;" ::: "memory");  // the stage is read: overwrite it
      store_split_part<KH>(base, base + kTile * K * 2, r, R, kTile, h * KH);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(op_full + s);
      ++j;
    }
    if (!ok && st == 0) atomicOr(a.status, 4u);
  } else {  // ---- warps 0-3: accumulators out, zero tiles
    const unsigned lane_off = static_cast<unsigned>(32 * warp) << 16;
    int j = 0, chunk = 0;
    for (long long t = t0; t < t1 && ok; ++t) {
      const int b = block_of(t);
      const LinTmaBlock& B = a.blk[b];
      const int node0 = static_cast<int>((t - B.first_tile) * B.nn);
      if (B.w_off < 0) {  // output irrep without a matching input irrep: zeros
        const int n = node0 + tid / B.dim;
        if (tid < B.dim * B.nn && n < a.nodes) {
          float* dst = a.y + static_cast<long long>(n) * a.dim_out + B.out_off + (tid % B.dim) * N;
          for (int q = 0; q < N; q += 4) *reinterpret_cast<float4*>(dst + q) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      ok = team_and(1, 128, mbar_wait(mma_done + (j & 1), (j >> 1) & 1));
      if (!ok) break;
      tc_after();
      for (int j0 = 0; j0 < N; j0 += 32) {
        float v[32];
        tmem_ld32(tmem + (j & 1) * a.tmem_half + lane_off + j0, v);
        if (j0 + 32 >= N) {  // the accumulator is read: free it for the tile after next
          tc_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tm_empty + (j & 1));
        }
        unsigned char* sg = stg + (chunk & 1) * kChunkBytes;
        if (tid == 0) bulk_wait_read_but<1>();  // the store issued from this staging tile has read it
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(sg + tid * 128 + ((i ^ (tid & 7)) << 4)) =
              make_float4(v[4 * i] * B.scale, v[4 * i + 1] * B.scale, v[4 * i + 2] * B.scale,
                          v[4 * i + 3] * B.scale);
        fence_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (tid == 0) {
          tma_store_3d(&a.out_map[b], sg, j0, 0, node0);
          bulk_commit();
        }
        ++chunk;
      }
      ++j;
    }
    if (tid == 0) bulk_wait_all();
    if (!ok && tid == 0) atomicOr(a.status, 4u);
  }
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * a.tmem_half)
                 : "memory");
}

}  // namespace

int linear_prepare(LinearPlan& lp, const std::vector<Irrep>& in, const std::vector<Irrep>& out,
                   double scale, std::string& err) {
  lp = LinearPlan{};
  if (in.empty() || out.empty()) {
    err = "irreps_in and irreps_out must not be empty";
    return E3CONV_ERR_IRREPS;
  }
  const int K = in[0].mul, N = out[0].mul;
  for (const auto& ir : in)
    if (ir.mul != K) {
      err = "all input multiplicities must be equal";
      return E3CONV_ERR_UNSUPPORTED;
    }
  for (const auto& ir : out)
    if (ir.mul != N) {
      err = "all output multiplicities must be equal";
      return E3CONV_ERR_UNSUPPORTED;
    }
  if (K != 32 && K != 64 && K != 128) {
    err = "input multiplicity must be 32, 64 or 128";
    return E3CONV_ERR_UNSUPPORTED;
  }
  if (N < 16 || N > 256 || N % 16) {
    err = "output multiplicity must be a multiple of 16 in [16, 256]";
    return E3CONV_ERR_UNSUPPORTED;
  }
  if (static_cast<int>(out.size()) > kLinMaxBlocks) {
    err = "too many output irreps";
    return E3CONV_ERR_UNSUPPORTED;
  }
  for (size_t q = 0; q < in.size(); ++q)
    for (size_t r = q + 1; r < in.size(); ++r)
      if (in[q].l == in[r].l && in[q].p == in[r].p) {
        err = "input irreps must be regrouped (each (l, parity) once)";
        return E3CONV_ERR_IRREPS;
      }
  for (size_t q = 0; q < out.size(); ++q)
    for (size_t r = q + 1; r < out.size(); ++r)
      if (out[q].l == out[r].l && out[q].p == out[r].p) {
        err = "output irreps must be regrouped (each (l, parity) once)";
        return E3CONV_ERR_IRREPS;
      }
  lp.in = in;
  lp.out = out;
  lp.K = K;
  lp.N = N;
  lp.scale = scale;
  int off = 0;
  for (const auto& ir : in) off += ir.dim() * ir.mul;
  lp.dim_in = off;
  off = 0;
  for (const auto& ir : out) {
    LinBlock b{};
    b.dim = ir.dim();
    b.out_off = off;
    b.in_off = -1;
    b.w_off = -1;
    int ioff = 0;
    for (const auto& jr : in) {
      if (jr.l == ir.l && jr.p == ir.p) {
        b.in_off = ioff;
        b.w_off = lp.num_weight_blocks++;  // packed offset fixed once weights are set
      }
      ioff += jr.dim() * jr.mul;
    }
    off += ir.dim() * ir.mul;
    lp.blocks.push_back(b);
  }
  lp.dim_out = off;
  return E3CONV_OK;
}

int linear_pack(LinearPlan& lp, const float* w, std::string& err) {
  const int K = lp.K, N = lp.N;
  const size_t per = static_cast<size_t>(K) * N;
  const int s = weight_scale_exp(w, per * lp.num_weight_blocks);
  const float f = std::ldexp(1.0f, s);
  const size_t bytes = 2 * static_cast<size_t>(N) * K * 2;
  lp.packed.assign(bytes * lp.num_weight_blocks, 0);
  for (auto& b : lp.blocks) {
    if (b.w_off < 0) continue;
    const float* wb = w + per * static_cast<size_t>(b.w_off);
    pack_kmajor(lp.packed, bytes * static_cast<size_t>(b.w_off), N, K,
                [&](int r, int k) { return wb[static_cast<size_t>(k) * N + r] * f; });
    b.scale = static_cast<float>(lp.scale / std::sqrt(static_cast<double>(K)) * std::ldexp(1.0, -s));
  }
  lp.scale_exp = s;
  (void)err;
  return E3CONV_OK;
}

size_t linear_smem_bytes(const LinearPlan& lp) {
  return 2 * static_cast<size_t>(lp.N) * lp.K * 2 + 2 * static_cast<size_t>(kTile) * lp.K * 2 + 64;
}

// stages of the tensor-map kernel that fit in shared memory next to the rest
static int linear_tma_stages(const LinearPlan& lp) {
  int s = 0;
  while (s < kTmaMaxStages && lin_tma_layout(lp.K, lp.N, s + 1).total <= 227 * 1024) ++s;
  return s;
}

bool linear_uses_tma(const LinearPlan& lp) {
  if (!lp.allow_tma || lp.N % 32 != 0 || static_cast<int>(lp.blocks.size()) > kTmaMaxBlocks) return false;
  for (const LinBlock& b : lp.blocks)
    if (b.dim > kTile) return false;
  return linear_tma_stages(lp) >= 2;  // one stage would serialise load, split and MMAs
}

static int encode_linear_args(const LinearPlan& lp, const void* dev_w, const float* x, long long nodes,
                              float* y, unsigned* status, TensorMapEncodeFn encode, LinTmaArgs& a,
                              std::string& err);

static int linear_launch_tma(const LinearPlan& lp, const void* dev_w, const float* x, long long nodes,
                             float* y, unsigned* status, int grid, cudaStream_t st,
                             TensorMapEncodeFn encode, std::string& err) {
  LinTmaArgs a;
  const bool cached = lp.tma_args.size() == sizeof a && lp.tma_x == x && lp.tma_y == y &&
                      lp.tma_w == dev_w && lp.tma_nodes == nodes;
  if (cached) {
    std::memcpy(&a, lp.tma_args.data(), sizeof a);
  } else {
    const int rc = encode_linear_args(lp, dev_w, x, nodes, y, status, encode, a, err);
    if (rc != E3CONV_OK) return rc;
    lp.tma_args.assign(reinterpret_cast<const unsigned char*>(&a),
                       reinterpret_cast<const unsigned char*>(&a) + sizeof a);
    lp.tma_x = x;
    lp.tma_y = y;
    lp.tma_w = dev_w;
    lp.tma_nodes = nodes;
  }
  const long long tiles = a.tiles_total;
  const size_t smem = lin_tma_layout(lp.K, lp.N, a.stages).total;
  // one CTA per SM (shared memory); as many as there are tiles, at most one per SM
  const unsigned blocks = static_cast<unsigned>(std::min<long long>(tiles, grid));
  auto launch = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kernel<<<blocks, kTmaThreads, smem, st>>>(a);
    return cudaGetLastError();
  };
  cudaError_t e = lp.K == 32 ? launch(k_linear_tma<32>) : lp.K == 64 ? launch(k_linear_tma<64>)
                                                                      : launch(k_linear_tma<128>);
  if (e != cudaSuccess) {
    err = "irreps linear kernel launch failed";
    return E3CONV_ERR_CUDA;
  }
  return E3CONV_OK;
}

// the tensor-map kernel's arguments: per irrep block its tile geometry and the tensor maps of
// its input rows and output rows
static int encode_linear_args(const LinearPlan& lp, const void* dev_w, const float* x, long long nodes,
                              float* y, unsigned* status, TensorMapEncodeFn encode, LinTmaArgs& a,
                              std::string& err) {
  std::memset(&a, 0, sizeof a);
  a.y = y;
  a.w = static_cast<const unsigned char*>(dev_w);
  a.nodes = nodes;
  a.dim_out = lp.dim_out;
  a.n_out = lp.N;
  a.nblocks = static_cast<int>(lp.blocks.size());
  a.status = status;
  a.stages = linear_tma_stages(lp);
  a.tmem_half = 32;
  while (a.tmem_half < static_cast<unsigned>(lp.N)) a.tmem_half *= 2;
  const size_t wbytes = 2 * static_cast<size_t>(lp.N) * lp.K * 2;
  long long tiles = 0, mma_tiles = 0;
  for (size_t q = 0; q < lp.blocks.size(); ++q) {
    const LinBlock& b = lp.blocks[q];
    LinTmaBlock& B = a.blk[q];
    B.dim = b.dim;
    B.nn = kTile / b.dim;
    B.first_tile = static_cast<int>(tiles);
    B.out_off = b.out_off;
    B.w_off = b.w_off >= 0 ? static_cast<long long>(wbytes) * b.w_off : -1;
    B.scale = b.scale;
    const long long nt = (nodes + B.nn - 1) / B.nn;
    tiles += nt;
    if (b.w_off >= 0) mma_tiles += nt;
    if (tiles >= (1ll << 31)) {
      err = "too many rows";
      return E3CONV_ERR_UNSUPPORTED;
    }
    // y viewed as [nodes][2l+1][mul_out] at the irrep; x as [nodes][2l+1][mul_in] at the match
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint64_t ostr[2] = {static_cast<cuuint64_t>(lp.N) * 4, static_cast<cuuint64_t>(lp.dim_out) * 4};
    const cuuint64_t odim[3] = {static_cast<cuuint64_t>(lp.N), static_cast<cuuint64_t>(b.dim),
                                static_cast<cuuint64_t>(nodes)};
    const cuuint32_t obox[3] = {32, static_cast<cuuint32_t>(b.dim), static_cast<cuuint32_t>(B.nn)};
    if (encode(&a.out_map[q], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, y + b.out_off, odim, ostr, obox, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      err = "cuTensorMapEncodeTiled failed for the linear output";
      return E3CONV_ERR_CUDA;
    }
    if (b.w_off >= 0) {
      const cuuint64_t istr[2] = {static_cast<cuuint64_t>(lp.K) * 4, static_cast<cuuint64_t>(lp.dim_in) * 4};
      const cuuint64_t idim[3] = {static_cast<cuuint64_t>(lp.K), static_cast<cuuint64_t>(b.dim),
                                  static_cast<cuuint64_t>(nodes)};
      if (encode(&a.in_map[q], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(x) + b.in_off, idim,
                 istr, obox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        err = "cuTensorMapEncodeTiled failed for the linear input";
        return E3CONV_ERR_CUDA;
      }
    }
  }
  a.tiles_total = static_cast<int>(tiles);
  (void)mma_tiles;
  return E3CONV_OK;
}

int linear_launch(const LinearPlan& lp, const void* dev_w, const float* x, long long nodes, float* y,
                  unsigned* status, int grid, cudaStream_t st, TensorMapEncodeFn encode,
                  std::string& err) {
  if (nodes == 0) return E3CONV_OK;
  if (encode && linear_uses_tma(lp))
    return linear_launch_tma(lp, dev_w, x, nodes, y, status, grid, st, encode, err);
  LinArgs a{};
  a.x = x;
  a.y = y;
  a.w = static_cast<const unsigned char*>(dev_w);
  a.nodes = nodes;
  a.dim_in = lp.dim_in;
  a.dim_out = lp.dim_out;
  a.n_out = lp.N;
  a.nblocks = static_cast<int>(lp.blocks.size());
  a.status = status;
  long long tiles = 0;
  const size_t wbytes = 2 * static_cast<size_t>(lp.N) * lp.K * 2;
  for (size_t q = 0; q < lp.blocks.size(); ++q) {
    LinBlock b = lp.blocks[q];
    b.first_tile = static_cast<int>(tiles);
    if (b.w_off >= 0) b.w_off = static_cast<long long>(wbytes) * b.w_off;
    a.blk[q] = b;
    tiles += (nodes * b.dim + kTile - 1) / kTile;
  }
  if (tiles >= (1ll << 31)) {
    err = "too many rows";
    return E3CONV_ERR_UNSUPPORTED;
  }
  a.tiles_total = static_cast<int>(tiles);
  const size_t smem = linear_smem_bytes(lp);
  a.tmem_cols = 32;
  while (a.tmem_cols < static_cast<unsigned>(lp.N)) a.tmem_cols *= 2;
  // CTAs per SM: shared memory (occupancy calculator, carveout at its maximum) and tensor
  // memory (512 columns per SM)
  auto launch = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    cudaFuncAttributes fa;
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    // by hand: 228 KB of shared memory per SM (1 KB reserved per block), 64K registers
    // (allocated per warp in units of 256), 512 tensor-memory columns
    const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
    const int by_smem = static_cast<int>((228 * 1024) / (smem + 1024));
    const int by_regs = 65536 / (regs_warp * 4);
    int per_sm = std::min({by_smem, by_regs, static_cast<int>(512 / a.tmem_cols), 8});
    per_sm = std::max(per_sm, 1);
    // several CTAs need the shared-memory carveout that holds them (the rest stays L1)
    if (per_sm > 1) {
      const int pct = static_cast<int>((per_sm * (smem + 1024) * 100 + 228 * 1024 - 1) / (228 * 1024));
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, std::min(pct, 100));
      if (e != cudaSuccess) return e;
    }
    const unsigned blocks =
        static_cast<unsigned>(std::min<long long>(tiles, static_cast<long long>(grid) * per_sm));
    kernel<<<blocks, 128, smem, st>>>(a);
    return cudaSuccess;
  };
  cudaError_t e = lp.K == 32 ? launch(k_linear<32>) : lp.K == 64 ? launch(k_linear<64>) : launch(k_linear<128>);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    err = "irreps linear kernel launch failed";
    return E3CONV_ERR_CUDA;
  }
  return E3CONV_OK;
}

}  // namespace e3c
