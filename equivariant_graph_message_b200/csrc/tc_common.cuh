// Device and host helpers shared by the tensor-core GEMM kernels (radial MLP,
// irreps linear): mbarrier waits with an iteration bound, bulk copies,
// tcgen05 MMA issue / commit / tensor-memory loads, K-major no-swizzle
// shared-memory operands of float16 hi + lo parts.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

namespace e3c {
namespace tc {

constexpr unsigned kSpinLimit = 1u << 22;

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(unsigned long long* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect(unsigned long long* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(unsigned long long* b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(unsigned long long* b, unsigned parity) {
  for (unsigned it = 0; it < kSpinLimit; ++it)
    if (mbar_try(b, parity)) return true;
  return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 2-D TMA tensor store of one box from shared memory at coordinates (x inner, y), in this
// thread's bulk async-group (commit with bulk_commit)
__device__ __forceinline__ void tma_store_2d(const void* map, const void* src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}
// 3-D TMA tensor load of one box into shared memory at coordinates (x inner, y, z); completes
// `bytes` of transaction on the mbarrier
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, unsigned long long* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 3-D TMA tensor store of one box from shared memory, in this thread's bulk async-group
__device__ __forceinline__ void tma_store_3d(const void* map, const void* src, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// this thread's bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major, no-swizzle shared-memory matrix descriptor: core matrices of 8 rows x
// 16 bytes; 128 bytes between the two K-adjacent core matrices of a 16-wide K
// slab, 256 bytes between row groups of 8.
__device__ __forceinline__ unsigned long long kmajor_desc(const void* p) {
  return static_cast<unsigned long long>((smem_u32(p) & 0x3FFFF) >> 4) | (8ull << 16) |
         (16ull << 32) | (1ull << 46);
}
// byte offset of element (row r, k) in a K-major operand of `rows` rows: K slab
// k / 16 of rows * 32 bytes, then the core-matrix layout inside the slab
__device__ __forceinline__ int kmajor_off(int r, int k, int rows) {
  return (k >> 4) * rows * 32 + (r >> 3) * 256 + ((k >> 3) & 1) * 128 + (r & 7) * 16 + (k & 7) * 2;
}
// instruction descriptor of kind::f16: float16 A and B (both K-major), float32 D
__device__ __forceinline__ unsigned idesc_f16(int m, int n) {
  return (1u << 4) | (static_cast<unsigned>(n >> 3) << 17) | (static_cast<unsigned>(m >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(unsigned tmem_d, unsigned long long a, unsigned long long b,
                                        unsigned idesc, unsigned accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(
          tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(unsigned addr, float* v) {
  unsigned r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(r[q]);
}

// all but the `n` most recent of this thread's bulk groups have finished reading shared memory
template <int n>
__device__ __forceinline__ void bulk_wait_read_but() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

// tcgen05.ld of 32 columns without the wait: the registers are valid only after tmem_wait32
// on the same array (which names them, so that no use can move above the wait)
__device__ __forceinline__ void tmem_ld32_async(unsigned addr, unsigned* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}
__device__ __forceinline__ void tmem_wait32(unsigned* r) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
        "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
        "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// SiLU(v) = v / (1 + e^-v): expf, then the correctly rounded reciprocal instead of a division
__device__ __forceinline__ float silu(float v) { return v * __frcp_rn(1.0f + expf(-v)); }

// two floats rounded to float16, low half first
__device__ __forceinline__ unsigned pack_half2(float lo, float hi) {
  unsigned r;
  asm("{ .reg .f16 a, b; cvt.rn.f16.f32 a, %1; cvt.rn.f16.f32 b, %2; mov.b32 %0, {a, b}; }"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}

// hi and lo float16 parts of v[0..8), packed as two 16-byte vectors (pairs converted by one
// cvt.rn.f16x2.f32 each, round to nearest like __float2half_rn)
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  unsigned h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[q]) : "f"(v[2 * q + 1]), "f"(v[2 * q]));
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[q]));
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(l[q]) : "f"(v[2 * q + 1] - f.y), "f"(v[2 * q] - f.x));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Writes row r's values v[0..K) of a K-major operand as float16 hi and lo parts: eight
// K-consecutive values are one 16-byte row of a core matrix, so a warp's 32 rows store
// 4 x 128 contiguous bytes per instruction.
template <int K>
__device__ __forceinline__ void store_split_row(unsigned char* hi, unsigned char* lo, int r,
                                                const float* v, int rows) {
  static_assert(K % 8 == 0, "K must be a multiple of 8");
#pragma unroll
  for (int k = 0; k < K; k += 8) {
    uint4 h, l;
    split8(v + k, h, l);
    const int off = kmajor_off(r, k, rows);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(lo + off) = l;
  }
}

// Writes values v[0..N) of row r at K columns k0 .. k0 + N - 1 (k0 a multiple of 16) of a
// K-major operand as float16 hi and lo parts.
template <int N>
__device__ __forceinline__ void store_split_part(unsigned char* hi, unsigned char* lo, int r,
                                                 const float* v, int rows, int k0) {
  static_assert(N % 8 == 0, "N must be a multiple of 8");
#pragma unroll
  for (int k = 0; k < N; k += 8) {
    uint4 h, l;
    split8(v + k, h, l);
    const int off = kmajor_off(r, k0 + k, rows);
    *reinterpret_cast<uint4*>(hi + off) = h;
    *reinterpret_cast<uint4*>(lo + off) = l;
  }
}

}  // namespace tc

namespace tc_host {

// ---- host: packing of float32 weights into K-major float16 hi / lo operands

// out[r][k] layout of kmajor_off for a [rows x K] operand from w(r, k) (row r = output).
template <typename F>
inline void pack_kmajor(std::vector<unsigned char>& buf, size_t base, int rows, int K, F w) {
  for (int r = 0; r < rows; ++r)
    for (int k = 0; k < K; ++k) {
      const int off = (k >> 4) * rows * 32 + (r >> 3) * 256 + ((k >> 3) & 1) * 128 + (r & 7) * 16 +
                      (k & 7) * 2;
      const float v = w(r, k);
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn(v - __half2float(h));
      std::memcpy(&buf[base + off], &h, 2);
      std::memcpy(&buf[base + rows * K * 2 + off], &l, 2);
    }
}

// power of two 2^s with max |w| 2^s <= 2^14 (so hi parts stay far from float16 overflow and
// lo parts are normal float16 numbers for the larger weights)
inline int weight_scale_exp(const float* w, size_t n) {
  float m = 0.f;
  for (size_t q = 0; q < n; ++q) m = std::max(m, std::fabs(w[q]));
  if (!(m > 0.f)) return 0;
  int e = 0;
  std::frexp(m, &e);  // m = f 2^e, f in [0.5, 1)
  return 14 - e;
}


}  // namespace tc_host
}  // namespace e3c
