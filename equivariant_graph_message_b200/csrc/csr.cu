// Receiver-sorted CSR indexing on the device, and a row gather.
//
// e3j.core.Convolution requires edges sorted by the endpoint of the graph
// ordering for its fused kernels ("__call__" note); with RECEIVER ordering
// the aggregation onto receivers is a segmented reduction.  This file builds
//   row_ptr[b] = #{e : receivers[e] < b}                       (histogram + scan)
//   perm       = stable counting sort of edges by receiver      (LSD radix sort)
// Both are integer-exact and deterministic: the radix sort is stable (ranks
// inside a chunk follow the item order; chunks follow the scan order), so
// edges of one receiver keep their original relative order.
//
// Out-of-range receivers are given the key num_nodes: they sort after every
// valid edge, are not counted in row_ptr, and set bit 1 of the status word
// at the start of the workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "../../include/e3conv.h"

namespace e3c {

namespace {

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanTile = kScanThreads * kScanItems;  // 4096 elements per block
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;
constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortRounds = 16;
constexpr int kChunk = kSortThreads * kSortRounds;  // 4096 items per chunk
constexpr int kHistThreads = 256;

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Scratch for an exclusive scan of n elements (block totals of every level).
size_t scan_scratch_ints(int64_t n) {
  size_t total = 0;
  while (n > kScanTile) {
    n = ceil_div(n, kScanTile);
    total += static_cast<size_t>(n);
  }
  return total;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// counts[key]++ for valid receivers; a warp adds once per distinct key.
__global__ void __launch_bounds__(kHistThreads) k_histogram(const int* __restrict__ recv, int E,
                                                           int N, int* __restrict__ counts,
                                                           unsigned* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  for (long long e0 = (long long)blockIdx.x * blockDim.x; e0 < E;
       e0 += (long long)gridDim.x * blockDim.x) {
    const long long e = e0 + threadIdx.x;
    int key = -1;
    if (e < E) {
      key = recv[e];
      if (key < 0 || key >= N) {
        atomicOr(status, 1u);
        key = -1;
      }
    }
    const unsigned active = __ballot_sync(0xffffffffu, true);
    const unsigned peers = __match_any_sync(active, key);
    const int leader = __ffs(peers) - 1;
    if (key >= 0 && lane == leader) atomicAdd(&counts[key], __popc(peers));
  }
}

// Exclusive scan of one tile of kScanThreads x ITEMS elements per block (thread t: the ITEMS
// consecutive elements from t x ITEMS); writes the tile total.  `in` and `out` may alias: every
// thread reads its items before the first barrier and writes them after it.
template <int ITEMS>
__global__ void __launch_bounds__(kScanThreads) k_scan_tile(const int* in, int* out, long long n,
                                                           int* __restrict__ totals) {
  __shared__ int warp_sums[kScanThreads / 32];
  const long long base = (long long)blockIdx.x * kScanThreads * ITEMS + (long long)threadIdx.x * ITEMS;
  int v[ITEMS];
  int sum = 0;
#pragma unroll
  for (int q = 0; q < ITEMS; ++q) {
    v[q] = (base + q < n) ? in[base + q] : 0;
    sum += v[q];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += t;
    }
    warp_sums[lane] = wi - w;
    if (lane == 31 && totals) totals[blockIdx.x] = wi;
  }
  __syncthreads();
  int run = warp_sums[warp] + incl - sum;
#pragma unroll
  for (int q = 0; q < ITEMS; ++q) {
    if (base + q < n) out[base + q] = run;
    run += v[q];
  }
}

// One block scans up to kScanThreads x kScanItemsOne elements in a single launch: coalesced
// loads into shared memory, each thread scans its consecutive run there, a block scan of the
// run totals, coalesced stores.  `in` and `out` may alias (every load precedes the first
// barrier, every store follows the last).
constexpr int kScanItemsOne = 32;
__global__ void __launch_bounds__(kScanThreads) k_scan_one(const int* in, int* out, int n) {
  extern __shared__ int sv[];  // n values
  __shared__ int warp_sums[kScanThreads / 32];
  for (int i = threadIdx.x; i < n; i += kScanThreads) sv[i] = in[i];
  __syncthreads();
  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int b0 = threadIdx.x * per, b1 = min(n, b0 + per);
  int sum = 0;
  for (int i = b0; i < b1; ++i) sum += sv[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += t;
    }
    warp_sums[lane] = wi - w;
  }
  __syncthreads();
  int run = warp_sums[warp] + incl - sum;
  for (int i = b0; i < b1; ++i) {
    const int v = sv[i];
    sv[i] = run;
    run += v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kScanThreads) out[i] = sv[i];
}

__global__ void __launch_bounds__(kScanThreads) k_scan_add(int* __restrict__ out, long long n,
                                                          const int* __restrict__ offsets) {
  const long long base = (long long)blockIdx.x * kScanTile + (long long)threadIdx.x * kScanItems;
  const int add = offsets[blockIdx.x];
#pragma unroll
  for (int q = 0; q < kScanItems; ++q)
    if (base + q < n) out[base + q] += add;
}

// Exclusive scan in -> out (may alias) of n ints; scratch holds the levels.
// With `count` set, only counts the kernels it would launch.
void exclusive_scan(const int* in, int* out, int64_t n, int* scratch, cudaStream_t st, int* count) {
  if (n <= 0) return;
  if (n <= static_cast<int64_t>(kScanThreads) * kScanItemsOne) {  // one launch
    if (count) {
      ++*count;
    } else if (n <= kScanTile) {
      k_scan_tile<kScanItems><<<1, kScanThreads, 0, st>>>(in, out, n, nullptr);
    } else {
      const int smem = static_cast<int>(n * sizeof(int));
      cudaFuncSetAttribute(k_scan_one, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      k_scan_one<<<1, kScanThreads, smem, st>>>(in, out, static_cast<int>(n));
    }
    return;
  }
  const int64_t blocks = ceil_div(n, kScanTile);
  int* totals = scratch;
  if (count) ++*count;
  else k_scan_tile<kScanItems><<<static_cast<unsigned>(blocks), kScanThreads, 0, st>>>(in, out, n, totals);
  exclusive_scan(totals, totals, blocks, scratch + blocks, st, count);
  if (count) ++*count;
  else k_scan_add<<<static_cast<unsigned>(blocks), kScanThreads, 0, st>>>(out, n, totals);
}

// Load the sort key of item e (first pass reads receivers, later passes the keys buffer).
__device__ __forceinline__ int load_key(const int* __restrict__ keys, bool first, long long e,
                                        int N) {
  int k = keys[e];
  if (first && (k < 0 || k >= N)) k = N;
  return k;
}

__global__ void __launch_bounds__(kSortThreads) k_radix_upsweep(const int* __restrict__ keys,
                                                               bool first, int E, int N,
                                                               int shift, int num_chunks,
                                                               int* __restrict__ hist) {
  __shared__ int h[kRadix];
  for (int d = threadIdx.x; d < kRadix; d += blockDim.x) h[d] = 0;
  __syncthreads();
  const long long base = (long long)blockIdx.x * kChunk;
  for (int r = 0; r < kSortRounds; ++r) {
    const long long e = base + (long long)r * kSortThreads + threadIdx.x;
    if (e < E) atomicAdd(&h[(load_key(keys, first, e, N) >> shift) & (kRadix - 1)], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < kRadix; d += blockDim.x)
    hist[(long long)d * num_chunks + blockIdx.x] = h[d];
}

// Stable scatter of one chunk: rank = chunk offset of the digit + items of
// the same digit in earlier rounds + earlier warps of this round + earlier
// lanes of this warp.
__global__ void __launch_bounds__(kSortThreads) k_radix_downsweep(
    const int* __restrict__ keys, const int* __restrict__ vals, bool first, int E, int N,
    int shift, int num_chunks, const int* __restrict__ offsets, int* __restrict__ keys_out,
    int* __restrict__ vals_out) {
  __shared__ int run[kRadix];
  __shared__ int warp_cnt[kSortWarps][kRadix];
  __shared__ int round_total[kRadix];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int d = tid; d < kRadix; d += kSortThreads)
    run[d] = offsets[(long long)d * num_chunks + blockIdx.x];
  const long long base = (long long)blockIdx.x * kChunk;
  for (int r = 0; r < kSortRounds; ++r) {
    for (int q = tid; q < kSortWarps * kRadix; q += kSortThreads) (&warp_cnt[0][0])[q] = 0;
    __syncthreads();
    const long long e = base + (long long)r * kSortThreads + tid;
    const bool valid = e < E;
    int key = 0, val = 0, digit = kRadix;  // kRadix: no digit (never counted)
    if (valid) {
      key = load_key(keys, first, e, N);
      val = first ? static_cast<int>(e) : vals[e];
      digit = (key >> shift) & (kRadix - 1);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, digit);
    const int rank = __popc(peers & lanemask_lt());
    if (valid && lane == __ffs(peers) - 1) warp_cnt[warp][digit] = __popc(peers);
    __syncthreads();
    for (int d = tid; d < kRadix; d += kSortThreads) {
      int acc = 0;
      for (int w = 0; w < kSortWarps; ++w) {
        int c = warp_cnt[w][d];
        warp_cnt[w][d] = acc;
        acc += c;
      }
      round_total[d] = acc;
    }
    __syncthreads();
    if (valid) {
      const int pos = run[digit] + warp_cnt[warp][digit] + rank;
      if (keys_out) keys_out[pos] = key;
      vals_out[pos] = val;
    }
    __syncthreads();
    for (int d = tid; d < kRadix; d += kSortThreads) run[d] += round_total[d];
    __syncthreads();
  }
}

__global__ void k_iota(int* __restrict__ out, int E) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < E;
       e += (long long)gridDim.x * blockDim.x)
    out[e] = static_cast<int>(e);
}

__global__ void k_flag_invalid(const int* __restrict__ recv, int E, int N,
                               unsigned* __restrict__ status) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < E;
       e += (long long)gridDim.x * blockDim.x)
    if (recv[e] < 0 || recv[e] >= N) atomicOr(status, 1u);
}

struct Layout {
  size_t status, counts, scan, hist, keys_a, vals_a, keys_b, vals_b, total;
};

Layout layout(int64_t E, int64_t N) {
  Layout L{};
  size_t off = 0;
  L.status = off;
  off += 256;
  L.counts = off;
  off += align256(sizeof(int) * static_cast<size_t>(N + 1));
  const int64_t chunks = ceil_div(E, kChunk);
  const int64_t hist_n = chunks * kRadix;
  const int64_t scan_n = hist_n > N + 1 ? hist_n : N + 1;
  L.scan = off;
  off += align256(sizeof(int) * (scan_scratch_ints(scan_n) + 1));
  L.hist = off;
  off += align256(sizeof(int) * static_cast<size_t>(hist_n > 0 ? hist_n : 1));
  L.keys_a = off;
  off += align256(sizeof(int) * static_cast<size_t>(E > 0 ? E : 1));
  L.vals_a = off;
  off += align256(sizeof(int) * static_cast<size_t>(E > 0 ? E : 1));
  L.keys_b = off;
  off += align256(sizeof(int) * static_cast<size_t>(E > 0 ? E : 1));
  L.vals_b = off;
  off += align256(sizeof(int) * static_cast<size_t>(E > 0 ? E : 1));
  L.total = off;
  return L;
}

}  // namespace

size_t csr_workspace_bytes(int64_t E, int64_t N) { return layout(E, N).total; }

int csr_build(const int* recv, int64_t E, int64_t N, int* row_ptr, int* perm, void* ws,
              size_t ws_bytes, cudaStream_t st, std::string& err, int* count) {
  const Layout L = layout(E, N);
  if (count) {
    *count = 0;
    ws = reinterpret_cast<void*>(uintptr_t(256));
    ws_bytes = L.total;
  }
  if (!ws || ws_bytes < L.total) {
    err = "workspace missing or smaller than e3conv_csr_workspace_size";
    return E3CONV_ERR_WORKSPACE;
  }
  char* w = static_cast<char*>(ws);
  unsigned* status = reinterpret_cast<unsigned*>(w + L.status);
  int* counts = reinterpret_cast<int*>(w + L.counts);
  int* scan = reinterpret_cast<int*>(w + L.scan);
  int* hist = reinterpret_cast<int*>(w + L.hist);
  int* keys_a = reinterpret_cast<int*>(w + L.keys_a);
  int* vals_a = reinterpret_cast<int*>(w + L.vals_a);
  int* keys_b = reinterpret_cast<int*>(w + L.keys_b);
  int* vals_b = reinterpret_cast<int*>(w + L.vals_b);
  const int e32 = static_cast<int>(E), n32 = static_cast<int>(N);

  // the status word and the counts are adjacent in the workspace: one memset clears both
  if (!count && cudaMemsetAsync(status, 0, L.counts - L.status + sizeof(int) * static_cast<size_t>(N + 1),
                                st) != cudaSuccess) {
    err = "cudaMemsetAsync failed";
    return E3CONV_ERR_CUDA;
  }
  if (E > 0) {
    const int64_t blocks = ceil_div(E, kHistThreads);
    if (count) ++*count;
    else
      k_histogram<<<static_cast<unsigned>(blocks < 65535 * 4 ? blocks : 65535 * 4), kHistThreads,
                    0, st>>>(recv, e32, n32, counts, status);
  }
  exclusive_scan(counts, row_ptr, N + 1, scan, st, count);

  if (E > 0) {
    int bits = 0;
    while ((int64_t(1) << bits) <= N) ++bits;  // keys are in [0, N]
    const int passes = (bits + kRadixBits - 1) / kRadixBits;
    const int chunks = static_cast<int>(ceil_div(E, kChunk));
    if (passes == 0) {
      if (count) {
        *count += 2;
      } else {
        k_flag_invalid<<<256, 256, 0, st>>>(recv, e32, n32, status);
        k_iota<<<256, 256, 0, st>>>(perm, e32);
      }
    }
    const int* kin = recv;
    const int* vin = nullptr;
    for (int pass = 0; pass < passes; ++pass) {
      const bool first = pass == 0, last = pass == passes - 1;
      int* kout = last ? nullptr : ((pass % 2 == 0) ? keys_a : keys_b);
      int* vout = last ? perm : ((pass % 2 == 0) ? vals_a : vals_b);
      const int shift = pass * kRadixBits;
      if (count) ++*count;
      else
        k_radix_upsweep<<<chunks, kSortThreads, 0, st>>>(kin, first, e32, n32, shift, chunks, hist);
      exclusive_scan(hist, hist, static_cast<int64_t>(chunks) * kRadix, scan, st, count);
      if (count) ++*count;
      else
        k_radix_downsweep<<<chunks, kSortThreads, 0, st>>>(kin, vin, first, e32, n32, shift,
                                                           chunks, hist, kout, vout);
      kin = kout;
      vin = vout;
    }
  }
  if (!count && cudaGetLastError() != cudaSuccess) {
    err = "kernel launch failed in e3conv_build_csr";
    return E3CONV_ERR_CUDA;
  }
  return E3CONV_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free CSR build: the same kernels with a fixed scratch area.
//
// For callers that must not allocate device memory themselves (see
// e3conv_build_csr_noalloc in e3conv.h).  The scratch is a file-scope device
// array, so every GPU that loads this library holds kStaticScratchBytes of it
// until the process exits.  Host code cannot use the array's name as a device
// address (it names a host-side shadow); its device address on the current
// device is looked up with cudaGetSymbolAddress on every call.

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_csr_scratch[kStaticScratchBytes];

size_t csr_static_scratch_bytes() { return kStaticScratchBytes; }

int csr_build_static(const int* recv, int64_t E, int64_t N, int* row_ptr, int* perm,
                     cudaStream_t st, std::string& err) {
  const size_t need = csr_workspace_bytes(E, N);
  if (need > kStaticScratchBytes) {
    err = "e3conv_build_csr_noalloc: these sizes need " + std::to_string(need) +
          " bytes of scratch, more than its fixed " + std::to_string(kStaticScratchBytes) +
          " bytes; use e3conv_build_csr with a caller-provided workspace";
    return E3CONV_ERR_WORKSPACE;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    err = "no current CUDA device";
    return E3CONV_ERR_CUDA;
  }
  // The array's device address on the current device, looked up on every call (the
  // lookup is cheap once the module is loaded, and a cached address would go stale if
  // the caller reset the device).
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_csr_scratch) != cudaSuccess || !ptr) {
    cudaGetLastError();
    err = "cudaGetSymbolAddress of the static CSR scratch failed";
    return E3CONV_ERR_CUDA;
  }
  return csr_build(recv, E, N, row_ptr, perm, ptr, kStaticScratchBytes, st, err, nullptr);
}

int csr_read_status(const void* ws, cudaStream_t st, unsigned* out) {
  if (cudaMemcpyAsync(out, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return E3CONV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return E3CONV_ERR_CUDA;
  return E3CONV_OK;
}

// ---------------------------------------------------------------------------
// dst[t] = src[perm[t]], rows of row_bytes bytes; one warp per row.

template <typename W>
__global__ void k_permute(const W* __restrict__ src, long long num_src, const int* __restrict__ perm,
                          long long rows, long long words, W* __restrict__ dst,
                          int* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long t = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < rows; t += warps) {
    const long long r = perm[t];
    W* d = dst + t * words;
    if (r < 0 || r >= num_src) {
      for (long long q = lane; q < words; q += 32) d[q] = W{};
      if (lane == 0 && status) atomicOr(reinterpret_cast<unsigned*>(status), 1u);
      continue;
    }
    const W* s = src + r * words;
    for (long long q = lane; q < words; q += 32) d[q] = s[q];
  }
}

int permute_rows(const void* src, int64_t num_src, const int* perm, int64_t rows,
                 int64_t row_bytes, void* dst, int* status, cudaStream_t st, std::string& err) {
  if (rows == 0 || row_bytes == 0) return E3CONV_OK;
  int64_t blocks = ceil_div(rows, 8);
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (row_bytes % 16 == 0) {
    k_permute<uint4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(src), num_src, perm, rows, row_bytes / 16,
        static_cast<uint4*>(dst), status);
  } else {
    k_permute<unsigned><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const unsigned*>(src), num_src, perm, rows, row_bytes / 4,
        static_cast<unsigned*>(dst), status);
  }
  if (cudaGetLastError() != cudaSuccess) {
    err = "kernel launch failed in e3conv_permute_rows";
    return E3CONV_ERR_CUDA;
  }
  return E3CONV_OK;
}

}  // namespace e3c
