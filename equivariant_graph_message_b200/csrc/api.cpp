// C ABI of libe3conv: plans, NVRTC compilation, launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <nvrtc.h>

#include <algorithm>
#include <utility>
#include <vector>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <regex>
#include <stdexcept>
#include <string>

#include "plan.h"

namespace e3c {
size_t csr_workspace_bytes(int64_t E, int64_t N);
int csr_build(const int* recv, int64_t E, int64_t N, int* row_ptr, int* perm, void* ws,
              size_t ws_bytes, cudaStream_t st, std::string& err, int* count);
int csr_read_status(const void* ws, cudaStream_t st, unsigned* out);
int csr_build_static(const int* recv, int64_t E, int64_t N, int* row_ptr, int* perm,
                     cudaStream_t st, std::string& err);
int permute_rows(const void* src, int64_t num_src, const int* perm, int64_t rows, int64_t row_bytes,
                 void* dst, int* status, cudaStream_t st, std::string& err);
}  // namespace e3c

using namespace e3c;

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

// Driver API entry points, resolved through the runtime so the library does
// not link libcuda (it must load on machines without a GPU driver).
struct Driver {
  CUresult (*ModuleLoadData)(CUmodule*, const void*) = nullptr;
  CUresult (*ModuleUnload)(CUmodule) = nullptr;
  CUresult (*ModuleGetFunction)(CUfunction*, CUmodule, const char*) = nullptr;
  CUresult (*LaunchKernel)(CUfunction, unsigned, unsigned, unsigned, unsigned, unsigned, unsigned,
                           unsigned, CUstream, void**, void**) = nullptr;
  CUresult (*FuncGetAttribute)(int*, CUfunction_attribute, CUfunction) = nullptr;
  CUresult (*CtxGetCurrent)(CUcontext*) = nullptr;
  CUresult (*FuncSetAttribute)(CUfunction, CUfunction_attribute, int) = nullptr;
  CUresult (*OccupancyMaxActiveBlocksPerMultiprocessor)(int*, CUfunction, int, size_t) = nullptr;
  CUresult (*TensorMapEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill) = nullptr;
  bool ok = false;
};

Driver& driver() {
  static Driver d;
  static std::once_flag once;
  std::call_once(once, [] {
    auto get = [](const char* name, void** fn) {
      cudaDriverEntryPointQueryResult q;
      return cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &q) == cudaSuccess &&
             q == cudaDriverEntryPointSuccess && *fn != nullptr;
    };
    d.ok = get("cuModuleLoadData", reinterpret_cast<void**>(&d.ModuleLoadData)) &&
           get("cuModuleUnload", reinterpret_cast<void**>(&d.ModuleUnload)) &&
           get("cuModuleGetFunction", reinterpret_cast<void**>(&d.ModuleGetFunction)) &&
           get("cuLaunchKernel", reinterpret_cast<void**>(&d.LaunchKernel)) &&
           get("cuFuncGetAttribute", reinterpret_cast<void**>(&d.FuncGetAttribute)) &&
           get("cuCtxGetCurrent", reinterpret_cast<void**>(&d.CtxGetCurrent)) &&
           get("cuFuncSetAttribute", reinterpret_cast<void**>(&d.FuncSetAttribute)) &&
           get("cuOccupancyMaxActiveBlocksPerMultiprocessor",
               reinterpret_cast<void**>(&d.OccupancyMaxActiveBlocksPerMultiprocessor)) &&
           get("cuTensorMapEncodeTiled", reinterpret_cast<void**>(&d.TensorMapEncodeTiled));
    cudaGetLastError();
  });
  return d;
}

bool has_device() {
  int n = 0;
  cudaError_t e = cudaGetDeviceCount(&n);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return n > 0;
}

// NVRTC, loaded from the toolkit the library was built with (E3CONV_NVRTC_PATH) rather
// than through the dynamic linker: a process may already hold another libnvrtc.so.12
// (PyTorch ships its own), and the generated kernels must not depend on which one was
// loaded first.  Falls back to the default search for libnvrtc.so.12.
struct Nvrtc {
  nvrtcResult (*CreateProgram)(nvrtcProgram*, const char*, const char*, int, const char* const*,
                               const char* const*) = nullptr;
  nvrtcResult (*CompileProgram)(nvrtcProgram, int, const char* const*) = nullptr;
  nvrtcResult (*GetProgramLogSize)(nvrtcProgram, size_t*) = nullptr;
  nvrtcResult (*GetProgramLog)(nvrtcProgram, char*) = nullptr;
  nvrtcResult (*GetCUBINSize)(nvrtcProgram, size_t*) = nullptr;
  nvrtcResult (*GetCUBIN)(nvrtcProgram, char*) = nullptr;
  nvrtcResult (*DestroyProgram)(nvrtcProgram*) = nullptr;
  nvrtcResult (*Version)(int*, int*) = nullptr;
  bool ok = false;
};

#ifndef E3CONV_NVRTC_PATH
#define E3CONV_NVRTC_PATH "libnvrtc.so.12"
#endif

Nvrtc& nvrtc() {
  static Nvrtc n;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen(E3CONV_NVRTC_PATH, RTLD_NOW | RTLD_LOCAL);
    if (!h) h = dlopen("libnvrtc.so.12", RTLD_NOW | RTLD_LOCAL);
    if (!h) return;
    auto get = [h](const char* name, auto** fn) {
      *reinterpret_cast<void**>(fn) = dlsym(h, name);
      return *fn != nullptr;
    };
    n.ok = get("nvrtcCreateProgram", &n.CreateProgram) &&
           get("nvrtcCompileProgram", &n.CompileProgram) &&
           get("nvrtcGetProgramLogSize", &n.GetProgramLogSize) &&
           get("nvrtcGetProgramLog", &n.GetProgramLog) &&
           get("nvrtcGetCUBINSize", &n.GetCUBINSize) && get("nvrtcGetCUBIN", &n.GetCUBIN) &&
           get("nvrtcDestroyProgram", &n.DestroyProgram) && get("nvrtcVersion", &n.Version);
  });
  return n;
}

// NVRTC compile of `source` for sm_100a; fills cubin, log, registers and local bytes
// (per thread: the stack frame, which is what the loaded function reports as
// CU_FUNC_ATTRIBUTE_LOCAL_SIZE_BYTES, or the spill stores if ptxas reports more).
int nvrtc_compile(const std::string& source, const char* name, std::vector<char>& cubin,
                  std::string& log, int& regs, int& local_bytes) {
  Nvrtc& nv = nvrtc();
  if (!nv.ok) return fail(E3CONV_ERR_COMPILE, "cannot load NVRTC (" E3CONV_NVRTC_PATH ")");
  nvrtcProgram prog;
  if (nv.CreateProgram(&prog, source.c_str(), name, 0, nullptr, nullptr) != NVRTC_SUCCESS)
    return fail(E3CONV_ERR_COMPILE, "nvrtcCreateProgram failed");
  const char* opts[] = {"--gpu-architecture=sm_100a", "--std=c++17", "-lineinfo",
                        "--ptxas-options=-v"};
  nvrtcResult rc = nv.CompileProgram(prog, 4, opts);
  size_t log_size = 0;
  nv.GetProgramLogSize(prog, &log_size);
  log.assign(log_size, '\0');
  if (log_size) nv.GetProgramLog(prog, &log[0]);
  if (rc != NVRTC_SUCCESS) {
    nv.DestroyProgram(&prog);
    return fail(E3CONV_ERR_COMPILE, "NVRTC compile failed: " + log.substr(0, 2000));
  }
  size_t n = 0;
  nv.GetCUBINSize(prog, &n);
  cubin.resize(n);
  nv.GetCUBIN(prog, cubin.data());
  nv.DestroyProgram(&prog);
  std::smatch m;
  regs = -1;
  if (std::regex_search(log, m, std::regex("Used ([0-9]+) registers"))) regs = std::stoi(m[1]);
  int stack = 0, spill = 0;
  if (std::regex_search(log, m, std::regex("([0-9]+) bytes stack frame"))) stack = std::stoi(m[1]);
  if (std::regex_search(log, m, std::regex("([0-9]+) bytes spill stores"))) spill = std::stoi(m[1]);
  local_bytes = std::max(stack, spill);
  return E3CONV_OK;
}

int compile_once(Plan& pl, int dtype) {
  Variant& v = pl.var[dtype];
  v = Variant{};
  v.shape = choose_shape(pl, dtype);
  v.source = generate_forward_source(pl, dtype, v.shape);
  const int rc = nvrtc_compile(v.source, "e3conv_fwd.cu", v.cubin, v.log, v.regs, v.local_bytes);
  if (rc != E3CONV_OK) return rc;
  // With a device, registers and local memory come from the loaded function: the NVRTC
  // log does not always carry ptxas' resource lines (a repeated compile of the same source
  // was seen to return none), and the launch-shape search must not read a missing line as
  // "no local memory".
  if (pl.device >= 0) {
    Driver& d = driver();
    CUmodule m = nullptr;
    CUfunction f = nullptr;
    if (d.ModuleLoadData(&m, v.cubin.data()) == CUDA_SUCCESS) {
      if (d.ModuleGetFunction(&f, m, "e3conv_fwd") == CUDA_SUCCESS) {
        int regs = 0, local = 0;
        if (d.FuncGetAttribute(&regs, CU_FUNC_ATTRIBUTE_NUM_REGS, f) == CUDA_SUCCESS) v.regs = regs;
        if (d.FuncGetAttribute(&local, CU_FUNC_ATTRIBUTE_LOCAL_SIZE_BYTES, f) == CUDA_SUCCESS)
          v.local_bytes = local;
      }
      d.ModuleUnload(m);
    }
  }
  pl.trace[dtype] += "compile: block=" + std::to_string(v.shape.block) + " V=" +
                     std::to_string(v.shape.V) + " team=" + std::to_string(v.shape.team) +
                     " stages=" + std::to_string(v.shape.stages) + " tc=" +
                     std::to_string(v.shape.tc ? 1 : 0) + " regs=" + std::to_string(v.regs) +
                     " local=" + std::to_string(v.local_bytes) + "\n";
  v.compiled = true;
  return E3CONV_OK;
}

// The backward kernels of the plan's current dtype: generated, compiled and (with a
// device) loaded on first use.
int prepare_backward(Plan& pl) {
  BwdVariant& bv = pl.bwd[pl.dtype];
  if (bv.compiled) return E3CONV_OK;
  if (pl.req_vec) return fail(E3CONV_ERR_UNSUPPORTED, "backward with edge vectors as input");
  BwdVariant v;
  v.shape = choose_backward_shape(pl, pl.dtype);
  if (!v.shape.ok)
    return fail(E3CONV_ERR_UNSUPPORTED, "backward needs C <= 128 (float32) or <= 256 (float16)");
  // modules 2 p + k: part p of the edges (k = 0) and nodes (k = 1) kernels; the nodes kernel
  // is split only when it is staged
  const int np_e = v.shape.eparts, np_n = v.shape.nstaged ? v.shape.eparts : 1;
  std::vector<int> mods;
  for (int p = 0; p < np_e; ++p) mods.push_back(2 * p);
  for (int p = 0; p < np_n; ++p) mods.push_back(2 * p + 1);
  for (int m : mods) {
    const int p = m / 2;
    const bool nodes = m % 2 == 1;
    v.source[m] = p == 0 ? generate_backward_source(pl, pl.dtype, v.shape, nodes)
                  : nodes ? generate_backward_nodes_part(pl, pl.dtype, v.shape, p)
                          : generate_backward_edges_part(pl, pl.dtype, v.shape, p);
    const std::string file = std::string(nodes ? "e3conv_bwd_nodes_" : "e3conv_bwd_edges_") +
                             std::to_string(p) + ".cu";
    const int rc = nvrtc_compile(v.source[m], file.c_str(), v.cubin[m], v.log[m], v.regs[m],
                                 v.local_bytes[m]);
    if (rc != E3CONV_OK) return rc;
  }
  if (pl.device >= 0) {
    Driver& d = driver();
    for (size_t q = 0; q < mods.size(); ++q) {
      const int m = mods[q];
      if (d.ModuleLoadData(&v.module[m], v.cubin[m].data()) != CUDA_SUCCESS ||
          d.ModuleGetFunction(&v.fn[m], v.module[m], m % 2 ? "e3conv_bwd_nodes" : "e3conv_bwd_edges") !=
              CUDA_SUCCESS) {
        for (size_t r = 0; r <= q; ++r)
          if (v.module[mods[r]]) d.ModuleUnload(v.module[mods[r]]);
        return fail(E3CONV_ERR_CUDA, "loading the backward kernels failed");
      }
    }
    bool ok = true;
    for (int m : mods) {
      const int p = m / 2;
      if (m % 2 == 0 && v.shape.staged)
        ok = ok && d.FuncSetAttribute(v.fn[m], CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES,
                                      v.shape.esmem[p]) == CUDA_SUCCESS;
      if (m % 2 == 1 && v.shape.nstaged)
        ok = ok && d.FuncSetAttribute(v.fn[m], CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES,
                                      np_n > 1 ? v.shape.nsmem_p[p] : v.shape.nsmem) == CUDA_SUCCESS;
    }
    if (!ok) {
      for (int m : mods) d.ModuleUnload(v.module[m]);
      return fail(E3CONV_ERR_CUDA, "cannot reserve the backward kernels' shared memory");
    }
  }
  v.compiled = true;
  bv = v;
  return E3CONV_OK;
}

void release_backward(BwdVariant& v) {
  for (int k = 0; k < 8; ++k)
    if (v.module[k]) driver().ModuleUnload(v.module[k]);
  v = BwdVariant{};
}

// Staged variant without a requested block size: a first compile gives the
// register count R; the block size is then the one that keeps the most warps
// resident per SM (228 KB of shared memory per SM with 1 KB reserved per
// block, 64K registers, 2048 threads, 32 blocks), larger blocks on ties; the
// launch bounds of the final compile keep R within budget.
int blocks_per_sm(const Shape& s, int regs, int block) {
  const int teams = block / (32 * s.team);
  const int smem = teams * s.warp_smem + 1024;
  const int r = (std::max(regs, 8) + 7) / 8 * 8;
  const int by_smem = (228 * 1024) / smem;
  const int by_regs = 65536 / (r * block);
  const int by_threads = 2048 / block;
  return std::min({by_smem, by_regs, by_threads, 32});
}

int compile_variant(Plan& pl, int dtype) {
  pl.trace[dtype].clear();
  pl.auto_block = 0;
  pl.tc_team_cap = 0;
  pl.tc_fallback = false;
  int rc = compile_once(pl, dtype);
  if (rc != E3CONV_OK) return rc;
  Variant& v = pl.var[dtype];
  // Tensor-core variant with local memory at three teams per block (168 registers): two
  // teams (255 registers); if that still uses local memory, the float32 staged variant,
  // kept for the rest of this compile (the block-size search below included).
  if (v.shape.tc && v.local_bytes > 0 && v.shape.tbufs > 2) {
    pl.tc_team_cap = 2;
    rc = compile_once(pl, dtype);
    if (rc != E3CONV_OK) return rc;
  }
  if (v.shape.tc && v.local_bytes > 0) {
    pl.tc_fallback = true;
    rc = compile_once(pl, dtype);
    if (rc != E3CONV_OK) return rc;
  }
  if (v.shape.stages > 0 && !v.shape.tc && pl.req_block == 0 && v.regs > 0) {
    const int tt = 32 * v.shape.team;
    const int first_block = v.shape.block;
    const bool first_spills = v.local_bytes > 0;
    std::vector<std::pair<int, int>> cand;  // (resident warps, block)
    for (int k = 1; k <= 15 && k * tt <= 1024; ++k) {
      if (k * v.shape.warp_smem > 227 * 1024) break;
      cand.push_back({blocks_per_sm(v.shape, v.regs, k * tt) * k * v.shape.team, k * tt});
    }
    std::sort(cand.begin(), cand.end(), [](const std::pair<int, int>& a, const std::pair<int, int>& b) {
      return a.first != b.first ? a.first > b.first : a.second > b.second;
    });
    bool done = false;
    for (size_t c = 0; c < cand.size() && c < 4 && !done; ++c) {
      if (cand[c].second == first_block && !first_spills) {
        rc = compile_once(pl, dtype);  // restore the first compile
        done = true;
        break;
      }
      pl.auto_block = cand[c].second;
      rc = compile_once(pl, dtype);
      if (rc != E3CONV_OK) break;
      done = v.local_bytes <= 0;  // keep only a spill-free choice
    }
    pl.auto_block = 0;
    if (rc == E3CONV_OK && !done) rc = compile_once(pl, dtype);
    if (rc != E3CONV_OK) return rc;
  }
  if (pl.device >= 0) {
    Driver& d = driver();
    if (d.ModuleLoadData(&v.module, v.cubin.data()) != CUDA_SUCCESS)
      return fail(E3CONV_ERR_CUDA, "cuModuleLoadData failed");
    if (d.ModuleGetFunction(&v.fn, v.module, "e3conv_fwd") != CUDA_SUCCESS)
      return fail(E3CONV_ERR_CUDA, "cuModuleGetFunction failed");
    int regs = 0, local = 0;
    d.FuncGetAttribute(&regs, CU_FUNC_ATTRIBUTE_NUM_REGS, v.fn);
    d.FuncGetAttribute(&local, CU_FUNC_ATTRIBUTE_LOCAL_SIZE_BYTES, v.fn);
    v.regs = regs;
    v.local_bytes = local;
    pl.trace[dtype] += "loaded: regs=" + std::to_string(regs) + " local=" + std::to_string(local) + "\n";
    if (v.shape.stages > 0) {
      const int smem = v.shape.tc ? v.shape.smem_request
                                  : v.shape.warp_smem * (v.shape.block / (32 * v.shape.team));
      if (d.FuncSetAttribute(v.fn, CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, smem) !=
          CUDA_SUCCESS)
        return fail(E3CONV_ERR_CUDA, "cannot reserve the shared-memory ring");
      int per_sm = 0, sms = 0;
      if (d.OccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, v.shape.block, smem) !=
              CUDA_SUCCESS ||
          per_sm < 1)
        return fail(E3CONV_ERR_CUDA, "staged kernel does not fit on an SM");
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pl.device) != cudaSuccess)
        return fail(E3CONV_ERR_CUDA, "cannot query the SM count");
      v.grid_blocks = per_sm * sms;
    }
  }
  return E3CONV_OK;
}

void release_variant(Variant& v) {
  if (v.module) driver().ModuleUnload(v.module);
  v.module = nullptr;
  v.fn = nullptr;
  v.compiled = false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Makes the plan's device current for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool changed = false;
  explicit DeviceGuard(int dev) {
    if (dev < 0) return;
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
      changed = cudaSetDevice(dev) == cudaSuccess;
    }
  }
  ~DeviceGuard() {
    if (changed) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" {

int e3conv_version(void) { return E3CONV_VERSION; }

const char* e3conv_strerror(int code) {
  switch (code) {
    case E3CONV_OK: return "ok";
    case E3CONV_ERR_INVALID_ARG: return "invalid argument";
    case E3CONV_ERR_IRREPS: return "invalid irreps";
    case E3CONV_ERR_UNSUPPORTED: return "unsupported";
    case E3CONV_ERR_CUDA: return "CUDA error";
    case E3CONV_ERR_NOMEM: return "out of memory";
    case E3CONV_ERR_COMPILE: return "kernel compilation failed";
    case E3CONV_ERR_NO_DEVICE: return "plan has no device module";
    case E3CONV_ERR_BAD_INDEX: return "out-of-range index met by a kernel";
    case E3CONV_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown error code";
  }
}

const char* e3conv_last_error(void) { return g_last_error.c_str(); }

int e3conv_create(e3conv_plan* out, const char* irreps_node, const char* irreps_sh,
                  const char* irreps_out, double avg_num_neighbors, int normalization) {
  if (!out) return fail(E3CONV_ERR_INVALID_ARG, "plan pointer is NULL");
  *out = nullptr;
  if (!(avg_num_neighbors > 0) || !std::isfinite(avg_num_neighbors))
    return fail(E3CONV_ERR_INVALID_ARG, "avg_num_neighbors must be positive and finite");
  if (normalization != E3CONV_NORM_SQRT_DIM_OUT && normalization != E3CONV_NORM_NONE)
    return fail(E3CONV_ERR_UNSUPPORTED, "unknown normalization");
  e3conv_plan h = new (std::nothrow) e3conv_plan_s;
  if (!h) return fail(E3CONV_ERR_NOMEM, "host allocation failed");
  Plan& pl = h->p;
  pl.avg = avg_num_neighbors;
  pl.norm = normalization;
  std::string err;
  std::vector<Irrep> sh;
  if (!parse_irreps(irreps_node, pl.node, err) || !parse_irreps(irreps_sh, sh, err) ||
      !parse_irreps(irreps_out, pl.filt, err)) {
    delete h;
    return fail(E3CONV_ERR_IRREPS, err);
  }
  for (size_t k = 0; k < sh.size(); ++k) {
    if (sh[k].mul != 1 || sh[k].l != static_cast<int>(k) || sh[k].p != ((k % 2) ? -1 : 1)) {
      delete h;
      return fail(E3CONV_ERR_IRREPS,
                  "irreps_sh must be 1x0e+1x1o+1x2e+... (consecutive l from 0, parity (-1)^l)");
    }
  }
  pl.lmax = static_cast<int>(sh.size()) - 1;
  if (pl.lmax > 6) {
    delete h;
    return fail(E3CONV_ERR_UNSUPPORTED, "spherical-harmonic degree above 6");
  }
  int rc;
  try {
    rc = build_paths(pl, err);
  } catch (const std::exception& ex) {
    rc = E3CONV_ERR_IRREPS;
    err = ex.what();
  }
  if (rc != E3CONV_OK) {
    delete h;
    return fail(rc, err);
  }
  if (pl.paths.empty()) {
    delete h;
    return fail(E3CONV_ERR_IRREPS, "no path produces any requested output irrep");
  }
  if (static_cast<long long>(pl.nx) * pl.C >= (1ll << 31) ||
      static_cast<long long>(pl.nout) * pl.C >= (1ll << 31)) {
    delete h;
    return fail(E3CONV_ERR_UNSUPPORTED, "feature row too large");
  }
  if (has_device()) {
    if (!driver().ok) {
      delete h;
      return fail(E3CONV_ERR_CUDA, "CUDA driver entry points unavailable");
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaFree(nullptr) != cudaSuccess) {
      cudaGetLastError();
      delete h;
      return fail(E3CONV_ERR_CUDA, "cannot initialise the CUDA context");
    }
    pl.device = dev;
    driver().CtxGetCurrent(&pl.ctx);
    if (cudaMalloc(&pl.status, sizeof(unsigned int)) != cudaSuccess) {
      cudaGetLastError();
      delete h;
      return fail(E3CONV_ERR_NOMEM, "cudaMalloc of the status word failed");
    }
    cudaMemset(pl.status, 0, sizeof(unsigned int));
  }
  rc = compile_variant(pl, E3CONV_F32);
  if (rc != E3CONV_OK) {
    std::string msg = g_last_error;
    e3conv_destroy(h);
    return fail(rc, msg);
  }
  *out = h;
  return E3CONV_OK;
}

void e3conv_destroy(e3conv_plan h) {
  if (!h) return;
  Plan& pl = h->p;
  {
    DeviceGuard g(pl.device);
    for (auto& v : pl.var) release_variant(v);
    for (auto& v : pl.bwd) release_backward(v);
    for (auto& v : pl.shk)
      if (v.module) driver().ModuleUnload(v.module);
    if (pl.status) cudaFree(pl.status);
    for (void* q : {pl.radial.d_w0, pl.radial.d_wh, pl.radial.d_wo})
      if (q) cudaFree(q);
  }
  delete h;
}

int e3conv_set_input_dtype(e3conv_plan h, int dtype) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  if (dtype != E3CONV_F32 && dtype != E3CONV_F16)
    return fail(E3CONV_ERR_UNSUPPORTED, "dtype must be E3CONV_F32 or E3CONV_F16");
  Plan& pl = h->p;
  if (!pl.var[dtype].compiled) {
    DeviceGuard g(pl.device);
    int rc = compile_variant(pl, dtype);
    if (rc != E3CONV_OK) return rc;
  }
  pl.dtype = dtype;
  return E3CONV_OK;
}

int e3conv_set_launch_config(e3conv_plan h, int channels_per_lane, int block_threads,
                             int stages) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  const int V = channels_per_lane;
  if (V != 0 && V != 1 && V != 2 && V != 4 && V != 8)
    return fail(E3CONV_ERR_INVALID_ARG, "channels_per_lane must be 0, 1, 2, 4 or 8");
  if (V > 0 && pl.C % V != 0)
    return fail(E3CONV_ERR_INVALID_ARG, "channels_per_lane must divide C");
  if (V * (pl.dtype == E3CONV_F16 ? 2 : 4) > 16)
    return fail(E3CONV_ERR_INVALID_ARG, "channels_per_lane exceeds one 16-byte load");
  if (block_threads != 0 && (block_threads < 32 || block_threads > 1024 || block_threads % 32))
    return fail(E3CONV_ERR_INVALID_ARG, "block_threads must be 0 or a multiple of 32 in [32, 1024]");
  if (stages < -1 || stages == 1 || stages > 8)
    return fail(E3CONV_ERR_INVALID_ARG, "stages must be -1 (automatic), 0 (direct) or 2..8");
  pl.req_V = V;
  pl.req_block = block_threads;
  pl.req_stages = stages;
  DeviceGuard g(pl.device);
  const int other = pl.dtype == E3CONV_F32 ? E3CONV_F16 : E3CONV_F32;
  release_variant(pl.var[other]);
  release_variant(pl.var[pl.dtype]);
  return compile_variant(pl, pl.dtype);
}

int e3conv_set_option(e3conv_plan h, int option, int value) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (option != E3CONV_OPT_CONTRACT_FIRST && option != E3CONV_OPT_TENSOR_CORES &&
      option != E3CONV_OPT_PATH_SPLIT && option != E3CONV_OPT_EDGE_VECTORS &&
      option != E3CONV_OPT_A_LAYOUT && option != E3CONV_OPT_COPY_GROUP &&
      option != E3CONV_OPT_DIRECT_PIPELINE && option != E3CONV_OPT_BACKWARD_PARTS)
    return fail(E3CONV_ERR_UNSUPPORTED, "unknown option");
  if (option == E3CONV_OPT_BACKWARD_PARTS) {  // backward kernels only: the forward stays
    if (value != -1 && (value < 1 || value > 4)) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1 or 1 .. 4");
    pl.req_bparts = value;
    DeviceGuard g(pl.device);
    for (auto& v : pl.bwd) release_backward(v);
    return E3CONV_OK;
  }
  if (option == E3CONV_OPT_DIRECT_PIPELINE) {
    if (value < -1 || value > 1) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1, 0 or 1");
    pl.req_dpipe = value;
  } else if (option == E3CONV_OPT_COPY_GROUP) {
    if (value != -1 && (value < 1 || value > 4)) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1 or 1 .. 4");
    pl.req_group = value;
  } else if (option == E3CONV_OPT_A_LAYOUT) {
    if (value < -1 || value > 3) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1 .. 3");
    pl.req_alayout = value;
  } else if (option == E3CONV_OPT_EDGE_VECTORS) {
    if (value != 0 && value != 1) return fail(E3CONV_ERR_INVALID_ARG, "value must be 0 or 1");
    pl.req_vec = value;
  } else if (option == E3CONV_OPT_PATH_SPLIT) {
    if (value < -1 || value > 8) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1 .. 8");
    pl.req_psplit = value;
  } else {
    if (value < -1 || value > 1) return fail(E3CONV_ERR_INVALID_ARG, "value must be -1, 0 or 1");
    if (option == E3CONV_OPT_CONTRACT_FIRST)
      pl.req_coop = value;
    else
      pl.req_tc = value;
  }
  DeviceGuard g(pl.device);
  const int other = pl.dtype == E3CONV_F32 ? E3CONV_F16 : E3CONV_F32;
  release_variant(pl.var[other]);
  release_variant(pl.var[pl.dtype]);
  for (auto& v : pl.bwd) release_backward(v);
  return compile_variant(pl, pl.dtype);
}

int e3conv_get_option(e3conv_plan h, int option, int* value) {
  if (!h || !value) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  const Plan& pl = h->p;
  switch (option) {
    case E3CONV_OPT_CONTRACT_FIRST: *value = pl.req_coop; return E3CONV_OK;
    case E3CONV_OPT_TENSOR_CORES: *value = pl.req_tc; return E3CONV_OK;
    case E3CONV_OPT_PATH_SPLIT: *value = pl.req_psplit; return E3CONV_OK;
    case E3CONV_OPT_EDGE_VECTORS: *value = pl.req_vec; return E3CONV_OK;
    case E3CONV_OPT_A_LAYOUT: *value = pl.req_alayout; return E3CONV_OK;
    case E3CONV_OPT_COPY_GROUP: *value = pl.req_group; return E3CONV_OK;
    case E3CONV_OPT_BACKWARD_PARTS: *value = pl.req_bparts; return E3CONV_OK;
    case E3CONV_OPT_DIRECT_PIPELINE: *value = pl.req_dpipe; return E3CONV_OK;
    default: return fail(E3CONV_ERR_UNSUPPORTED, "unknown option");
  }
}

int e3conv_spherical_harmonics(e3conv_plan h, const double* vec, double* out) {
  if (!h || !vec || !out) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  const Plan& pl = h->p;
  const double r2 = vec[0] * vec[0] + vec[1] * vec[1] + vec[2] * vec[2];
  if (!(r2 > 0.0)) {
    for (int j = 0; j < pl.ny; ++j) out[j] = j == 0 ? 1.0 : 0.0;
    return E3CONV_OK;
  }
  const double inv = 1.0 / std::sqrt(r2);
  const double u[3] = {vec[0] * inv, vec[1] * inv, vec[2] * inv};
  const auto polys = sh_polynomials(pl.lmax);
  for (int j = 0; j < pl.ny; ++j) {
    double v = 0.0;
    for (const auto& m : polys[j])
      v += m.coef * std::pow(u[0], m.px) * std::pow(u[1], m.py) * std::pow(u[2], m.pz);
    out[j] = v;
  }
  return E3CONV_OK;
}

int e3conv_edge_harmonics(e3conv_plan h, const float* edge_vectors, int64_t num_edges,
                          void* edge_sh, e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (num_edges < 0) return fail(E3CONV_ERR_INVALID_ARG, "num_edges < 0");
  if (num_edges == 0) return E3CONV_OK;
  if (!edge_vectors || !edge_sh) return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if (!aligned16(edge_vectors) || !aligned16(edge_sh))
    return fail(E3CONV_ERR_INVALID_ARG, "edge_vectors and edge_sh must be 16-byte aligned");
  // generated and compiled on the first call (also without a device, so a host can
  // check the kernel builds); loaded once a device is there
  ShVariant& v = pl.shk[pl.dtype];
  if (v.cubin.empty()) {
    ShVariant n;
    n.source = generate_sh_source(pl, pl.dtype);
    int rc = nvrtc_compile(n.source, "e3conv_edge_sh.cu", n.cubin, n.log, n.regs, n.local_bytes);
    if (rc != E3CONV_OK) return rc;
    v = n;
  }
  if (pl.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "plan has no device");
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != pl.device)
    return fail(E3CONV_ERR_INVALID_ARG, "current device differs from the plan's device");
  if (!v.compiled) {
    Driver& d = driver();
    if (d.ModuleLoadData(&v.module, v.cubin.data()) != CUDA_SUCCESS)
      return fail(E3CONV_ERR_CUDA, "cuModuleLoadData failed (harmonics)");
    if (d.ModuleGetFunction(&v.fn, v.module, "e3conv_edge_sh") != CUDA_SUCCESS) {
      d.ModuleUnload(v.module);
      v.module = nullptr;
      return fail(E3CONV_ERR_CUDA, "cuModuleGetFunction failed (harmonics)");
    }
    v.compiled = true;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pl.device) != cudaSuccess)
    return fail(E3CONV_ERR_CUDA, "cannot query the SM count");
  const long long need = (num_edges + 255) / 256;
  const long long blocks = std::min<long long>(need, static_cast<long long>(sms) * 8);
  long long ne = num_edges;
  void* args[] = {const_cast<float**>(&edge_vectors), &ne, &edge_sh};
  if (driver().LaunchKernel(v.fn, static_cast<unsigned>(blocks), 1, 1, 256, 1, 1, 0,
                            reinterpret_cast<CUstream>(stream), args, nullptr) != CUDA_SUCCESS)
    return fail(E3CONV_ERR_CUDA, "cuLaunchKernel failed (harmonics)");
  return E3CONV_OK;
}

int e3conv_query(e3conv_plan h, int* C, int* nx, int* ny, int* nout, int* num_paths) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  const Plan& pl = h->p;
  if (C) *C = pl.C;
  if (nx) *nx = pl.nx;
  if (ny) *ny = pl.ny;
  if (nout) *nout = pl.nout;
  if (num_paths) *num_paths = static_cast<int>(pl.paths.size());
  return E3CONV_OK;
}

int e3conv_path(e3conv_plan h, int p, int* l1, int* p1, int* l2, int* l3, int* p3, int* x_off,
                int* out_off) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  const Plan& pl = h->p;
  if (p < 0 || p >= static_cast<int>(pl.paths.size()))
    return fail(E3CONV_ERR_INVALID_ARG, "path index out of range");
  const Path& q = pl.paths[p];
  if (l1) *l1 = q.l1;
  if (p1) *p1 = q.p1;
  if (l2) *l2 = q.l2;
  if (l3) *l3 = q.l3;
  if (p3) *p3 = q.p3;
  if (x_off) *x_off = q.x_off;
  if (out_off) *out_off = q.out_off;
  return E3CONV_OK;
}

int e3conv_num_outputs(e3conv_plan h, int* count) {
  if (!h || !count) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  *count = static_cast<int>(h->p.outputs.size());
  return E3CONV_OK;
}

int e3conv_output_irrep(e3conv_plan h, int k, int* l, int* p, int* offset) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  const Plan& pl = h->p;
  if (k < 0 || k >= static_cast<int>(pl.outputs.size()))
    return fail(E3CONV_ERR_INVALID_ARG, "output index out of range");
  if (l) *l = pl.outputs[k].l;
  if (p) *p = pl.outputs[k].p;
  if (offset) *offset = pl.outputs[k].off;
  return E3CONV_OK;
}

int e3conv_cg(e3conv_plan h, int p, double* dense_out) {
  if (!h || !dense_out) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  const Plan& pl = h->p;
  if (p < 0 || p >= static_cast<int>(pl.paths.size()))
    return fail(E3CONV_ERR_INVALID_ARG, "path index out of range");
  std::memcpy(dense_out, pl.paths[p].cg.data(), sizeof(double) * pl.paths[p].cg.size());
  return E3CONV_OK;
}

int e3conv_kernel_info(e3conv_plan h, int dtype, int* V, int* TL, int* block, int* stages,
                       int* contract_first, int* tensor_cores, int* regs, int* local_bytes) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  if (dtype != E3CONV_F32 && dtype != E3CONV_F16)
    return fail(E3CONV_ERR_UNSUPPORTED, "unknown dtype");
  const Variant& v = h->p.var[dtype];
  if (!v.compiled) return fail(E3CONV_ERR_INVALID_ARG, "variant not compiled (set_input_dtype)");
  if (V) *V = v.shape.V;
  if (TL) *TL = v.shape.TL;
  if (block) *block = v.shape.block;
  if (stages) *stages = v.shape.stages;
  if (contract_first) *contract_first = (v.shape.coop || v.shape.tc) ? 1 : 0;
  if (tensor_cores) *tensor_cores = v.shape.tc ? 1 : 0;
  if (regs) *regs = v.regs;
  if (local_bytes) *local_bytes = v.local_bytes;
  return E3CONV_OK;
}

int e3conv_kernel_log(e3conv_plan h, int dtype, char* buf, size_t buf_len, size_t* needed) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  if (dtype != E3CONV_F32 && dtype != E3CONV_F16)
    return fail(E3CONV_ERR_UNSUPPORTED, "unknown dtype");
  const Variant& v = h->p.var[dtype];
  if (!v.compiled) return fail(E3CONV_ERR_INVALID_ARG, "variant not compiled (set_input_dtype)");
  const std::string text = h->p.trace[dtype] + v.log;
  if (needed) *needed = text.size() + 1;
  if (buf && buf_len >= text.size() + 1) std::memcpy(buf, text.c_str(), text.size() + 1);
  return E3CONV_OK;
}

int e3conv_kernel_source(e3conv_plan h, int dtype, char* buf, size_t buf_len, size_t* needed) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  if (dtype != E3CONV_F32 && dtype != E3CONV_F16)
    return fail(E3CONV_ERR_UNSUPPORTED, "unknown dtype");
  const Variant& v = h->p.var[dtype];
  if (!v.compiled) return fail(E3CONV_ERR_INVALID_ARG, "variant not compiled (set_input_dtype)");
  if (needed) *needed = v.source.size() + 1;
  if (buf && buf_len >= v.source.size() + 1) std::memcpy(buf, v.source.c_str(), v.source.size() + 1);
  return E3CONV_OK;
}

}  // extern "C"

namespace {

// One launch of the plan's forward kernel over the receiver rows
// [row_begin, row_end) of row_ptr; x holds num_nodes node rows (the senders' table).
int launch_forward(e3conv_plan h, const void* x, int64_t num_nodes, const void* Y, const void* s,
                   const int32_t* senders, const int32_t* row_ptr, int64_t row_begin,
                   int64_t row_end, float* out, e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (num_nodes < 0 || num_nodes >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "num_nodes out of range");
  if (row_begin < 0 || row_end < row_begin || row_end >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "rows must satisfy 0 <= row_begin <= row_end < 2^31");
  if (row_end == row_begin) return E3CONV_OK;
  if (!x || !row_ptr || !out)
    return fail(E3CONV_ERR_INVALID_ARG, "node_features, receiver_row_ptr and out are required");
  // (edge buffers may be NULL only for a graph without edges in these rows: the edge
  // count lives on the device, so this is the caller's promise, not a host check)
  if (!aligned16(x) || !aligned16(out) || !aligned16(Y) || !aligned16(s))
    return fail(E3CONV_ERR_INVALID_ARG, "feature buffers must be 16-byte aligned");
  const Variant& v = pl.var[pl.dtype];
  if (pl.device < 0 || !v.fn) return fail(E3CONV_ERR_NO_DEVICE, "plan has no device module");
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != pl.device)
    return fail(E3CONV_ERR_INVALID_ARG, "current device differs from the plan's device");
  const Shape& sh = v.shape;
  const long long rows = row_end - row_begin;
  long long blocks;
  unsigned smem = 0;
  CUtensorMap xmap;
  std::memset(&xmap, 0, sizeof xmap);
  if (sh.tc) {
    // x viewed as a 4-D tensor {64 channels, nx components, C / 64 channel halves, nodes}
    // (strides C * 2, 128 and nx * C * 2 bytes).  One box {64, 16, 2, 1} is a sender's
    // whole tile: two 128B-swizzled 64-channel halves of 16 rows each, 2048 bytes apart;
    // rows nx..15 lie outside the tensor and are filled with zeros.
    const cuuint64_t gdim[4] = {64, static_cast<cuuint64_t>(pl.nx), static_cast<cuuint64_t>(pl.C / 64),
                                static_cast<cuuint64_t>(num_nodes)};
    const cuuint64_t gstride[3] = {static_cast<cuuint64_t>(pl.C) * 2, 128,
                                   static_cast<cuuint64_t>(pl.nx) * pl.C * 2};
    const cuuint32_t box[4] = {64, 16, static_cast<cuuint32_t>(pl.C / 64), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (driver().TensorMapEncodeTiled(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(x),
                                      gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(E3CONV_ERR_CUDA, "cuTensorMapEncodeTiled failed for node_features");
    blocks = std::min<long long>(v.grid_blocks, rows);
    smem = static_cast<unsigned>(sh.smem_request);
  } else if (sh.stages > 0) {
    const long long tpb = sh.block / (32 * sh.team);  // teams per block
    blocks = std::min<long long>(v.grid_blocks, (rows + tpb - 1) / tpb);
    smem = static_cast<unsigned>(sh.warp_smem * tpb);
  } else {
    const long long items = rows * sh.tiles;
    const long long warps = (items + sh.ipw - 1) / sh.ipw;
    blocks = (warps * 32 + sh.block - 1) / sh.block;
  }
  if (blocks >= (1ll << 31)) return fail(E3CONV_ERR_UNSUPPORTED, "grid too large");
  int n32 = static_cast<int>(num_nodes), b32 = static_cast<int>(row_begin),
      r32 = static_cast<int>(row_end);
  float inv_avg = static_cast<float>(1.0 / pl.avg);
  void* args[] = {const_cast<void**>(&x), const_cast<void**>(&Y), const_cast<void**>(&s),
                  const_cast<int32_t**>(&senders), const_cast<int32_t**>(&row_ptr),
                  &n32, &b32, &r32, &out, &inv_avg, &pl.status, &xmap};
  CUresult r = driver().LaunchKernel(v.fn, static_cast<unsigned>(blocks), 1, 1,
                                     static_cast<unsigned>(sh.block), 1, 1, smem,
                                     reinterpret_cast<CUstream>(stream), args, nullptr);
  if (r != CUDA_SUCCESS) return fail(E3CONV_ERR_CUDA, "cuLaunchKernel failed");
  return E3CONV_OK;
}

}  // namespace

extern "C" {

int e3conv_forward(e3conv_plan h, const void* x, const void* Y, const void* s,
                   const int32_t* senders, const int32_t* row_ptr, int64_t num_nodes, float* out,
                   e3conv_stream stream) {
  return launch_forward(h, x, num_nodes, Y, s, senders, row_ptr, 0, num_nodes, out, stream);
}

int e3conv_forward_rows(e3conv_plan h, const void* x, int64_t num_nodes, const void* Y,
                        const void* s, const int32_t* senders, const int32_t* row_ptr,
                        int64_t row_begin, int64_t row_end, float* out, e3conv_stream stream) {
  return launch_forward(h, x, num_nodes, Y, s, senders, row_ptr, row_begin, row_end, out, stream);
}

int e3conv_set_radial_mlp(e3conv_plan h, int num_basis, double r_max, int hidden, int layers,
                          const float* w0, const float* w_hidden, const float* w_out) {
  if (!h || !w0 || !w_out || (layers > 1 && !w_hidden))
    return fail(E3CONV_ERR_INVALID_ARG, "NULL weights");
  Plan& pl = h->p;
  const int nout = static_cast<int>(pl.paths.size()) * pl.C;
  std::vector<const float*> wh;
  for (int l = 1; l < layers; ++l)
    wh.push_back(w_hidden + static_cast<size_t>(l - 1) * hidden * hidden);
  RadialPlan rp;
  std::string err;
  int rc = radial_prepare(rp, num_basis, r_max, hidden, layers, w0, wh.data(), w_out, nout, err);
  if (rc != E3CONV_OK) return fail(rc, err);
  if (pl.device >= 0) {
    DeviceGuard g(pl.device);
    struct Up { void** dst; const void* src; size_t n; };
    const Up ups[3] = {{&rp.d_w0, rp.w0.data(), rp.w0.size()},
                       {&rp.d_wh, rp.wh.data(), rp.wh.size()},
                       {&rp.d_wo, rp.wo.data(), rp.wo.size()}};
    for (const Up& u : ups) {
      bool good = cudaMalloc(u.dst, std::max<size_t>(u.n, 16)) == cudaSuccess;
      if (good && u.n) good = cudaMemcpy(*u.dst, u.src, u.n, cudaMemcpyHostToDevice) == cudaSuccess;
      if (!good) {
        cudaGetLastError();
        for (void* q : {rp.d_w0, rp.d_wh, rp.d_wo}) if (q) cudaFree(q);
        return fail(E3CONV_ERR_NOMEM, "allocating or copying the radial weights failed");
      }
    }
  }
  for (void* q : {pl.radial.d_w0, pl.radial.d_wh, pl.radial.d_wo})
    if (q) {
      DeviceGuard g(pl.device);
      cudaFree(q);
    }
  rp.set = true;
  pl.radial = std::move(rp);
  return E3CONV_OK;
}

int e3conv_radial_scalars(e3conv_plan h, const float* edge_vectors, int64_t num_edges,
                          void* edge_scalars, e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (!pl.radial.set) return fail(E3CONV_ERR_INVALID_ARG, "no radial MLP set (e3conv_set_radial_mlp)");
  if (num_edges < 0 || num_edges >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "num_edges out of range");
  if (num_edges == 0) return E3CONV_OK;
  if (!edge_vectors || !edge_scalars) return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if (!aligned16(edge_vectors) || !aligned16(edge_scalars))
    return fail(E3CONV_ERR_INVALID_ARG, "edge_vectors and edge_scalars must be 16-byte aligned");
  if (pl.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "plan has no device");
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != pl.device)
    return fail(E3CONV_ERR_INVALID_ARG, "current device differs from the plan's device");
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pl.device) != cudaSuccess)
    return fail(E3CONV_ERR_CUDA, "cannot query the SM count");
  std::string err;
  // the output as a 2-D tensor [num_edges][P*C] for the kernel's TMA stores: boxes of 128 edge
  // rows x 128 bytes, 128-byte swizzle; rows whose byte length is not a multiple of 16 cannot
  // be described (the kernel then stores element by element)
  const int elem = pl.dtype == E3CONV_F16 ? 2 : 4;
  const int nout = static_cast<int>(pl.paths.size()) * pl.C;
  CUtensorMap smap;
  std::memset(&smap, 0, sizeof smap);
  bool tma = (static_cast<long long>(nout) * elem) % 16 == 0 && num_edges < (1ll << 31) - 256 &&
             driver().ok;
  if (tma) {
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(nout), static_cast<cuuint64_t>(num_edges)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(nout) * elem};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), 128};
    const cuuint32_t estr[2] = {1, 1};
    tma = driver().TensorMapEncodeTiled(&smap, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                        2, edge_scalars, gdim, gstride, box, estr,
                                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                        CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const int rc = radial_launch(pl.radial, pl.radial.d_w0, pl.radial.d_wh, pl.radial.d_wo,
                               edge_vectors, num_edges, edge_scalars, pl.dtype == E3CONV_F16 ? 1 : 0,
                               pl.status, sms, reinterpret_cast<cudaStream_t>(stream), err,
                               tma ? &smap : nullptr);
  return rc == E3CONV_OK ? rc : fail(rc, err);
}

int e3conv_linear_create(e3conv_linear* out, const char* irreps_in, const char* irreps_out,
                         double scale) {
  if (!out) return fail(E3CONV_ERR_INVALID_ARG, "linear pointer is NULL");
  *out = nullptr;
  if (!std::isfinite(scale)) return fail(E3CONV_ERR_INVALID_ARG, "scale must be finite");
  std::vector<Irrep> in, o;
  std::string err;
  if (!parse_irreps(irreps_in, in, err) || !parse_irreps(irreps_out, o, err))
    return fail(E3CONV_ERR_IRREPS, err);
  e3conv_linear h = new (std::nothrow) e3conv_linear_s;
  if (!h) return fail(E3CONV_ERR_NOMEM, "host allocation failed");
  const int rc = linear_prepare(h->p, in, o, scale, err);
  if (rc != E3CONV_OK) {
    delete h;
    return fail(rc, err);
  }
  if (has_device()) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaMalloc(&h->p.status, sizeof(unsigned)) != cudaSuccess) {
      cudaGetLastError();
      delete h;
      return fail(E3CONV_ERR_NOMEM, "cudaMalloc of the status word failed");
    }
    cudaMemset(h->p.status, 0, sizeof(unsigned));
    h->p.device = dev;
  }
  *out = h;
  return E3CONV_OK;
}

void e3conv_linear_destroy(e3conv_linear h) {
  if (!h) return;
  {
    DeviceGuard g(h->p.device);
    if (h->p.d_w) cudaFree(h->p.d_w);
    if (h->p.status) cudaFree(h->p.status);
  }
  delete h;
}

int e3conv_linear_query(e3conv_linear h, int* dim_in, int* dim_out, int* num_weight_blocks,
                        int* mul_in, int* mul_out) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "linear is NULL");
  if (dim_in) *dim_in = h->p.dim_in;
  if (dim_out) *dim_out = h->p.dim_out;
  if (num_weight_blocks) *num_weight_blocks = h->p.num_weight_blocks;
  if (mul_in) *mul_in = h->p.K;
  if (mul_out) *mul_out = h->p.N;
  return E3CONV_OK;
}

int e3conv_linear_uses_tma(e3conv_linear h, int* uses_tma) {
  if (!h || !uses_tma) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  *uses_tma = linear_uses_tma(h->p) ? 1 : 0;
  return E3CONV_OK;
}

int e3conv_linear_set_tma(e3conv_linear h, int enable) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "linear is NULL");
  if (enable != 0 && enable != 1) return fail(E3CONV_ERR_INVALID_ARG, "enable must be 0 or 1");
  h->p.allow_tma = enable == 1;
  h->p.tma_args.clear();
  return E3CONV_OK;
}

int e3conv_linear_set_weights(e3conv_linear h, const float* w) {
  if (!h || (!w && h->p.num_weight_blocks > 0)) return fail(E3CONV_ERR_INVALID_ARG, "NULL argument");
  LinearPlan& lp = h->p;
  std::string err;
  int rc = linear_pack(lp, w, err);
  if (rc != E3CONV_OK) return fail(rc, err);
  lp.tma_args.clear();  // the block scales of the kernel arguments follow the weights
  if (lp.device >= 0 && !lp.packed.empty()) {
    DeviceGuard g(lp.device);
    if (!lp.d_w && cudaMalloc(&lp.d_w, lp.packed.size()) != cudaSuccess) {
      cudaGetLastError();
      lp.d_w = nullptr;
      return fail(E3CONV_ERR_NOMEM, "cudaMalloc of the packed weights failed");
    }
    if (cudaMemcpy(lp.d_w, lp.packed.data(), lp.packed.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      return fail(E3CONV_ERR_CUDA, "copying the packed weights failed");
    }
  }
  lp.weights_set = true;
  return E3CONV_OK;
}

int e3conv_linear_forward(e3conv_linear h, const float* x, int64_t num_nodes, float* y,
                          e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "linear is NULL");
  LinearPlan& lp = h->p;
  if (num_nodes < 0 || num_nodes >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "num_nodes out of range");
  if (num_nodes == 0) return E3CONV_OK;
  if (!lp.weights_set) return fail(E3CONV_ERR_INVALID_ARG, "weights not set (e3conv_linear_set_weights)");
  if (!x || !y) return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if (!aligned16(x) || !aligned16(y)) return fail(E3CONV_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  if (lp.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "no CUDA device");
  int cur = -1, sms = 0;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != lp.device)
    return fail(E3CONV_ERR_INVALID_ARG, "current device differs from the linear layer's device");
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, lp.device) != cudaSuccess)
    return fail(E3CONV_ERR_CUDA, "cannot query the SM count");
  std::string err;
  const int rc = linear_launch(lp, lp.d_w, x, num_nodes, y, lp.status, sms,
                               reinterpret_cast<cudaStream_t>(stream),
                               driver().ok ? driver().TensorMapEncodeTiled : nullptr, err);
  return rc == E3CONV_OK ? rc : fail(rc, err);
}

int e3conv_linear_check(e3conv_linear h, e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "linear is NULL");
  if (h->p.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "no device");
  unsigned st = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, h->p.status, sizeof st, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return fail(E3CONV_ERR_CUDA, "reading the status word failed");
  if (st) {
    cudaMemsetAsync(h->p.status, 0, sizeof st, s);
    cudaStreamSynchronize(s);
    return fail(E3CONV_ERR_CUDA, "a pipeline wait of the linear layer timed out");
  }
  return E3CONV_OK;
}

int e3conv_partition_rows(const int32_t* row_ptr, int64_t num_nodes, int parts, int64_t* bounds) {
  if (!row_ptr || !bounds) return fail(E3CONV_ERR_INVALID_ARG, "row_ptr and bounds are required");
  if (parts < 1) return fail(E3CONV_ERR_INVALID_ARG, "parts must be at least 1");
  if (num_nodes < 0 || num_nodes >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "num_nodes out of range");
  if (row_ptr[0] < 0) return fail(E3CONV_ERR_INVALID_ARG, "row_ptr[0] is negative");
  for (int64_t b = 0; b < num_nodes; ++b)
    if (row_ptr[b + 1] < row_ptr[b]) return fail(E3CONV_ERR_INVALID_ARG, "row_ptr decreases");
  // cost of the rows before b: their edges plus one per row (every row stores an output
  // row); strictly increasing in b.  Boundary r is the row whose prefix cost is nearest to
  // r/parts of the total (of the first row that reaches it and the one before).
  auto cost = [&](int64_t b) { return static_cast<int64_t>(row_ptr[b]) - row_ptr[0] + b; };
  const int64_t total = cost(num_nodes);
  bounds[0] = 0;
  for (int r = 1; r < parts; ++r) {
    const int64_t target = static_cast<int64_t>((static_cast<__int128>(total) * r) / parts);
    int64_t lo = bounds[r - 1], hi = num_nodes;
    while (lo < hi) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (cost(mid) >= target) hi = mid; else lo = mid + 1;
    }
    if (lo > bounds[r - 1] && target - cost(lo - 1) < cost(lo) - target) --lo;
    bounds[r] = lo;
  }
  bounds[parts] = num_nodes;
  return E3CONV_OK;
}

int e3conv_prepare_backward(e3conv_plan h) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  DeviceGuard g(h->p.device);
  return prepare_backward(h->p);
}

int e3conv_backward(e3conv_plan h, const void* x, const void* Y, const void* s,
                    const int32_t* senders, const int32_t* receivers, const int32_t* row_ptr,
                    const int32_t* sender_row_ptr, const int32_t* sender_perm, int64_t num_nodes,
                    const float* grad_out, float* grad_x, float* grad_sh, float* grad_scalars,
                    e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (num_nodes < 0 || num_nodes >= (1ll << 31))
    return fail(E3CONV_ERR_INVALID_ARG, "num_nodes out of range");
  if (num_nodes == 0) return E3CONV_OK;
  if ((grad_sh == nullptr) != (grad_scalars == nullptr))
    return fail(E3CONV_ERR_INVALID_ARG, "grad_sh and grad_scalars are computed together: give both or neither");
  if (!row_ptr || !grad_out) return fail(E3CONV_ERR_INVALID_ARG, "receiver_row_ptr and grad_out are required");
  if (grad_sh && !x) return fail(E3CONV_ERR_INVALID_ARG, "node_features is required for grad_sh / grad_scalars");
  if (grad_x && (!receivers || !sender_row_ptr || !sender_perm))
    return fail(E3CONV_ERR_INVALID_ARG, "grad_x needs receivers, sender_row_ptr and sender_perm");
  if (!aligned16(x) || !aligned16(Y) || !aligned16(s) || !aligned16(grad_out) ||
      !aligned16(grad_x) || !aligned16(grad_scalars))
    return fail(E3CONV_ERR_INVALID_ARG, "feature and gradient buffers must be 16-byte aligned");
  if (pl.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "plan has no device module");
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != pl.device)
    return fail(E3CONV_ERR_INVALID_ARG, "current device differs from the plan's device");
  int rc = prepare_backward(pl);
  if (rc != E3CONV_OK) return rc;
  const BwdVariant& bv = pl.bwd[pl.dtype];
  const BwdShape& b = bv.shape;
  int n32 = static_cast<int>(num_nodes);
  float inv_avg = static_cast<float>(1.0 / pl.avg);
  const long long warps = (num_nodes + b.ipw - 1) / b.ipw;
  const long long blocks = (warps * 32 + b.block - 1) / b.block;
  if (blocks >= (1ll << 31)) return fail(E3CONV_ERR_UNSUPPORTED, "grid too large");
  CUstream st = reinterpret_cast<CUstream>(stream);
  if (grad_sh) {
    void* args[] = {const_cast<void**>(&x), const_cast<void**>(&Y), const_cast<void**>(&s),
                    const_cast<int32_t**>(&senders), const_cast<int32_t**>(&row_ptr), &n32,
                    const_cast<float**>(&grad_out), &grad_sh, &grad_scalars, &inv_avg, &pl.status};
    for (int p = 0; p < b.eparts; ++p)
      if (driver().LaunchKernel(bv.fn[2 * p], static_cast<unsigned>(blocks), 1, 1, b.block, 1, 1,
                                b.staged ? static_cast<unsigned>(b.esmem[p]) : 0u, st, args,
                                nullptr) != CUDA_SUCCESS)
        return fail(E3CONV_ERR_CUDA, "cuLaunchKernel failed (backward, edges)");
  }
  if (grad_x) {
    void* args[] = {const_cast<void**>(&Y), const_cast<void**>(&s),
                    const_cast<int32_t**>(&receivers), const_cast<int32_t**>(&row_ptr),
                    const_cast<int32_t**>(&sender_row_ptr), const_cast<int32_t**>(&sender_perm),
                    &n32, const_cast<float**>(&grad_out), &grad_x, &inv_avg, &pl.status};
    const int nparts = b.nstaged ? b.eparts : 1;
    for (int p = 0; p < nparts; ++p)
      if (driver().LaunchKernel(bv.fn[2 * p + 1], static_cast<unsigned>(blocks), 1, 1, b.block, 1, 1,
                                b.nstaged ? static_cast<unsigned>(nparts > 1 ? b.nsmem_p[p] : b.nsmem) : 0u,
                                st, args, nullptr) != CUDA_SUCCESS)
        return fail(E3CONV_ERR_CUDA, "cuLaunchKernel failed (backward, nodes)");
  }
  return E3CONV_OK;
}

int e3conv_backward_source(e3conv_plan h, int which, char* buf, size_t buf_len, size_t* needed) {
  if (!h || which < 0 || which > 7) return fail(E3CONV_ERR_INVALID_ARG, "bad argument");
  DeviceGuard g(h->p.device);
  int rc = prepare_backward(h->p);
  if (rc != E3CONV_OK) return rc;
  if (which >= 2 && h->p.bwd[h->p.dtype].source[which].empty())
    return fail(E3CONV_ERR_INVALID_ARG, "this plan's backward kernels are not split");
  const std::string& src = h->p.bwd[h->p.dtype].source[which];
  if (needed) *needed = src.size() + 1;
  if (buf && buf_len >= src.size() + 1) std::memcpy(buf, src.c_str(), src.size() + 1);
  return E3CONV_OK;
}

int e3conv_check(e3conv_plan h, e3conv_stream stream) {
  if (!h) return fail(E3CONV_ERR_INVALID_ARG, "plan is NULL");
  Plan& pl = h->p;
  if (pl.device < 0) return fail(E3CONV_ERR_NO_DEVICE, "plan has no device");
  unsigned st = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, pl.status, sizeof st, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return fail(E3CONV_ERR_CUDA, "reading the status word failed");
  if (st) {
    cudaMemsetAsync(pl.status, 0, sizeof st, s);
    cudaStreamSynchronize(s);
    if (st & 4u) return fail(E3CONV_ERR_CUDA, "a forward's shared-memory pipeline wait timed out");
    return fail(E3CONV_ERR_BAD_INDEX, std::string("forward met ") +
                                          ((st & 1u) ? "an invalid receiver_row_ptr range " : "") +
                                          ((st & 2u) ? "an out-of-range sender" : ""));
  }
  return E3CONV_OK;
}

int e3conv_csr_workspace_size(int64_t num_edges, int64_t num_nodes, size_t* bytes) {
  if (!bytes) return fail(E3CONV_ERR_INVALID_ARG, "bytes is NULL");
  if (num_edges < 0 || num_nodes < 0 || num_edges >= (1ll << 31) || num_nodes >= (1ll << 31) - 1)
    return fail(E3CONV_ERR_INVALID_ARG, "sizes out of range");
  *bytes = csr_workspace_bytes(num_edges, num_nodes);
  return E3CONV_OK;
}

int e3conv_build_csr(const int32_t* receivers, int64_t num_edges, int64_t num_nodes,
                     int32_t* row_ptr, int32_t* perm, void* workspace, size_t workspace_bytes,
                     e3conv_stream stream) {
  if (num_edges < 0 || num_nodes < 0 || num_edges >= (1ll << 31) || num_nodes >= (1ll << 31) - 1)
    return fail(E3CONV_ERR_INVALID_ARG, "sizes out of range");
  if (!row_ptr || (num_edges > 0 && (!receivers || !perm)))
    return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(E3CONV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (!has_device()) return fail(E3CONV_ERR_NO_DEVICE, "no CUDA device");
  std::string err;
  int rc = csr_build(receivers, num_edges, num_nodes, row_ptr, perm, workspace, workspace_bytes,
                     reinterpret_cast<cudaStream_t>(stream), err, nullptr);
  return rc == E3CONV_OK ? rc : fail(rc, err);
}

int e3conv_build_csr_noalloc(const int32_t* receivers, int64_t num_edges, int64_t num_nodes,
                             int32_t* row_ptr, int32_t* perm, e3conv_stream stream) {
  if (num_edges < 0 || num_nodes < 0 || num_edges >= (1ll << 31) || num_nodes >= (1ll << 31) - 1)
    return fail(E3CONV_ERR_INVALID_ARG, "sizes out of range");
  if (!row_ptr || (num_edges > 0 && (!receivers || !perm)))
    return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if (!has_device()) return fail(E3CONV_ERR_NO_DEVICE, "no CUDA device");
  std::string err;
  int rc = csr_build_static(receivers, num_edges, num_nodes, row_ptr, perm,
                            reinterpret_cast<cudaStream_t>(stream), err);
  return rc == E3CONV_OK ? rc : fail(rc, err);
}

int e3conv_csr_kernel_count(int64_t num_edges, int64_t num_nodes, int* count) {
  if (!count) return fail(E3CONV_ERR_INVALID_ARG, "count is NULL");
  if (num_edges < 0 || num_nodes < 0 || num_edges >= (1ll << 31) || num_nodes >= (1ll << 31) - 1)
    return fail(E3CONV_ERR_INVALID_ARG, "sizes out of range");
  std::string err;
  return csr_build(nullptr, num_edges, num_nodes, nullptr, nullptr, nullptr, 0, nullptr, err,
                   count);
}

int e3conv_csr_check(const void* workspace, e3conv_stream stream) {
  if (!workspace) return fail(E3CONV_ERR_INVALID_ARG, "workspace is NULL");
  unsigned st = 0;
  if (csr_read_status(workspace, reinterpret_cast<cudaStream_t>(stream), &st) != E3CONV_OK)
    return fail(E3CONV_ERR_CUDA, "reading the CSR status word failed");
  if (st) return fail(E3CONV_ERR_BAD_INDEX, "receivers outside [0, num_nodes)");
  return E3CONV_OK;
}

int e3conv_permute_rows(const void* src, int64_t num_src_rows, const int32_t* perm,
                        int64_t num_rows, int64_t row_bytes, void* dst, int32_t* status,
                        e3conv_stream stream) {
  if (num_rows < 0 || num_src_rows < 0 || row_bytes < 0 || row_bytes % 4)
    return fail(E3CONV_ERR_INVALID_ARG, "bad sizes (row_bytes must be a multiple of 4)");
  if (num_rows == 0 || row_bytes == 0) return E3CONV_OK;
  if (!src || !dst || !perm) return fail(E3CONV_ERR_INVALID_ARG, "NULL buffer");
  if (!aligned16(src) || !aligned16(dst))
    return fail(E3CONV_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  if (!has_device()) return fail(E3CONV_ERR_NO_DEVICE, "no CUDA device");
  std::string err;
  int rc = permute_rows(src, num_src_rows, perm, num_rows, row_bytes, dst, status,
                        reinterpret_cast<cudaStream_t>(stream), err);
  return rc == E3CONV_OK ? rc : fail(rc, err);
}

}  // extern "C"
