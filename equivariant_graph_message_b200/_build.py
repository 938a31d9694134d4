"""Builds libe3conv.so in-tree with nvcc for sm_100a.

Host sources (plans, Racah CG tables, kernel code generation, NVRTC and the
C ABI) and the device sources (CSR indexing, row gather) are compiled with
`-gencode arch=compute_100a,code=sm_100a -lineinfo`; the forward kernel is
generated per plan and compiled by NVRTC for sm_100a at plan creation.
The CUDA runtime is linked statically; NVRTC is found through the rpath of
the CUDA toolkit; the driver is reached through cudaGetDriverEntryPoint, so
the library loads on machines without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libe3conv.so")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
SOURCES = ["api.cpp", "irreps.cpp", "cg.cpp", "sh.cpp", "codegen.cpp", "csr.cu", "radial.cu", "linear.cu"]


def _nvcc() -> str:
    p = os.path.join(CUDA_HOME, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def sources() -> list[str]:
    return [os.path.join(CSRC, s) for s in SOURCES] + \
        [os.path.join(CSRC, "plan.h"), os.path.join(CSRC, "tc_common.cuh"),
         os.path.join(CSRC, "exports.map"),
         os.path.join(os.path.dirname(PKG), "include", "e3conv.h")]


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(verbose: bool = False, jobs: int = 8) -> str:
    nvcc = _nvcc()
    tmp = tempfile.mkdtemp(prefix="e3conv_build_")
    try:
        objs, procs = [], []
        for s in SOURCES:
            src = os.path.join(CSRC, s)
            obj = os.path.join(tmp, s + ".o")
            cmd = [nvcc, "-c", src, "-o", obj, "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                   "-Xcompiler", "-fvisibility=hidden", "-lineinfo", *ARCH,
                   "-I", os.path.join(CUDA_HOME, "include"),
                   '-DE3CONV_NVRTC_PATH="%s"' % os.path.join(CUDA_HOME, "lib64", "libnvrtc.so.12")]
            if verbose:
                print(" ".join(cmd))
            procs.append(subprocess.Popen(cmd))
            objs.append(obj)
        for p in procs:
            if p.wait() != 0:
                raise RuntimeError("nvcc failed while building libe3conv.so")
        out_tmp = LIB + ".tmp"
        cmd = [nvcc, "-shared", "-o", out_tmp, *objs, *ARCH, "-cudart", "static",
               "-ldl",
               "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map")]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        os.replace(out_tmp, LIB)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))
