"""Builds oracle/liboracle.so from forward.c and backward.c with gcc and OpenMP (test
infrastructure)."""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def build(verbose: bool = False) -> str:
    srcs = [os.path.join(_HERE, "forward.c"), os.path.join(_HERE, "backward.c")]
    out = os.path.join(_HERE, "liboracle.so")
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", *srcs, "-o", out + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose=True))
