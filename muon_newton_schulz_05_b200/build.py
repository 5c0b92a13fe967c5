"""Build libmuonb200.so in-tree with nvcc for sm_100a.

Usage: python muon_newton_schulz_05_b200/build.py [--verbose-ptxas] [--check]
(--check builds libmuonb200_check.so with device-side bounds checks, -DMUON_CHECK;
the binding loads it instead when MUON_B200_CHECK=1)
(run by path: the script does not import the package, so it works before
the library exists)
The CUDA runtime is linked statically; the driver entry point used for TMA
descriptors is looked up at run time, so the library has no -lcuda dependency.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmuonb200.so")
LIB_CHECK = os.path.join(PKG, "libmuonb200_check.so")
SOURCES = ["api.cu", "elementwise.cu", "ns_gemm.cu"]
HEADERS = ["plan.cuh", "ptx.cuh", "tiles.cuh", "update_math.cuh", "check.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(INCLUDE, "muon_b200.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, check: bool = False,
          out: str = None, defines=()) -> str:
    """Compile the library. out/defines build a variant elsewhere (tuning
    constants such as MUON_STAGES=5) without touching the in-tree library."""
    lib = out or (LIB_CHECK if check else LIB)
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp"]
    if check:
        cmd += ["-DMUON_CHECK"]
    cmd += [f"-D{d}" for d in defines]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if ptxas_verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    args = sys.argv[1:]
    out = args[args.index("--out") + 1] if "--out" in args else None
    defines = [a[2:] for a in args if a.startswith("-D")]
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in args, check="--check" in args,
                out=out, defines=defines))
