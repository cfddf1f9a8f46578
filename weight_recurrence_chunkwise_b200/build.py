"""Build ``libdeltarule.so`` (the C-ABI library) in-tree with nvcc for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdeltarule.so")
MAIN = os.path.join(CSRC, "deltarule_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]


def _sources():
    out = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    return out


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile the library unless it is newer than every source; return its path."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, MAIN, "-o", LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in args else []
    print(build(force=True, verbose=True, extra=extra))
