"""Build libtok.so (the C-ABI library of include/tok.h) in-tree with nvcc for sm_100a.

    python -m haar_wavelet_patching_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled to an object in _build/ and linked into
haar_wavelet_patching_b200/libtok.so with a static CUDA runtime, so the library
loads on machines without a GPU (calls then fail with TOK_ERR_CUDA).
"""
import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
TARGET = os.path.join(PKG, "libtok.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


_INCLUDE_RE = re.compile(r'^\s*#\s*include\s*"([^"]+)"', re.M)


def local_headers(path, seen=None):
    """The repository headers a source includes, directly or through other repository headers."""
    seen = set() if seen is None else seen
    with open(path) as f:
        text = f.read()
    for name in _INCLUDE_RE.findall(text):
        for d in (os.path.dirname(path), CSRC, INCLUDE):
            cand = os.path.join(d, name)
            if os.path.exists(cand) and cand not in seen:
                seen.add(cand)
                local_headers(cand, seen)
                break
    return seen


def build(force: bool = False, verbose: bool = False) -> str:
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    objs, rebuilt = [], False
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        deps = [src, *local_headers(src)]
        if not force and os.path.exists(obj) and \
                os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps):
            continue
        cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        rebuilt = True
    if not rebuilt and os.path.exists(TARGET) and \
            os.path.getmtime(TARGET) >= max(os.path.getmtime(o) for o in objs):
        return TARGET
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
                    "-o", TARGET + ".tmp", *objs], check=True)
    os.replace(TARGET + ".tmp", TARGET)
    return TARGET


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
