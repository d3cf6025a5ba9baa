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


# Files whose kernels come from CUTLASS's sm100 templates (header-only, vendored in the image).
CUTLASS_SOURCES = ("conv.cu",)


def cutlass_includes():
    """Include directories of the CUTLASS tree vendored with flashinfer in this image."""
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")
    roots = [os.path.join(os.path.dirname(spec.origin), "data", "cutlass")] if spec and spec.origin else []
    for root in roots:
        inc, util = os.path.join(root, "include"), os.path.join(root, "tools", "util", "include")
        if os.path.exists(os.path.join(inc, "cutlass", "conv", "collective", "builders", "sm100_umma_builder.inl")):
            return [inc, util]
    raise RuntimeError("CUTLASS headers with the sm100 convolution builders were not found")


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
        if os.path.basename(src) in CUTLASS_SOURCES:
            for inc in cutlass_includes():
                cmd += ["-I", inc]
            cmd += ["-diag-suppress", "20012"]  # CUTLASS's defaulted host-device constructors
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
