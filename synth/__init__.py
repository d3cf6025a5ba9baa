"""Seeded synthetic workloads for the tests and the benchmark.

This module holds no arithmetic of the patcher or the quantizer: it draws
counter-based random numbers (``gen.c``), evaluates the smooth-field recipe and
rounds to the stored type.  Both the CUDA path and the CPU oracle read the
buffers it returns.

bf16 data is returned as numpy ``uint16`` bit patterns (numpy has no bf16);
``bf16_bits_to_f64`` widens them exactly.
"""
import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(HERE, "_synth.so")
_lib = None

F32, BF16, F64 = 0, 1, 2
_NP = {F32: np.float32, BF16: np.uint16, F64: np.float64}

# Stream ids: one per kind of draw, so workloads never share random numbers.
STREAM_PIXELS, STREAM_LATENT, STREAM_SCALE, STREAM_WEIGHT = 1, 2, 3, 4
WEIGHT_SEED = 0x5EED


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.run(["gcc", "-std=c11", "-O3", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        "-Wall", "-o", _SO + ".tmp", src, "-lm"], check=True)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i32, i64, u64, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        lib.synth_uniform.argtypes = [vp, i32, i64, u64, u64, d, d]
        lib.synth_normal.argtypes = [vp, i32, i64, u64, u64, d, d]
        lib.synth_smooth_field.argtypes = [vp, i32, i64, i64, i64, i64, i64, u64, d]
        for f in (lib.synth_uniform, lib.synth_normal, lib.synth_smooth_field):
            f.restype = None
        _lib = lib
    return _lib


def _alloc(shape, dtype, out=None):
    if out is not None:
        assert out.dtype == _NP[dtype] and out.flags.c_contiguous and out.shape == tuple(shape)
        return out
    return np.empty(shape, dtype=_NP[dtype])


def uniform(shape, seed, lo=-1.0, hi=1.0, dtype=F32, stream=STREAM_PIXELS, out=None):
    a = _alloc(shape, dtype, out)
    _load().synth_uniform(a.ctypes.data, dtype, a.size, seed, stream, lo, hi)
    return a


def normal(shape, seed, mean=0.0, std=1.0, dtype=F32, stream=STREAM_LATENT, out=None):
    a = _alloc(shape, dtype, out)
    _load().synth_normal(a.ctypes.data, dtype, a.size, seed, stream, mean, std)
    return a


def smooth_field(shape, seed, dtype=BF16, noise=0.05, out=None):
    """[B, C, T, H, W]: eight seeded sinusoids per (b, c) plus U[-noise, noise], clipped to [-1, 1]."""
    B, C, T, H, W = shape
    a = _alloc(shape, dtype, out)
    _load().synth_smooth_field(a.ctypes.data, dtype, B, C, T, H, W, seed, noise)
    return a


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    return bf16_bits_to_f64(a) if dtype == BF16 else a.astype(np.float64)


# ---------------------------------------------------------------------------
# The five workloads.  Shapes follow the pages' workloads: 121-frame 704x1280
# (and 1088x1920) clips, 16-channel latents on 8x16x16 grids (16x44x80 per
# 704x1280 clip), 6-channel FSQ.  Config k uses seed k.
# ---------------------------------------------------------------------------
HAAR_CONFIGS = {
    1: dict(shape=(1, 3, 9, 64, 64), dtype=F32, kind="uniform"),
    2: dict(shape=(16, 3, 1, 1024, 1024), dtype=BF16, kind="uniform"),
    3: dict(shape=(1, 3, 121, 704, 1280), dtype=BF16, kind="smooth"),
    5: dict(shape=(4, 3, 121, 1088, 1920), dtype=BF16, kind="smooth"),
}

FSQ_CONFIGS = {
    1: dict(B=1, C=16, S=4096, kind="normal", std=1.0),
    2: dict(B=16, C=16, S=64 * 64, kind="normal", std=1.5),
    4: dict(B=64, C=16, S=16 * 44 * 80, kind="scaled", std_lo=0.5, std_hi=2.0),
    5: dict(B=4, C=16, S=16 * 68 * 120, kind="normal", std=1.0),
}


def haar_input(cfg: int, out=None):
    c = HAAR_CONFIGS[cfg]
    if c["kind"] == "uniform":
        return uniform(c["shape"], seed=cfg, dtype=c["dtype"], out=out)
    return smooth_field(c["shape"], seed=cfg, dtype=c["dtype"], out=out)


def fsq_weight(C: int = 16, seed: int = WEIGHT_SEED) -> np.ndarray:
    """Projection weight W [6, C] ~ N(0, 1/C) (std 1/4 for C = 16), fp32."""
    return normal((6, C), seed=seed, std=1.0 / np.sqrt(C), stream=STREAM_WEIGHT)


def fsq_input(cfg: int, out=None) -> np.ndarray:
    """Latent u [B, C, S] fp32."""
    c = FSQ_CONFIGS[cfg]
    shape = (c["B"], c["C"], c["S"])
    if c["kind"] == "normal":
        return normal(shape, seed=cfg, std=c["std"], out=out)
    # N(0,1) scaled per (batch item, channel) by sigma ~ U[std_lo, std_hi].
    n = normal(shape, seed=cfg, dtype=F64)
    sigma = uniform(shape[:2], seed=cfg, lo=c["std_lo"], hi=c["std_hi"], dtype=F64, stream=STREAM_SCALE)
    u = (n * sigma[:, :, None]).astype(np.float32)
    if out is not None:
        out[...] = u
        return out
    return u
