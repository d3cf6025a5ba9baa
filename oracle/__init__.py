"""CPU oracle for the Haar patcher and the FSQ quantizer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product (``haar_wavelet_patching_b200``) never imports it and has no CPU
fallback.

The arithmetic lives in plain C (``haar.c``, ``fsq.c``) in double precision;
this module only marshals numpy arrays through ctypes.  Each C function cites
the page and section it follows.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None

FSQ_LEVELS = (8, 8, 8, 5, 5, 5)
FSQ_CODEBOOK = 64000


def _load():
    global _lib
    if _lib is None:
        # ORACLE_SO lets the mutation test load a copy of the oracle with a planted mistake.
        path = os.environ.get("ORACLE_SO") or _build()
        lib = ctypes.CDLL(path)
        i64, dp, fp = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_float)
        for name in ("oracle_haar_fwd", "oracle_haar_inv", "oracle_haar_fwd_blockform"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [dp, dp, i64, i64, i64, i64, i64]
        for name in ("oracle_haar_fwd_adjoint", "oracle_haar_inv_adjoint"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [dp, dp, i64, i64, i64, i64, i64]
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_haar_padded_extents.restype = ctypes.c_int
        lib.oracle_haar_padded_extents.argtypes = [i64, i64, i64, i64, i64, i64p, i64p, i64p]
        lib.oracle_haar_pad.restype = ctypes.c_int
        lib.oracle_haar_pad.argtypes = [dp, dp, i64, i64, i64, i64, i64, i64, i64, i64]
        for name in ("oracle_haar_fwd_padded", "oracle_haar_inv_cropped"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [dp, dp, i64, i64, i64, i64, i64, i64, i64]
        for name in ("oracle_haar_fwd_chunk", "oracle_haar_inv_chunk"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [dp, dp, i64, i64, i64, i64, i64, ctypes.c_int]
        for name in ("oracle_haar_level_fwd", "oracle_haar_level_inv"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [dp, dp, i64, i64, i64, i64]
        lib.oracle_haar_out_frames.restype = i64
        lib.oracle_haar_out_frames.argtypes = [i64]
        lib.oracle_fsq_levels.restype = ctypes.c_int
        lib.oracle_fsq_levels.argtypes = [ctypes.c_int]
        lib.oracle_fsq_basis.restype = i64
        lib.oracle_fsq_basis.argtypes = [ctypes.c_int]
        lib.oracle_fsq_bound.restype = ctypes.c_double
        lib.oracle_fsq_bound.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_fsq_quantize.restype = ctypes.c_int
        lib.oracle_fsq_quantize.argtypes = [ctypes.c_float, ctypes.c_int]
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_fsq_pack.restype = i64
        lib.oracle_fsq_pack.argtypes = [ip]
        lib.oracle_fsq_unpack.restype = None
        lib.oracle_fsq_unpack.argtypes = [i64, ip]
        i32p = ctypes.POINTER(ctypes.c_int32)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_fsq_encode.restype = i64
        lib.oracle_fsq_encode.argtypes = [fp, fp, i64, i64, i64, i32p, dp, u8p]
        lib.oracle_fsq_decode.restype = i64
        lib.oracle_fsq_decode.argtypes = [i32p, fp, i64, i64, i64, dp]
        lib.oracle_fsq_ste_slope.restype = ctypes.c_double
        lib.oracle_fsq_ste_slope.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.oracle_fsq_encode_backward.restype = None
        lib.oracle_fsq_encode_backward.argtypes = [fp, fp, fp, i64, i64, i64, dp, dp]
        lib.oracle_fsq_decode_backward.restype = None
        lib.oracle_fsq_decode_backward.argtypes = [i32p, fp, fp, i64, i64, i64, dp, dp]
        _lib = lib
    return _lib


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected the shape (code {rc})")


def out_frames(T: int) -> int:
    """Latent frames of the two-level patcher: 1 + (T-1)/4, or 1 for an image."""
    return int(_load().oracle_haar_out_frames(T))


def haar_out_shape(B, C, T, H, W):
    if T == 1:
        return (B, 16 * C, 1, H // 4, W // 4)
    return (B, 64 * C, out_frames(T), H // 4, W // 4)


def haar_fwd(x: np.ndarray) -> np.ndarray:
    """Two-level causal full-packet Haar patcher, level by level, in double.

    x: [B, C, T, H, W] (any real dtype; converted exactly to float64).
    Returns y: [B, 64C, 1+(T-1)/4, H/4, W/4], or [B, 16C, 1, H/4, W/4] if T == 1.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, C, T, H, W = x.shape
    y = np.zeros(haar_out_shape(B, C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_fwd(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double), B, C, T, H, W),
           "haar_fwd")
    return y


def haar_fwd_blockform(x: np.ndarray) -> np.ndarray:
    """Same transform through its derived 4x4x4 Walsh-Hadamard block form (pins only)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, C, T, H, W = x.shape
    y = np.zeros(haar_out_shape(B, C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_fwd_blockform(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double),
                                             B, C, T, H, W), "haar_fwd_blockform")
    return y


def haar_inv(y: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Two-level unpatcher; T, H, W are the pixel-space extents.  Returns [B, C, T, H, W]."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    B = y.shape[0]
    C = y.shape[1] // (16 if T == 1 else 64)
    if y.shape != haar_out_shape(B, C, T, H, W):
        raise ValueError(f"haar_inv: coefficient shape {y.shape} does not match T,H,W={T},{H},{W}")
    x = np.zeros((B, C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_inv(_ptr(y, ctypes.c_double), _ptr(x, ctypes.c_double), B, C, T, H, W),
           "haar_inv")
    return x


def haar_fwd_adjoint(gy: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Gradient of the patcher: coefficient-shaped gy -> pixel-shaped gx = M^T gy (video only)."""
    gy = np.ascontiguousarray(gy, dtype=np.float64)
    B = gy.shape[0]
    C = gy.shape[1] // 64
    if gy.shape != haar_out_shape(B, C, T, H, W):
        raise ValueError("haar_fwd_adjoint: shape mismatch")
    gx = np.zeros((B, C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_fwd_adjoint(_ptr(gy, ctypes.c_double), _ptr(gx, ctypes.c_double), B, C, T, H, W),
           "haar_fwd_adjoint")
    return gx


def haar_inv_adjoint(gx: np.ndarray) -> np.ndarray:
    """Gradient of the unpatcher: pixel-shaped gx -> coefficient-shaped gy (video only)."""
    gx = np.ascontiguousarray(gx, dtype=np.float64)
    B, C, T, H, W = gx.shape
    gy = np.zeros(haar_out_shape(B, C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_inv_adjoint(_ptr(gx, ctypes.c_double), _ptr(gy, ctypes.c_double), B, C, T, H, W),
           "haar_inv_adjoint")
    return gy


def haar_level_fwd(x: np.ndarray) -> np.ndarray:
    """One level: [C, T, H, W] -> [8C, (T+1)/2, H/2, W/2] (T odd > 1) or [4C, 1, H/2, W/2] (T == 1)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    C, T, H, W = x.shape
    shape = (4 * C, 1, H // 2, W // 2) if T == 1 else (8 * C, (T + 1) // 2, H // 2, W // 2)
    y = np.zeros(shape, dtype=np.float64)
    _check(_load().oracle_haar_level_fwd(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double), C, T, H, W),
           "haar_level_fwd")
    return y


def haar_level_inv(y: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    """Inverse of one level, T, H, W the pixel extents: -> [C, T, H, W]."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    C = y.shape[0] // (4 if T == 1 else 8)
    x = np.zeros((C, T, H, W), dtype=np.float64)
    _check(_load().oracle_haar_level_inv(_ptr(y, ctypes.c_double), _ptr(x, ctypes.c_double), C, T, H, W),
           "haar_level_inv")
    return x


def single_out_shape(B, C, T, H, W):
    """The single-level patcher (patch_size=2): [B, 8C, (T+1)/2, H/2, W/2], images [B, 4C, 1, H/2, W/2]."""
    return (B, 4 * C, 1, H // 2, W // 2) if T == 1 else (B, 8 * C, (T + 1) // 2, H // 2, W // 2)


def haar_single_fwd(x: np.ndarray) -> np.ndarray:
    """The single-level patcher on a batch [B, C, T, H, W]: one level per item."""
    return np.stack([haar_level_fwd(xb) for xb in np.asarray(x, dtype=np.float64)])


def haar_single_inv(y: np.ndarray, T: int, H: int, W: int) -> np.ndarray:
    return np.stack([haar_level_inv(yb, T, H, W) for yb in np.asarray(y, dtype=np.float64)])


def fsq_basis():
    return tuple(int(_load().oracle_fsq_basis(i)) for i in range(6))


def fsq_bound(z: float, i: int) -> float:
    return float(_load().oracle_fsq_bound(float(z), i))


def fsq_quantize(z: float, i: int) -> int:
    return int(_load().oracle_fsq_quantize(float(z), i))


def fsq_pack(digits) -> int:
    d = (ctypes.c_int * 6)(*[int(v) for v in digits])
    return int(_load().oracle_fsq_pack(d))


def fsq_unpack(idx: int):
    d = (ctypes.c_int * 6)()
    _load().oracle_fsq_unpack(int(idx), d)
    return tuple(d)


def fsq_encode(u: np.ndarray, w: np.ndarray):
    """Projection C->6 (fp32 fmaf chain) + tanh bound + round + index pack.

    u: [B, C, S] float32; w: [6, C] float32.
    Returns (idx [B,S] int32, codes [B,6,S] float64, near [B,S] bool).
    """
    u = np.ascontiguousarray(u, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    B, C, S = u.shape
    if w.shape != (6, C):
        raise ValueError(f"fsq_encode: weight shape {w.shape} != (6, {C})")
    idx = np.zeros((B, S), dtype=np.int32)
    codes = np.zeros((B, 6, S), dtype=np.float64)
    near = np.zeros((B, S), dtype=np.uint8)
    _load().oracle_fsq_encode(_ptr(u, ctypes.c_float), _ptr(w, ctypes.c_float), B, C, S,
                              _ptr(idx, ctypes.c_int32), _ptr(codes, ctypes.c_double),
                              _ptr(near, ctypes.c_uint8))
    return idx, codes, near.astype(bool)


def fsq_decode(idx: np.ndarray, w: np.ndarray):
    """Index unpack -> normalized codes -> 6->C projection, in double.

    idx: [B, S] int32; w: [6, C].  Returns (out [B, C, S] float64, n_bad).
    """
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    B, S = idx.shape
    C = w.shape[1]
    out = np.zeros((B, C, S), dtype=np.float64)
    bad = _load().oracle_fsq_decode(_ptr(idx, ctypes.c_int32), _ptr(w, ctypes.c_float), B, C, S,
                                    _ptr(out, ctypes.c_double))
    return out, int(bad)


def fsq_ste_slope(z: float, i: int) -> float:
    return float(_load().oracle_fsq_ste_slope(float(z), i))


def fsq_encode_backward(u: np.ndarray, w: np.ndarray, g: np.ndarray):
    """Straight-through encode backward: (grad_u [B,C,S], grad_w [6,C]) in float64."""
    u = np.ascontiguousarray(u, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    B, C, S = u.shape
    gu = np.zeros((B, C, S), dtype=np.float64)
    gw = np.zeros((6, C), dtype=np.float64)
    _load().oracle_fsq_encode_backward(_ptr(u, ctypes.c_float), _ptr(w, ctypes.c_float), _ptr(g, ctypes.c_float),
                                       B, C, S, _ptr(gu, ctypes.c_double), _ptr(gw, ctypes.c_double))
    return gu, gw


def fsq_decode_backward(idx: np.ndarray, w: np.ndarray, g: np.ndarray):
    """Decode backward: (grad_codes [B,6,S], grad_w [6,C]) in float64."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    g = np.ascontiguousarray(g, dtype=np.float32)
    B, C, S = g.shape
    gc = np.zeros((B, 6, S), dtype=np.float64)
    gw = np.zeros((6, C), dtype=np.float64)
    _load().oracle_fsq_decode_backward(_ptr(idx, ctypes.c_int32), _ptr(w, ctypes.c_float), _ptr(g, ctypes.c_float),
                                       B, C, S, _ptr(gc, ctypes.c_double), _ptr(gw, ctypes.c_double))
    return gc, gw


def padded_extents(T: int, H: int, W: int, ms: int = 4, mt: int = 4):
    """(Tp, Hp, Wp): zeros to multiples of ms in space, reflection to Tp = 1 (mod mt) in time."""
    Tp, Hp, Wp = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    if not _load().oracle_haar_padded_extents(T, H, W, ms, mt, ctypes.byref(Tp), ctypes.byref(Hp), ctypes.byref(Wp)):
        raise ValueError("padded_extents: invalid multiples or shape")
    return Tp.value, Hp.value, Wp.value


def haar_pad(x: np.ndarray, ms: int = 4, mt: int = 4) -> np.ndarray:
    """The padded clip [B, C, Tp, Hp, Wp] the padded patcher transforms."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, C, T, H, W = x.shape
    Tp, Hp, Wp = padded_extents(T, H, W, ms, mt)
    xp = np.zeros((B, C, Tp, Hp, Wp))
    _check(_load().oracle_haar_pad(_ptr(x, ctypes.c_double), _ptr(xp, ctypes.c_double), B, C, T, H, W, Tp, Hp, Wp),
           "haar_pad")
    return xp


def haar_fwd_padded(x: np.ndarray, ms: int = 4, mt: int = 4) -> np.ndarray:
    """Patcher on a clip of any extents: pad (zeros in space, reflection in time), then transform."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, C, T, H, W = x.shape
    Tp, Hp, Wp = padded_extents(T, H, W, ms, mt)
    y = np.zeros(haar_out_shape(B, C, Tp, Hp, Wp))
    _check(_load().oracle_haar_fwd_padded(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double), B, C, T, H, W, ms, mt),
           "haar_fwd_padded")
    return y


def haar_inv_cropped(y: np.ndarray, T: int, H: int, W: int, ms: int = 4, mt: int = 4) -> np.ndarray:
    """Unpatcher on the padded extents, cropped to [B, C, T, H, W]."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    Tp, Hp, Wp = padded_extents(T, H, W, ms, mt)
    B = y.shape[0]
    C = y.shape[1] // (16 if Tp == 1 else 64)
    if y.shape != haar_out_shape(B, C, Tp, Hp, Wp):
        raise ValueError("haar_inv_cropped: coefficient shape does not match the padded extents")
    x = np.zeros((B, C, T, H, W))
    _check(_load().oracle_haar_inv_cropped(_ptr(y, ctypes.c_double), _ptr(x, ctypes.c_double), B, C, T, H, W, ms, mt),
           "haar_inv_cropped")
    return x


def chunk_out_shape(B, C, T, H, W, first):
    """Streaming chunks are always video: 64C channels, (T + 3) // 4 latent frames (first) or T // 4."""
    return (B, 64 * C, (T + 3) // 4 if first else T // 4, H // 4, W // 4)


def haar_fwd_chunk(x: np.ndarray, first: bool) -> np.ndarray:
    """Streaming chunk of a video: first -> T = 1 + 4k frames with the frame-0 replicas (3D even
    for one frame); else 4k frames, no replica."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, C, T, H, W = x.shape
    y = np.zeros(chunk_out_shape(B, C, T, H, W, first))
    _check(_load().oracle_haar_fwd_chunk(_ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double), B, C, T, H, W,
                                         int(bool(first))), "haar_fwd_chunk")
    return y


def haar_inv_chunk(y: np.ndarray, T: int, H: int, W: int, first: bool) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    B = y.shape[0]
    C = y.shape[1] // 64
    if y.shape != chunk_out_shape(B, C, T, H, W, first):
        raise ValueError("haar_inv_chunk: shape mismatch")
    x = np.zeros((B, C, T, H, W))
    _check(_load().oracle_haar_inv_chunk(_ptr(y, ctypes.c_double), _ptr(x, ctypes.c_double), B, C, T, H, W,
                                         int(bool(first))), "haar_inv_chunk")
    return x


def haar_fwd_channels_last(x: np.ndarray) -> np.ndarray:
    """The patcher's coefficients in channels-last order [B, T', h, w, 64C]: haar_fwd with the
    channel axis moved last (a layout of the same values; numpy does the permutation)."""
    return np.ascontiguousarray(np.moveaxis(haar_fwd(x), 1, -1))
