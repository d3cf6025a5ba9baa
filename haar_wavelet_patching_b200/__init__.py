"""B200 Haar patcher / unpatcher and FSQ quantizer: Python binding of libtok.so.

The functions named like the C ABI (``tok_haar_fwd`` ...) marshal torch CUDA
tensors into the C calls of ``include/tok.h`` and nothing else: every step of
the computation runs in the library's sm_100a kernels.  There is no CPU path;
a missing library or a CPU tensor raises.

Convenience wrappers (``haar_fwd``, ``haar_inv``, ``fsq_encode``,
``fsq_decode``) allocate outputs with torch and call the same entry points.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtok.so")

(TOK_OK, TOK_ERR_NULL, TOK_ERR_SHAPE, TOK_ERR_ALIGN, TOK_ERR_DTYPE, TOK_ERR_ALIAS, TOK_ERR_CUDA,
 TOK_ERR_TIMEOUT, TOK_ERR_TOO_LARGE) = range(9)
TOK_F32, TOK_BF16 = 0, 1
FSQ_CODEBOOK = 64000
FSQ_DIM = 6

# Every symbol include/tok.h declares.
ABI_SYMBOLS = ("tok_abi_version", "tok_status_str", "tok_last_cuda_error", "tok_check_device",
               "tok_selftest_wait_timeout", "tok_haar_fwd",
               "tok_haar_inv", "tok_haar_fwd_adjoint", "tok_haar_inv_adjoint", "tok_haar_fwd_windows",
               "tok_haar_inv_windows", "tok_haar_fwd_single", "tok_haar_inv_single", "tok_haar_fwd_channels_last", "tok_haar_padded_extents", "tok_haar_fwd_padded", "tok_haar_inv_cropped",
               "tok_haar_fwd_chunk", "tok_haar_inv_chunk", "tok_conv_spatial", "tok_conv_temporal_causal",
               "tok_conv_factorized", "tok_patch_embed_pack_weights", "tok_patch_embed_spatial", "tok_fsq_encode", "tok_fsq_decode", "tok_fsq_backward_workspace_size",
               "tok_fsq_encode_backward", "tok_fsq_encode_backward_noalloc", "tok_fsq_decode_backward")

_lib = None


class TokError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        msg = lib().tok_status_str(status).decode()
        if status == TOK_ERR_CUDA:
            msg += f" (cudaError {lib().tok_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


def lib():
    """The loaded libtok.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m haar_wavelet_patching_b200.build` "
                              "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.tok_abi_version.restype = i32
        L.tok_abi_version.argtypes = []
        L.tok_status_str.restype = ctypes.c_char_p
        L.tok_status_str.argtypes = [i32]
        L.tok_last_cuda_error.restype = i32
        L.tok_last_cuda_error.argtypes = []
        L.tok_check_device.restype = i32
        L.tok_check_device.argtypes = [vp]
        L.tok_selftest_wait_timeout.restype = i32
        L.tok_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
        for f in (L.tok_haar_fwd, L.tok_haar_inv, L.tok_haar_fwd_adjoint, L.tok_haar_inv_adjoint,
                  L.tok_haar_fwd_single, L.tok_haar_inv_single, L.tok_haar_fwd_channels_last):
            f.restype = i32
            f.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, vp]
        L.tok_fsq_backward_workspace_size.restype = i64
        L.tok_fsq_backward_workspace_size.argtypes = [i64, i64, i64]
        for f in (L.tok_fsq_encode_backward, L.tok_fsq_decode_backward):
            f.restype = i32
            f.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
        L.tok_fsq_encode_backward_noalloc.restype = i32
        L.tok_fsq_encode_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
        for f in (L.tok_haar_fwd_windows, L.tok_haar_inv_windows):
            f.restype = i32
            f.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, i64, i64, vp]
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.tok_haar_padded_extents.restype = i32
        L.tok_haar_padded_extents.argtypes = [i64, i64, i64, i64, i64, i64p, i64p, i64p]
        for f in (L.tok_haar_fwd_padded, L.tok_haar_inv_cropped):
            f.restype = i32
            f.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, i64, i64, vp]
        for f in (L.tok_haar_fwd_chunk, L.tok_haar_inv_chunk):
            f.restype = i32
            f.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, i32, vp]
        for f in (L.tok_conv_spatial, L.tok_conv_temporal_causal):
            f.restype = i32
            f.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, vp]
        L.tok_patch_embed_pack_weights.restype = i32
        L.tok_patch_embed_pack_weights.argtypes = [vp, vp, i64, i64, vp]
        L.tok_patch_embed_spatial.restype = i32
        L.tok_patch_embed_spatial.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, vp]
        L.tok_conv_factorized.restype = i32
        L.tok_conv_factorized.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, i64, vp]
        L.tok_fsq_encode.restype = i32
        L.tok_fsq_encode.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
        L.tok_fsq_decode.restype = i32
        L.tok_fsq_decode.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
        _lib = L
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TOK_F32
    if t.dtype == torch.bfloat16:
        return TOK_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: the patcher takes float32 or bfloat16")


def _cuda(t: torch.Tensor, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(t: torch.Tensor, stream):
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check(status, what):
    if status != TOK_OK:
        raise TokError(status, what)


# ---------------------------------------------------------------------------
# Shape rules (host logic).
# ---------------------------------------------------------------------------
def latent_frames(T: int) -> int:
    """1 + (T-1)/4 latent frames for T = 1 + 4k video frames; 1 for an image."""
    if T == 1:
        return 1
    if T < 1 or T % 4 != 1:
        raise ValueError(f"T={T}: the causal two-level patcher needs T == 1 or T % 4 == 1")
    return 1 + (T - 1) // 4


def haar_coeff_shape(B, C, T, H, W):
    if H % 4 or W % 4:
        raise ValueError(f"H={H}, W={W} must be multiples of 4")
    return (B, (16 if T == 1 else 64) * C, latent_frames(T), H // 4, W // 4)


# ---------------------------------------------------------------------------
# C-ABI calls.
# ---------------------------------------------------------------------------
def tok_check_device(device=None, stream=None):
    """Synchronize the stream; raise TokError if a kernel stopped after a bounded wait ran out."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    _check(lib().tok_check_device(ctypes.c_void_p(stream.cuda_stream)), "tok_check_device")


def tok_selftest_wait_timeout(polls: int, device=None, stream=None):
    """Launch the failure-channel self-test: a kernel whose barrier wait runs out after
    `polls` polls and counts a timeout (the next tok_check_device raises TOK_ERR_TIMEOUT)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    _check(lib().tok_selftest_wait_timeout(polls, ctypes.c_void_p(stream.cuda_stream)), "tok_selftest_wait_timeout")


def tok_haar_fwd(x: torch.Tensor, y: torch.Tensor, stream=None):
    """x [B,C,T,H,W] -> y [B,64C,T',H/4,W/4] (T == 1: [B,16C,1,H/4,W/4]); same dtype."""
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5:
        raise ValueError("x must be [B, C, T, H, W]")
    if y.dtype != x.dtype:
        raise TypeError("x and y must have the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != haar_coeff_shape(B, C, T, H, W):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {haar_coeff_shape(B, C, T, H, W)}")
    _check(lib().tok_haar_fwd(_ptr(x), _ptr(y), _dtype_code(x), B, C, T, H, W, _stream(x, stream)), "tok_haar_fwd")
    return y


def tok_haar_inv(y: torch.Tensor, x: torch.Tensor, stream=None):
    """Coefficients y -> x [B,C,T,H,W] (the output's shape gives T, H, W)."""
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5:
        raise ValueError("x must be [B, C, T, H, W]")
    if y.dtype != x.dtype:
        raise TypeError("x and y must have the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != haar_coeff_shape(B, C, T, H, W):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {haar_coeff_shape(B, C, T, H, W)}")
    _check(lib().tok_haar_inv(_ptr(y), _ptr(x), _dtype_code(x), B, C, T, H, W, _stream(x, stream)), "tok_haar_inv")
    return x


def _haar_windows(fwd, x, y, t_begin, t_end, stream):
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != haar_coeff_shape(B, C, T, H, W):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {haar_coeff_shape(B, C, T, H, W)}")
    f = lib().tok_haar_fwd_windows if fwd else lib().tok_haar_inv_windows
    src, dst = (x, y) if fwd else (y, x)
    _check(f(_ptr(src), _ptr(dst), _dtype_code(x), B, C, T, H, W, int(t_begin), int(t_end), _stream(x, stream)),
           "tok_haar_fwd_windows" if fwd else "tok_haar_inv_windows")


def tok_haar_fwd_windows(x: torch.Tensor, y: torch.Tensor, t_begin: int, t_end: int, stream=None):
    """Forward restricted to latent frames [t_begin, t_end) of the full tensors x, y."""
    _haar_windows(True, x, y, t_begin, t_end, stream)
    return y


def tok_haar_inv_windows(y: torch.Tensor, x: torch.Tensor, t_begin: int, t_end: int, stream=None):
    """Inverse restricted to latent frames [t_begin, t_end): writes only those windows' pixel frames."""
    _haar_windows(False, x, y, t_begin, t_end, stream)
    return x


def channels_last_shape(B, C, T, H, W):
    """tok_haar_fwd_channels_last's output: [B, T', H/4, W/4, 64C] (images [B, 1, H/4, W/4, 16C])."""
    b, k, t, h, w = haar_coeff_shape(B, C, T, H, W)
    return (b, t, h, w, k)


def tok_haar_fwd_channels_last(x: torch.Tensor, y: torch.Tensor, stream=None):
    """x [B,C,T,H,W] -> y [B,T',H/4,W/4,64C]: the patcher's coefficients, channels last."""
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != channels_last_shape(B, C, T, H, W):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {channels_last_shape(B, C, T, H, W)}")
    _check(lib().tok_haar_fwd_channels_last(_ptr(x), _ptr(y), _dtype_code(x), B, C, T, H, W, _stream(x, stream)),
           "tok_haar_fwd_channels_last")
    return y


def haar_fwd_channels_last(x: torch.Tensor, stream=None) -> torch.Tensor:
    y = torch.empty(channels_last_shape(*x.shape), dtype=x.dtype, device=x.device)
    return tok_haar_fwd_channels_last(x, y, stream)


def single_coeff_shape(B, C, T, H, W):
    """The single-level patcher's output: [B, 8C, (T+1)/2, H/2, W/2], images [B, 4C, 1, H/2, W/2]."""
    return (B, 4 * C, 1, H // 2, W // 2) if T == 1 else (B, 8 * C, (T + 1) // 2, H // 2, W // 2)


def _haar_single(fwd, x, y, stream):
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != single_coeff_shape(B, C, T, H, W):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {single_coeff_shape(B, C, T, H, W)}")
    f = lib().tok_haar_fwd_single if fwd else lib().tok_haar_inv_single
    src, dst = (x, y) if fwd else (y, x)
    _check(f(_ptr(src), _ptr(dst), _dtype_code(x), B, C, T, H, W, _stream(x, stream)),
           "tok_haar_fwd_single" if fwd else "tok_haar_inv_single")


def tok_haar_fwd_single(x: torch.Tensor, y: torch.Tensor, stream=None):
    """The single-level patcher (patch_size=2): x [B,C,T,H,W] -> y (single_coeff_shape)."""
    _haar_single(True, x, y, stream)
    return y


def tok_haar_inv_single(y: torch.Tensor, x: torch.Tensor, stream=None):
    _haar_single(False, x, y, stream)
    return x


def padded_extents(T: int, H: int, W: int, spatial_multiple: int = 4, temporal_multiple: int = 4):
    """(Tp, Hp, Wp) of tok_haar_fwd_padded: zeros in space, a mirrored tail in time."""
    Tp, Hp, Wp = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().tok_haar_padded_extents(T, H, W, spatial_multiple, temporal_multiple, ctypes.byref(Tp),
                                         ctypes.byref(Hp), ctypes.byref(Wp)), "tok_haar_padded_extents")
    return Tp.value, Hp.value, Wp.value


def padded_coeff_shape(B, C, T, H, W, spatial_multiple=4, temporal_multiple=4):
    Tp, Hp, Wp = padded_extents(T, H, W, spatial_multiple, temporal_multiple)
    return haar_coeff_shape(B, C, Tp, Hp, Wp)


def tok_haar_fwd_padded(x: torch.Tensor, y: torch.Tensor, spatial_multiple: int = 4, temporal_multiple: int = 4,
                        stream=None):
    """x [B,C,T,H,W] of any extents -> y, the patcher of the padded clip (see padded_coeff_shape)."""
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != padded_coeff_shape(B, C, T, H, W, spatial_multiple, temporal_multiple):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected "
                         f"{padded_coeff_shape(B, C, T, H, W, spatial_multiple, temporal_multiple)}")
    _check(lib().tok_haar_fwd_padded(_ptr(x), _ptr(y), _dtype_code(x), B, C, T, H, W, spatial_multiple,
                                     temporal_multiple, _stream(x, stream)), "tok_haar_fwd_padded")
    return y


def tok_haar_inv_cropped(y: torch.Tensor, x: torch.Tensor, spatial_multiple: int = 4, temporal_multiple: int = 4,
                         stream=None):
    """Coefficients of a padded clip -> x [B,C,T,H,W], the unpatcher cropped to x's extents."""
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != padded_coeff_shape(B, C, T, H, W, spatial_multiple, temporal_multiple):
        raise ValueError("y does not have the padded coefficient shape of x")
    _check(lib().tok_haar_inv_cropped(_ptr(y), _ptr(x), _dtype_code(x), B, C, T, H, W, spatial_multiple,
                                      temporal_multiple, _stream(x, stream)), "tok_haar_inv_cropped")
    return x


def chunk_coeff_shape(B, C, T, H, W, first):
    """Streaming chunks are video: 64C channels, (T + 3) // 4 latent frames (first) or T // 4."""
    return (B, 64 * C, (T + 3) // 4 if first else T // 4, H // 4, W // 4)


def _haar_chunk(fwd, x, y, first, stream):
    _cuda(x, "x"), _cuda(y, "y")
    if x.dim() != 5 or y.dtype != x.dtype:
        raise ValueError("x must be [B, C, T, H, W] and y of the same dtype")
    B, C, T, H, W = x.shape
    if tuple(y.shape) != chunk_coeff_shape(B, C, T, H, W, first):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {chunk_coeff_shape(B, C, T, H, W, first)}")
    f = lib().tok_haar_fwd_chunk if fwd else lib().tok_haar_inv_chunk
    src, dst = (x, y) if fwd else (y, x)
    _check(f(_ptr(src), _ptr(dst), _dtype_code(x), B, C, T, H, W, int(bool(first)), _stream(x, stream)),
           "tok_haar_fwd_chunk" if fwd else "tok_haar_inv_chunk")


def tok_haar_fwd_chunk(x: torch.Tensor, y: torch.Tensor, first: bool, stream=None):
    """A chunk of a video: first -> T = 1 + 4k frames with the frame-0 replicas; else 4k frames, none."""
    _haar_chunk(True, x, y, first, stream)
    return y


def tok_haar_inv_chunk(y: torch.Tensor, x: torch.Tensor, first: bool, stream=None):
    _haar_chunk(False, x, y, first, stream)
    return x


def _conv_dims(x, name):
    _cuda(x, name)
    if x.dim() != 5 or x.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be a channels-last bf16 tensor [B, T, h, w, C]")
    return x.shape


def tok_conv_spatial(x: torch.Tensor, ws: torch.Tensor, y: torch.Tensor, stream=None):
    """1 x k x k convolution, 'same' zero padding: x [B,T,h,w,Cin], ws [Cout,k,k,Cin] -> y [B,T,h,w,Cout]."""
    B, T, h, w, Cin = _conv_dims(x, "x")
    _conv_dims(y, "y"), _cuda(ws, "ws")
    Cout, k = ws.shape[0], ws.shape[1]
    if tuple(ws.shape) != (Cout, k, k, Cin) or tuple(y.shape) != (B, T, h, w, Cout) or ws.dtype != torch.bfloat16:
        raise ValueError("ws must be bf16 [Cout, k, k, Cin] and y [B, T, h, w, Cout]")
    _check(lib().tok_conv_spatial(_ptr(x), _ptr(ws), _ptr(y), B, T, h, w, Cin, Cout, k, _stream(x, stream)),
           "tok_conv_spatial")
    return y


def tok_conv_temporal_causal(x: torch.Tensor, wt: torch.Tensor, y: torch.Tensor, stream=None):
    """k x 1 x 1 convolution over time, frame t reading t-k+1 .. t: wt [Cout, k, Cin]."""
    B, T, h, w, Cin = _conv_dims(x, "x")
    _conv_dims(y, "y"), _cuda(wt, "wt")
    Cout, k = wt.shape[0], wt.shape[1]
    if tuple(wt.shape) != (Cout, k, Cin) or tuple(y.shape) != (B, T, h, w, Cout) or wt.dtype != torch.bfloat16:
        raise ValueError("wt must be bf16 [Cout, k, Cin] and y [B, T, h, w, Cout]")
    _check(lib().tok_conv_temporal_causal(_ptr(x), _ptr(wt), _ptr(y), B, T, h, w, Cin, Cout, k,
                                          _stream(x, stream)), "tok_conv_temporal_causal")
    return y


def tok_conv_factorized(x, ws, wt, mid, y, stream=None):
    """The spatial convolution into mid, then the causal temporal convolution into y."""
    B, T, h, w, Cin = _conv_dims(x, "x")
    _conv_dims(mid, "mid"), _conv_dims(y, "y"), _cuda(ws, "ws"), _cuda(wt, "wt")
    Cmid, k, Cout = ws.shape[0], ws.shape[1], wt.shape[0]
    if (tuple(ws.shape) != (Cmid, k, k, Cin) or tuple(wt.shape) != (Cout, k, Cmid)
            or tuple(mid.shape) != (B, T, h, w, Cmid) or tuple(y.shape) != (B, T, h, w, Cout)):
        raise ValueError("shapes: ws [Cmid,k,k,Cin], wt [Cout,k,Cmid], mid [B,T,h,w,Cmid], y [B,T,h,w,Cout]")
    _check(lib().tok_conv_factorized(_ptr(x), _ptr(ws), _ptr(wt), _ptr(mid), _ptr(y), B, T, h, w, Cin, Cmid, Cout,
                                     k, _stream(x, stream)), "tok_conv_factorized")
    return y


def tok_patch_embed_pack_weights(ws: torch.Tensor, wp: torch.Tensor, stream=None):
    """Reorder the spatial filter ws [Cmid, 3, 3, 64C] for the fused call: wp [Cmid, 9C, 64]."""
    _cuda(ws, "ws"), _cuda(wp, "wp")
    Cmid, C = ws.shape[0], ws.shape[3] // 64
    if (ws.dim() != 4 or tuple(ws.shape[1:3]) != (3, 3) or ws.shape[3] != 64 * C or ws.dtype != torch.bfloat16
            or tuple(wp.shape) != (Cmid, 9 * C, 64) or wp.dtype != torch.bfloat16):
        raise ValueError("ws must be bf16 [Cmid, 3, 3, 64C] and wp bf16 [Cmid, 9C, 64]")
    _check(lib().tok_patch_embed_pack_weights(_ptr(ws), _ptr(wp), C, Cmid, _stream(ws, stream)),
           "tok_patch_embed_pack_weights")
    return wp


def tok_patch_embed_spatial(x: torch.Tensor, wp: torch.Tensor, y: torch.Tensor, stream=None):
    """The patcher fused into the 1 x 3 x 3 convolution: x [B,C,T,H,W] bf16 pixels, wp the packed
    filter [Cmid, 9C, 64] -> y [B, T', H/4, W/4, Cmid] bf16."""
    _cuda(x, "x"), _cuda(wp, "wp"), _cuda(y, "y")
    if x.dim() != 5 or x.dtype != torch.bfloat16 or wp.dtype != torch.bfloat16 or y.dtype != torch.bfloat16:
        raise ValueError("x [B, C, T, H, W], wp and y must be bf16")
    B, C, T, H, W = x.shape
    Cmid = wp.shape[0]
    if tuple(wp.shape) != (Cmid, 9 * C, 64) or tuple(y.shape) != (B, latent_frames(T), H // 4, W // 4, Cmid):
        raise ValueError("wp must be [Cmid, 9C, 64] and y [B, T', H/4, W/4, Cmid]")
    _check(lib().tok_patch_embed_spatial(_ptr(x), _ptr(wp), _ptr(y), B, C, T, H, W, Cmid, _stream(x, stream)),
           "tok_patch_embed_spatial")
    return y


def patch_embed_pack_weights(ws, stream=None):
    Cmid, C = ws.shape[0], ws.shape[3] // 64
    wp = torch.empty((Cmid, 9 * C, 64), dtype=torch.bfloat16, device=ws.device)
    return tok_patch_embed_pack_weights(ws, wp, stream)


def patch_embed_spatial(x, wp, stream=None):
    B, C, T, H, W = x.shape
    y = torch.empty((B, latent_frames(T), H // 4, W // 4, wp.shape[0]), dtype=torch.bfloat16, device=x.device)
    return tok_patch_embed_spatial(x, wp, y, stream)


def conv_factorized(x, ws, wt, stream=None):
    B, T, h, w, _ = x.shape
    mid = torch.empty((B, T, h, w, ws.shape[0]), dtype=torch.bfloat16, device=x.device)
    y = torch.empty((B, T, h, w, wt.shape[0]), dtype=torch.bfloat16, device=x.device)
    return tok_conv_factorized(x, ws, wt, mid, y, stream)


def tok_haar_fwd_adjoint(gy: torch.Tensor, gx: torch.Tensor, stream=None):
    """Gradient of the patcher: gy (coefficient shape) -> gx [B,C,T,H,W]."""
    _cuda(gx, "gx"), _cuda(gy, "gy")
    B, C, T, H, W = gx.shape
    if gy.dtype != gx.dtype or tuple(gy.shape) != haar_coeff_shape(B, C, T, H, W):
        raise ValueError("gy must have the coefficient shape and dtype of gx")
    _check(lib().tok_haar_fwd_adjoint(_ptr(gy), _ptr(gx), _dtype_code(gx), B, C, T, H, W, _stream(gx, stream)),
           "tok_haar_fwd_adjoint")
    return gx


def tok_haar_inv_adjoint(gx: torch.Tensor, gy: torch.Tensor, stream=None):
    """Gradient of the unpatcher: gx [B,C,T,H,W] -> gy (coefficient shape)."""
    _cuda(gx, "gx"), _cuda(gy, "gy")
    B, C, T, H, W = gx.shape
    if gy.dtype != gx.dtype or tuple(gy.shape) != haar_coeff_shape(B, C, T, H, W):
        raise ValueError("gy must have the coefficient shape and dtype of gx")
    _check(lib().tok_haar_inv_adjoint(_ptr(gx), _ptr(gy), _dtype_code(gx), B, C, T, H, W, _stream(gx, stream)),
           "tok_haar_inv_adjoint")
    return gy


def _latent_dims(u: torch.Tensor):
    if u.dim() < 2:
        raise ValueError("latent must be [B, C, ...]")
    B, C = u.shape[0], u.shape[1]
    S = 1
    for d in u.shape[2:]:
        S *= d
    return B, C, S


def tok_fsq_encode(u: torch.Tensor, w: torch.Tensor, idx: torch.Tensor, codes: torch.Tensor = None, stream=None):
    """u [B,C,...] fp32, w [6,C] fp32 -> idx [B,...] int32 (+ codes [B,6,...] fp32)."""
    for t, n in ((u, "u"), (w, "w"), (idx, "idx"), (codes, "codes")):
        _cuda(t, n)
    B, C, S = _latent_dims(u)
    if u.dtype != torch.float32 or w.dtype != torch.float32 or idx.dtype != torch.int32:
        raise TypeError("u and w must be float32, idx int32")
    if tuple(w.shape) != (FSQ_DIM, C):
        raise ValueError(f"w must be [6, {C}]")
    if idx.numel() != B * S or (codes is not None and (codes.numel() != B * FSQ_DIM * S or codes.dtype != torch.float32)):
        raise ValueError("idx must hold B*S int32 and codes B*6*S float32")
    _check(lib().tok_fsq_encode(_ptr(u), _ptr(w), _ptr(idx), _ptr(codes), B, C, S, _stream(u, stream)),
           "tok_fsq_encode")
    return idx, codes


def tok_fsq_decode(idx: torch.Tensor, w: torch.Tensor, out: torch.Tensor, bad_count: torch.Tensor = None,
                   stream=None):
    """idx [B,...] int32, w [6,C] -> out [B,C,...] fp32; bad_count: optional 1-element int32 CUDA tensor."""
    for t, n in ((idx, "idx"), (w, "w"), (out, "out"), (bad_count, "bad_count")):
        _cuda(t, n)
    B, C, S = _latent_dims(out)
    if idx.dtype != torch.int32 or w.dtype != torch.float32 or out.dtype != torch.float32:
        raise TypeError("idx must be int32, w and out float32")
    if tuple(w.shape) != (FSQ_DIM, C) or idx.numel() != B * S:
        raise ValueError(f"w must be [6, {C}] and idx hold B*S = {B * S} indices")
    if bad_count is not None and (bad_count.dtype != torch.int32 or bad_count.numel() < 1):
        raise ValueError("bad_count must be an int32 CUDA tensor")
    _check(lib().tok_fsq_decode(_ptr(idx), _ptr(w), _ptr(out), _ptr(bad_count), B, C, S, _stream(idx, stream)),
           "tok_fsq_decode")
    return out


def fsq_backward_workspace_size(B: int, C: int, S: int) -> int:
    n = int(lib().tok_fsq_backward_workspace_size(B, C, S))
    if n < 0:
        raise ValueError(f"no FSQ backward for B={B}, C={C}, S={S} (1 <= C <= 16)")
    return n


def tok_fsq_encode_backward(u, w, grad_codes, grad_u, grad_w, workspace, stream=None):
    """Straight-through encode backward into grad_u [B,C,...] and grad_w [6,C]; workspace: uint8 CUDA tensor."""
    for t, n in ((u, "u"), (w, "w"), (grad_codes, "grad_codes"), (grad_u, "grad_u"), (grad_w, "grad_w"),
                 (workspace, "workspace")):
        _cuda(t, n)
    B, C, S = _latent_dims(u)
    if grad_u.shape != u.shape or grad_codes.numel() != B * FSQ_DIM * S or tuple(grad_w.shape) != (FSQ_DIM, C):
        raise ValueError("shapes: grad_u like u, grad_codes [B,6,...], grad_w [6,C]")
    _check(lib().tok_fsq_encode_backward(_ptr(u), _ptr(w), _ptr(grad_codes), _ptr(grad_u), _ptr(grad_w),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(), B, C, S,
                                         _stream(u, stream)), "tok_fsq_encode_backward")
    return grad_u, grad_w


def tok_fsq_encode_backward_noalloc(u, w, grad_codes, grad_u, grad_w, stream=None):
    """tok_fsq_encode_backward using the library's fixed scratch instead of a workspace (allocates nothing;
    its 3 MB scratch holds at most 8,388,608 tokens at C = 16; concurrent calls must be serialized by the caller)."""
    for t, n in ((u, "u"), (w, "w"), (grad_codes, "grad_codes"), (grad_u, "grad_u"), (grad_w, "grad_w")):
        _cuda(t, n)
    B, C, S = _latent_dims(u)
    if grad_u.shape != u.shape or grad_codes.numel() != B * FSQ_DIM * S or tuple(grad_w.shape) != (FSQ_DIM, C):
        raise ValueError("shapes: grad_u like u, grad_codes [B,6,...], grad_w [6,C]")
    _check(lib().tok_fsq_encode_backward_noalloc(_ptr(u), _ptr(w), _ptr(grad_codes), _ptr(grad_u), _ptr(grad_w),
                                                 B, C, S, _stream(u, stream)), "tok_fsq_encode_backward_noalloc")
    return grad_u, grad_w


def tok_fsq_decode_backward(idx, w, grad_out, grad_codes, grad_w, workspace, stream=None):
    """Decode backward into grad_codes [B,6,...] and grad_w [6,C]; workspace: uint8 CUDA tensor."""
    for t, n in ((idx, "idx"), (w, "w"), (grad_out, "grad_out"), (grad_codes, "grad_codes"), (grad_w, "grad_w"),
                 (workspace, "workspace")):
        _cuda(t, n)
    B, C, S = _latent_dims(grad_out)
    if idx.numel() != B * S or grad_codes.numel() != B * FSQ_DIM * S or tuple(grad_w.shape) != (FSQ_DIM, C):
        raise ValueError("shapes: idx [B,...], grad_codes [B,6,...], grad_w [6,C]")
    _check(lib().tok_fsq_decode_backward(_ptr(idx), _ptr(w), _ptr(grad_out), _ptr(grad_codes), _ptr(grad_w),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(), B, C, S,
                                         _stream(idx, stream)), "tok_fsq_decode_backward")
    return grad_codes, grad_w


# ---------------------------------------------------------------------------
# Allocating wrappers.
# ---------------------------------------------------------------------------
def haar_fwd(x: torch.Tensor, stream=None) -> torch.Tensor:
    y = torch.empty(haar_coeff_shape(*x.shape), dtype=x.dtype, device=x.device)
    return tok_haar_fwd(x, y, stream)


def haar_inv(y: torch.Tensor, T: int, H: int, W: int, stream=None) -> torch.Tensor:
    B = y.shape[0]
    C = y.shape[1] // (16 if T == 1 else 64)
    x = torch.empty((B, C, T, H, W), dtype=y.dtype, device=y.device)
    return tok_haar_inv(y, x, stream)


def fsq_encode(u: torch.Tensor, w: torch.Tensor, with_codes: bool = False, stream=None):
    B = u.shape[0]
    idx = torch.empty((B,) + tuple(u.shape[2:]), dtype=torch.int32, device=u.device)
    codes = torch.empty((B, FSQ_DIM) + tuple(u.shape[2:]), dtype=torch.float32, device=u.device) if with_codes else None
    tok_fsq_encode(u, w, idx, codes, stream)
    return (idx, codes) if with_codes else idx


def fsq_decode(idx: torch.Tensor, w: torch.Tensor, bad_count: torch.Tensor = None, stream=None) -> torch.Tensor:
    out = torch.empty((idx.shape[0], w.shape[1]) + tuple(idx.shape[1:]), dtype=torch.float32, device=idx.device)
    return tok_fsq_decode(idx, w, out, bad_count, stream)


def haar_fwd_single(x: torch.Tensor, stream=None) -> torch.Tensor:
    y = torch.empty(single_coeff_shape(*x.shape), dtype=x.dtype, device=x.device)
    return tok_haar_fwd_single(x, y, stream)


def haar_inv_single(y: torch.Tensor, T: int, H: int, W: int, stream=None) -> torch.Tensor:
    x = torch.empty((y.shape[0], y.shape[1] // (4 if T == 1 else 8), T, H, W), dtype=y.dtype, device=y.device)
    return tok_haar_inv_single(y, x, stream)


def haar_fwd_padded(x: torch.Tensor, spatial_multiple: int = 4, temporal_multiple: int = 4,
                    stream=None) -> torch.Tensor:
    y = torch.empty(padded_coeff_shape(*x.shape, spatial_multiple, temporal_multiple), dtype=x.dtype, device=x.device)
    return tok_haar_fwd_padded(x, y, spatial_multiple, temporal_multiple, stream)


def haar_inv_cropped(y: torch.Tensor, T: int, H: int, W: int, spatial_multiple: int = 4, temporal_multiple: int = 4,
                     stream=None) -> torch.Tensor:
    B = y.shape[0]
    C = y.shape[1] // (16 if T == 1 else 64)
    x = torch.empty((B, C, T, H, W), dtype=y.dtype, device=y.device)
    return tok_haar_inv_cropped(y, x, spatial_multiple, temporal_multiple, stream)


def haar_fwd_chunk(x: torch.Tensor, first: bool, stream=None) -> torch.Tensor:
    y = torch.empty(chunk_coeff_shape(*x.shape, first), dtype=x.dtype, device=x.device)
    return tok_haar_fwd_chunk(x, y, first, stream)


def haar_inv_chunk(y: torch.Tensor, T: int, H: int, W: int, first: bool, stream=None) -> torch.Tensor:
    x = torch.empty((y.shape[0], y.shape[1] // 64, T, H, W), dtype=y.dtype, device=y.device)
    return tok_haar_inv_chunk(y, x, first, stream)


def haar_fwd_adjoint(gy: torch.Tensor, T: int, H: int, W: int, stream=None) -> torch.Tensor:
    B = gy.shape[0]
    C = gy.shape[1] // (16 if T == 1 else 64)
    gx = torch.empty((B, C, T, H, W), dtype=gy.dtype, device=gy.device)
    return tok_haar_fwd_adjoint(gy, gx, stream)


def haar_inv_adjoint(gx: torch.Tensor, stream=None) -> torch.Tensor:
    gy = torch.empty(haar_coeff_shape(*gx.shape), dtype=gx.dtype, device=gx.device)
    return tok_haar_inv_adjoint(gx, gy, stream)


def _workspace(B, C, S, device):
    return torch.empty(max(fsq_backward_workspace_size(B, C, S), 1), dtype=torch.uint8, device=device)


def fsq_encode_backward(u: torch.Tensor, w: torch.Tensor, grad_codes: torch.Tensor, stream=None):
    B, C, S = _latent_dims(u)
    grad_u = torch.empty_like(u)
    grad_w = torch.empty_like(w)
    return tok_fsq_encode_backward(u, w, grad_codes, grad_u, grad_w, _workspace(B, C, S, u.device), stream)


def fsq_decode_backward(idx: torch.Tensor, w: torch.Tensor, grad_out: torch.Tensor, stream=None):
    B, C, S = _latent_dims(grad_out)
    grad_codes = torch.empty((B, FSQ_DIM) + tuple(grad_out.shape[2:]), dtype=torch.float32, device=idx.device)
    grad_w = torch.empty_like(w)
    return tok_fsq_decode_backward(idx, w, grad_out, grad_codes, grad_w, _workspace(B, C, S, idx.device), stream)
