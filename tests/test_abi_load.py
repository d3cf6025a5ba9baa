"""libtok.so loads on a machine without a GPU, exports every symbol tok.h declares,
and rejects bad arguments on the host before anything is launched.

No call here reaches a kernel launch: each case fails validation (or is empty)
first, so the tests run on CPU-only machines.
"""
import ctypes
import os
import re

import pytest

import haar_wavelet_patching_b200 as hwp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from haar_wavelet_patching_b200.build import build
    build()
    return hwp.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tok_\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names, "no declarations found in include/*.h"
    assert names == set(hwp.ABI_SYMBOLS)
    for n in names:
        assert hasattr(lib, n), f"libtok.so does not export {n}"


def test_version_and_status_strings(lib):
    assert lib.tok_abi_version() == 1
    for code in range(9):
        assert lib.tok_status_str(code).decode().startswith("TOK_")
    assert lib.tok_last_cuda_error() == 0


F = ctypes.c_void_p
NULL = F(0)
A = F(0x10000)      # stand-in device addresses: never dereferenced on these paths
Bp = F(0x8000000)


def fwd(lib, x, y, dt, B, C, T, H, W):
    return lib.tok_haar_fwd(x, y, dt, B, C, T, H, W, NULL)


def test_selftest_poll_range(lib):
    # out-of-range poll counts are rejected before any launch
    assert lib.tok_selftest_wait_timeout(0, NULL) == hwp.TOK_ERR_SHAPE
    assert lib.tok_selftest_wait_timeout((1 << 22) + 1, NULL) == hwp.TOK_ERR_SHAPE


def test_haar_shape_rules(lib):
    assert fwd(lib, A, Bp, 0, 1, 3, 3, 64, 64) == hwp.TOK_ERR_SHAPE    # T % 4 != 1
    assert fwd(lib, A, Bp, 0, 1, 3, 5, 62, 64) == hwp.TOK_ERR_SHAPE    # H % 4
    assert fwd(lib, A, Bp, 0, 1, 3, 5, 64, 66) == hwp.TOK_ERR_SHAPE    # W % 4
    assert fwd(lib, A, Bp, 0, -1, 3, 5, 64, 64) == hwp.TOK_ERR_SHAPE
    assert fwd(lib, A, Bp, 0, 1, 3, 0, 64, 64) == hwp.TOK_ERR_SHAPE    # T >= 1
    assert fwd(lib, A, Bp, 0, 1 << 40, 1 << 20, 5, 1 << 20, 1 << 20) == hwp.TOK_ERR_SHAPE  # overflow
    assert fwd(lib, A, Bp, 7, 1, 3, 5, 64, 64) == hwp.TOK_ERR_DTYPE


def test_haar_empty_is_ok_without_pointers(lib):
    assert fwd(lib, NULL, NULL, 1, 0, 3, 5, 64, 64) == hwp.TOK_OK
    assert fwd(lib, NULL, NULL, 1, 2, 0, 5, 64, 64) == hwp.TOK_OK
    assert fwd(lib, NULL, NULL, 0, 2, 3, 1, 0, 64) == hwp.TOK_OK
    assert lib.tok_haar_inv(NULL, NULL, 0, 0, 3, 5, 8, 8, NULL) == hwp.TOK_OK


def test_haar_null_alignment_alias(lib):
    assert fwd(lib, NULL, Bp, 1, 1, 3, 5, 64, 64) == hwp.TOK_ERR_NULL
    assert fwd(lib, A, NULL, 1, 1, 3, 5, 64, 64) == hwp.TOK_ERR_NULL
    assert fwd(lib, F(0x10001), Bp, 1, 1, 3, 5, 64, 64) == hwp.TOK_ERR_ALIGN   # bf16 needs 2 bytes
    assert fwd(lib, F(0x10002), Bp, 0, 1, 3, 5, 64, 64) == hwp.TOK_ERR_ALIGN   # fp32 needs 4 bytes
    assert fwd(lib, A, A, 1, 1, 3, 5, 64, 64) == hwp.TOK_ERR_ALIAS
    # x occupies 3*5*64*64*2 = 122880 bytes; y starting inside it overlaps
    assert fwd(lib, A, F(0x10000 + 122880 - 16), 1, 1, 3, 5, 64, 64) == hwp.TOK_ERR_ALIAS
    assert lib.tok_haar_inv(A, F(0x10000 + 64), 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_ALIAS


def test_haar_window_rules(lib):
    fw, iw = lib.tok_haar_fwd_windows, lib.tok_haar_inv_windows
    # clip T = 9 -> 3 latent frames
    assert fw(A, Bp, 1, 1, 3, 9, 64, 64, 2, 1, NULL) == hwp.TOK_ERR_SHAPE     # begin > end
    assert fw(A, Bp, 1, 1, 3, 9, 64, 64, 0, 4, NULL) == hwp.TOK_ERR_SHAPE     # end > T'
    assert fw(A, Bp, 1, 1, 3, 9, 64, 64, -1, 2, NULL) == hwp.TOK_ERR_SHAPE
    assert fw(A, Bp, 1, 1, 3, 9, 64, 64, 0, -1, NULL) == hwp.TOK_ERR_SHAPE    # no open-ended range
    assert fw(NULL, NULL, 1, 1, 3, 9, 64, 64, 2, 2, NULL) == hwp.TOK_OK       # empty range touches nothing
    assert iw(NULL, NULL, 1, 1, 3, 9, 64, 64, 3, 3, NULL) == hwp.TOK_OK
    assert fw(A, Bp, 1, 1, 3, 1, 64, 64, 0, 2, NULL) == hwp.TOK_ERR_SHAPE     # images have one latent frame
    assert iw(A, A, 1, 1, 3, 9, 64, 64, 0, 1, NULL) == hwp.TOK_ERR_ALIAS


def test_backward_argument_rules(lib):
    ws = lib.tok_fsq_backward_workspace_size
    def rows(B, S):  # register path: 2048 tokens per row; TMA path: 8 tiles of 128 tokens of a batch row
        return max((B * S + 2047) // 2048, (B * ((S + 127) // 128) + 7) // 8)
    assert ws(64, 16, 56320) == rows(64, 56320) * 96 * 4 == 3520 * 384
    assert ws(3, 16, 1000) == rows(3, 1000) * 96 * 4 == 3 * 384
    assert ws(1, 5, 4097) == rows(1, 4097) * 30 * 4 == 5 * 120
    assert ws(1, 17, 8) == -1 and ws(1, 0, 8) == -1 and ws(-1, 16, 8) == -1
    assert ws(0, 16, 8) == 0
    eb, db = lib.tok_fsq_encode_backward, lib.tok_fsq_decode_backward
    U, Wt, G, GU, GW, WS = F(0x100000), F(0x200000), F(0x300000), F(0x400000), F(0x500000), F(0x600000)
    need = ws(1, 16, 128)
    assert eb(U, Wt, G, GU, GW, WS, need - 4, 1, 16, 128, NULL) == hwp.TOK_ERR_SHAPE    # workspace too small
    assert eb(U, Wt, G, GU, GW, WS, need, 1, 17, 128, NULL) == hwp.TOK_ERR_SHAPE        # C > 16
    assert eb(U, Wt, G, NULL, GW, WS, need, 1, 16, 128, NULL) == hwp.TOK_ERR_NULL
    assert eb(U, Wt, G, F(0x100000 + 64), GW, WS, need, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIAS  # grad_u in u
    assert eb(U, Wt, G, GU, GW, F(0x400000 + 8), need, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIAS   # workspace in grad_u
    assert eb(U, Wt, G, GU, GW, F(0x600000 + 2), need, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIGN
    assert db(U, Wt, G, GU, GW, F(0x600000 + 2), need, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIGN
    assert db(U, Wt, G, GU, GW, WS, need - 4, 1, 16, 128, NULL) == hwp.TOK_ERR_SHAPE
    assert db(U, Wt, G, F(0x300000 + 4), GW, WS, need, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIAS
    nb = lib.tok_fsq_encode_backward_noalloc
    assert nb(U, Wt, G, GU, GW, 1, 16, 4096 * 2048 + 1, NULL) == hwp.TOK_ERR_TOO_LARGE     # beyond the fixed scratch
    assert nb(U, Wt, G, GU, GW, 2, 16, 4096 * 1024 + 1, NULL) == hwp.TOK_ERR_TOO_LARGE
    assert nb(U, Wt, G, GU, GW, 1, 17, 128, NULL) == hwp.TOK_ERR_SHAPE
    assert nb(U, Wt, G, NULL, GW, 1, 16, 128, NULL) == hwp.TOK_ERR_NULL
    assert nb(U, Wt, G, F(0x100000 + 64), GW, 1, 16, 128, NULL) == hwp.TOK_ERR_ALIAS


def test_fsq_argument_rules(lib):
    enc, dec = lib.tok_fsq_encode, lib.tok_fsq_decode
    assert enc(A, Bp, F(0x20000000), NULL, 1, 0, 16, NULL) == hwp.TOK_ERR_SHAPE       # C >= 1
    assert enc(A, Bp, F(0x20000000), NULL, 1, 5000, 16, NULL) == hwp.TOK_ERR_SHAPE    # C <= 1024
    assert enc(A, Bp, F(0x20000000), NULL, -1, 16, 16, NULL) == hwp.TOK_ERR_SHAPE
    assert enc(NULL, NULL, NULL, NULL, 0, 16, 16, NULL) == hwp.TOK_OK                   # empty
    assert enc(NULL, Bp, F(0x20000000), NULL, 1, 16, 16, NULL) == hwp.TOK_ERR_NULL
    assert enc(A, Bp, F(0x20000002), NULL, 1, 16, 16, NULL) == hwp.TOK_ERR_ALIGN
    assert enc(A, Bp, F(0x10000 + 64), NULL, 1, 16, 16, NULL) == hwp.TOK_ERR_ALIAS     # idx inside u
    assert enc(A, Bp, F(0x20000000), F(0x20000000 + 16), 1, 16, 16, NULL) == hwp.TOK_ERR_ALIAS  # codes/idx
    assert dec(A, Bp, NULL, NULL, 1, 16, 16, NULL) == hwp.TOK_ERR_NULL
    assert dec(A, Bp, F(0x10000), NULL, 1, 16, 16, NULL) == hwp.TOK_ERR_ALIAS
    assert dec(A, Bp, F(0x20000000), F(0x20000000 + 8), 1, 16, 16, NULL) == hwp.TOK_ERR_ALIAS  # counter in out
    assert dec(NULL, NULL, NULL, NULL, 3, 16, 0, NULL) == hwp.TOK_OK


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 5, 8, 8)
    with pytest.raises(ValueError, match="CUDA"):
        hwp.tok_haar_fwd(x, torch.zeros(1, 64, 2, 2, 2))


def test_host_shape_logic():
    assert hwp.haar_coeff_shape(1, 3, 121, 704, 1280) == (1, 192, 31, 176, 320)
    assert hwp.haar_coeff_shape(16, 3, 1, 1024, 1024) == (16, 48, 1, 256, 256)
    with pytest.raises(ValueError):
        hwp.latent_frames(7)


def test_padded_and_chunk_rules(lib):
    T, H, W = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    ext = lib.tok_haar_padded_extents
    assert ext(10, 5, 6, 4, 4, ctypes.byref(T), ctypes.byref(H), ctypes.byref(W)) == hwp.TOK_OK
    assert (T.value, H.value, W.value) == (13, 8, 8)
    assert ext(10, 5, 6, 16, 8, ctypes.byref(T), ctypes.byref(H), ctypes.byref(W)) == hwp.TOK_OK
    assert (T.value, H.value, W.value) == (17, 16, 16)
    assert ext(1, 1080, 1920, 16, 8, ctypes.byref(T), ctypes.byref(H), ctypes.byref(W)) == hwp.TOK_OK
    assert (T.value, H.value, W.value) == (1, 1088, 1920)
    for bad in [(10, 5, 6, 6, 4), (10, 5, 6, 4, 0), (10, 5, 6, 0, 4), (0, 5, 6, 4, 4), (10, -1, 6, 4, 4)]:
        assert ext(*bad, ctypes.byref(T), ctypes.byref(H), ctypes.byref(W)) == hwp.TOK_ERR_SHAPE
    assert ext(10, 5, 6, 4, 4, None, ctypes.byref(H), ctypes.byref(W)) == hwp.TOK_ERR_NULL
    fp, ic = lib.tok_haar_fwd_padded, lib.tok_haar_inv_cropped
    assert fp(A, Bp, 1, 1, 3, 10, 5, 6, 6, 4, NULL) == hwp.TOK_ERR_SHAPE      # spatial multiple 6
    assert fp(A, Bp, 7, 1, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_ERR_DTYPE
    assert fp(NULL, Bp, 1, 1, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_ERR_NULL
    assert fp(F(0x10001), Bp, 1, 1, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_ERR_ALIGN
    assert fp(A, A, 1, 1, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_ERR_ALIAS
    assert ic(A, A, 1, 1, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_ERR_ALIAS
    assert fp(NULL, NULL, 1, 0, 3, 10, 5, 6, 4, 4, NULL) == hwp.TOK_OK        # empty: nothing to do
    fc, iv = lib.tok_haar_fwd_chunk, lib.tok_haar_inv_chunk
    assert fc(A, Bp, 1, 1, 3, 8, 64, 64, 1, NULL) == hwp.TOK_ERR_SHAPE        # first chunk: 1 + 4k frames
    assert fc(A, Bp, 1, 1, 3, 6, 64, 64, 0, NULL) == hwp.TOK_ERR_SHAPE        # continuation: 4k frames
    assert fc(A, Bp, 1, 1, 3, 0, 64, 64, 0, NULL) == hwp.TOK_ERR_SHAPE
    assert fc(A, Bp, 1, 1, 3, 8, 62, 64, 0, NULL) == hwp.TOK_ERR_SHAPE       # H % 4
    assert fc(NULL, Bp, 1, 1, 3, 8, 64, 64, 0, NULL) == hwp.TOK_ERR_NULL
    assert iv(A, A, 1, 1, 3, 8, 64, 64, 0, NULL) == hwp.TOK_ERR_ALIAS


def test_single_level_rules(lib):
    fs, iv = lib.tok_haar_fwd_single, lib.tok_haar_inv_single
    assert fs(A, Bp, 1, 1, 3, 4, 64, 64, NULL) == hwp.TOK_ERR_SHAPE    # T even
    assert fs(A, Bp, 1, 1, 3, 5, 63, 64, NULL) == hwp.TOK_ERR_SHAPE    # H odd
    assert fs(A, Bp, 7, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_DTYPE
    assert fs(NULL, Bp, 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_NULL
    assert fs(A, A, 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_ALIAS
    assert iv(A, A, 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_ALIAS
    assert fs(NULL, NULL, 1, 0, 3, 5, 64, 64, NULL) == hwp.TOK_OK      # empty


def test_channels_last_rules(lib):
    f = lib.tok_haar_fwd_channels_last
    assert f(A, Bp, 1, 1, 3, 8, 64, 64, NULL) == hwp.TOK_ERR_SHAPE     # T % 4 != 1
    assert f(A, Bp, 1, 1, 3, 5, 62, 64, NULL) == hwp.TOK_ERR_SHAPE     # H % 4
    assert f(A, Bp, 9, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_DTYPE
    assert f(NULL, Bp, 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_NULL
    assert f(A, A, 1, 1, 3, 5, 64, 64, NULL) == hwp.TOK_ERR_ALIAS
    assert f(NULL, NULL, 1, 1, 0, 5, 64, 64, NULL) == hwp.TOK_OK         # empty


def test_conv_rules(lib):
    sp, tp, fz = lib.tok_conv_spatial, lib.tok_conv_temporal_causal, lib.tok_conv_factorized
    X, Wg, Y, M = F(0x100000), F(0x200000), F(0x300000), F(0x400000)
    assert sp(X, Wg, Y, 1, 2, 8, 8, 32, 64, 3, NULL) == hwp.TOK_ERR_SHAPE    # Cin not a multiple of 64
    assert sp(X, Wg, Y, 1, 2, 8, 8, 64, 48, 3, NULL) == hwp.TOK_ERR_SHAPE    # Cout not a multiple of 32
    assert tp(X, Wg, Y, 1, 2, 8, 8, 64, 288, 3, NULL) == hwp.TOK_ERR_SHAPE   # above 256, not a multiple of 256
    assert sp(X, Wg, Y, 1, 2, 8, 8, 64, 64, 2, NULL) == hwp.TOK_ERR_SHAPE    # even spatial k
    assert tp(X, Wg, Y, 1, 2, 8, 8, 64, 64, 0, NULL) == hwp.TOK_ERR_SHAPE
    assert fz(X, Wg, Wg, M, Y, 1, 2, 8, 8, 64, 96, 64, 3, NULL) == hwp.TOK_ERR_SHAPE  # Cmid feeds a Cin
    assert sp(NULL, Wg, Y, 1, 2, 8, 8, 64, 64, 3, NULL) == hwp.TOK_ERR_NULL
    assert sp(F(0x100008), Wg, Y, 1, 2, 8, 8, 64, 64, 3, NULL) == hwp.TOK_ERR_ALIGN
    assert sp(X, Wg, X, 1, 2, 8, 8, 64, 64, 3, NULL) == hwp.TOK_ERR_ALIAS
    assert fz(X, Wg, Wg, M, X, 1, 2, 8, 8, 64, 64, 64, 3, NULL) == hwp.TOK_ERR_ALIAS
    assert sp(NULL, NULL, NULL, 0, 2, 8, 8, 64, 64, 3, NULL) == hwp.TOK_OK     # empty


def test_patch_embed_rules(lib):
    pe, pk = lib.tok_patch_embed_spatial, lib.tok_patch_embed_pack_weights
    X, Wp, Y = F(0x100000), F(0x800000), F(0x1000000)
    assert pe(X, Wp, Y, 1, 3, 7, 64, 64, 256, NULL) == hwp.TOK_ERR_SHAPE    # T % 4 != 1
    assert pe(X, Wp, Y, 1, 3, 1, 64, 64, 256, NULL) == hwp.TOK_ERR_SHAPE    # images: video only
    assert pe(X, Wp, Y, 1, 3, 9, 64, 60, 256, NULL) == hwp.TOK_ERR_SHAPE    # W % 8 != 0
    assert pe(X, Wp, Y, 1, 3, 9, 62, 64, 256, NULL) == hwp.TOK_ERR_SHAPE    # H % 4 != 0
    assert pe(X, Wp, Y, 1, 3, 9, 64, 64, 48, NULL) == hwp.TOK_ERR_SHAPE     # Cmid not a multiple of 32
    assert pe(X, Wp, Y, 1, 3, 9, 64, 64, 288, NULL) == hwp.TOK_ERR_SHAPE    # above 256, not a multiple of 256
    assert pe(X, Wp, Y, 1, 9, 9, 64, 64, 256, NULL) == hwp.TOK_ERR_SHAPE    # C > 8
    assert pe(NULL, Wp, Y, 1, 3, 9, 64, 64, 256, NULL) == hwp.TOK_ERR_NULL
    assert pe(F(0x100008), Wp, Y, 1, 3, 9, 64, 64, 256, NULL) == hwp.TOK_ERR_ALIGN
    assert pe(X, Wp, X, 1, 3, 9, 64, 64, 256, NULL) == hwp.TOK_ERR_ALIAS
    assert pe(NULL, NULL, NULL, 0, 3, 9, 64, 64, 256, NULL) == hwp.TOK_OK      # empty
    assert pk(X, Wp, 3, 48, NULL) == hwp.TOK_ERR_SHAPE
    assert pk(NULL, Wp, 3, 256, NULL) == hwp.TOK_ERR_NULL
    assert pk(X, F(0x800008), 3, 256, NULL) == hwp.TOK_ERR_ALIGN
    assert pk(X, X, 3, 256, NULL) == hwp.TOK_ERR_ALIAS


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every call raises: there is no CPU fallback to land on."""
    import torch
    monkeypatch.setattr(hwp, "LIB_PATH", str(tmp_path / "libtok.so"))
    monkeypatch.setattr(hwp, "_lib", None)
    with pytest.raises(ImportError, match="no CPU fallback"):
        hwp.lib()
    with pytest.raises((ImportError, ValueError)):
        hwp.tok_fsq_encode(torch.zeros(1, 16, 4), torch.zeros(6, 16), torch.zeros(1, 4, dtype=torch.int32))
