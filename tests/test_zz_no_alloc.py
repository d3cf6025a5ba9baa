"""The allocation-free encode backward (tok_fsq_encode_backward_noalloc).

It exists for callers that cannot allocate device memory when they need the
gradient (a host framework that owns all device allocations, a service with a
memory budget fixed at start-up, a pipeline without an allocator): its scratch
is a fixed array inside the library instead of a caller-provided workspace.
This file is named so that pytest collects it last.  The tests call the entry
point through the C ABI: twice in a row (the second call reuses the scratch the
first one left), each result bit for bit equal to tok_fsq_encode_backward (the
workspace form runs the same kernels in the same order); once at exactly the
8,388,608-token limit, which writes and reads every row of the array, against
the workspace form and the oracle; and once 128 tokens past it, which must be
refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth

pytestmark = pytest.mark.gpu

LEVELS = (8, 8, 8, 5, 5, 5)
SCALE = np.array([(L - 1) * 1.001 / 2 / (L // 2) for L in LEVELS])  # largest straight-through slope
MAX_TOKENS = 8192 * 1024  # the array's 8192 rows of 1024 tokens at C = 16


def call_noalloc(lib, ud, wd, gd, gu, gw, B, C, S):
    stream = torch.cuda.current_stream()
    return lib.tok_fsq_encode_backward_noalloc(
        ctypes.c_void_p(ud.data_ptr()), ctypes.c_void_p(wd.data_ptr()), ctypes.c_void_p(gd.data_ptr()),
        ctypes.c_void_p(gu.data_ptr()), ctypes.c_void_p(gw.data_ptr()), B, C, S,
        ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_matches_workspace_form_on_two_calls_in_a_row():
    lib = hwp.lib()
    B, C, S = 4, 16, 56320
    for seed in (61, 67):
        u = synth.normal((B, C, S), seed=seed, std=1.2)
        w = synth.fsq_weight(C, seed=seed)
        g = synth.normal((B, 6, S), seed=seed + 1)
        ud, wd, gd = (torch.from_numpy(a).cuda() for a in (u, w, g))
        ref_u, ref_w = hwp.fsq_encode_backward(ud, wd, gd)
        gu = torch.full_like(ud, float("nan"))
        gw = torch.full_like(wd, float("nan"))
        st = call_noalloc(lib, ud, wd, gd, gu, gw, B, C, S)
        assert st == hwp.TOK_OK, lib.tok_status_str(st).decode()
        hwp.tok_check_device()
        assert torch.equal(gu, ref_u) and torch.equal(gw, ref_w)


def test_noalloc_at_its_token_limit():
    """B = 1, C = 16, S = 8,388,608 (u is 537 MB): every row of the fixed array is used."""
    lib = hwp.lib()
    B, C, S = 1, 16, MAX_TOKENS
    u = synth.normal((B, C, S), seed=71, std=1.2)
    w = synth.fsq_weight(C, seed=71)
    g = synth.normal((B, 6, S), seed=72)
    ud, wd, gd = (torch.from_numpy(a).cuda() for a in (u, w, g))
    gu = torch.full_like(ud, float("nan"))
    gw = torch.full_like(wd, float("nan"))
    st = call_noalloc(lib, ud, wd, gd, gu, gw, B, C, S)
    assert st == hwp.TOK_OK, lib.tok_status_str(st).decode()
    hwp.tok_check_device()
    ref_u, ref_w = hwp.fsq_encode_backward(ud, wd, gd)
    assert torch.equal(gu, ref_u) and torch.equal(gw, ref_w)
    o_u, o_w = oracle.fsq_encode_backward(u, w, g)
    gs = np.abs(g.astype(np.float64)) * SCALE[None, :, None]
    tol_u = 1e-5 * np.einsum("ic,bis->bcs", np.abs(w.astype(np.float64)), gs) + 1e-30
    tol_w = 1e-5 * np.einsum("bis,bcs->ic", gs, np.abs(u.astype(np.float64))) + 1e-30
    assert (np.abs(gu.double().cpu().numpy() - o_u) <= tol_u).all()
    assert (np.abs(gw.double().cpu().numpy() - o_w) <= tol_w).all()


def test_noalloc_refuses_128_tokens_past_its_limit():
    """Refused before any launch.  Null pointers: if the size check ever stopped refusing, the
    call would stop at TOK_ERR_NULL and still launch nothing."""
    lib = hwp.lib()
    null = ctypes.c_void_p(None)
    st = lib.tok_fsq_encode_backward_noalloc(null, null, null, null, null, 1, 16, MAX_TOKENS + 128, null)
    assert st == hwp.TOK_ERR_TOO_LARGE
