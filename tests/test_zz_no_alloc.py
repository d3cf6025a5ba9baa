"""The allocation-free encode backward (tok_fsq_encode_backward_noalloc).

It exists for callers that cannot allocate device memory when they need the
gradient (a host framework that owns all device allocations, a service with a
memory budget fixed at start-up, a pipeline without an allocator): its scratch
is a fixed array inside the library instead of a caller-provided workspace.
This file is named so that pytest collects it last.  The test calls the entry
point through the C ABI twice in a row (the second call reuses the scratch the
first one left) and checks each result against tok_fsq_encode_backward, the
workspace form, within the backward tests' tolerance.
"""
import ctypes

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import synth

pytestmark = pytest.mark.gpu

LEVELS = (8, 8, 8, 5, 5, 5)
SCALE = np.array([(L - 1) * 1.001 / 2 / (L // 2) for L in LEVELS])  # largest straight-through slope


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
        stream = torch.cuda.current_stream()
        st = lib.tok_fsq_encode_backward_noalloc(
            ctypes.c_void_p(ud.data_ptr()), ctypes.c_void_p(wd.data_ptr()), ctypes.c_void_p(gd.data_ptr()),
            ctypes.c_void_p(gu.data_ptr()), ctypes.c_void_p(gw.data_ptr()), B, C, S,
            ctypes.c_void_p(stream.cuda_stream))
        assert st == hwp.TOK_OK, lib.tok_status_str(st).decode()
        hwp.tok_check_device()
        gs = np.abs(g.astype(np.float64)) * SCALE[None, :, None]
        tol_u = 1e-5 * np.einsum("ic,bis->bcs", np.abs(w.astype(np.float64)), gs) + 1e-30
        tol_w = 1e-5 * np.einsum("bis,bcs->ic", gs, np.abs(u.astype(np.float64))) + 1e-30
        du = np.abs(gu.double().cpu().numpy() - ref_u.double().cpu().numpy())
        dw = np.abs(gw.double().cpu().numpy() - ref_w.double().cpu().numpy())
        assert (du <= tol_u).all() and (dw <= tol_w).all()


def test_noalloc_rejects_more_tokens_than_its_scratch():
    lib = hwp.lib()
    too_many = 4096 * 2048 + 1
    st = lib.tok_fsq_encode_backward_noalloc(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
                                             ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 16, too_many,
                                             ctypes.c_void_p(0))
    assert st == hwp.TOK_ERR_TOO_LARGE
