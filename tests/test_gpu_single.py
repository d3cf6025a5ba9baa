"""GPU parity of the single-level patcher / unpatcher (patch_size=2).

Tolerances: fp32 1e-5; bf16 one ulp plus the fp32 bound of the block, d * 2^-24 *
sum|block| * scale * 1.01, with d = 5 on video (three butterfly stages, the rounding of the
fp32 constant 1/(2 sqrt 2) and of the product) and scale 2^-1.5, d = 2 and the exact scale
1/2 on images.
"""
import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import U, check_bf16, to_device, to_f64

pytestmark = pytest.mark.gpu


def single_block_sums(x64):
    """sum |x| over the pixels each single-level coefficient reads: [B, C, Tq, h, w]."""
    B, C, T, H, W = x64.shape
    sp = np.abs(x64).reshape(B, C, T, H // 2, 2, W // 2, 2).sum(axis=(4, 6))
    if T == 1:
        return sp
    out = np.empty((B, C, (T + 1) // 2) + sp.shape[3:])
    out[:, :, 0] = 2.0 * sp[:, :, 0]
    out[:, :, 1:] = sp[:, :, 1::2] + sp[:, :, 2::2]
    return out


def single_fp32_bound(sums, video):
    """fp32 error of a single-level output: three butterfly stages and the fp32 constant 1/(2*sqrt 2)
    with its product on video (d = 5, scale 2^-1.5), two stages and the exact 1/2 on images."""
    d, scale = (5, 2 ** -1.5) if video else (2, 0.5)
    return d * U * sums * scale * 1.01


CASES = [
    ((1, 3, 9, 32, 64), synth.BF16, "TMA bf16"),
    ((2, 2, 7, 20, 48), synth.F32, "TMA fp32, partial tiles"),
    ((1, 2, 5, 36, 160), synth.BF16, "TMA bf16, ragged block rows"),
    ((2, 3, 1, 40, 96), synth.BF16, "TMA image"),
    ((1, 2, 1, 18, 24), synth.F32, "TMA image fp32"),
    ((1, 2, 5, 12, 24), synth.BF16, "TMA forward (w = 12: coefficient rows not 16-byte units), row-form inverse"),
    ((1, 2, 9, 10, 22), synth.BF16, "row form bf16, odd w"),
    ((1, 1, 3, 6, 14), synth.F32, "row form fp32, odd w"),
    ((2, 2, 1, 6, 10), synth.BF16, "row form image, odd w"),
    ((1, 1, 5, 8, 1276), synth.BF16, "row form bf16, long odd rows"),
    ((1, 1, 1, 2, 2), synth.F32, "smallest image"),
    ((1, 1, 3, 2, 2), synth.F32, "smallest video"),
]


@pytest.mark.parametrize("shape,dtype,note", CASES, ids=[c[2] for c in CASES])
def test_single_level_matches_oracle(shape, dtype, note):
    B, C, T, H, W = shape
    video = T > 1
    G = 8 if video else 4
    x_np = synth.uniform(shape, seed=sum(shape) + 7, dtype=dtype)
    x64 = synth.to_f64(x_np, dtype)
    y = hwp.haar_fwd_single(to_device(x_np, dtype))
    hwp.tok_check_device()
    ref = oracle.haar_single_fwd(x64)
    got = to_f64(y)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    if dtype == synth.F32:
        assert err.max() <= 1e-5, f"{note}: {err.max():.3g}"
    else:
        check_bf16(got, ref, single_fp32_bound(np.concatenate([single_block_sums(x64)] * G, axis=1), video), note)
    # inverse of the GPU coefficients against the oracle inverse of the same coefficients
    y64 = got
    xr = hwp.haar_inv_single(y, T, H, W)
    hwp.tok_check_device()
    ref_x = oracle.haar_single_inv(y64, T, H, W)
    err = np.abs(to_f64(xr) - ref_x)
    if dtype == synth.F32:
        assert err.max() <= 1e-5
    else:
        s = np.abs(y64).reshape(B, G, C, *y64.shape[2:]).sum(axis=1)          # [B, C, Tq, h, w]
        s = np.repeat(np.repeat(s, 2, axis=3), 2, axis=4)
        if video:
            s = s[:, :, [0] + [1 + (f - 1) // 2 for f in range(1, T)]]
        check_bf16(to_f64(xr), ref_x, single_fp32_bound(s, video), note + " (inverse)")


@pytest.mark.parametrize("shape", [(1, 2, 9, 32, 64), (2, 1, 1, 16, 32)])
def test_two_single_levels_are_the_two_level_call(shape):
    x = torch.rand(shape, device="cuda") * 2 - 1
    y2 = hwp.haar_fwd_single(hwp.haar_fwd_single(x))
    assert torch.allclose(y2, hwp.haar_fwd(x), atol=1e-5, rtol=0)


def test_single_bad_arguments_raise():
    with pytest.raises(hwp.TokError):
        hwp.haar_fwd_single(torch.zeros(1, 1, 4, 8, 8, device="cuda"))   # T even
    with pytest.raises(hwp.TokError):
        hwp.tok_haar_fwd_single(torch.zeros(1, 1, 3, 7, 8, device="cuda"),
                                torch.zeros(1, 8, 2, 3, 4, device="cuda"))  # H odd


@pytest.mark.parametrize("shape,dtype", [((1, 2, 9, 10, 22), torch.bfloat16), ((1, 1, 3, 6, 14), torch.float32),
                                         ((2, 2, 1, 6, 10), torch.bfloat16), ((1, 2, 5, 12, 24), torch.bfloat16)])
def test_single_rows_form_equals_register_kernels(shape, dtype):
    """The row form (16-byte-aligned sources whose rows are not 16-byte units) against the register
    kernels (a view one element past a 16-byte boundary), bit for bit, both directions."""
    from tests.test_gpu_rows import empty_off, off_view
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y = hwp.haar_fwd_single(x)
    y_reg = empty_off(y.shape, dtype)
    hwp.tok_haar_fwd_single(off_view(x), y_reg)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg)
    xr = hwp.haar_inv_single(y, *shape[2:])
    xr_reg = empty_off(shape, dtype)
    hwp.tok_haar_inv_single(off_view(y), xr_reg)
    hwp.tok_check_device()
    assert torch.equal(xr, xr_reg)


@pytest.mark.parametrize("shape", [(0, 3, 9, 16, 16), (1, 2, 5, 0, 8), (2, 1, 1, 8, 0)])
def test_single_empty_is_noop(shape):
    x = torch.empty(shape, device="cuda", dtype=torch.bfloat16)
    y = hwp.haar_fwd_single(x)
    assert y.shape == hwp.single_coeff_shape(*shape)
    xr = hwp.haar_inv_single(y, *shape[2:])
    hwp.tok_check_device()
    assert xr.shape == x.shape
