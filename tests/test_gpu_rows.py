"""GPU parity of the row form of the TMA Haar kernels.

The row form takes the planar calls whose rows are not whole 16-byte units (bf16 W % 8 != 0
or w % 8 != 0, fp32 W % 4 != 0 or w % 4 != 0, odd w) on 16-byte-aligned sources: each source
row of a tile is staged by a bulk copy from the 16-byte boundary at or below it and read
back realigned; stores take the widest width the destination address allows.  An inverse
whose source rows are whole 16-byte units but whose pixel rows are not keeps the box loads
and takes only the run-time store widths.

Checked here: the oracle, element by element (same tolerances as the other Haar parity
tests), and bit-for-bit agreement with the register kernels, which a view one element past
a 16-byte boundary forces (both paths round the same fp32 operations in the same order).
"""
import zlib

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import to_device, to_f64
from tests.test_gpu_haar import TOL_F32, check_fwd, check_inv

pytestmark = pytest.mark.gpu

# (shape, dtype, note); the forms each direction takes are in the note.
CASES = [
    ((1, 2, 9, 16, 44), synth.BF16, "bf16 video, rows both ways, odd w"),
    ((1, 2, 9, 16, 80), synth.BF16, "bf16 video, boxes forward, rows inverse (w = 20)"),
    ((2, 3, 13, 24, 52), synth.F32, "fp32 video, rows both ways, odd w"),
    ((1, 1, 5, 8, 1300), synth.BF16, "bf16 video, six tiles per row, odd w"),
    ((1, 2, 17, 12, 296), synth.F32, "fp32 video, boxes forward, rows inverse (w = 74)"),
    ((2, 3, 1, 36, 40), synth.BF16, "bf16 image, boxes forward, rows inverse"),
    ((1, 2, 1, 20, 52), synth.F32, "fp32 image, rows both ways, odd w"),
    ((3, 1, 1, 12, 1036), synth.BF16, "bf16 image, odd w, three block rows"),
]

def off_view(t: torch.Tensor, k: int = 1) -> torch.Tensor:
    """A contiguous copy of t that starts k elements past a 16-byte boundary."""
    buf = torch.empty(t.numel() + k, dtype=t.dtype, device=t.device)
    v = buf[k:].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 16 != 0
    return v


def empty_off(shape, dtype, k: int = 1) -> torch.Tensor:
    n = int(np.prod(shape))
    return torch.empty(n + k, dtype=dtype, device="cuda")[k:].view(shape)


@pytest.mark.parametrize("shape,dtype,note", CASES, ids=[c[2] for c in CASES])
def test_rows_form_matches_oracle(shape, dtype, note):
    x = synth.uniform(shape, seed=zlib.crc32(note.encode()), dtype=dtype)
    y, _ = check_fwd(x, dtype, note)
    B, C, T, H, W = shape
    xr = check_inv(y, T, H, W, note)
    if dtype == synth.F32:
        assert np.abs(to_f64(xr) - synth.to_f64(x, dtype)).max() <= 1e-6


@pytest.mark.parametrize("shape,dtype,note", CASES, ids=[c[2] for c in CASES])
def test_rows_form_equals_register_kernels(shape, dtype, note):
    B, C, T, H, W = shape
    x = to_device(synth.uniform(shape, seed=7, dtype=dtype), dtype)
    y = hwp.haar_fwd(x)
    y_reg = empty_off(y.shape, y.dtype)
    hwp.tok_haar_fwd(off_view(x), y_reg)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg)
    xr = hwp.haar_inv(y, T, H, W)
    xr_reg = empty_off(x.shape, x.dtype)
    hwp.tok_haar_inv(off_view(y), xr_reg)
    hwp.tok_check_device()
    assert torch.equal(xr, xr_reg)


@pytest.mark.parametrize("shape,dtype", [((1, 2, 9, 16, 64), torch.bfloat16), ((1, 2, 9, 16, 44), torch.bfloat16),
                                         ((2, 1, 5, 8, 48), torch.float32), ((1, 3, 1, 8, 64), torch.float32)])
def test_misaligned_destination_only(shape, dtype):
    """An aligned source with a destination one element off a 16-byte boundary takes the row form
    (run-time store widths, down to single elements) and gives the aligned call's bits."""
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y = hwp.haar_fwd(x)
    yo = empty_off(y.shape, dtype)
    hwp.tok_haar_fwd(x, yo)
    hwp.tok_check_device()
    assert torch.equal(yo, y)
    xo = empty_off(shape, dtype)
    hwp.tok_haar_inv(y, xo)
    hwp.tok_check_device()
    assert torch.equal(xo, hwp.haar_inv(y, *shape[2:]))
    if shape[2] > 1:
        # The adjoints the same way (the patcher's adjoint writes pixels like the inverse).
        ao = empty_off(shape, dtype)
        hwp.tok_haar_fwd_adjoint(y, ao)
        bo = empty_off(y.shape, dtype)
        hwp.tok_haar_inv_adjoint(x, bo)
        hwp.tok_check_device()
        assert torch.equal(ao, hwp.haar_fwd_adjoint(y, *shape[2:]))
        assert torch.equal(bo, hwp.haar_inv_adjoint(x))


@pytest.mark.parametrize("shape,dtype", [((1, 2, 9, 16, 44), torch.bfloat16), ((2, 1, 13, 8, 52), torch.float32)])
def test_rows_form_adjoints(shape, dtype):
    """The adjoints in the row form: against the oracle and bit for bit against the register kernels."""
    B, C, T, H, W = shape
    rng = np.random.default_rng(sum(shape))
    gy = torch.from_numpy(rng.uniform(-1, 1, oracle.haar_out_shape(B, C, T, H, W))).cuda().to(dtype)
    gx = torch.from_numpy(rng.uniform(-1, 1, shape)).cuda().to(dtype)
    ax = hwp.haar_fwd_adjoint(gy, T, H, W)
    ay = hwp.haar_inv_adjoint(gx)
    ax_reg, ay_reg = empty_off(shape, dtype), empty_off(gy.shape, dtype)
    hwp.tok_haar_fwd_adjoint(off_view(gy), ax_reg)
    hwp.tok_haar_inv_adjoint(off_view(gx), ay_reg)
    hwp.tok_check_device()
    assert torch.equal(ax, ax_reg) and torch.equal(ay, ay_reg)
    if dtype == torch.float32:
        ref_x = oracle.haar_fwd_adjoint(gy.double().cpu().numpy(), T, H, W)
        ref_y = oracle.haar_inv_adjoint(gx.double().cpu().numpy())
        assert np.abs(ax.double().cpu().numpy() - ref_x).max() <= TOL_F32
        assert np.abs(ay.double().cpu().numpy() - ref_y).max() <= TOL_F32


@pytest.mark.parametrize("shape,dtype,ms,mt", [((1, 2, 7, 21, 45), torch.bfloat16, 4, 4),
                                               ((1, 2, 11, 13, 30), torch.float32, 8, 8),
                                               ((2, 3, 1, 30, 50), torch.bfloat16, 4, 4),
                                               ((1, 1, 6, 9, 1277), torch.bfloat16, 16, 8),
                                               ((1, 2, 9, 12, 54), torch.bfloat16, 32, 4)])
def test_rows_form_padded_and_cropped_equal_register_kernels(shape, dtype, ms, mt):
    """Padding (zeros past the clip's rows and columns, mirrored frames) and cropping in the row form;
    where the padded coefficient rows are whole 16-byte units (w = 8, 16, 320 here) the cropped
    inverse loads boxes and stores its odd-width pixel rows at run-time widths."""
    B, C, T, H, W = shape
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y = hwp.haar_fwd_padded(x, ms, mt)
    y_reg = empty_off(y.shape, dtype)
    hwp.tok_haar_fwd_padded(off_view(x), y_reg, ms, mt)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg)
    xr = hwp.haar_inv_cropped(y, T, H, W, ms, mt)
    xr_reg = empty_off(shape, dtype)
    hwp.tok_haar_inv_cropped(off_view(y), xr_reg, ms, mt)
    hwp.tok_check_device()
    assert torch.equal(xr, xr_reg)


def test_rows_form_padded_matches_oracle_long_odd_row():
    """A 1277-pixel row (odd: every staged row at a different 2-byte offset) against the oracle."""
    shape, ms, mt = (1, 1, 6, 9, 1277), 16, 8
    x_np = synth.uniform(shape, seed=1277, dtype=synth.F32)
    y = hwp.haar_fwd_padded(to_device(x_np, synth.F32), ms, mt)
    hwp.tok_check_device()
    ref = oracle.haar_fwd_padded(synth.to_f64(x_np, synth.F32), ms, mt)
    assert np.abs(to_f64(y) - ref).max() <= TOL_F32
    xr = hwp.haar_inv_cropped(y, *shape[2:], ms, mt)
    ref_x = oracle.haar_inv_cropped(to_f64(y), *shape[2:], ms, mt)
    assert np.abs(to_f64(xr) - ref_x).max() <= TOL_F32


@pytest.mark.parametrize("shape,dtype,first", [((1, 2, 13, 8, 20), torch.float32, True),
                                               ((1, 2, 8, 12, 44), torch.bfloat16, False)])
def test_rows_form_chunks_equal_register_kernels(shape, dtype, first):
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y = hwp.haar_fwd_chunk(x, first)
    y_reg = empty_off(y.shape, dtype)
    hwp.tok_haar_fwd_chunk(off_view(x), y_reg, first)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg)
    xr = hwp.haar_inv_chunk(y, *shape[2:], first)
    xr_reg = empty_off(xr.shape, dtype)
    hwp.tok_haar_inv_chunk(off_view(y), xr_reg, first)
    hwp.tok_check_device()
    assert torch.equal(xr, xr_reg)
