"""GPU parity of the grouped-row form of the bf16 video patcher, and of the padded row form.

A bf16 video whose pixel rows are 8-byte units (W % 8 == 4) and whose coefficient rows have an
odd number w of blocks takes the grouped-row form: two consecutive pixel rows together are a
16-byte multiple, so tensor boxes read rows of 2W elements, and the 8 elements after the box of
the part that starts off a 16-byte boundary come from a tail box.  The tiles of a block row may
start one block left of a pair boundary, so that their coefficient-pair stores are aligned (up
to whole 32-byte sectors); a lane whose pair then straddles column 0 or the last column stores
its one block alone.  Padded calls whose padded w is even keep the row form, whose lanes at the
tensor's edge now also store their one block alone.

Checked here: bit for bit against the register kernels (a source one element past a 16-byte
boundary forces them; both round the same fp32 operations in the same order) across the
shift units the plane sizes allow (16, 8, 4, 2 and none), continuation chunks, padded calls
(zero rows and columns, mirrored frames) and the unpatcher's adjoint; and against the oracle
on a subset.
"""
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import block_abs_sums, check_bf16, expand_to_channels, haar_fp32_bound, to_device, to_f64
from tests.test_gpu_haar import check_fwd
from tests.test_gpu_rows import empty_off, off_view

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16

# (shape, note); plane = T' h w decides the shift unit of the tiles.
PLAIN = [
    ((1, 1, 9, 64, 1300), "plane % 16 == 0 (sector shifts), six tiles per row"),
    ((1, 2, 13, 8, 76), "plane % 16 == 8 (shifts of 8)"),
    ((2, 1, 9, 8, 44), "plane % 4 == 2 (shifts of 2)"),
    ((1, 2, 9, 12, 44), "odd plane (no shift; element stores on odd block rows)"),
    ((1, 1, 5, 16, 1276), "w = 319"),
]

# (shape, spatial multiple, temporal multiple, note): padded calls.
PADDED = [
    ((1, 2, 7, 20, 44), 4, 4, "grouped rows, odd padded w, mirrored frames"),
    ((1, 1, 10, 22, 1276), 4, 8, "grouped rows, zero rows, mirrored frames"),
    ((1, 2, 6, 16, 54), 8, 4, "row form, W % 8 == 6, mirrored frames"),
    ((1, 1, 10, 20, 1286), 16, 8, "row form, long rows, zero rows and columns"),
    ((2, 1, 1, 16, 50), 4, 4, "row form, W % 8 == 2, images"),
    ((1, 2, 7, 20, 44), 16, 4, "row form, even padded w, zero columns"),
]


@pytest.mark.parametrize("shape,note", PLAIN, ids=[p[1] for p in PLAIN])
def test_grouped_form_equals_register_kernels(shape, note):
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(BF16)
    y = hwp.haar_fwd(x)
    y_reg = empty_off(y.shape, BF16)
    hwp.tok_haar_fwd(off_view(x), y_reg)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg), note


@pytest.mark.parametrize("shape,note", [PLAIN[0], PLAIN[3]], ids=[PLAIN[i][1] for i in (0, 3)])
def test_grouped_form_matches_oracle(shape, note):
    x = synth.uniform(shape, seed=sum(shape), dtype=synth.BF16)
    check_fwd(x, synth.BF16, note)


@pytest.mark.parametrize("shape,ms,mt,note", PADDED, ids=[p[3] for p in PADDED])
def test_padded_equals_register_kernels(shape, ms, mt, note):
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(BF16)
    y = hwp.haar_fwd_padded(x, ms, mt)
    y_reg = empty_off(y.shape, BF16)
    hwp.tok_haar_fwd_padded(off_view(x), y_reg, ms, mt)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg), note


@pytest.mark.parametrize("shape,ms,mt,note", [PADDED[0], PADDED[1], PADDED[2]], ids=[PADDED[i][3] for i in (0, 1, 2)])
def test_padded_matches_oracle(shape, ms, mt, note):
    x_np = synth.uniform(shape, seed=sum(shape) + ms, dtype=synth.BF16)
    x64 = synth.to_f64(x_np, synth.BF16)
    y = hwp.haar_fwd_padded(to_device(x_np, synth.BF16), ms, mt)
    hwp.tok_check_device()
    ref = oracle.haar_fwd_padded(x64, ms, mt)
    assert tuple(y.shape) == ref.shape
    video = shape[2] > 1
    sums = expand_to_channels(block_abs_sums(oracle.haar_pad(x64, ms, mt)), 64 if video else 16)
    check_bf16(to_f64(y), ref, haar_fp32_bound(sums, video), note)


def test_grouped_chunk_equals_register_kernels():
    shape = (1, 2, 8, 20, 1276)
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(BF16)
    y = hwp.haar_fwd_chunk(x, False)
    y_reg = empty_off(y.shape, BF16)
    hwp.tok_haar_fwd_chunk(off_view(x), y_reg, False)
    hwp.tok_check_device()
    assert torch.equal(y, y_reg)


def test_grouped_unpatcher_adjoint_equals_register_kernels():
    """The unpatcher's adjoint maps pixels to coefficients with the forward's kernel."""
    shape = (1, 2, 9, 16, 1300)
    gx = (torch.rand(shape, device="cuda") * 2 - 1).to(BF16)
    ay = hwp.haar_inv_adjoint(gx)
    ay_reg = empty_off(ay.shape, BF16)
    hwp.tok_haar_inv_adjoint(off_view(gx), ay_reg)
    hwp.tok_check_device()
    assert torch.equal(ay, ay_reg)
