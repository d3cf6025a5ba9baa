"""GPU parity of the channels-last patcher: the same coefficients as tok_haar_fwd, laid out
[B, T', h, w, 64C].  The kernels run the same butterflies as the planar ones, so the result
equals the planar call's output permuted, bit for bit; one case is also checked against
the oracle with the planar tolerances."""
import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import block_abs_sums, check_bf16, expand_to_channels, haar_fp32_bound, to_device, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    ((1, 3, 9, 32, 64), torch.bfloat16, "TMA, C = 3"),
    ((2, 1, 5, 16, 96), torch.bfloat16, "TMA, C = 1, partial tile"),
    ((1, 2, 13, 20, 64), torch.float32, "TMA fp32, C = 2"),
    ((1, 4, 5, 8, 32), torch.bfloat16, "TMA, C = 4"),
    ((2, 3, 1, 36, 64), torch.bfloat16, "TMA image, partial block rows"),
    ((1, 3, 9, 16, 72), torch.bfloat16, "TMA, w = 18 (coefficient rows not whole 16-byte units)"),
    ((1, 2, 5, 8, 40), torch.float32, "TMA fp32, w = 10"),
    ((1, 3, 9, 12, 44), torch.float32, "TMA fp32, odd w = 11"),
    ((1, 1, 1, 20, 28), torch.float32, "TMA fp32 image, odd w = 7"),
    ((1, 3, 9, 16, 76), torch.bfloat16, "pair rows, w = 19"),
    ((2, 1, 5, 8, 1292), torch.bfloat16, "pair rows, w = 323 (six tiles, odd last)"),
    ((1, 4, 13, 12, 300), torch.bfloat16, "pair rows, C = 4, w = 75"),
    ((1, 1, 5, 4, 4), torch.bfloat16, "pair rows, w = 1"),
    ((1, 3, 5, 8, 260), torch.bfloat16, "pair rows, w = 65 (a one-block last tile)"),
    ((2, 2, 9, 8, 516), torch.bfloat16, "pair rows, B = 2, w = 129"),
    ((1, 2, 1, 8, 20), torch.bfloat16, "row form image, w = 5"),
    ((2, 3, 1, 36, 52), torch.bfloat16, "row form image, partial block rows, w = 13"),
    ((1, 5, 9, 16, 64), torch.bfloat16, "register, C = 5"),
    ((1, 5, 5, 8, 44), torch.bfloat16, "register, C = 5, odd w"),
]


@pytest.mark.parametrize("shape,dtype,note", CASES, ids=[c[2] for c in CASES])
def test_channels_last_is_the_planar_result_permuted(shape, dtype, note):
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y_cl = hwp.haar_fwd_channels_last(x)
    hwp.tok_check_device()
    assert torch.equal(y_cl, hwp.haar_fwd(x).permute(0, 2, 3, 4, 1))


@pytest.mark.parametrize("shape", [(1, 3, 9, 32, 64), (1, 2, 9, 16, 76)], ids=["box form", "pair rows, odd w"])
def test_channels_last_matches_oracle(shape):
    x_np = synth.uniform(shape, seed=17, dtype=synth.BF16)
    x64 = synth.to_f64(x_np, synth.BF16)
    got = to_f64(hwp.haar_fwd_channels_last(to_device(x_np, synth.BF16)))
    ref = oracle.haar_fwd_channels_last(x64)
    E = np.moveaxis(haar_fp32_bound(expand_to_channels(block_abs_sums(x64), 64), True), 1, -1)
    assert got.shape == ref.shape
    check_bf16(got, ref, E, "channels-last")


@pytest.mark.parametrize("shape,dtype", [((1, 3, 9, 16, 76), torch.bfloat16), ((2, 2, 1, 12, 36), torch.bfloat16),
                                         ((1, 3, 5, 8, 44), torch.float32)])
def test_channels_last_tile_kernels_equal_register_kernel(shape, dtype):
    """A source one element past a 16-byte boundary takes the register kernel: same bits."""
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    buf = torch.empty(x.numel() + 1, dtype=dtype, device="cuda")
    xo = buf[1:].view(shape)
    xo.copy_(x)
    assert xo.data_ptr() % 16 != 0
    assert torch.equal(hwp.haar_fwd_channels_last(x), hwp.haar_fwd_channels_last(xo))
    hwp.tok_check_device()


def test_channels_last_bad_arguments_raise():
    with pytest.raises(ValueError):
        hwp.tok_haar_fwd_channels_last(torch.zeros(1, 3, 9, 32, 64, device="cuda"),
                                       torch.zeros(1, 192, 3, 8, 16, device="cuda"))
    with pytest.raises((ValueError, hwp.TokError)):  # T % 4 != 1: the shape helper or the library refuses
        hwp.haar_fwd_channels_last(torch.zeros(1, 3, 8, 32, 64, device="cuda"))


@pytest.mark.parametrize("shape", [(0, 3, 9, 32, 64), (1, 2, 5, 0, 76), (2, 1, 1, 8, 0)])
def test_channels_last_empty_is_noop(shape):
    y = hwp.haar_fwd_channels_last(torch.empty(shape, device="cuda", dtype=torch.bfloat16))
    hwp.tok_check_device()
    assert y.shape == hwp.channels_last_shape(*shape) and y.numel() == 0
