"""GPU parity of the padded patcher, the cropped unpatcher and the streaming chunks.

Against the oracle's padded / chunk forms (pinned in test_oracle_padding.py), with the
tolerances of the plain transform (fp32 1e-5; bf16 one ulp, or the fp32 butterfly bound of
the block, computed over the padded clip, in the cancellation regime); and bit for bit against the plain
transform where the two must agree: chunks of a video concatenate to the whole-video
call, and a clip that needs no padding gives the plain call's output.
"""
import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import (block_abs_sums, check_bf16, expand_blocks_to_pixels, expand_to_channels, haar_fp32_bound,
                           inv_block_abs_sums, to_device, to_f64)

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5


def assert_close(got, ref, dtype, bound_sums, video, label):
    err = np.abs(got - ref)
    if dtype == synth.F32:
        assert err.max() <= TOL_F32, f"{label}: max |err| {err.max():.3g}"
    else:
        check_bf16(got, ref, haar_fp32_bound(bound_sums, video), label)


PADDED = [
    # (shape, dtype, spatial multiple, temporal multiple, note)
    ((1, 2, 10, 36, 64), synth.BF16, 4, 4, "TMA bf16, 3 mirrored frames"),
    ((2, 1, 6, 30, 256), synth.BF16, 16, 8, "TMA bf16, zero rows, mirrored frames"),
    ((1, 2, 7, 20, 32), synth.F32, 8, 4, "TMA fp32, zero rows"),
    ((1, 1, 2, 8, 64), synth.BF16, 4, 8, "TMA bf16, mirror longer than the clip"),
    ((1, 2, 7, 21, 45), synth.BF16, 4, 4, "row form bf16, ragged rows and columns"),
    ((1, 2, 11, 13, 30), synth.F32, 8, 8, "row form fp32"),
    ((2, 3, 1, 30, 50), synth.BF16, 4, 4, "image, row form"),
    ((1, 2, 1, 24, 64), synth.F32, 16, 4, "image, TMA, zero rows"),
    ((1, 2, 5, 15, 88), synth.BF16, 4, 4, "TMA bf16, sector-shifted tiles (w = 22), zero rows"),
]


@pytest.mark.parametrize("shape,dtype,ms,mt,note", PADDED, ids=[p[4] for p in PADDED])
def test_padded_forward_and_cropped_inverse_match_oracle(shape, dtype, ms, mt, note):
    B, C, T, H, W = shape
    x_np = synth.uniform(shape, seed=sum(shape), dtype=dtype)
    x64 = synth.to_f64(x_np, dtype)
    video = T > 1
    G = 64 if video else 16
    y = hwp.haar_fwd_padded(to_device(x_np, dtype), ms, mt)
    hwp.tok_check_device()
    ref = oracle.haar_fwd_padded(x64, ms, mt)
    assert tuple(y.shape) == ref.shape
    xp64 = oracle.haar_pad(x64, ms, mt)
    assert_close(to_f64(y), ref, dtype, expand_to_channels(block_abs_sums(xp64), G), video, note + " (fwd)")

    y64 = to_f64(y)
    xr = hwp.haar_inv_cropped(y, T, H, W, ms, mt)
    hwp.tok_check_device()
    ref_x = oracle.haar_inv_cropped(y64, T, H, W, ms, mt)
    Tp = xp64.shape[2]
    sums = expand_blocks_to_pixels(inv_block_abs_sums(y64, C, video), Tp)[:, :, :T, :H, :W]
    assert_close(to_f64(xr), ref_x, dtype, sums, video, note + " (inv)")


@pytest.mark.parametrize("shape,dtype", [((1, 2, 9, 16, 64), synth.BF16), ((2, 1, 1, 8, 32), synth.F32),
                                         ((1, 1, 5, 8, 44), synth.BF16)])
def test_no_padding_needed_is_the_plain_call_bit_for_bit(shape, dtype):
    x = to_device(synth.uniform(shape, seed=3, dtype=dtype), dtype)
    y = hwp.haar_fwd_padded(x)
    assert torch.equal(y, hwp.haar_fwd(x))
    B, C, T, H, W = shape
    assert torch.equal(hwp.haar_inv_cropped(y, T, H, W), hwp.haar_inv(y, T, H, W))


CHUNKS = [
    # (shape of the whole video, dtype, frames per chunk: 1 + 4k first, then multiples of 4)
    ((2, 2, 21, 16, 64), synth.BF16, [1, 8, 4, 8]),      # TMA path; a one-frame first chunk
    ((1, 2, 13, 8, 20), synth.F32, [5, 4, 4]),           # row form (w * 4 bytes not a multiple of 16)
    ((1, 3, 25, 12, 96), synth.BF16, [9, 16]),
]


@pytest.mark.parametrize("shape,dtype,frames", CHUNKS)
def test_chunks_concatenate_to_the_whole_video(shape, dtype, frames):
    B, C, T, H, W = shape
    assert sum(frames) == T
    x = to_device(synth.uniform(shape, seed=T, dtype=dtype), dtype)
    y = hwp.haar_fwd(x)
    parts, start = [], 0
    for k, n in enumerate(frames):
        parts.append(hwp.haar_fwd_chunk(x[:, :, start:start + n].contiguous(), first=(k == 0)))
        start += n
    hwp.tok_check_device()
    assert torch.equal(torch.cat(parts, dim=2), y)
    # and back: each chunk's inverse is its frames of the whole-video inverse
    xr = hwp.haar_inv(y, T, H, W)
    q, start = 0, 0
    for k, n in enumerate(frames):
        nq = (n + 3) // 4 if k == 0 else n // 4
        back = hwp.haar_inv_chunk(y[:, :, q:q + nq].contiguous(), n, H, W, first=(k == 0))
        assert torch.equal(back, xr[:, :, start:start + n])
        q, start = q + nq, start + n
    hwp.tok_check_device()


@pytest.mark.parametrize("shape,dtype", [((2, 2, 8, 16, 64), synth.BF16), ((1, 1, 12, 8, 20), synth.F32)])
def test_continuation_chunk_matches_oracle(shape, dtype):
    x_np = synth.uniform(shape, seed=5, dtype=dtype)
    x64 = synth.to_f64(x_np, dtype)
    y = hwp.haar_fwd_chunk(to_device(x_np, dtype), first=False)
    hwp.tok_check_device()
    ref = oracle.haar_fwd_chunk(x64, first=False)
    B, C, T, H, W = shape
    # a continuation block reads 4 distinct frames: the block sums are those of windows 1..k of a
    # clip that starts one frame earlier
    sums = np.abs(x64).reshape(B, C, T // 4, 4, H // 4, 4, W // 4, 4).sum(axis=(3, 5, 7))
    assert_close(to_f64(y), ref, dtype, expand_to_channels(sums, 64), True, "continuation chunk")
    y64 = to_f64(y)
    xr = hwp.haar_inv_chunk(y, T, H, W, first=False)
    ref_x = oracle.haar_inv_chunk(y64, T, H, W, first=False)
    isums = np.repeat(np.repeat(np.repeat(inv_block_abs_sums(y64, C, True), 4, axis=2), 4, axis=3), 4, axis=4)
    assert_close(to_f64(xr), ref_x, dtype, isums, True, "continuation chunk (inv)")


def test_padded_bad_arguments_raise():
    x = torch.zeros(1, 1, 5, 8, 8, device="cuda")
    with pytest.raises(hwp.TokError):
        hwp.padded_extents(5, 8, 8, 6, 4)
    with pytest.raises(hwp.TokError):
        hwp.haar_fwd_chunk(torch.zeros(1, 1, 6, 8, 8, device="cuda"), first=False)
    with pytest.raises(ValueError):
        hwp.tok_haar_fwd_padded(x, torch.zeros(1, 64, 1, 2, 2, device="cuda"))
