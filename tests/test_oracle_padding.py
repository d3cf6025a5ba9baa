"""Pins for the oracle's arbitrary-extent and streaming forms of the patcher.

"NVIDIA Cosmos Tokenizer 完全指南", section 6.3: clips of any size are padded (zeros
in space, reflection at the temporal edge) to aligned extents, transformed, and
cropped back; long clips run window by window.  Checked against numpy's own padding
routine, against the unpadded transform (which its own pins fix), and against
identities that hold for any correct implementation: perfect reconstruction, zero
coefficients over all-zero blocks, and the composition of streaming chunks into
the whole-clip transform.
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(11)


@pytest.mark.parametrize("T,H,W,ms,mt", [(2, 4, 4, 4, 4), (3, 5, 7, 4, 4), (6, 8, 9, 8, 8), (10, 3, 4, 4, 16),
                                         (8, 6, 6, 4, 8), (1, 5, 6, 4, 4)])
def test_padding_is_numpy_reflect_in_time_and_zeros_in_space(T, H, W, ms, mt):
    x = RNG.normal(size=(2, 2, T, H, W))
    Tp, Hp, Wp = oracle.padded_extents(T, H, W, ms, mt)
    expect = x
    if Tp > T:
        expect = np.pad(expect, ((0, 0), (0, 0), (0, Tp - T), (0, 0), (0, 0)), mode="reflect")
    expect = np.pad(expect, ((0, 0), (0, 0), (0, 0), (0, Hp - H), (0, Wp - W)), mode="constant")
    assert np.array_equal(oracle.haar_pad(x, ms, mt), expect)


def test_padded_extents():
    assert oracle.padded_extents(9, 8, 8) == (9, 8, 8)
    assert oracle.padded_extents(10, 5, 6) == (13, 8, 8)
    assert oracle.padded_extents(10, 5, 6, 16, 8) == (17, 16, 16)
    assert oracle.padded_extents(120, 720, 1280, 16, 8) == (121, 720, 1280)
    assert oracle.padded_extents(1, 1080, 1920, 16, 8) == (1, 1088, 1920)  # images: no temporal padding
    for bad in [(9, 8, 8, 6, 4), (9, 8, 8, 4, 2), (0, 8, 8, 4, 4)]:
        with pytest.raises(ValueError):
            oracle.padded_extents(*bad)


@pytest.mark.parametrize("shape", [(1, 2, 9, 8, 8), (2, 1, 1, 8, 12)])
def test_no_padding_needed_is_the_plain_patcher(shape):
    x = RNG.normal(size=shape)
    assert np.array_equal(oracle.haar_fwd_padded(x), oracle.haar_fwd(x))


@pytest.mark.parametrize("shape,ms,mt", [((1, 2, 6, 5, 7), 4, 4), ((2, 1, 11, 9, 6), 4, 8), ((1, 1, 2, 4, 4), 4, 4),
                                         ((1, 3, 1, 10, 5), 8, 4), ((1, 1, 13, 4, 4), 4, 4)])
def test_cropped_inverse_reconstructs_the_clip(shape, ms, mt):
    x = RNG.normal(size=shape)
    y = oracle.haar_fwd_padded(x, ms, mt)
    _, _, T, H, W = shape
    np.testing.assert_allclose(oracle.haar_inv_cropped(y, T, H, W, ms, mt), x, atol=1e-12)


def test_blocks_of_spatial_padding_are_zero():
    x = RNG.normal(size=(1, 2, 7, 5, 9))  # padded to 9 x 16 x 16 with ms = 16
    y = oracle.haar_fwd_padded(x, 16, 4)
    # block rows i with 4i >= 5 and block columns j with 4j >= 9 hold only padding
    assert np.all(y[:, :, :, 2:, :] == 0.0)
    assert np.all(y[:, :, :, :, 3:] == 0.0)
    assert np.any(y[:, :, :, 1, 2] != 0.0)


def test_temporal_padding_mirrors_the_last_frames():
    """With T = 6 (padded to 9), padded frames 6, 7, 8 are frames 4, 3, 2: the last window
    equals the transform of an explicitly mirrored window."""
    x = RNG.normal(size=(1, 1, 6, 4, 4))
    y = oracle.haar_fwd_padded(x)
    mirrored = np.concatenate([x, x[:, :, [4, 3, 2]]], axis=2)
    np.testing.assert_allclose(y, oracle.haar_fwd(mirrored), atol=0)


@pytest.mark.parametrize("K,a,b", [(4, 1, 3), (4, 2, 5), (3, 1, 4), (5, 4, 6)])
def test_continuation_chunks_compose_into_the_whole_clip(K, a, b):
    """Latent frames [a, b) of the whole clip (T = 1 + 4K) come from frames 4a-3 .. 4b-4 alone."""
    x = RNG.normal(size=(2, 2, 1 + 4 * K, 8, 4))
    y = oracle.haar_fwd(x)
    chunk = oracle.haar_fwd_chunk(x[:, :, 4 * a - 3:4 * b - 3], first=False)
    np.testing.assert_allclose(chunk, y[:, :, a:b], atol=1e-12)
    first = oracle.haar_fwd_chunk(x[:, :, :1 + 4 * (a - 1)], first=True)
    np.testing.assert_allclose(first, y[:, :, :a], atol=1e-12)
    # and the inverse of a continuation chunk gives back those frames of the whole-clip inverse
    xr = oracle.haar_inv(y, 1 + 4 * K, 8, 4)
    np.testing.assert_allclose(oracle.haar_inv_chunk(y[:, :, a:b], 4 * (b - a), 8, 4, first=False),
                               xr[:, :, 4 * a - 3:4 * b - 3], atol=1e-12)


def test_continuation_chunk_is_orthonormal():
    x = RNG.normal(size=(1, 2, 12, 8, 8))
    y = oracle.haar_fwd_chunk(x, first=False)
    assert y.shape == (1, 128, 3, 2, 2)
    np.testing.assert_allclose(np.sum(y * y), np.sum(x * x), rtol=1e-12)  # no replica: plain Parseval
    np.testing.assert_allclose(oracle.haar_inv_chunk(y, 12, 8, 8, first=False), x, atol=1e-12)


def test_one_frame_first_chunk_is_video_latent_frame_0():
    x = RNG.normal(size=(1, 2, 9, 8, 8))
    np.testing.assert_allclose(oracle.haar_fwd_chunk(x[:, :, :1], first=True), oracle.haar_fwd(x)[:, :, :1],
                               atol=1e-12)


def test_chunk_shape_rules():
    with pytest.raises(ValueError):
        oracle.haar_fwd_chunk(np.zeros((1, 1, 6, 4, 4)), first=False)   # 4k frames
    with pytest.raises(ValueError):
        oracle.haar_fwd_chunk(np.zeros((1, 1, 8, 4, 4)), first=True)    # 1 + 4k frames
