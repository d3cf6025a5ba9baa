"""Pins for the single-level patcher / unpatcher (patch_size=2: one DWT, "NVIDIA Cosmos
Tokenizer 完全指南", section 7.1: one 2D DWT turns c channels into 4c at half size, one 3D
DWT into 8c with frame 0 repeated; patch_size=4 stacks two).

The forward level is the building block of the two-level patcher, whose own pins fix it;
here: the level applied twice is the two-level transform, the inverse level undoes it,
energy is kept up to the causal replica, and a constant input has the closed form.
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(21)
S = 2 ** -0.5


@pytest.mark.parametrize("shape", [(2, 1, 8, 8), (3, 9, 8, 12), (1, 5, 4, 4)])
def test_two_single_levels_are_the_two_level_patcher(shape):
    x = RNG.normal(size=shape)
    y2 = oracle.haar_level_fwd(oracle.haar_level_fwd(x))
    np.testing.assert_allclose(y2, oracle.haar_fwd(x[None])[0], atol=1e-12)


@pytest.mark.parametrize("shape", [(2, 1, 6, 10), (3, 7, 4, 6), (1, 3, 2, 2)])
def test_single_level_inverse(shape):
    x = RNG.normal(size=shape)
    C, T, H, W = shape
    np.testing.assert_allclose(oracle.haar_level_inv(oracle.haar_level_fwd(x), T, H, W), x, atol=1e-12)


def test_single_level_parseval_with_the_replica():
    x = RNG.normal(size=(2, 7, 4, 6))
    y = oracle.haar_level_fwd(x)
    # the replica adds one copy of frame 0's energy (video); images keep it exactly
    np.testing.assert_allclose(np.sum(y * y), np.sum(x * x) + np.sum(x[:, 0] ** 2), rtol=1e-12)
    xi = RNG.normal(size=(2, 1, 4, 6))
    yi = oracle.haar_level_fwd(xi)
    np.testing.assert_allclose(np.sum(yi * yi), np.sum(xi * xi), rtol=1e-12)


def test_single_level_constant_input():
    y = oracle.haar_level_fwd(np.full((2, 5, 4, 4), 1.5))
    np.testing.assert_allclose(y[:2], 1.5 * 2 * np.sqrt(2), atol=1e-12)  # (1/sqrt2)^3 * 8 * k
    assert np.all(np.abs(y[2:]) < 1e-12)
    yi = oracle.haar_level_fwd(np.full((1, 1, 4, 4), 1.5))
    np.testing.assert_allclose(yi[:1], 3.0, atol=1e-12)                   # (1/sqrt2)^2 * 4 * k
    assert np.all(np.abs(yi[1:]) < 1e-12)


def test_single_level_window_0_reads_frame_0_twice():
    x = RNG.normal(size=(1, 5, 2, 2))
    y = oracle.haar_level_fwd(x)
    # window 0 is the pair (frame 0, frame 0): its temporal high bands (s >= 4) are zero
    assert np.all(np.abs(y[4:, 0]) < 1e-12)
    # window t >= 1 reads frames 2t-1, 2t: changing frame 3 changes window 2 only
    x2 = x.copy()
    x2[0, 3] += 1.0
    d = np.abs(oracle.haar_level_fwd(x2) - y).max(axis=(0, 2, 3))
    assert d[2] > 0 and d[0] == 0 and d[1] == 0
