"""Pins for the oracle's gradients: the Haar adjoints and the FSQ straight-through backward.

Checked against the definitions, not the oracle's own code: dot-product identities
<A x, g> = <x, A^T g>, the explicit operator matrix transposed, the closed forms
M^T M = I + 3 E0 and L L^T = I, and central finite differences of the smooth
surrogate that the straight-through estimator differentiates (the bound before
rounding, [guide] section 7.2: round_ste passes the gradient through the round).
"""
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_haar import full_matrix

RNG = np.random.default_rng(7)
LEVELS = (8, 8, 8, 5, 5, 5)


@pytest.mark.parametrize("shape", [(2, 3, 9, 8, 8), (1, 2, 13, 4, 12), (1, 1, 5, 4, 4)])
def test_patcher_adjoint_dot_product(shape):
    B, C, T, H, W = shape
    x = RNG.normal(size=shape)
    g = RNG.normal(size=oracle.haar_out_shape(B, C, T, H, W))
    lhs = np.sum(oracle.haar_fwd(x) * g)
    rhs = np.sum(x * oracle.haar_fwd_adjoint(g, T, H, W))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


@pytest.mark.parametrize("shape", [(2, 3, 9, 8, 8), (1, 2, 13, 4, 12)])
def test_unpatcher_adjoint_dot_product(shape):
    B, C, T, H, W = shape
    y = RNG.normal(size=oracle.haar_out_shape(B, C, T, H, W))
    g = RNG.normal(size=shape)
    lhs = np.sum(oracle.haar_inv(y, T, H, W) * g)
    rhs = np.sum(y * oracle.haar_inv_adjoint(g))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


def test_patcher_adjoint_is_the_transposed_matrix():
    T, H, W = 5, 4, 8
    M = full_matrix(T, H, W)
    g = RNG.normal(size=M.shape[0])
    gx = oracle.haar_fwd_adjoint(g.reshape(oracle.haar_out_shape(1, 1, T, H, W)), T, H, W)
    np.testing.assert_allclose(gx.ravel(), M.T @ g, atol=1e-12)


def test_adjoint_of_patcher_after_patcher_multiplies_frame0_by_four():
    """M^T M = I + 3 E0: frame 0 is read four times by the forward."""
    x = RNG.normal(size=(1, 2, 9, 8, 8))
    back = oracle.haar_fwd_adjoint(oracle.haar_fwd(x), 9, 8, 8)
    expect = x.copy()
    expect[:, :, 0] *= 4.0
    np.testing.assert_allclose(back, expect, atol=1e-12)


def test_unpatcher_after_its_adjoint_is_identity():
    """L L^T = I: the unpatcher's adjoint puts each pixel gradient where the unpatcher reads it."""
    g = RNG.normal(size=(2, 1, 13, 4, 8))
    np.testing.assert_allclose(oracle.haar_inv(oracle.haar_inv_adjoint(g), 13, 4, 8), g, atol=1e-12)


def test_unpatcher_adjoint_gives_no_gradient_to_replicas():
    """Window 0 of L^T g is the block transform of the time samples (0, 0, 0, g0): per spatial
    coefficient, (1/2)(-1)^popcount(kt) times the 2D transform of frame 0's block."""
    g = RNG.normal(size=(1, 1, 5, 4, 4))
    gy = oracle.haar_inv_adjoint(g)
    y2d = oracle.haar_fwd(g[:, :, :1])[0, :, 0, 0, 0]  # image path: 16 channels, C = 1
    for kt in range(4):
        time_coeff = 0.5 * (-1) ** bin(kt).count("1")
        for s in range(16):
            ky, kx = 2 * ((s >> 2) >> 1) + ((s & 3) >> 1), 2 * ((s >> 2) & 1) + (s & 1)
            s2 = 4 * (kt >> 1) + 2 * (ky >> 1) + (kx >> 1)
            s1 = 4 * (kt & 1) + 2 * (ky & 1) + (kx & 1)
            np.testing.assert_allclose(gy[0, 8 * s2 + s1, 0, 0, 0], time_coeff * y2d[s], atol=1e-12)


# --------------------------------------------------------------------------
# FSQ straight-through backward.
# --------------------------------------------------------------------------
def surrogate(u64, w64, g):
    """sum over tokens and channels of g_i * bound_i(z_i) / floor(L_i / 2), z in double."""
    z = np.einsum("ic,bcs->bis", w64, u64)
    total = 0.0
    for i, L in enumerate(LEVELS):
        half = (L - 1) * 1.001 / 2
        off = 0.5 if L % 2 == 0 else 0.0
        v = np.tanh(z[:, i] + math.atanh(off / half)) * half - off
        total += np.sum(g[:, i] * v / (L // 2))
    return total


@pytest.mark.parametrize("ch", range(6))
def test_ste_slope_is_the_derivative_of_the_bound(ch):
    L = LEVELS[ch]
    for z in (-2.5, -0.7, 0.0, 0.3, 1.9, 4.0):
        h = 1e-5
        fd = (oracle.fsq_bound(z + h, ch) - oracle.fsq_bound(z - h, ch)) / (2 * h) / (L // 2)
        assert abs(fd - oracle.fsq_ste_slope(z, ch)) < 1e-8


def test_encode_backward_matches_finite_differences():
    B, C, S = 2, 5, 7
    u = RNG.normal(0, 1.2, (B, C, S)).astype(np.float32)
    w = RNG.normal(0, 0.4, (6, C)).astype(np.float32)
    g = RNG.normal(size=(B, 6, S)).astype(np.float32)
    gu, gw = oracle.fsq_encode_backward(u, w, g)
    u64, w64, g64 = u.astype(np.float64), w.astype(np.float64), g.astype(np.float64)
    h = 1e-6
    for (b, c, s) in [(0, 0, 0), (1, 4, 6), (0, 2, 3), (1, 1, 1)]:
        up, um = u64.copy(), u64.copy()
        up[b, c, s] += h
        um[b, c, s] -= h
        fd = (surrogate(up, w64, g64) - surrogate(um, w64, g64)) / (2 * h)
        assert abs(fd - gu[b, c, s]) < 1e-5 * (1 + abs(fd))
    for (i, c) in [(0, 0), (3, 4), (5, 2), (2, 1)]:
        wp, wm = w64.copy(), w64.copy()
        wp[i, c] += h
        wm[i, c] -= h
        fd = (surrogate(u64, wp, g64) - surrogate(u64, wm, g64)) / (2 * h)
        assert abs(fd - gw[i, c]) < 1e-5 * (1 + abs(fd))


def test_decode_backward_dot_products():
    """decode is linear in the codes and in W: both gradients are exact dot-product identities."""
    B, C, S = 2, 6, 9
    idx = RNG.integers(0, 64000, (B, S)).astype(np.int32)
    idx[0, 3] = -5                         # invalid: no gradient either way
    w = RNG.normal(0, 0.3, (6, C)).astype(np.float32)
    g = RNG.normal(size=(B, C, S)).astype(np.float32)
    gc, gw = oracle.fsq_decode_backward(idx, w, g)
    zhat = np.zeros((B, 6, S))
    for b in range(B):
        for s in range(S):
            if 0 <= idx[b, s] < 64000:
                d = oracle.fsq_unpack(int(idx[b, s]))
                zhat[b, :, s] = [(d[i] - L // 2) / (L // 2) for i, L in enumerate(LEVELS)]
    out = np.einsum("ic,bis->bcs", w.astype(np.float64), zhat)
    assert abs(np.sum(out * g) - np.sum(zhat * gc)) < 1e-10
    assert np.all(gc[0, :, 3] == 0)
    # linear in W: the change of <out, g> when W[i][c] grows by 1 is grad_w[i][c]
    for (i, c) in [(0, 0), (4, 5), (2, 3)]:
        e = np.zeros((6, C))
        e[i, c] = 1.0
        delta = np.sum(np.einsum("ic,bis->bcs", e, zhat) * g)
        assert abs(delta - gw[i, c]) < 1e-10
