"""Pins for the Haar oracle, none of which re-uses the oracle's own code.

Each test checks the level-by-level oracle against something the pages or the
mathematics fix: the pages' printed shapes, an explicit operator matrix built
here from the definition with Kronecker products, perfect reconstruction,
energy (Parseval with the causal frame-0 term), constant input, and the causal
structure.  A dropped term, a wrong sign, a swapped subband or a misplaced
replica frame fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle

S = 1.0 / math.sqrt(2.0)
RNG = np.random.default_rng(20241202)


# --------------------------------------------------------------------------
# Brute force: the operator as an explicit matrix.
# --------------------------------------------------------------------------
def pair_matrix(n):
    """n samples -> n/2 low bands (a+b)/sqrt2 followed by n/2 high bands (a-b)/sqrt2."""
    P = np.zeros((n, n))
    for k in range(n // 2):
        P[k, 2 * k] = S
        P[k, 2 * k + 1] = S
        P[n // 2 + k, 2 * k] = S
        P[n // 2 + k, 2 * k + 1] = -S
    return P


def replicate_first(T):
    """T frames -> T+1 frames, a copy of frame 0 in front."""
    R = np.zeros((T + 1, T))
    R[0, 0] = 1.0
    for t in range(T):
        R[t + 1, t] = 1.0
    return R


def level_matrix(T, H, W):
    """One level on a single [T, H, W] channel; rows ordered [bt][j][by][i][bx][k] (2D: [by][i][bx][k])."""
    if T == 1:
        return np.kron(pair_matrix(H), pair_matrix(W))
    return np.kron(np.kron(pair_matrix(T + 1) @ replicate_first(T), pair_matrix(H)), pair_matrix(W))


def brute_level(v):
    """v [C, T, H, W] -> [nsub*C, T1, H/2, W/2] with channel s*C + c, through the explicit matrix."""
    C, T, H, W = v.shape
    M = level_matrix(T, H, W)
    out = (M @ v.reshape(C, -1).T).T  # [C, rows]
    Ho, Wo = H // 2, W // 2
    if T == 1:
        out = out.reshape(C, 2, Ho, 2, Wo).transpose(1, 3, 0, 2, 4).reshape(4 * C, 1, Ho, Wo)
    else:
        T1 = (T + 1) // 2
        out = out.reshape(C, 2, T1, 2, Ho, 2, Wo).transpose(1, 3, 5, 0, 2, 4, 6).reshape(8 * C, T1, Ho, Wo)
    return out


def brute_fwd(x):
    return np.stack([brute_level(brute_level(xb)) for xb in x])


def full_matrix(T, H, W):
    """The whole two-level operator on one channel, as a matrix, by probing unit vectors."""
    n = T * H * W
    cols = []
    for k in range(n):
        e = np.zeros(n)
        e[k] = 1.0
        cols.append(brute_fwd(e.reshape(1, 1, T, H, W)).ravel())
    return np.array(cols).T


@pytest.mark.parametrize("shape", [(1, 1, 5, 4, 4), (2, 2, 9, 8, 8), (1, 3, 13, 4, 8), (1, 2, 1, 8, 8),
                                   (2, 1, 1, 4, 12)])
def test_oracle_matches_explicit_matrix(shape):
    x = RNG.uniform(-1, 1, shape)
    np.testing.assert_allclose(oracle.haar_fwd(x), brute_fwd(x), rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,H,W", [(5, 4, 4), (9, 8, 4)])
def test_matrix_energy_identity_3d(T, H, W):
    """M^T M = I + 3 E0: every frame except frame 0 keeps its energy, frame 0 counts four times."""
    M = full_matrix(T, H, W)
    E0 = np.zeros(T * H * W)
    E0[: H * W] = 1.0
    np.testing.assert_allclose(M.T @ M, np.eye(T * H * W) + 3.0 * np.diag(E0), atol=1e-12)


def test_matrix_orthogonal_2d():
    M = full_matrix(1, 8, 8)
    assert M.shape == (64, 64)
    np.testing.assert_allclose(M.T @ M, np.eye(64), atol=1e-12)
    np.testing.assert_allclose(M @ M.T, np.eye(64), atol=1e-12)


# --------------------------------------------------------------------------
# Closed form: the level-by-level definition equals the block form.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(2, 3, 9, 16, 24), (1, 2, 21, 8, 8), (3, 2, 1, 16, 8), (1, 1, 5, 4, 4)])
def test_level_by_level_equals_block_form(shape):
    x = RNG.normal(size=shape)
    np.testing.assert_allclose(oracle.haar_fwd(x), oracle.haar_fwd_blockform(x), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Perfect reconstruction and energy.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(2, 3, 9, 16, 24), (1, 1, 5, 4, 4), (2, 2, 1, 12, 8), (1, 3, 17, 8, 16)])
def test_perfect_reconstruction(shape):
    x = RNG.uniform(-1, 1, shape)
    B, C, T, H, W = shape
    np.testing.assert_allclose(oracle.haar_inv(oracle.haar_fwd(x), T, H, W), x, rtol=0, atol=1e-12)


def test_inverse_drops_the_replica_not_the_data():
    """On coefficients outside the forward's range, frame 0 comes from the LAST sample of window 0.

    Window 0 of the inverse yields four frames; the first three are replicas.  A
    coefficient vector whose window-0 reconstruction is (0, 0, 0, 1) must give
    x_0 = 1 (the kept copy), and (1, 1, 1, 0) must give x_0 = 0.
    """
    T, H, W = 5, 4, 4
    # Coefficients of the block form for a time-only signal r_a at window 0, constant over y, x.
    for r, expect in [((0, 0, 0, 1.0), 1.0), ((1.0, 1.0, 1.0, 0), 0.0)]:
        y = np.zeros((1, 64, 2, 1, 1))
        # window 0: coefficient (kt, ky=0, kx=0) = (1/8) * sum_a (-1)^popcount(kt&a) r_a * 16
        for kt in range(4):
            val = sum(((-1) ** bin(kt & a).count("1")) * r[a] for a in range(4)) * 16 / 8.0
            s2, s1 = 4 * (kt >> 1), 4 * (kt & 1)
            y[0, 8 * s2 + s1, 0, 0, 0] = val
        x = oracle.haar_inv(y, T, H, W)
        np.testing.assert_allclose(x[0, 0, 0], expect, atol=1e-12)


@pytest.mark.parametrize("shape", [(2, 3, 9, 16, 24), (1, 2, 25, 8, 8)])
def test_parseval_with_causal_term(shape):
    """||fwd(x)||^2 = ||x||^2 + 3 ||x[:, :, 0]||^2 on video."""
    x = RNG.normal(size=shape)
    y = oracle.haar_fwd(x)
    lhs = np.sum(y * y)
    rhs = np.sum(x * x) + 3.0 * np.sum(x[:, :, 0] ** 2)
    assert abs(lhs - rhs) <= 1e-10 * rhs


def test_parseval_2d():
    x = RNG.normal(size=(3, 2, 1, 16, 20))
    y = oracle.haar_fwd(x)
    assert abs(np.sum(y * y) - np.sum(x * x)) <= 1e-10 * np.sum(x * x)


# --------------------------------------------------------------------------
# Constant input and causal structure.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 5, 13])
def test_constant_input(T):
    """A constant k puts 8k (2D: 4k) in the all-low channels and exactly 0 everywhere else."""
    C, k = 3, 0.37
    x = np.full((2, C, T, 8, 12), k)
    y = oracle.haar_fwd(x)
    gain = 4.0 if T == 1 else 8.0
    np.testing.assert_allclose(y[:, :C], gain * k, rtol=1e-14)
    assert np.all(y[:, C:] == 0.0)


def test_first_latent_frame_has_no_temporal_high_band():
    """At t' = 0 both time bands are built from copies of frame 0, so every channel with bt1 or bt2 set is 0."""
    C = 2
    x = RNG.normal(size=(1, C, 9, 8, 8))
    y = oracle.haar_fwd(x)
    for s2 in range(8):
        for s1 in range(8):
            if (s2 >> 2) or (s1 >> 2):
                ch = (8 * s2 + s1) * C
                assert np.all(y[0, ch:ch + C, 0] == 0.0)


def test_frame_dependence_is_causal_and_local():
    """Changing frame f changes output frame ceil(f/4) only (frame 0 -> output frame 0)."""
    x = RNG.normal(size=(1, 1, 13, 4, 8))
    y = oracle.haar_fwd(x)
    for f in range(13):
        x2 = x.copy()
        x2[0, 0, f] += 1.0
        d = np.abs(oracle.haar_fwd(x2) - y).max(axis=(0, 1, 3, 4))
        changed = set(np.nonzero(d > 1e-12)[0].tolist())
        assert changed == {(f + 3) // 4}, (f, changed)


def test_first_window_is_twice_the_image_transform():
    """Output frame 0 of the video path, on its all-low time channels, is 2 x the 2D transform of frame 0."""
    C = 2
    x = RNG.normal(size=(1, C, 5, 8, 8))
    y3 = oracle.haar_fwd(x)
    y2 = oracle.haar_fwd(x[:, :, :1])
    for s2 in range(4):
        for s1 in range(4):
            ch3 = (8 * s2 + s1) * C  # bt2 = bt1 = 0: s = 2*by + bx
            ch2 = (4 * s2 + s1) * C
            np.testing.assert_allclose(y3[0, ch3:ch3 + C, 0], 2.0 * y2[0, ch2:ch2 + C, 0], atol=1e-12)


def test_one_dimensional_subband_signs():
    """A single x-axis ramp: the 4-point two-level transform is H4/2 in natural order (k = 2*b2 + b1)."""
    x = np.zeros((1, 1, 1, 4, 4))
    x[0, 0, 0, :, :] = np.array([1.0, 2.0, 4.0, 8.0])  # constant along y
    y = oracle.haar_fwd(x)[0, :, 0, 0, 0]  # 16 channels, C = 1
    # along y constant -> only ky = 0 (by2 = by1 = 0); along x: k = 2*bx2 + bx1 -> channel 4*bx2 + bx1
    xs = np.array([1.0, 2.0, 4.0, 8.0])
    h4 = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=float)
    coeff_x = h4 @ xs / 2.0
    expect = np.zeros(16)
    for k in range(4):
        expect[4 * (k >> 1) + (k & 1)] = coeff_x[k] * 2.0  # the y axis contributes (1+1+1+1)/2 = 2
    np.testing.assert_allclose(y, expect, atol=1e-12)


# --------------------------------------------------------------------------
# The pages' printed shapes.
# --------------------------------------------------------------------------
def test_page_example_2d_shapes(golden):
    shapes = golden["haar_2d_two_levels"]["shapes"]
    C, H, W = shapes[0]
    x = RNG.normal(size=(C, 1, H, W))
    y1 = oracle.haar_level_fwd(x)
    assert (y1.shape[0], y1.shape[2], y1.shape[3]) == tuple(shapes[1])
    y2 = oracle.haar_level_fwd(y1)
    assert (y2.shape[0], y2.shape[2], y2.shape[3]) == tuple(shapes[2])
    full = oracle.haar_fwd(x[None])
    assert full.shape == (1, shapes[2][0], 1, shapes[2][1], shapes[2][2])
    np.testing.assert_allclose(full[0, :, 0], y2[:, 0], atol=1e-12)


def test_page_3d_level_shape(golden):
    f = golden["haar_3d_one_level"]["channel_factor"]
    y = oracle.haar_level_fwd(RNG.normal(size=(3, 9, 8, 8)))
    assert y.shape == (3 * f, 5, 4, 4)


def test_page_causal_frame_count(golden):
    p = golden["causal_frames"]
    assert oracle.out_frames(p["T"]) == p["t"]
    enc = golden["discrete_encode_shapes"]
    assert oracle.out_frames(enc["input"][2]) == enc["indices"][1] == enc["codes"][2]
    for T in (1, 5, 9, 17, 121):
        assert oracle.out_frames(T) == 1 + (T - 1) // 4


def test_page_haar_taps(golden):
    taps = golden["haar_taps"]["value"]
    # the printed taps are 1/sqrt(2) rounded to four decimals
    assert all(abs(t - S) < 0.5 * 10 ** -golden["haar_taps"]["printed_decimals"] for t in taps)
    # one level on a pair of equal samples gives sqrt(2) * a in the low band, 0 in the high band
    x = np.ones((1, 1, 2, 2))
    y = oracle.haar_level_fwd(x)[:, 0, 0, 0]
    np.testing.assert_allclose(y, [2.0, 0, 0, 0], atol=1e-15)  # (1+1)/sqrt2 twice = 2


def test_workload_shapes():
    assert oracle.haar_out_shape(1, 3, 9, 64, 64) == (1, 192, 3, 16, 16)
    assert oracle.haar_out_shape(1, 3, 121, 704, 1280) == (1, 192, 31, 176, 320)
    assert oracle.haar_out_shape(4, 3, 121, 1088, 1920) == (4, 192, 31, 272, 480)
    assert oracle.haar_out_shape(16, 3, 1, 1024, 1024) == (16, 48, 1, 256, 256)


def test_bad_shapes_rejected():
    with pytest.raises(ValueError):
        oracle.haar_fwd(np.zeros((1, 1, 3, 4, 4)))
    with pytest.raises(ValueError):
        oracle.haar_fwd(np.zeros((1, 1, 5, 6, 4)))
