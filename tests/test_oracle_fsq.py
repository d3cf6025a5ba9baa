"""Pins for the FSQ oracle, checked against closed forms and exhaustive enumeration.

The pages fix the levels (8,8,8,5,5,5), the codebook size 64000, a tanh bound
followed by rounding, and a mixed-radix index.  The constants of the bound
(eps = 1e-3, the even-level offset) are a reading of the published FSQ method
and are pinned here only through what follows from them: exactly L levels per
channel, z = 0 at the centre code, monotonicity, odd-level symmetry, and the
code centres mapping back to themselves.
"""
import math

import numpy as np
import pytest

import oracle

LEVELS = (8, 8, 8, 5, 5, 5)
EPS = 1e-3


def half_and_offset(L):
    return (L - 1) * (1 + EPS) / 2.0, (0.5 if L % 2 == 0 else 0.0)


def test_levels_and_codebook_from_pages(golden):
    g = golden["fsq_levels"]
    assert tuple(g["levels"]) == LEVELS == oracle.FSQ_LEVELS
    assert math.prod(g["levels"]) == g["codebook"] == oracle.FSQ_CODEBOOK


def test_mixed_radix_basis():
    # place value of channel i = product of the levels of channels below it
    expect = tuple(math.prod(LEVELS[:i]) for i in range(6))
    assert oracle.fsq_basis() == expect == (1, 8, 64, 512, 2560, 12800)


def test_index_bijection_exhaustive():
    """Every index in [0, 64000) unpacks to in-range digits and packs back to itself."""
    seen = set()
    for idx in range(64000):
        d = oracle.fsq_unpack(idx)
        assert all(0 <= d[i] < LEVELS[i] for i in range(6))
        assert oracle.fsq_pack(d) == idx
        seen.add(d)
    assert len(seen) == 64000


@pytest.mark.parametrize("ch", range(6))
def test_each_channel_reaches_exactly_L_levels(ch):
    L = LEVELS[ch]
    zs = np.linspace(-8, 8, 40001)
    qs = [oracle.fsq_quantize(float(np.float32(z)), ch) for z in zs]
    assert sorted(set(qs)) == list(range(-(L // 2), (L + 1) // 2))
    assert all(a <= b for a, b in zip(qs, qs[1:]))  # monotone in z


@pytest.mark.parametrize("ch", range(6))
def test_zero_maps_to_centre_code(ch):
    assert oracle.fsq_quantize(0.0, ch) == 0
    assert abs(oracle.fsq_bound(0.0, ch)) < 1e-15


@pytest.mark.parametrize("ch", [3, 4, 5])
def test_odd_levels_are_symmetric(ch):
    for z in np.linspace(-5, 5, 2001):
        z = float(np.float32(z))
        assert oracle.fsq_quantize(-z, ch) == -oracle.fsq_quantize(z, ch)


@pytest.mark.parametrize("ch", range(6))
def test_code_centres_round_trip(ch):
    """z at the centre of code q, atanh((q + off)/half) - shift, quantizes back to q."""
    L = LEVELS[ch]
    half, off = half_and_offset(L)
    shift = math.atanh(off / half)
    for q in range(-(L // 2), (L + 1) // 2):
        z = math.atanh((q + off) / half) - shift
        assert oracle.fsq_quantize(float(np.float32(z)), ch) == q
        assert abs(oracle.fsq_bound(z, ch) - q) < 1e-12


def test_index_of_zero_and_extremes():
    """z = 0 -> digits (4,4,4,2,2,2) -> 4 + 4*8 + 4*64 + 2*512 + 2*2560 + 2*12800 = 32036."""
    C, S = 6, 3
    u = np.zeros((1, C, S), np.float32)
    u[0, :, 1] = 1e6
    u[0, :, 2] = -1e6
    w = np.eye(6, dtype=np.float32)
    idx, codes, near = oracle.fsq_encode(u, w)
    assert idx.tolist() == [[32036, 63999, 0]]
    np.testing.assert_array_equal(codes[0, :, 1], [0.75, 0.75, 0.75, 1, 1, 1])
    np.testing.assert_array_equal(codes[0, :, 2], [-1, -1, -1, -1, -1, -1])
    assert not near.any()


def test_projection_uses_rows_of_w():
    """W with one 1 per row (row i picks channel perm[i]) makes z_i = u[perm[i]] exactly.

    A transposed operand or a wrong channel index would quantize the wrong inputs.
    """
    rng = np.random.default_rng(7)
    C, S = 16, 4000
    perm = [11, 2, 7, 0, 15, 5]
    w = np.zeros((6, C), np.float32)
    for i, c in enumerate(perm):
        w[i, c] = 1.0
    u = rng.normal(0, 1.5, (2, C, S)).astype(np.float32)
    idx, codes, _ = oracle.fsq_encode(u, w)
    basis = oracle.fsq_basis()
    for b in range(2):
        for s in range(0, S, 97):
            digits = [oracle.fsq_quantize(float(u[b, perm[i], s]), i) + LEVELS[i] // 2 for i in range(6)]
            assert idx[b, s] == sum(d * p for d, p in zip(digits, basis))
            for i in range(6):
                assert codes[b, i, s] == (digits[i] - LEVELS[i] // 2) / (LEVELS[i] // 2)


def test_projection_is_fp32_fused_chain():
    """z is the fp32 chain z = fma(w_c, u_c, z) from 0, so the decision follows the fp32 sum.

    With w = (1, 1) and u = (a, b), b below half an ulp of a, the fp32 chain
    gives z = a exactly while the real sum a + b lies on the other side of a
    decision threshold of channel 3 (L = 5).  An oracle that accumulated in
    double would pick the other code.
    """
    half, off = half_and_offset(5)
    theta = math.atanh((0.5 + off) / half) - math.atanh(off / half)  # boundary between q = 0 and q = 1
    below = np.float32(theta)
    if float(below) > theta:
        below = np.nextafter(below, np.float32(-np.inf))
    above = np.nextafter(below, np.float32(np.inf))
    ulp = float(above) - float(below)
    if theta - float(below) < ulp / 2:
        a = below                                   # fp32 says q = 0 ...
        b = np.float32((theta - float(below) + ulp / 2) / 2)  # ... the real sum says q = 1
        expect_q = 0
    else:
        a = above                                   # fp32 says q = 1 ...
        b = -np.float32((float(above) - theta + ulp / 2) / 2)  # ... the real sum says q = 0
        expect_q = 1
    assert np.float32(a + b) == a and (float(a) + float(b) > theta) != (expect_q == 1)
    w = np.zeros((6, 2), np.float32)
    w[3] = [1.0, 1.0]
    u = np.array([[[a], [b]]], np.float32)
    idx, _, _ = oracle.fsq_encode(u, w)
    assert (int(idx[0, 0]) // 512) % 5 - 2 == expect_q


def test_near_boundary_flag():
    half, off = half_and_offset(8)
    shift = math.atanh(off / half)
    theta = math.atanh((0.5 + off) / half) - shift  # v = 0.5 there
    u = np.zeros((1, 6, 2), np.float32)
    u[0, 0, 0] = np.float32(theta)
    u[0, 0, 1] = np.float32(theta + 0.01)
    _, _, near = oracle.fsq_encode(u, np.eye(6, dtype=np.float32))
    assert near.tolist() == [[True, False]]


def test_decode_of_extremes_and_one_hot():
    rng = np.random.default_rng(3)
    C = 16
    w = rng.normal(0, 0.25, (6, C)).astype(np.float32)
    out, bad = oracle.fsq_decode(np.array([[0, 63999, 32036]], np.int32), w)
    assert bad == 0
    z0 = np.array([-1.0] * 6)
    z1 = np.array([0.75, 0.75, 0.75, 1, 1, 1])
    np.testing.assert_allclose(out[0, :, 0], w.astype(np.float64).T @ z0, atol=1e-15)
    np.testing.assert_allclose(out[0, :, 1], w.astype(np.float64).T @ z1, atol=1e-15)
    np.testing.assert_allclose(out[0, :, 2], 0.0, atol=1e-15)  # centre code is all zeros
    # one-hot W: decode places zhat_i in channel perm[i]
    perm = [3, 9, 0, 14, 6, 1]
    wp = np.zeros((6, C), np.float32)
    for i, c in enumerate(perm):
        wp[i, c] = 1.0
    idx = 5 + 3 * 8 + 7 * 64 + 1 * 512 + 4 * 2560 + 0 * 12800  # digits (5,3,7,1,4,0)
    out, _ = oracle.fsq_decode(np.array([[idx]], np.int32), wp)
    zhat = [(5 - 4) / 4, (3 - 4) / 4, (7 - 4) / 4, (1 - 2) / 2, (4 - 2) / 2, (0 - 2) / 2]
    for i, c in enumerate(perm):
        assert out[0, c, 0] == zhat[i]


def test_decode_flags_invalid_indices():
    w = np.ones((6, 4), np.float32)
    out, bad = oracle.fsq_decode(np.array([[-1, 64000, 5, 2 ** 31 - 1]], np.int32), w)
    assert bad == 3
    assert np.isnan(out[0, :, [0, 1, 3]]).all()
    assert not np.isnan(out[0, :, 2]).any()


def test_decode_inverts_encode_on_centres():
    """With W = I (C = 6), encoding the code centres and decoding returns the normalized codes."""
    rng = np.random.default_rng(11)
    S = 500
    q = np.stack([rng.integers(-(L // 2), (L + 1) // 2, S) for L in LEVELS])  # [6, S]
    z = np.zeros((6, S))
    for i, L in enumerate(LEVELS):
        half, off = half_and_offset(L)
        z[i] = np.arctanh((q[i] + off) / half) - math.atanh(off / half)
    u = z.astype(np.float32)[None]
    w = np.eye(6, dtype=np.float32)
    idx, codes, _ = oracle.fsq_encode(u, w)
    out, bad = oracle.fsq_decode(idx, w)
    assert bad == 0
    zhat = q / np.array([L // 2 for L in LEVELS])[:, None]
    np.testing.assert_array_equal(codes[0], zhat)
    np.testing.assert_allclose(out[0], zhat, atol=0)


def test_discrete_shapes_from_pages(golden):
    """A latent [B, 16, t, h, w] gives indices [B, t, h, w] and codes [B, 6, t, h, w]."""
    enc = golden["discrete_encode_shapes"]
    B, t, h, w = enc["indices"]
    u = np.zeros((B, 16, t * h * w), np.float32)
    idx, codes, _ = oracle.fsq_encode(u, np.zeros((6, 16), np.float32))
    assert idx.reshape(B, t, h, w).shape == tuple(enc["indices"])
    assert codes.reshape(B, 6, t, h, w).shape == tuple(enc["codes"])
