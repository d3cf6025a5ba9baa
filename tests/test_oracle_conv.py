"""Pins for the oracle of the causal factorized convolution (oracle/conv.py).

Against plain loops written out per output element on tiny inputs (a second,
independent statement of the two sums), torch's own bf16 rounding, and properties
any correct implementation has: identity taps, causality, zero padding at the borders,
linearity.
"""
import numpy as np
import pytest
import torch

from oracle import conv

RNG = np.random.default_rng(31)


def spatial_loops(x, ws):
    B, T, h, w, Cin = x.shape
    Cmid, k, _, _ = ws.shape
    p = (k - 1) // 2
    out = np.zeros((B, T, h, w, Cmid))
    for b in range(B):
        for t in range(T):
            for i in range(h):
                for j in range(w):
                    for m in range(Cmid):
                        acc = 0.0
                        for dy in range(k):
                            for dx in range(k):
                                y, xx = i + dy - p, j + dx - p
                                if 0 <= y < h and 0 <= xx < w:
                                    acc += float(np.dot(ws[m, dy, dx], x[b, t, y, xx]))
                        out[b, t, i, j, m] = acc
    return out


def temporal_loops(s, wt):
    B, T, h, w, Cmid = s.shape
    Cout, k, _ = wt.shape
    out = np.zeros((B, T, h, w, Cout))
    for b in range(B):
        for t in range(T):
            for n in range(Cout):
                acc = np.zeros((h, w))
                for dt in range(k):
                    f = t - (k - 1) + dt
                    if f >= 0:
                        acc += np.einsum("ijm,m->ij", s[b, f], wt[n, dt])
                out[b, t, :, :, n] = acc
    return out


def test_spatial_matches_loops():
    x = RNG.normal(size=(2, 2, 4, 5, 3))
    ws = RNG.normal(size=(4, 3, 3, 3))
    np.testing.assert_allclose(conv.spatial_conv(x, ws), spatial_loops(x, ws), atol=1e-12)


def test_temporal_matches_loops():
    s = RNG.normal(size=(2, 5, 2, 3, 4))
    wt = RNG.normal(size=(3, 3, 4))
    np.testing.assert_allclose(conv.temporal_causal_conv(s, wt), temporal_loops(s, wt), atol=1e-12)


def test_identity_taps():
    x = RNG.normal(size=(1, 3, 4, 4, 5))
    ws = np.zeros((5, 3, 3, 5))
    ws[:, 1, 1, :] = np.eye(5)
    np.testing.assert_allclose(conv.spatial_conv(x, ws), x, atol=0)
    wt = np.zeros((5, 3, 5))
    wt[:, 2, :] = np.eye(5)           # tap 2 multiplies the current frame
    np.testing.assert_allclose(conv.temporal_causal_conv(x, wt), x, atol=0)
    wt = np.zeros((5, 3, 5))
    wt[:, 1, :] = np.eye(5)           # tap 1: the previous frame, zero before frame 0
    shifted = np.concatenate([np.zeros_like(x[:, :1]), x[:, :-1]], axis=1)
    np.testing.assert_allclose(conv.temporal_causal_conv(x, wt), shifted, atol=0)


def test_causality():
    s = RNG.normal(size=(1, 6, 2, 2, 3))
    wt = RNG.normal(size=(2, 3, 3))
    s2 = s.copy()
    s2[:, 3] += 1.0
    d = np.abs(conv.temporal_causal_conv(s2, wt) - conv.temporal_causal_conv(s, wt)).max(axis=(0, 2, 3, 4))
    assert np.all(d[:3] == 0) and np.all(d[3:6] > 0)   # frames 3, 4, 5 read frame 3


def test_zero_padding_at_the_border():
    x = np.zeros((1, 1, 4, 4, 1))
    x[0, 0, 0, 0, 0] = 1.0
    ws = RNG.normal(size=(1, 3, 3, 1))
    out = conv.spatial_conv(x, ws)[0, 0, :, :, 0]
    # a unit at (0, 0) reaches (0, 0), (0, 1), (1, 0), (1, 1) through taps (1,1), (1,0), (0,1), (0,0)
    np.testing.assert_allclose(out[:2, :2], [[ws[0, 1, 1, 0], ws[0, 1, 0, 0]], [ws[0, 0, 1, 0], ws[0, 0, 0, 0]]])
    assert np.all(out[2:] == 0) and np.all(out[:, 2:] == 0)


def test_round_bf16_is_torch_rounding_on_float32_values():
    a = (RNG.normal(size=100000) * np.exp(RNG.uniform(-30, 30, 100000))).astype(np.float32)
    a[:8] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, 1.0, -2.5, 3.0 + 2 ** -7, 1e-20]  # ties
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(conv.round_bf16(a.astype(np.float64)), ref)


def test_layer_is_linear():
    x = RNG.normal(size=(1, 4, 3, 3, 2))
    ws = RNG.normal(size=(3, 3, 3, 2))
    wt = RNG.normal(size=(2, 3, 3))
    f = lambda v: conv.temporal_causal_conv(conv.spatial_conv(v, ws), wt)  # noqa: E731
    np.testing.assert_allclose(f(2.0 * x) , 2.0 * f(x), atol=1e-12)
