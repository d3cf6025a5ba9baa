"""Oracle for the first causal factorized convolution after the patcher.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): only tests/, the smoke check and
bench.py's CPU-baseline legs use it; it shares nothing with the CUDA library.

"Cosmos World Foundation Model Platform for Physical AI (Cosmos-Predict1)" notes,
model architecture item 1 (the wavelet space operation): after the 2-level Haar
transform the encoder's convolutions are factorized in space and time -- first a
1 x k x k spatial convolution, then a k x 1 x 1 temporal convolution padded by k - 1
on the left (past) side only, so an output frame depends on its own and earlier
frames.

Readings where the pages are silent (parity unpinned by the pages for all of them;
they are conventions shared with the CUDA path):
  - k = 3; the spatial convolution is padded by (k - 1)/2 zeros on every side ("same");
  - no bias, no activation between the two convolutions (one factorized 3D layer);
  - channels: C_in = 64 C (the patcher's output), C_mid = C_out = 256 at the measured
    size (the oracle takes any counts); weights layout [C_mid][k][k][C_in] (spatial)
    and [C_out][k][C_mid] (temporal), tap dt multiplying frame t - (k - 1) + dt;
  - activations are channels-last [B, T', h, w, C] (the patcher's channels-last output);
  - the network stores activations in bf16: the spatial result is rounded to bf16
    (nearest-even) before the temporal convolution; arithmetic here is float64.
"""
import numpy as np


def spatial_conv(x: np.ndarray, ws: np.ndarray) -> np.ndarray:
    """x [B, T, h, w, Cin], ws [Cmid, k, k, Cin] -> [B, T, h, w, Cmid]; zero 'same' padding."""
    x = np.asarray(x, dtype=np.float64)
    ws = np.asarray(ws, dtype=np.float64)
    B, T, h, w, Cin = x.shape
    Cmid, k, k2, Cin2 = ws.shape
    assert k == k2 and Cin == Cin2 and k % 2 == 1
    p = (k - 1) // 2
    xp = np.zeros((B, T, h + 2 * p, w + 2 * p, Cin))
    xp[:, :, p:p + h, p:p + w] = x
    out = np.zeros((B, T, h, w, Cmid))
    for dy in range(k):
        for dx in range(k):
            out += np.einsum("btijc,mc->btijm", xp[:, :, dy:dy + h, dx:dx + w], ws[:, dy, dx, :])
    return out


def temporal_causal_conv(s: np.ndarray, wt: np.ndarray) -> np.ndarray:
    """s [B, T, h, w, Cmid], wt [Cout, k, Cmid] -> [B, T, h, w, Cout]; output frame t reads
    frames t - (k - 1) .. t, frames before 0 are zero (left padding k - 1)."""
    s = np.asarray(s, dtype=np.float64)
    wt = np.asarray(wt, dtype=np.float64)
    B, T, h, w, Cmid = s.shape
    Cout, k, Cmid2 = wt.shape
    assert Cmid == Cmid2
    sp = np.concatenate([np.zeros((B, k - 1, h, w, Cmid)), s], axis=1)
    out = np.zeros((B, T, h, w, Cout))
    for dt in range(k):
        out += np.einsum("btijm,nm->btijn", sp[:, dt:dt + T], wt[:, dt, :])
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float64 -> the nearest bf16 value (8 significant bits, ties to even), as float64.
    frexp splits a = m * 2^e with 0.5 <= |m| < 1; m * 256 holds the 8 kept bits in its
    integer part, rint rounds it half to even, and the scaling back is exact.  (Normal
    bf16 range only: the activations here are far from 2^-126 and from overflow.)"""
    m, e = np.frexp(np.asarray(a, dtype=np.float64))
    return np.ldexp(np.rint(m * 256.0), e - 8)


def factorized_conv(x: np.ndarray, ws: np.ndarray, wt: np.ndarray) -> np.ndarray:
    """The layer: spatial convolution, bf16 rounding of the intermediate, causal temporal convolution."""
    return temporal_causal_conv(round_bf16(spatial_conv(x, ws)), wt)
