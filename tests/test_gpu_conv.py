"""GPU parity of the causal factorized convolution (tensor cores) against the oracle.

Tolerance, from the arithmetic: the products of bf16 values are exact in fp32 and the
tensor cores accumulate K of them in fp32, so |acc - exact| <= 2 K 2^-24 sum|terms| (a
factor 2 of headroom for the accumulator's internal rounding); the bf16 result adds one
bf16 ulp.  For the two-layer chain, the intermediate's own error (one bf16 ulp plus its
accumulation bound) is carried through the temporal weights.
"""
import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from oracle import conv as oconv
from tests.helpers import U, check_bf16, to_device, ulp_bf16

pytestmark = pytest.mark.gpu


def bf16_input(shape, seed, std=1.0):
    a = synth.normal(shape, seed=seed, std=std, dtype=synth.BF16)
    return a, synth.to_f64(a, synth.BF16)


def as_f64(t):
    return t.to(torch.float64).cpu().numpy()


@pytest.mark.parametrize("shape,Cout", [((1, 3, 12, 20, 64), 64), ((2, 2, 9, 33, 192), 256), ((1, 1, 1, 1, 64), 128)])
def test_spatial_matches_oracle(shape, Cout):
    B, T, h, w, Cin = shape
    x, x64 = bf16_input(shape, seed=101)
    ws, ws64 = bf16_input((Cout, 3, 3, Cin), seed=103, std=(9 * Cin) ** -0.5)
    y = torch.empty((B, T, h, w, Cout), dtype=torch.bfloat16, device="cuda")
    hwp.tok_conv_spatial(to_device(x, synth.BF16), to_device(ws, synth.BF16), y)
    hwp.tok_check_device()
    ref = oconv.spatial_conv(x64, ws64)
    check_bf16(as_f64(y), ref, 2 * 9 * Cin * U * oconv.spatial_conv(np.abs(x64), np.abs(ws64)), "spatial")


@pytest.mark.parametrize("shape,Cout", [((2, 7, 6, 10, 64), 128), ((1, 4, 16, 16, 256), 256), ((1, 1, 4, 4, 64), 64)])
def test_temporal_causal_matches_oracle(shape, Cout):
    B, T, h, w, Cin = shape
    x, x64 = bf16_input(shape, seed=107)
    wt, wt64 = bf16_input((Cout, 3, Cin), seed=109, std=(3 * Cin) ** -0.5)
    y = torch.empty((B, T, h, w, Cout), dtype=torch.bfloat16, device="cuda")
    hwp.tok_conv_temporal_causal(to_device(x, synth.BF16), to_device(wt, synth.BF16), y)
    hwp.tok_check_device()
    ref = oconv.temporal_causal_conv(x64, wt64)
    check_bf16(as_f64(y), ref, 2 * 3 * Cin * U * oconv.temporal_causal_conv(np.abs(x64), np.abs(wt64)), "temporal")


def factorized_tolerance(x64, ws64, wt64):
    """The oracle chain and the fp32 error of the kernels' value before the final bf16 rounding:
    the temporal layer's accumulation plus the intermediate's own error (its bf16 rounding and
    accumulation bound) carried through the temporal weights."""
    Cin, Cmid = x64.shape[-1], ws64.shape[0]
    s = oconv.spatial_conv(x64, ws64)
    s_err = ulp_bf16(s) + 2 * 9 * Cin * U * oconv.spatial_conv(np.abs(x64), np.abs(ws64))
    ref = oconv.temporal_causal_conv(oconv.round_bf16(s), wt64)
    E = (2 * 3 * Cmid * U * oconv.temporal_causal_conv(np.abs(s), np.abs(wt64))
         + oconv.temporal_causal_conv(s_err, np.abs(wt64)))
    return ref, E


def test_factorized_matches_oracle():
    B, T, h, w, Cin, Cmid, Cout = 1, 5, 8, 16, 192, 256, 256
    x, x64 = bf16_input((B, T, h, w, Cin), seed=113)
    ws, ws64 = bf16_input((Cmid, 3, 3, Cin), seed=127, std=(9 * Cin) ** -0.5)
    wt, wt64 = bf16_input((Cout, 3, Cmid), seed=131, std=(3 * Cmid) ** -0.5)
    y = hwp.conv_factorized(to_device(x, synth.BF16), to_device(ws, synth.BF16), to_device(wt, synth.BF16))
    hwp.tok_check_device()
    ref, E = factorized_tolerance(x64, ws64, wt64)
    check_bf16(as_f64(y), ref, E, "factorized")


def test_patcher_then_convolution():
    """Pixels -> channels-last patcher -> factorized convolution, against the oracle chain.
    The patcher's bf16 coefficients may differ from the oracle's rounded ones by one ulp plus
    its butterfly bound; that difference is carried through both convolutions."""
    B, C, T, H, W = 1, 3, 9, 32, 64
    xp = synth.uniform((B, C, T, H, W), seed=137, dtype=synth.BF16)
    xp64 = synth.to_f64(xp, synth.BF16)
    Cin, Cmid, Cout = 192, 64, 64
    ws, ws64 = bf16_input((Cmid, 3, 3, Cin), seed=139, std=(9 * Cin) ** -0.5)
    wt, wt64 = bf16_input((Cout, 3, Cmid), seed=149, std=(3 * Cmid) ** -0.5)
    y_cl = hwp.haar_fwd_channels_last(to_device(xp, synth.BF16))
    out = hwp.conv_factorized(y_cl, to_device(ws, synth.BF16), to_device(wt, synth.BF16))
    hwp.tok_check_device()
    coeff = oconv.round_bf16(oracle.haar_fwd_channels_last(xp64))
    # the patcher's error per coefficient: one bf16 ulp plus 6 butterfly stages on the block's 64 pixels
    blocks = np.abs(xp64).reshape(B, C, T, H // 4, 4, W // 4, 4).sum(axis=(4, 6))
    Tq = 1 + (T - 1) // 4
    bs = np.empty((B, C, Tq, H // 4, W // 4))
    bs[:, :, 0] = 4 * blocks[:, :, 0]
    bs[:, :, 1:] = blocks[:, :, 1:].reshape(B, C, Tq - 1, 4, H // 4, W // 4).sum(axis=3)
    c_err = 2 * ulp_bf16(coeff) + 6 * U * np.moveaxis(np.concatenate([bs] * 64, axis=1), 1, -1) / 8 * 1.01
    ref, E = factorized_tolerance(coeff, ws64, wt64)
    carried = oconv.temporal_causal_conv(oconv.spatial_conv(c_err, np.abs(ws64)), np.abs(wt64))
    check_bf16(as_f64(out), ref, E + carried, "patcher -> factorized")


# ---------------------------------------------------------------------------
# The hand-written tensor-core kernels: more tile shapes, several output-channel tiles, k = 5.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape,Cout,k", [((1, 3, 20, 24, 128), 512, 3), ((2, 2, 17, 9, 64), 96, 3),
                                          ((1, 2, 12, 16, 64), 32, 5)],
                         ids=["two channel tiles", "ragged tiles", "k=5"])
def test_spatial_tile_shapes(shape, Cout, k):
    B, T, h, w, Cin = shape
    x, x64 = bf16_input(shape, seed=151)
    ws, ws64 = bf16_input((Cout, k, k, Cin), seed=157, std=(k * k * Cin) ** -0.5)
    y = torch.empty((B, T, h, w, Cout), dtype=torch.bfloat16, device="cuda")
    hwp.tok_conv_spatial(to_device(x, synth.BF16), to_device(ws, synth.BF16), y)
    hwp.tok_check_device()
    ref = oconv.spatial_conv(x64, ws64)
    check_bf16(as_f64(y), ref, 2 * k * k * Cin * U * oconv.spatial_conv(np.abs(x64), np.abs(ws64)), "spatial")


@pytest.mark.parametrize("shape,Cout,k", [((2, 5, 17, 9, 64), 96, 3), ((1, 6, 8, 8, 128), 512, 3),
                                          ((2, 7, 4, 12, 64), 64, 5)],
                         ids=["ragged tiles, two clips", "two channel tiles", "k=5"])
def test_temporal_tile_shapes(shape, Cout, k):
    B, T, h, w, Cin = shape
    x, x64 = bf16_input(shape, seed=163)
    wt, wt64 = bf16_input((Cout, k, Cin), seed=167, std=(k * Cin) ** -0.5)
    y = torch.empty((B, T, h, w, Cout), dtype=torch.bfloat16, device="cuda")
    hwp.tok_conv_temporal_causal(to_device(x, synth.BF16), to_device(wt, synth.BF16), y)
    hwp.tok_check_device()
    ref = oconv.temporal_causal_conv(x64, wt64)
    check_bf16(as_f64(y), ref, 2 * k * Cin * U * oconv.temporal_causal_conv(np.abs(x64), np.abs(wt64)), "temporal")


# ---------------------------------------------------------------------------
# The patcher fused into the spatial convolution.
# ---------------------------------------------------------------------------
def patcher_coeff_error(xp64, coeff):
    """Per coefficient: how far the kernel's bf16 coefficient may be from the oracle's coefficient
    rounded to bf16 -- two bf16 ulps plus the 6-stage butterfly bound of its block's 64 pixels."""
    B, C, T, H, W = xp64.shape
    blocks = np.abs(xp64).reshape(B, C, T, H // 4, 4, W // 4, 4).sum(axis=(4, 6))
    Tq = 1 + (T - 1) // 4
    bs = np.empty((B, C, Tq, H // 4, W // 4))
    bs[:, :, 0] = 4 * blocks[:, :, 0]
    bs[:, :, 1:] = blocks[:, :, 1:].reshape(B, C, Tq - 1, 4, H // 4, W // 4).sum(axis=3)
    return 2 * ulp_bf16(coeff) + 6 * U * np.moveaxis(np.concatenate([bs] * 64, axis=1), 1, -1) / 8 * 1.01


EMBED = [((1, 3, 9, 64, 64), 256, "three colours, whole tiles"),
         ((2, 2, 13, 36, 72), 64, "ragged tiles, two clips"),
         ((1, 1, 5, 16, 32), 512, "two channel tiles"),
         ((1, 4, 5, 68, 40), 128, "four colours, ragged rows"),
         ((1, 8, 9, 16, 24), 32, "eight colours, the smallest channel tile")]


@pytest.mark.parametrize("shape,Cmid,note", EMBED, ids=[e[2] for e in EMBED])
def test_patch_embed_matches_oracle_chain(shape, Cmid, note):
    """Pixels -> fused patcher + 1x3x3 convolution, against the oracle patcher (rounded to bf16, as the
    kernel rounds its coefficients) and the oracle convolution.  The kernel's coefficients may differ
    from the oracle's rounded ones by patcher_coeff_error, carried through the filter."""
    B, C, T, H, W = shape
    xp = synth.uniform(shape, seed=173 + C, dtype=synth.BF16)
    xp64 = synth.to_f64(xp, synth.BF16)
    Cin = 64 * C
    ws, ws64 = bf16_input((Cmid, 3, 3, Cin), seed=179, std=(9 * Cin) ** -0.5)
    wp = hwp.patch_embed_pack_weights(to_device(ws, synth.BF16))
    y = hwp.patch_embed_spatial(to_device(xp, synth.BF16), wp)
    hwp.tok_check_device()
    coeff = oconv.round_bf16(oracle.haar_fwd_channels_last(xp64))
    ref = oconv.spatial_conv(coeff, ws64)
    E = (2 * 9 * Cin * U * oconv.spatial_conv(np.abs(coeff), np.abs(ws64))
         + oconv.spatial_conv(patcher_coeff_error(xp64, coeff), np.abs(ws64)))
    strict = check_bf16(as_f64(y), ref, E, note)
    print(f"{note}: {strict} of {y.numel()} outputs beyond a plain 1 bf16 ulp")


def test_packed_filter_layout():
    """wp[n][(c*3 + dx)*3 + dy][g] = ws[n][dy][dx][g*C + c], bit for bit."""
    C, Cmid = 3, 64
    ws = torch.randn((Cmid, 3, 3, 64 * C), device="cuda").to(torch.bfloat16)
    wp = hwp.patch_embed_pack_weights(ws)
    torch.cuda.synchronize()
    ref = ws.view(Cmid, 3, 3, 64, C).permute(0, 4, 2, 1, 3).reshape(Cmid, 9 * C, 64)
    assert torch.equal(wp, ref)
