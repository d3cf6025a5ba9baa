"""Parity at the sizes bench.py times, for the calls it measures beyond the headline step.

Each sampled expected value comes from the oracle on a small crop of the full input,
which is exact because of the transform's structure (pinned in the oracle tests): a
latent window depends only on its own 4 (2) frames and 4x4 (2x2) pixels, a continuation
chunk of 4 frames is exactly one window, and a 3x3 convolution's output depends only on
a one-block margin.  The FSQ gradients at the full 64-grid latent are compared in full.
"""
import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from oracle import conv as oconv
from tests.helpers import U, check_bf16, haar_fp32_bound, to_device, ulp_bf16

pytestmark = pytest.mark.gpu

CLIP = (1, 3, 121, 704, 1280)
SAMPLES = [(0, 0, 0), (0, 87, 160), (1, 175, 319), (2, 40, 1), (3, 0, 319), (15, 88, 160), (30, 175, 0),
           (30, 1, 318), (17, 120, 250), (8, 64, 64)]


@pytest.fixture(scope="module")
def clip():
    x = synth.haar_input(3)
    return x, to_device(x, synth.BF16)


def pixels(x, f0, f1, r0, r1, c0, c1):
    return synth.bf16_bits_to_f64(x[:, :, f0:f1, r0:r1, c0:c1])


def window_coeffs(x, tq, i, j, frames=None):
    """Oracle coefficients [1, 64C] of latent window tq at block (i, j); frames: source frame of each
    of the window's 4 samples (default 4tq-3 .. 4tq)."""
    if tq == 0 and frames is None:
        crop = pixels(x, 0, 1, 4 * i, 4 * i + 4, 4 * j, 4 * j + 4)
        return oracle.haar_fwd_chunk(crop, first=True)[:, :, 0, 0, 0]
    fr = frames if frames is not None else list(range(4 * tq - 3, 4 * tq + 1))
    crop = np.concatenate([pixels(x, f, f + 1, 4 * i, 4 * i + 4, 4 * j, 4 * j + 4) for f in fr], axis=2)
    return oracle.haar_fwd_chunk(crop, first=False)[:, :, 0, 0, 0]


def test_conv_chain_full_size_sampled(clip):
    """Headline clip -> channels-last patcher -> factorized convolution (bench.py patch_embed)."""
    x, xd = clip
    y_cl = hwp.haar_fwd_channels_last(xd)
    assert torch.equal(y_cl, hwp.haar_fwd(xd).permute(0, 2, 3, 4, 1))
    Cin, Cmid, Cout = 192, 256, 256
    ws = synth.normal((Cmid, 3, 3, Cin), seed=211, std=(9 * Cin) ** -0.5, dtype=synth.BF16)
    wt = synth.normal((Cout, 3, Cmid), seed=223, std=(3 * Cmid) ** -0.5, dtype=synth.BF16)
    ws64, wt64 = synth.to_f64(ws, synth.BF16), synth.to_f64(wt, synth.BF16)
    out = hwp.conv_factorized(y_cl, to_device(ws, synth.BF16), to_device(wt, synth.BF16))
    hwp.tok_check_device()
    _, Tq, h, w, _ = y_cl.shape
    for (t, i, j) in SAMPLES:
        i0, i1, j0, j1 = max(0, i - 1), min(h, i + 2), max(0, j - 1), min(w, j + 2)
        a = max(0, t - 2)
        # oracle coefficients of latent frames a..t over the blocks (i0..i1, j0..j1)
        if a == 0:
            crop = pixels(x, 0, 4 * t + 1, 4 * i0, 4 * i1, 4 * j0, 4 * j1)
            cf = oracle.haar_fwd_chunk(crop, first=True)
        else:
            crop = pixels(x, 4 * a - 3, 4 * t + 1, 4 * i0, 4 * i1, 4 * j0, 4 * j1)
            cf = oracle.haar_fwd_chunk(crop, first=False)
        coeff = np.moveaxis(cf, 1, -1)                                   # [1, nt, nh, nw, 192]
        cb = oconv.round_bf16(coeff)
        # the patcher's own error per coefficient, carried through both convolutions
        blk = np.abs(crop).reshape(1, 3, crop.shape[2], i1 - i0, 4, j1 - j0, 4).sum(axis=(4, 6))
        nt = coeff.shape[1]
        if a == 0:
            bs = np.concatenate([4 * blk[:, :, :1], blk[:, :, 1:].reshape(1, 3, nt - 1, 4, i1 - i0, j1 - j0).sum(axis=3)],
                                axis=2) if nt > 1 else 4 * blk[:, :, :1]
        else:
            bs = blk.reshape(1, 3, nt, 4, i1 - i0, j1 - j0).sum(axis=3)
        c_err = 2 * ulp_bf16(cb) + 6 * U * np.moveaxis(np.concatenate([bs] * 64, axis=1), 1, -1) / 8 * 1.01
        s = oconv.spatial_conv(cb, ws64)[0, :, i - i0, j - j0]           # [nt, Cmid]
        s_abs = oconv.spatial_conv(np.abs(cb), np.abs(ws64))[0, :, i - i0, j - j0]
        s_err = (ulp_bf16(s) + 2 * 9 * Cin * U * s_abs
                 + oconv.spatial_conv(c_err, np.abs(ws64))[0, :, i - i0, j - j0])
        sb = oconv.round_bf16(s)
        ref = np.zeros(Cout)
        t_abs = np.zeros(Cout)
        carried = np.zeros(Cout)
        for dt in range(3):
            f = t - 2 + dt
            if f < 0:
                continue
            ref += wt64[:, dt, :] @ sb[f - a]
            t_abs += np.abs(wt64[:, dt, :]) @ np.abs(sb[f - a])
            carried += np.abs(wt64[:, dt, :]) @ s_err[f - a]
        got = out[0, t, i, j].double().cpu().numpy()
        check_bf16(got, ref, 2 * 3 * Cmid * U * t_abs + carried, f"sample {(t, i, j)}")


def test_patch_embed_full_size(clip):
    """Headline clip through the fused patcher + 1x3x3 convolution (bench.py patch_embed_fused):
    every output against the two-call chain (channels-last patcher, then tok_conv_spatial) -- the
    same bf16 coefficients summed in another order, so each pair differs by at most two fp32
    accumulation bounds plus the bf16 rounding -- and sampled outputs against the oracle chain."""
    import torch.nn.functional as F
    x, xd = clip
    Cin, Cmid = 192, 256
    ws = synth.normal((Cmid, 3, 3, Cin), seed=211, std=(9 * Cin) ** -0.5, dtype=synth.BF16)
    ws64 = synth.to_f64(ws, synth.BF16)
    wsd = to_device(ws, synth.BF16)
    y = hwp.patch_embed_spatial(xd, hwp.patch_embed_pack_weights(wsd))
    y_cl = hwp.haar_fwd_channels_last(xd)
    mid = torch.empty_like(y)
    hwp.tok_conv_spatial(y_cl, wsd, mid)
    hwp.tok_check_device()
    _, Tq, h, w, _ = y_cl.shape
    with torch.backends.cudnn.flags(enabled=True, allow_tf32=False):
        a = y_cl[0].float().abs().permute(0, 3, 1, 2)                        # [Tq, Cin, h, w]
        S = F.conv2d(a, wsd.float().abs().permute(0, 3, 1, 2), padding=1)     # sum |c| |w| per output
    E = (2 * 2 * 9 * Cin * U * 1.01) * S.permute(0, 2, 3, 1).double()
    m = mid[0].double()
    tol = torch.maximum(torch.ldexp(torch.ones_like(m), torch.frexp((m.abs() + E).clamp(min=2.0 ** -126))[1] - 8),
                        torch.zeros_like(m)) + E
    bad = int(((y[0].double() - m).abs() > tol).sum())
    assert bad == 0, f"{bad} fused outputs differ from the two-call chain beyond the accumulation bounds"
    del a, S, E, m, tol
    for (t, i, j) in SAMPLES:
        i0, i1, j0, j1 = max(0, i - 1), min(h, i + 2), max(0, j - 1), min(w, j + 2)
        if t == 0:
            crop = pixels(x, 0, 1, 4 * i0, 4 * i1, 4 * j0, 4 * j1)
            cf = oracle.haar_fwd_chunk(crop, first=True)
        else:
            crop = pixels(x, 4 * t - 3, 4 * t + 1, 4 * i0, 4 * i1, 4 * j0, 4 * j1)
            cf = oracle.haar_fwd_chunk(crop, first=False)
        cb = oconv.round_bf16(np.moveaxis(cf, 1, -1))                      # [1, 1, nh, nw, 192]
        blk = np.abs(crop).reshape(1, 3, crop.shape[2], i1 - i0, 4, j1 - j0, 4).sum(axis=(4, 6))
        bs = 4 * blk if t == 0 else blk.reshape(1, 3, 1, 4, i1 - i0, j1 - j0).sum(axis=3)
        c_err = 2 * ulp_bf16(cb) + 6 * U * np.moveaxis(np.concatenate([bs] * 64, axis=1), 1, -1) / 8 * 1.01
        ref = oconv.spatial_conv(cb, ws64)[0, 0, i - i0, j - j0]
        E = (2 * 9 * Cin * U * oconv.spatial_conv(np.abs(cb), np.abs(ws64))[0, 0, i - i0, j - j0]
             + oconv.spatial_conv(c_err, np.abs(ws64))[0, 0, i - i0, j - j0])
        check_bf16(y[0, t, i, j].double().cpu().numpy(), ref, E, f"fused sample {(t, i, j)}")


def test_padded_and_chunk_full_size_sampled():
    """bench.py streaming: [1,3,120,720,1280] padded to 121 frames (spatial 16, temporal 8), and as one
    continuation chunk."""
    shape = (1, 3, 120, 720, 1280)
    x = synth.uniform(shape, seed=233, dtype=synth.BF16)
    xd = to_device(x, synth.BF16)
    yp = hwp.haar_fwd_padded(xd, 16, 8)
    yc = hwp.haar_fwd_chunk(xd, first=False)
    hwp.tok_check_device()
    assert tuple(yp.shape) == (1, 192, 31, 180, 320) and tuple(yc.shape) == (1, 192, 30, 180, 320)
    for (tq, i, j) in [(0, 0, 0), (1, 90, 100), (29, 179, 319), (30, 0, 319), (30, 100, 5)]:
        frames = None if tq < 30 else [117, 118, 119, 118]  # frame 120 mirrors frame 118
        ref = window_coeffs(x, tq, i, j, frames)[0]
        got = yp[0, :, tq, i, j].double().cpu().numpy()
        bsum = np.abs(pixels(x, 0, 1, 4 * i, 4 * i + 4, 4 * j, 4 * j + 4)).sum() * 4 if tq == 0 else \
            sum(np.abs(pixels(x, f, f + 1, 4 * i, 4 * i + 4, 4 * j, 4 * j + 4)).sum()
                for f in (frames or range(4 * tq - 3, 4 * tq + 1)))
        check_bf16(got, ref, haar_fp32_bound(bsum, True), f"padded window {(tq, i, j)}")
        if tq < 30:  # continuation window q reads frames 4q .. 4q + 3
            refc = window_coeffs(x, 0, i, j, list(range(4 * tq, 4 * tq + 4)))[0]
            gotc = yc[0, :, tq, i, j].double().cpu().numpy()
            bs = sum(np.abs(pixels(x, f, f + 1, 4 * i, 4 * i + 4, 4 * j, 4 * j + 4)).sum() for f in range(4 * tq, 4 * tq + 4))
            check_bf16(gotc, refc, haar_fp32_bound(bs, True), f"chunk window {(tq, i, j)}")
    # the cropped inverse: the last window rebuilds frames 117..119 (its fourth sample is cropped)
    xr = hwp.haar_inv_cropped(yp, 120, 720, 1280, 16, 8)
    hwp.tok_check_device()
    for (i, j) in [(0, 0), (179, 319), (60, 200)]:
        coef = yp[0, :, 30, i, j].double().cpu().numpy().reshape(1, 192, 1, 1, 1)
        ref = oracle.haar_inv_chunk(coef, 4, 4, 4, first=False)[0, :, :3]
        got = xr[0, :, 117:120, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
        per_c = np.abs(coef).reshape(64, 3).sum(axis=0)[:, None, None, None]  # channel c's 64 coefficients
        check_bf16(got, ref, haar_fp32_bound(per_c, True), f"cropped inverse block {(i, j)}")


def test_single_level_full_size_sampled(clip):
    x, xd = clip
    y1 = hwp.haar_fwd_single(xd)
    hwp.tok_check_device()
    assert tuple(y1.shape) == (1, 24, 61, 352, 640)
    for (tq, i, j) in [(0, 0, 0), (1, 100, 200), (60, 351, 639), (33, 17, 300)]:
        f0 = 0 if tq == 0 else 2 * tq - 2
        crop = pixels(x, f0, f0 + 3, 2 * i, 2 * i + 2, 2 * j, 2 * j + 2)[0]      # [3, 3 frames, 2, 2]
        ref = oracle.haar_level_fwd(crop)[:, 0 if tq == 0 else 1, 0, 0]
        got = y1[0, :, tq, i, j].double().cpu().numpy()
        s = np.abs(crop[:, [0, 0]] if tq == 0 else crop[:, 1:]).sum(axis=(1, 2, 3))
        check_bf16(got, ref, 5 * U * np.tile(s, 8) * 2 ** -1.5 * 1.01, f"single-level window {(tq, i, j)}")


def test_adjoints_full_size_sampled():
    """bench.py gradients: the adjoints at the headline sizes, sampled blocks."""
    T, H, W = 121, 704, 1280
    gy = (torch.rand((1, 192, 31, 176, 320), device="cuda") * 2 - 1).to(torch.bfloat16)
    gx = hwp.haar_fwd_adjoint(gy, T, H, W)
    g2 = (torch.rand((1, 3, T, H, W), device="cuda") * 2 - 1).to(torch.bfloat16)
    gyy = hwp.haar_inv_adjoint(g2)
    hwp.tok_check_device()
    for (tq, i, j) in [(0, 0, 0), (1, 50, 60), (30, 175, 319), (12, 3, 7)]:
        cw = gy[0, :, tq, i, j].double().cpu().numpy().reshape(1, 192, 1, 1, 1)
        if tq == 0:  # frame 0 collects window 0's four samples: the adjoint on a 5-frame crop
            two = np.zeros((1, 192, 2, 1, 1))
            two[:, :, 0] = cw[:, :, 0]
            ref = oracle.haar_fwd_adjoint(two, 5, 4, 4)[0, :, :1]
            got = gx[0, :, :1, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
            d = 36
        else:        # an orthonormal window: the adjoint is the inverse of the window
            ref = oracle.haar_inv_chunk(cw, 4, 4, 4, first=False)[0]
            got = gx[0, :, 4 * tq - 3:4 * tq + 1, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
            d = 6
        check_bf16(got, ref, d * U * np.abs(cw).reshape(64, 3).sum(axis=0)[:, None, None, None] / 8 * 1.01,
                   f"patcher adjoint window {(tq, i, j)}")
        # the unpatcher's adjoint: window tq >= 1 is the forward transform of its 4 frames; window 0 sees
        # (0, 0, 0, frame 0)
        px = g2[:, :, max(0, 4 * tq - 3):4 * tq + 1, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
        if tq == 0:
            five = np.zeros((1, 3, 5, 4, 4))
            five[:, :, 0] = px[:, :, 0]
            ref = oracle.haar_inv_adjoint(five)[0, :, 0, 0, 0]
            s = np.tile(np.abs(px[0, :, 0]).sum(axis=(1, 2)), 64)
        else:
            ref = oracle.haar_fwd_chunk(px, first=False)[0, :, 0, 0, 0]
            s = np.tile(np.abs(px[0]).sum(axis=(1, 2, 3)), 64)
        got = gyy[0, :, tq, i, j].double().cpu().numpy()
        check_bf16(got, ref, 6 * U * s / 8 * 1.01, f"unpatcher adjoint {(tq, i, j)}")


def test_fsq_backward_full_latent():
    """bench.py gradients: the FSQ backward on the full [64, 16, 56320] latent, every output."""
    u = synth.fsq_input(4)
    w = synth.fsq_weight()
    g = synth.normal((64, 6, 56320), seed=239)
    gu, gw = hwp.fsq_encode_backward(torch.from_numpy(u).cuda(), torch.from_numpy(w).cuda(),
                                     torch.from_numpy(g).cuda())
    hwp.tok_check_device()
    ref_u, ref_w = oracle.fsq_encode_backward(u, w, g)
    scale = np.array([(L - 1) * 1.001 / 2 / (L // 2) for L in (8, 8, 8, 5, 5, 5)])
    gs = np.abs(g.astype(np.float64)) * scale[None, :, None]
    tol_u = 1e-5 * np.einsum("ic,bis->bcs", np.abs(w.astype(np.float64)), gs) + 1e-30
    assert (np.abs(gu.double().cpu().numpy() - ref_u) <= tol_u).all()
    tol_w = 1e-5 * np.einsum("bis,bcs->ic", gs, np.abs(u.astype(np.float64))) + 1e-30
    assert (np.abs(gw.double().cpu().numpy() - ref_w) <= tol_w).all()


def test_image_beyond_the_tile_kernels_limits():
    """A [1,1,1,32768,32768] bf16 image (2 GB): its 2^26 latent pixels put the 64 planes of a
    channel past the 32-bit element offsets the TMA kernels use, so the vectorized register
    kernels take it.  Checked bit for bit against the TMA kernels on 4096-row strips (tensors of
    their own), and on sampled blocks against the oracle."""
    H = W = 32768
    g = torch.Generator(device="cuda").manual_seed(7)
    x = (torch.rand((1, 1, 1, H, W), generator=g, device="cuda") * 2 - 1).to(torch.bfloat16)
    y = hwp.haar_fwd(x)
    xr = hwp.haar_inv(y, 1, H, W)
    hwp.tok_check_device()
    assert y.shape == (1, 16, 1, H // 4, W // 4)
    for r0 in (0, H - 4096):
        strip = x[:, :, :, r0:r0 + 4096].contiguous()
        ys = hwp.haar_fwd(strip)
        assert torch.equal(ys, y[:, :, :, r0 // 4:r0 // 4 + 1024])
        xs = hwp.haar_inv(ys, 1, 4096, W)
        assert torch.equal(xs, xr[:, :, :, r0:r0 + 4096])
        del strip, ys, xs
    rng = np.random.default_rng(7)
    pos = [(int(rng.integers(H // 4)), int(rng.integers(W // 4))) for _ in range(400)]
    pos += [(0, 0), (0, W // 4 - 1), (H // 4 - 1, 0), (H // 4 - 1, W // 4 - 1)]
    blocks = np.stack([x[0, 0, 0, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy() for i, j in pos])
    ref = oracle.haar_fwd(blocks[:, None, None])  # [n, 16, 1, 1, 1]
    got = np.stack([y[0, :, 0, i, j].double().cpu().numpy() for i, j in pos])
    check_bf16(got, ref[:, :, 0, 0, 0], haar_fp32_bound(np.abs(blocks).sum(axis=(1, 2))[:, None], False),
               "32768x32768 image")
    del x, y, xr
    torch.cuda.empty_cache()
