"""GPU parity of tok_fsq_encode / tok_fsq_decode against the CPU oracle.

Indices must match bit for bit except on tokens the oracle flags as lying
within 1e-5 of a rounding boundary; those mismatches are counted and capped at
1e-6 of the tokens.  Codes must equal q / floor(L/2) of the GPU's own digits
and match the oracle where the index does.  Decode is compared with the
oracle's double-precision projection within the fp32 bound of a 6-term chain.
"""
import math

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import U

pytestmark = pytest.mark.gpu

LEVELS = (8, 8, 8, 5, 5, 5)
BASIS = (1, 8, 64, 512, 2560, 12800)


def encode_gpu(u_np, w_np, with_codes=True):
    u = torch.from_numpy(u_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    idx, codes = hwp.fsq_encode(u, w, with_codes=True) if with_codes else (hwp.fsq_encode(u, w), None)
    hwp.tok_check_device()
    return idx.cpu().numpy(), (codes.cpu().numpy() if codes is not None else None)


def check_encode(u_np, w_np, label):
    ref_idx, ref_codes, near = oracle.fsq_encode(u_np, w_np)
    idx, codes = encode_gpu(u_np, w_np)
    idx = idx.reshape(ref_idx.shape)
    codes = codes.reshape(ref_codes.shape)
    mism = idx != ref_idx
    n = idx.size
    assert not (mism & ~near).any(), f"{label}: {(mism & ~near).sum()} index mismatches away from a boundary"
    assert mism.sum() <= math.floor(1e-6 * n), f"{label}: {mism.sum()} near-boundary mismatches of {n} tokens"
    assert ((idx >= 0) & (idx < 64000)).all()
    # codes agree with the GPU's own digits, and with the oracle where the index agrees
    digits = np.stack([(idx // BASIS[i]) % LEVELS[i] for i in range(6)], axis=1)
    half = np.array([L // 2 for L in LEVELS])[None, :, None]
    np.testing.assert_array_equal(codes, (digits - half) / half)
    np.testing.assert_array_equal(codes.transpose(0, 2, 1)[~mism], ref_codes.transpose(0, 2, 1)[~mism])
    return idx, int(near.sum()), int(mism.sum())


def check_decode(idx_np, w_np, label):
    ref, bad_ref = oracle.fsq_decode(idx_np, w_np)
    idx = torch.from_numpy(idx_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = hwp.fsq_decode(idx, w, bad_count=bad)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    assert int(bad.item()) == bad_ref, label
    nan_ref = np.isnan(ref)
    assert (np.isnan(got) == nan_ref).all(), label
    # bound of the fp32 chain: 8 u sum_i |w_ic zhat_i| <= 8 u sum_i |w_ic| (|zhat| <= 1)
    tol = 8 * U * np.abs(w_np.astype(np.float64)).sum(axis=0)[None, :, None] + 1e-30
    err = np.where(nan_ref, 0.0, np.abs(got - np.where(nan_ref, 0.0, ref)))
    assert (err <= tol).all(), f"{label}: decode max err {err.max():.3g}"
    return got


LATENTS = {1: "latent [1,16,4096]", 2: "latent [16,16,4096] (image batch)", 4: "latent [64,16,56320]",
           5: "latent [4,16,130560] (stress clips)"}  # synth workload keys


@pytest.mark.parametrize("cfg", list(LATENTS), ids=[LATENTS[k] for k in LATENTS])
def test_encode_decode_latents(cfg):
    u = synth.fsq_input(cfg)
    w = synth.fsq_weight(u.shape[1])
    idx, n_near, n_mism = check_encode(u, w, LATENTS[cfg])
    print(f"{LATENTS[cfg]}: {idx.size} tokens, {n_near} near a boundary, {n_mism} mismatches")
    check_decode(idx, w, LATENTS[cfg])


@pytest.mark.parametrize("B,C,S", [(3, 16, 4100), (2, 16, 132), (1, 16, 128), (3, 16, 4097), (2, 16, 1), (1, 3, 1000),
                                   (2, 40, 512), (1, 1, 8), (5, 6, 999)])
def test_encode_decode_shapes(B, C, S):
    """C = 16 with S % 4 == 0 takes the TMA encode (ragged last tile when S % 128 != 0); odd S takes the
    element-wise kernels; C != 16 the runtime-channel kernels; tiny sizes."""
    u = synth.normal((B, C, S), seed=B * 1000 + C * 10 + S, std=1.5)
    w = synth.fsq_weight(C, seed=C)
    idx, _, _ = check_encode(u, w, f"B={B} C={C} S={S}")
    check_decode(idx, w, f"B={B} C={C} S={S}")


def test_thresholds_exactly_at_boundaries():
    """z equal to the fp32 values around every rounding boundary, with W = I (z_i = u_i exactly)."""
    zs = []
    for L in (8, 5):
        half = (L - 1) * (1 + 1e-3) / 2
        off = 0.5 if L % 2 == 0 else 0.0
        shift = math.atanh(off / half)
        for m in range(L - 1):
            theta = math.atanh((-(L // 2) + m + 0.5 + off) / half) - shift
            f = np.float32(theta)
            for k in range(-3, 4):
                v = f
                for _ in range(abs(k)):
                    v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf))
                zs.append(v)
    # (no infinities: 0 * inf in the projection chain would be NaN, which has no code)
    zs += [np.float32(0.0), np.float32(-0.0), np.float32(1e30), np.float32(-1e30)]
    zs = np.array(zs, np.float32)
    u = np.zeros((1, 6, zs.size), np.float32)
    for i in range(6):
        u[0, i] = np.roll(zs, 7 * i)
    w = np.eye(6, dtype=np.float32)
    ref_idx, _, near = oracle.fsq_encode(u, w)
    idx, _ = encode_gpu(u, w)
    assert (idx.reshape(ref_idx.shape) == ref_idx).all()


def test_one_hot_projection_and_extremes():
    C = 16
    perm = [11, 2, 7, 0, 15, 5]
    w = np.zeros((6, C), np.float32)
    for i, c in enumerate(perm):
        w[i, c] = 1.0
    u = synth.normal((2, C, 1024), seed=77, std=1.5)
    u[0, :, 0] = 0.0
    u[0, :, 1] = 1e6
    u[0, :, 2] = -1e6
    idx, _, _ = check_encode(u, w, "one-hot")
    assert idx[0, :3].tolist() == [32036, 63999, 0]


def test_decode_invalid_indices_give_nan_and_count():
    w = synth.fsq_weight(16)
    idx = np.array([[0, -1, 64000, 63999, 2 ** 31 - 1, 32036, -(2 ** 31), 12345]], np.int32)
    got = check_decode(idx, w, "invalid")
    assert np.isnan(got[0, :, [1, 2, 4, 6]]).all() and not np.isnan(got[0, :, [0, 3, 5, 7]]).any()


def test_decode_inverts_encode_on_centres():
    rng = np.random.default_rng(5)
    S = 4096
    q = np.stack([rng.integers(-(L // 2), (L + 1) // 2, S) for L in LEVELS])
    z = np.zeros((6, S))
    for i, L in enumerate(LEVELS):
        half = (L - 1) * (1 + 1e-3) / 2
        off = 0.5 if L % 2 == 0 else 0.0
        z[i] = np.arctanh((q[i] + off) / half) - math.atanh(off / half)
    u = z.astype(np.float32)[None]
    w = np.eye(6, dtype=np.float32)
    idx, codes = encode_gpu(u, w)
    out = hwp.fsq_decode(torch.from_numpy(idx).cuda(), torch.from_numpy(w).cuda())
    zhat = q / np.array([L // 2 for L in LEVELS])[:, None]
    np.testing.assert_array_equal(out.cpu().numpy()[0], zhat)
    np.testing.assert_array_equal(codes[0], zhat)


def test_tma_and_register_encode_agree_bitwise():
    """The TMA encode (aligned, C = 16) and the register encode (a misaligned view) give identical results."""
    u = synth.fsq_input(2)
    w = torch.from_numpy(synth.fsq_weight()).cuda()
    ud = torch.from_numpy(u).cuda()
    idx_tma, codes_tma = hwp.fsq_encode(ud, w, with_codes=True)
    buf = torch.empty(ud.numel() + 1, device="cuda")
    buf[1:].copy_(ud.reshape(-1))
    idx_reg, codes_reg = hwp.fsq_encode(buf[1:].view(ud.shape), w, with_codes=True)
    hwp.tok_check_device()
    assert torch.equal(idx_tma, idx_reg) and torch.equal(codes_tma, codes_reg)


def test_encode_without_codes_and_empty():
    u = synth.fsq_input(1)
    w = synth.fsq_weight()
    idx, _ = encode_gpu(u, w, with_codes=False)
    ref, _, _ = oracle.fsq_encode(u, w)
    assert (idx.reshape(ref.shape) == ref).all()
    e = hwp.fsq_encode(torch.empty(0, 16, 5, device="cuda"), torch.from_numpy(w).cuda())
    assert e.shape == (0, 5)
