"""GPU parity of the gradients: Haar adjoints and FSQ straight-through backward, against the oracle.

Tolerances, from the arithmetic of the kernels:
  Haar adjoints, fp32: 1e-5 absolute (as the forward); bf16: one bf16 ulp plus the fp32
    accumulation bound of the block, d * 2^-24 * sum|block| / 8 with d = 6 butterfly stages;
    window 0 of the patcher's adjoint adds up four rebuilt values (each within the 6-stage
    bound) with three more additions of values up to sum|block| / 2: d = 4*6 + 3*4 = 36.
  FSQ encode backward: t_i = g_i * slope_i(z_i) carries the rounding of z + shift and of the
    exp-based sech^2 (a few 1e-7 relative, amplified by at most 2|x| ~ 20); grad_u is a 6-term
    fp32 chain: |err| <= 1e-5 * sum_i |w_ic| |g_i| scale_i (scale_i = max slope);
    grad_w sums 16 terms per thread, a 5-level shuffle tree, 4 warps, then rows in double:
    |err| <= 1e-5 * sum_tokens |g_i| scale_i |u_c|.
  FSQ decode backward: grad_codes is a C-term fp32 chain: <= 20 * 2^-24 * sum_c |w_ic| |g_c|;
    grad_w: <= 1e-5 * sum_tokens |g_c| (|zhat| <= 1).
"""

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import U, check_bf16, expand_blocks_to_pixels, expand_to_channels

pytestmark = pytest.mark.gpu

LEVELS = (8, 8, 8, 5, 5, 5)
SCALE = np.array([(L - 1) * 1.001 / 2 / (L // 2) for L in LEVELS])


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


@pytest.mark.parametrize("shape,dtype", [((2, 3, 13, 40, 96), torch.float32),     # TMA path
                                         ((1, 2, 9, 16, 44), torch.float32),      # register path
                                         ((2, 2, 17, 64, 128), torch.bfloat16),   # TMA bf16
                                         ((1, 3, 9, 24, 72), torch.bfloat16)])    # register bf16
def test_haar_adjoints_match_oracle(shape, dtype):
    B, C, T, H, W = shape
    rng = np.random.default_rng(sum(shape))
    gy = rng.uniform(-1, 1, oracle.haar_out_shape(B, C, T, H, W))
    gx = rng.uniform(-1, 1, shape)
    gy_d, gx_d = dev(gy, dtype), dev(gx, dtype)
    gy64 = gy_d.double().cpu().numpy()  # the values the kernel sees
    gx64 = gx_d.double().cpu().numpy()
    out_x = hwp.haar_fwd_adjoint(gy_d, T, H, W)
    out_y = hwp.haar_inv_adjoint(gx_d)
    hwp.tok_check_device()
    ref_x = oracle.haar_fwd_adjoint(gy64, T, H, W)
    ref_y = oracle.haar_inv_adjoint(gx64)
    got_x, got_y = out_x.double().cpu().numpy(), out_y.double().cpu().numpy()
    if dtype == torch.float32:
        assert np.abs(got_x - ref_x).max() <= 1e-5
        assert np.abs(got_y - ref_y).max() <= 1e-5
    else:
        # coefficient-block sums |gy| per block, for the pixel-side result
        a = np.abs(gy64).reshape(B, 64, C, *gy64.shape[2:]).sum(axis=1)
        check_bf16(got_x, ref_x, 36 * U * expand_blocks_to_pixels(a, T) / 8 * 1.01, "patcher adjoint")
        # pixel-block sums |gx| per block, for the coefficient-side result (window 0 reads one frame)
        ax = np.abs(gx64)
        sp = ax.reshape(B, C, T, H // 4, 4, W // 4, 4).sum(axis=(4, 6))
        Tq = 1 + (T - 1) // 4
        blk = np.empty((B, C, Tq) + sp.shape[3:])
        blk[:, :, 0] = sp[:, :, 0]
        blk[:, :, 1:] = sp[:, :, 1:].reshape(B, C, Tq - 1, 4, *sp.shape[3:]).sum(axis=3)
        check_bf16(got_y, ref_y, 6 * U * expand_to_channels(blk, 64) / 8 * 1.01, "unpatcher adjoint")


def test_haar_adjoint_dot_product_on_gpu():
    """<fwd(x), g> = <x, fwd_adjoint(g)> and <inv(y), h> = <y, inv_adjoint(h)>, through the kernels."""
    x = torch.rand(1, 3, 21, 32, 64, device="cuda") * 2 - 1
    g = torch.rand(hwp.haar_coeff_shape(1, 3, 21, 32, 64), device="cuda") * 2 - 1
    lhs = (hwp.haar_fwd(x).double() * g.double()).sum()
    rhs = (x.double() * hwp.haar_fwd_adjoint(g, 21, 32, 64).double()).sum()
    assert abs(float(lhs - rhs)) < 1e-4 * float((x.abs().sum() + g.abs().sum()))
    h = torch.rand_like(x) * 2 - 1
    lhs = (hwp.haar_inv(g, 21, 32, 64).double() * h.double()).sum()
    rhs = (g.double() * hwp.haar_inv_adjoint(h).double()).sum()
    assert abs(float(lhs - rhs)) < 1e-4 * float((h.abs().sum() + g.abs().sum()))


def test_image_adjoints_are_the_other_direction():
    x = torch.rand(2, 3, 1, 32, 64, device="cuda")
    assert torch.equal(hwp.haar_inv_adjoint(x), hwp.haar_fwd(x))
    y = hwp.haar_fwd(x)
    assert torch.equal(hwp.haar_fwd_adjoint(y, 1, 32, 64), hwp.haar_inv(y, 1, 32, 64))


# C = 16 with S % 4 == 0 takes the TMA kernels (ragged last tile at S = 1000, a single
# mostly empty tile at S = 4, workspace rows spanning batch rows at B = 3); S = 1001 and
# C = 4, 5 take the register kernels.  6C % 8 == 0 (C = 4, 16) sums the rows in groups of
# 8 entries, C = 5 entry by entry.
CASES = [(2, 16, 4096), (3, 16, 1000), (1, 16, 4), (2, 16, 1001), (2, 4, 1000), (1, 5, 777), (16, 16, 56320)]


@pytest.mark.parametrize("B,C,S", CASES)
def test_fsq_encode_backward_matches_oracle(B, C, S):
    u = synth.normal((B, C, S), seed=41 + C, std=1.3)
    w = synth.fsq_weight(C)
    g = synth.normal((B, 6, S), seed=43, std=1.0)
    gu, gw = hwp.fsq_encode_backward(dev(u), dev(w), dev(g))
    hwp.tok_check_device()
    ref_u, ref_w = oracle.fsq_encode_backward(u, w, g)
    got_u, got_w = gu.double().cpu().numpy(), gw.double().cpu().numpy()
    gs = np.abs(g.astype(np.float64)) * SCALE[None, :, None]            # |g_i| * max slope
    tol_u = 1e-5 * np.einsum("ic,bis->bcs", np.abs(w.astype(np.float64)), gs) + 1e-30
    assert (np.abs(got_u - ref_u) <= tol_u).all(), np.abs(got_u - ref_u).max()
    tol_w = 1e-5 * np.einsum("bis,bcs->ic", gs, np.abs(u.astype(np.float64))) + 1e-30
    assert (np.abs(got_w - ref_w) <= tol_w).all(), (np.abs(got_w - ref_w) / tol_w).max()


@pytest.mark.parametrize("B,C,S", CASES)
def test_fsq_decode_backward_matches_oracle(B, C, S):
    idx = synth.uniform((B, S), seed=47, lo=0, hi=64000, dtype=synth.F64).astype(np.int32)
    idx.reshape(-1)[::997] = -3                                          # some invalid indices
    w = synth.fsq_weight(C)
    g = synth.normal((B, C, S), seed=53, std=1.0)
    gc, gw = hwp.fsq_decode_backward(dev(idx), dev(w), dev(g))
    hwp.tok_check_device()
    ref_c, ref_w = oracle.fsq_decode_backward(idx, w, g)
    got_c, got_w = gc.double().cpu().numpy(), gw.double().cpu().numpy()
    g64 = np.abs(g.astype(np.float64))
    tol_c = 20 * U * np.einsum("ic,bcs->bis", np.abs(w.astype(np.float64)), g64) + 1e-30
    assert (np.abs(got_c - ref_c) <= tol_c).all()
    tol_w = 1e-5 * g64.sum(axis=(0, 2))[None, :] + 1e-30
    assert (np.abs(got_w - ref_w) <= tol_w).all()


def misaligned(a):
    """A contiguous device copy of `a` whose address is 4 bytes past a 16-byte boundary, so the
    library takes its register kernels instead of the TMA kernels."""
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    buf = torch.empty(t.numel() + 4, dtype=t.dtype, device="cuda")
    out = buf[1:1 + t.numel()].view(t.shape)
    out.copy_(t)
    assert out.data_ptr() % 16 != 0
    return out


def test_fsq_backward_paths_agree_bit_for_bit():
    """The TMA kernels and the register kernels round the same fp32 operations in the same
    order per token, so grad_u and grad_codes agree bit for bit; grad_w differs only in the
    partition of its sums."""
    B, C, S = 2, 16, 4096
    u = synth.normal((B, C, S), seed=71, std=1.4)
    w = synth.fsq_weight(C)
    g = synth.normal((B, 6, S), seed=73)
    gu_a, gw_a = hwp.fsq_encode_backward(dev(u), dev(w), dev(g))
    gu_b, gw_b = hwp.fsq_encode_backward(misaligned(u), dev(w), misaligned(g))
    assert torch.equal(gu_a, gu_b)
    gs = np.abs(g.astype(np.float64)) * SCALE[None, :, None]
    tol_w = 2e-5 * np.einsum("bis,bcs->ic", gs, np.abs(u.astype(np.float64)))  # each side within 1e-5
    assert (np.abs(gw_a.double().cpu().numpy() - gw_b.double().cpu().numpy()) <= tol_w).all()
    idx = synth.uniform((B, S), seed=79, lo=0, hi=64000, dtype=synth.F64).astype(np.int32)
    go = synth.normal((B, C, S), seed=83)
    gc_a, gw_a = hwp.fsq_decode_backward(dev(idx), dev(w), dev(go))
    gc_b, gw_b = hwp.fsq_decode_backward(misaligned(idx), dev(w), misaligned(go))
    assert torch.equal(gc_a, gc_b)
    tol_w = 2e-5 * np.abs(go.astype(np.float64)).sum(axis=(0, 2))[None, :]
    assert (np.abs(gw_a.double().cpu().numpy() - gw_b.double().cpu().numpy()) <= tol_w).all()


def test_fsq_backward_is_deterministic():
    u = dev(synth.fsq_input(4)[:8])
    w = dev(synth.fsq_weight())
    g = torch.randn(8, 6, u.shape[2], device="cuda")
    a = hwp.fsq_encode_backward(u, w, g)
    b = hwp.fsq_encode_backward(u, w, g)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    idx = hwp.fsq_encode(u, w)
    go = torch.randn_like(u)
    c = hwp.fsq_decode_backward(idx, w, go)
    d = hwp.fsq_decode_backward(idx, w, go)
    assert torch.equal(c[0], d[0]) and torch.equal(c[1], d[1])


def test_fsq_backward_empty_zeroes_grad_w():
    w = dev(synth.fsq_weight())
    gu, gw = hwp.fsq_encode_backward(torch.empty(0, 16, 8, device="cuda"), w, torch.empty(0, 6, 8, device="cuda"))
    torch.cuda.synchronize()
    assert gw.abs().sum().item() == 0
