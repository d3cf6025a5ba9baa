"""GPU parity of tok_haar_fwd / tok_haar_inv against the CPU oracle.

Small cases are compared element by element against the oracle on the same
seeded inputs (both vector and element-wise kernel paths, several CTAs and a
ragged tail).  The full workloads are compared on sampled blocks, computed by
the oracle one 4x4x4 window at a time (output frame t' depends only on frames
4t'-3..4t', or on frame 0 for t' = 0), plus energy and round-trip properties
that hold at any size.
"""
import zlib

import numpy as np
import pytest
import torch

import haar_wavelet_patching_b200 as hwp
import oracle
import synth
from tests.helpers import (block_abs_sums, expand_blocks_to_pixels, expand_to_channels, haar_bf16_tolerance,
                           inv_block_abs_sums, to_device, to_f64, ulp_bf16)

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5


def run_fwd(xd: torch.Tensor) -> torch.Tensor:
    y = hwp.haar_fwd(xd)
    hwp.tok_check_device()
    return y


def check_fwd(x_np, dtype, label):
    """Whole-tensor comparison of the forward against the oracle; returns (gpu y, oracle y)."""
    x64 = synth.to_f64(x_np, dtype)
    ref = oracle.haar_fwd(x64)
    y = run_fwd(to_device(x_np, dtype))
    got = to_f64(y)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    if dtype == synth.F32:
        assert err.max() <= TOL_F32, f"{label}: max |err| {err.max():.3g}"
    else:
        video = x_np.shape[2] > 1
        bs = expand_to_channels(block_abs_sums(x64), 64 if video else 16)
        tol = haar_bf16_tolerance(ref, bs, video)
        bad = err > tol
        assert not bad.any(), f"{label}: {bad.sum()} outputs beyond tolerance, worst {(err - tol).max():.3g}"
        # Outputs beyond a plain 1 ulp are near-zero coefficients of blocks whose fp32 sums were
        # inexact (tiny inputs next to large ones); they are inside E above.  Reported, and kept rare.
        strict = int((err > ulp_bf16(ref)).sum())
        print(f"{label}: {strict} of {err.size} outputs beyond a plain 1 bf16 ulp (all within the fp32 bound)")
        assert strict <= max(1, int(5e-3 * err.size)), f"{label}: {strict} outputs beyond 1 bf16 ulp"
    return y, ref


def check_inv(y: torch.Tensor, T, H, W, label):
    """The GPU inverse of the GPU coefficients against the oracle inverse of the same coefficients."""
    y64 = to_f64(y)
    ref = oracle.haar_inv(y64, T, H, W)
    x = hwp.haar_inv(y, T, H, W)
    hwp.tok_check_device()
    got = to_f64(x)
    err = np.abs(got - ref)
    if y.dtype == torch.float32:
        assert err.max() <= TOL_F32, f"{label}: max |err| {err.max():.3g}"
    else:
        video = T > 1
        C = got.shape[1]
        bs = expand_blocks_to_pixels(inv_block_abs_sums(y64, C, video), T)
        tol = haar_bf16_tolerance(ref, bs, video)
        assert not (err > tol).any(), f"{label}: {(err > tol).sum()} pixels beyond tolerance"
    return x


SMALL = [
    # (shape, dtype, note).  TMA box form: the source's rows are whole 16-byte units (forward:
    # W * elem, with w even; inverse: w * elem and W * elem); other 16-byte-aligned sources take
    # the TMA row form.  The register kernels take misaligned views (tests below).
    ((1, 3, 9, 64, 64), synth.F32, "config 1"),
    ((2, 3, 13, 40, 96), synth.BF16, "TMA bf16, partial tiles in x and y"),
    ((1, 2, 9, 36, 80), synth.F32, "TMA fp32, partial tiles"),
    ((2, 2, 17, 64, 544), synth.BF16, "TMA bf16, several tiles per row, ragged last"),
    ((1, 1, 5, 4, 32), synth.BF16, "TMA bf16, one block row"),
    ((3, 2, 1, 24, 160), synth.BF16, "TMA image path, partial tiles"),
    ((2, 1, 1, 20, 48), synth.F32, "TMA image path fp32"),
    ((2, 3, 13, 64, 264), synth.F32, "box forward, row-form inverse, ragged tail"),
    ((2, 3, 13, 64, 264), synth.BF16, "box forward, row-form inverse, bf16"),
    ((1, 2, 9, 16, 44), synth.BF16, "W % 8 == 4: row form, odd w"),
    ((1, 2, 9, 16, 44), synth.F32, "row form fp32, odd w"),
    ((1, 1, 5, 4, 4), synth.F32, "smallest video"),
    ((3, 2, 1, 64, 192), synth.BF16, "image path, boxes both ways"),
    ((3, 2, 1, 64, 192), synth.F32, "image path fp32"),
    ((2, 3, 1, 36, 40), synth.BF16, "image path, W % 16 == 8: row-form inverse"),
    ((1, 1, 1, 4, 4), synth.F32, "smallest image"),
    ((1, 5, 21, 24, 1032), synth.BF16, "odd channel count, long row"),
]


@pytest.mark.parametrize("shape,dtype,note", SMALL, ids=[s[2] for s in SMALL])
def test_fwd_inv_small(shape, dtype, note):
    x = synth.uniform(shape, seed=zlib.crc32(note.encode()), dtype=dtype)
    y, _ = check_fwd(x, dtype, note)
    B, C, T, H, W = shape
    xr = check_inv(y, T, H, W, note)
    if dtype == synth.F32:
        # perfect reconstruction through the GPU, fp32
        assert np.abs(to_f64(xr) - synth.to_f64(x, dtype)).max() <= 1e-6


def test_smooth_field_small():
    x = synth.smooth_field((1, 3, 17, 32, 128), seed=3)
    y, _ = check_fwd(x, synth.BF16, "smooth field")
    check_inv(y, 17, 32, 128, "smooth field inverse")


def test_misaligned_pointers_take_elementwise_path():
    """Views offset by one element are not 16-byte aligned: results must not change."""
    shape = (1, 2, 9, 16, 64)
    x = synth.uniform(shape, seed=99, dtype=synth.BF16)
    xd = to_device(x, synth.BF16)
    n = xd.numel()
    buf = torch.empty(n + 1, dtype=torch.bfloat16, device="cuda")
    buf[1:].copy_(xd.reshape(-1))
    xo = buf[1:].view(shape)
    assert xo.data_ptr() % 16 != 0
    ybuf = torch.empty(hwp.haar_coeff_shape(*shape)).numel() + 1
    ybuf = torch.empty(ybuf, dtype=torch.bfloat16, device="cuda")
    yo = ybuf[1:].view(hwp.haar_coeff_shape(*shape))
    hwp.tok_haar_fwd(xo, yo)
    yv = hwp.haar_fwd(xd)
    torch.cuda.synchronize()
    assert torch.equal(yo, yv)
    xr = torch.empty_like(buf)
    hwp.tok_haar_inv(yo, xr[1:].view(shape))
    torch.cuda.synchronize()
    assert torch.equal(xr[1:].view(shape), hwp.haar_inv(yv, 9, 16, 64))


@pytest.mark.parametrize("shape,dtype", [((2, 3, 13, 40, 96), torch.bfloat16), ((1, 2, 9, 36, 80), torch.float32),
                                         ((3, 2, 1, 24, 160), torch.bfloat16)])
def test_tma_and_register_paths_agree_bitwise(shape, dtype):
    """The TMA kernels and the register kernels (taken for a misaligned view) give identical bits."""
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y_tma = hwp.haar_fwd(x)
    buf = torch.empty(x.numel() + 1, dtype=dtype, device="cuda")
    buf[1:].copy_(x.reshape(-1))
    ybuf = torch.empty(y_tma.numel() + 1, dtype=dtype, device="cuda")
    hwp.tok_haar_fwd(buf[1:].view(shape), ybuf[1:].view(y_tma.shape))
    hwp.tok_check_device()
    assert torch.equal(ybuf[1:].view(y_tma.shape), y_tma)
    xr_tma = hwp.haar_inv(y_tma, *shape[2:])
    xbuf = torch.empty_like(buf)
    hwp.tok_haar_inv(ybuf[1:].view(y_tma.shape), xbuf[1:].view(shape))
    hwp.tok_check_device()
    assert torch.equal(xbuf[1:].view(shape), xr_tma)


@pytest.mark.parametrize("shape,dtype,chunks", [
    ((1, 3, 41, 64, 128), torch.bfloat16, [(0, 1), (1, 4), (4, 7), (7, 11)]),    # TMA path
    ((2, 2, 29, 40, 72), torch.bfloat16, [(0, 3), (3, 8)]),                      # row-form inverse (W % 32 != 0)
    ((1, 2, 21, 32, 64), torch.float32, [(0, 2), (2, 2), (2, 6)]),               # fp32, an empty chunk
    ((2, 3, 1, 32, 64), torch.bfloat16, [(0, 1)]),                               # image: one window
])
def test_windows_compose_to_the_full_call(shape, dtype, chunks):
    """Chunks of latent frames, processed separately, give exactly the full result; each chunk
    writes only its own frames (everything else keeps a sentinel)."""
    B, C, T, H, W = shape
    x = (torch.rand(shape, device="cuda") * 2 - 1).to(dtype)
    y_full = hwp.haar_fwd(x)
    x_full = hwp.haar_inv(y_full, T, H, W)
    y = torch.full_like(y_full, float("nan"))
    xr = torch.full_like(x, float("nan"))
    for a, b in chunks:
        before = y.clone()
        hwp.tok_haar_fwd_windows(x, y, a, b)
        hwp.tok_check_device()
        changed = (y != before) & ~(torch.isnan(y) & torch.isnan(before))
        outside = torch.ones(y.shape[2], dtype=torch.bool, device="cuda")
        outside[a:b] = False
        assert not changed[:, :, outside].any(), f"forward chunk {(a, b)} wrote outside its frames"
        hwp.tok_haar_inv_windows(y, xr, a, b)
        hwp.tok_check_device()
    assert torch.equal(y, y_full)
    assert torch.equal(xr, x_full)


def test_constant_and_causal_structure_on_gpu():
    C = 3
    x = torch.full((2, C, 9, 16, 32), 0.375, device="cuda")
    y = run_fwd(x)
    assert torch.all(y[:, :C] == 3.0)          # 8 * 0.375, exact
    assert torch.all(y[:, C:] == 0)
    xr = torch.randn(1, C, 9, 16, 32, device="cuda")
    y = run_fwd(xr)
    for g in range(64):
        if (g >> 3) >> 2 or (g & 7) >> 2:         # a temporal high band at level 2 or 1
            assert torch.all(y[0, g * C:(g + 1) * C, 0] == 0)


def test_empty_is_noop():
    x = torch.empty(0, 3, 9, 16, 16, device="cuda")
    y = hwp.haar_fwd(x)
    assert y.shape == (0, 192, 3, 4, 4)
    xr = hwp.haar_inv(y, 9, 16, 16)
    assert xr.shape == x.shape


def test_bad_arguments_raise_before_launch():
    buf = torch.zeros(8192, device="cuda")
    x = buf[:2304].view(1, 1, 9, 16, 16)
    y = buf[1024:1024 + 3072].view(1, 64, 3, 4, 4)  # overlaps x
    with pytest.raises(hwp.TokError, match="ALIAS"):
        hwp.tok_haar_fwd(x, y)
    with pytest.raises(ValueError):
        hwp.haar_fwd(torch.zeros(1, 1, 7, 16, 16, device="cuda"))


def test_stream_ordering():
    """Work goes on the given stream and is ordered after earlier work on it."""
    s = torch.cuda.Stream()
    x = synth.uniform((1, 3, 13, 64, 128), seed=5, dtype=synth.BF16)
    with torch.cuda.stream(s):
        xd = to_device(x, synth.BF16)
        y = hwp.haar_fwd(xd, stream=s)
        xr = hwp.haar_inv(y, 13, 64, 128, stream=s)
    s.synchronize()
    ref = hwp.haar_fwd(to_device(x, synth.BF16))
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    assert xr.shape == xd.shape


# ---------------------------------------------------------------------------
# Full workloads: sampled blocks + properties.
# ---------------------------------------------------------------------------
def sample_positions(B, C, Tq, h, w, n, seed):
    rng = np.random.default_rng(seed)
    pos = [(rng.integers(B), rng.integers(C), rng.integers(Tq), rng.integers(h), rng.integers(w)) for _ in range(n)]
    # corners and the first / last latent frame
    for tq in (0, Tq - 1):
        for i in (0, h - 1):
            for j in (0, w - 1):
                pos.append((B - 1, C - 1, tq, i, j))
                pos.append((0, 0, tq, i, j))
    return pos


def window_batch(x64_getter, pos):
    """Per sampled block: a 5-frame, 4x4 window whose output frame (0 or 1) is that block's."""
    wins = np.empty((len(pos), 1, 5, 4, 4))
    for k, (b, c, tq, i, j) in enumerate(pos):
        f0 = 0 if tq == 0 else 4 * tq - 4
        wins[k, 0] = x64_getter(b, c, slice(f0, f0 + 5), slice(4 * i, 4 * i + 4), slice(4 * j, 4 * j + 4))
    return wins


@pytest.mark.parametrize("cfg", [3, 5])
def test_full_workload_sampled(cfg):
    c = synth.HAAR_CONFIGS[cfg]
    B, C, T, H, W = c["shape"]
    x = synth.haar_input(cfg)
    xd = to_device(x, synth.BF16)
    y = run_fwd(xd)
    Tq, h, w = y.shape[2:]
    assert y.shape == (B, 64 * C, Tq, H // 4, W // 4)
    pos = sample_positions(B, C, Tq, h, w, 4000, seed=cfg)

    def getx(b, cc, ft, fy, fx):
        return synth.bf16_bits_to_f64(x[b, cc, ft, fy, fx])

    wins = window_batch(getx, pos)
    ref_w = oracle.haar_fwd(wins)  # [n, 64, 2, 1, 1]
    sel = torch.tensor(pos, device="cuda")
    b_, c_, t_, i_, j_ = sel.unbind(1)
    groups = torch.arange(64, device="cuda")
    got = y[b_[:, None], groups[None, :] * C + c_[:, None], t_[:, None], i_[:, None], j_[:, None]]
    got = got.double().cpu().numpy()
    ref = np.stack([ref_w[k, :, 0 if p[2] == 0 else 1, 0, 0] for k, p in enumerate(pos)])
    bsum = np.array([np.abs(wins[k, 0, (0 if p[2] == 0 else 1):]).sum() if p[2] else 4 * np.abs(wins[k, 0, 0]).sum()
                     for k, p in enumerate(pos)])
    tol = haar_bf16_tolerance(ref, bsum[:, None], True)
    err = np.abs(got - ref)
    assert not (err > tol).any(), f"config {cfg}: {(err > tol).sum()} sampled outputs beyond tolerance"

    # Inverse on the same sampled blocks, against the oracle inverse of the GPU coefficients.
    xr = hwp.haar_inv(y, T, H, W)
    torch.cuda.synchronize()
    ycoef = np.zeros((len(pos), 64, 2, 1, 1))
    y0 = y[b_[:, None], groups[None, :] * C + c_[:, None], 0, i_[:, None], j_[:, None]].double().cpu().numpy()
    ycoef[:, :, 0, 0, 0] = y0
    ycoef[:, :, 1, 0, 0] = got
    xw = oracle.haar_inv(ycoef, 5, 4, 4)  # [n, 1, 5, 4, 4]
    for k, (b, cc, tq, i, j) in enumerate(pos[:600]):
        if tq == 0:
            g = xr[b, cc, 0, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
            r = xw[k, 0, 0]
        else:
            g = xr[b, cc, 4 * tq - 3:4 * tq + 1, 4 * i:4 * i + 4, 4 * j:4 * j + 4].double().cpu().numpy()
            r = xw[k, 0, 1:]
        tol = haar_bf16_tolerance(r, np.abs(ycoef[k, :, 1 if tq else 0]).sum(), True)
        assert (np.abs(g - r) <= tol).all(), f"config {cfg}: inverse block {(b, cc, tq, i, j)}"

    # Properties at full size, one (b, c) slab at a time: energy (video Parseval) and the round trip.
    e_in = e_out = 0.0
    rt_max = 0.0
    for b in range(B):
        for cc in range(C):
            xs = xd[b, cc].double()
            e_in += float((xs * xs).sum() + 3.0 * (xs[0] ** 2).sum())
            rt_max = max(rt_max, float((xr[b, cc].double() - xs).abs().max()))
        e_out += float((y[b].double() ** 2).sum())
    assert abs(e_out / e_in - 1.0) < 2e-3
    assert rt_max < 0.05  # bf16 coefficients: a few bf16 ulps of the block's range
    del y, xr, xd


def test_config2_images_full():
    """Image batch [16,3,1024,1024] bf16 compared element by element with the oracle."""
    x = synth.haar_input(2)
    y, _ = check_fwd(x, synth.BF16, "config 2")
    check_inv(y, 1, 1024, 1024, "config 2 inverse")
