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
from tests.helpers import (block_abs_sums, check_bf16, check_bf16_t, expand_blocks_to_pixels, expand_to_channels,
                           haar_fp32_bound, inv_block_abs_sums, to_device, to_f64)

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
        E = haar_fp32_bound(expand_to_channels(block_abs_sums(x64), 64 if video else 16), video)
        strict = check_bf16(got, ref, E, label)
        print(f"{label}: {strict} of {got.size} outputs beyond a plain 1 bf16 ulp, each in the cancellation regime")
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
        E = haar_fp32_bound(expand_blocks_to_pixels(inv_block_abs_sums(y64, C, video), T), video)
        strict = check_bf16(got, ref, E, label)
        print(f"{label}: {strict} of {got.size} pixels beyond a plain 1 bf16 ulp, each in the cancellation regime")
    return x


SMALL = [
    # (shape, dtype, note).  TMA box form: the source's rows are whole 16-byte units (forward:
    # W * elem, with w even; inverse: w * elem and W * elem); other 16-byte-aligned sources take
    # the TMA row form.  The register kernels take misaligned views (tests below).
    ((1, 3, 9, 64, 64), synth.F32, "clip [1,3,9,64,64] fp32"),
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
    ((1, 2, 25, 64, 1300), torch.bfloat16, [(0, 2), (2, 5), (5, 7)]),            # grouped rows, shifted tiles
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
# Full workloads, element by element.
# ---------------------------------------------------------------------------
def _window_sums(a: torch.Tensor, T: int) -> torch.Tensor:
    """[T, H, W] float64 |pixels| -> [Tq, h, w] sums over each output's 4x4x4 input window
    (window 0 reads frame 0 four times)."""
    _, H, W = a.shape
    sp = a.view(T, H // 4, 4, W // 4, 4).sum(dim=(2, 4))
    Tq = 1 + (T - 1) // 4
    out = torch.empty((Tq,) + sp.shape[1:], dtype=a.dtype, device=a.device)
    out[0] = 4.0 * sp[0]
    out[1:] = sp[1:].view(Tq - 1, 4, *sp.shape[1:]).sum(dim=1)
    return out


def _slab_oracle(x_bits, y_host, T, H, W):
    """The oracle's forward of one (b, c) pixel slab, and its inverse of the GPU's coefficients
    of that slab: ([1, 64, Tq, h, w], [1, 1, T, H, W]) in float64."""
    x64 = synth.bf16_bits_to_f64(x_bits)
    return oracle.haar_fwd(x64), oracle.haar_inv(y_host, T, H, W)


FULL_WORKLOADS = {3: "clip [1,3,121,704,1280]", 5: "clips [4,3,121,1088,1920]"}  # synth workload keys


@pytest.mark.parametrize("cfg", [3, 5], ids=["headline_clip", "stress_clips"])
def test_full_workload_elementwise(cfg):
    """The 121-frame 704x1280 clip and the four 121-frame 1088x1920 throughput-stress clips
    in full: every coefficient of the forward and every pixel of the inverse compared with the
    oracle, one (b, c) slab at a time (the oracle on host threads, the comparison on the device).
    The inverse is compared with the oracle inverse of the same bf16 coefficients.  Also the
    video Parseval identity and the round trip at full size."""
    from concurrent.futures import ThreadPoolExecutor

    c = synth.HAAR_CONFIGS[cfg]
    B, C, T, H, W = c["shape"]
    x = synth.haar_input(cfg)
    xd = to_device(x, synth.BF16)
    y = run_fwd(xd)
    Tq, h, w = y.shape[2:]
    assert y.shape == (B, 64 * C, Tq, H // 4, W // 4)
    xr = hwp.haar_inv(y, T, H, W)
    hwp.tok_check_device()
    frames = torch.tensor([0] + [1 + (f - 1) // 4 for f in range(1, T)], device="cuda")
    slabs = [(b, cc) for b in range(B) for cc in range(C)]
    strict_f = strict_i = 0
    e_in = e_out = rt_max = 0.0
    with ThreadPoolExecutor(max_workers=3) as pool:
        futs = {}

        def submit(k):
            b, cc = slabs[k]
            ys = y[b:b + 1, cc::C].double().cpu().numpy()
            futs[k] = pool.submit(_slab_oracle, x[b:b + 1, cc:cc + 1], ys, T, H, W)

        for k in range(min(3, len(slabs))):
            submit(k)
        for k, (b, cc) in enumerate(slabs):
            ref_y, ref_x = futs.pop(k).result()
            if k + 3 < len(slabs):
                submit(k + 3)
            label = f"{FULL_WORKLOADS[cfg]} (b={b}, c={cc})"
            xs = xd[b, cc].double()
            E = haar_fp32_bound(_window_sums(xs.abs(), T), True)           # [Tq, h, w]
            ys = y[b, cc::C]
            strict_f += check_bf16_t(ys, torch.from_numpy(ref_y[0]).cuda(), E, label + " forward")
            a = ys.double().abs().sum(dim=0)                                # sum |y| over a block's 64 coefficients
            Ei = haar_fp32_bound(a.repeat_interleave(4, 1).repeat_interleave(4, 2)[frames], True)
            strict_i += check_bf16_t(xr[b, cc], torch.from_numpy(ref_x[0, 0]).cuda(), Ei, label + " inverse")
            e_in += float((xs * xs).sum() + 3.0 * (xs[0] ** 2).sum())
            e_out += float((ys.double() ** 2).sum())
            rt_max = max(rt_max, float((xr[b, cc].double() - xs).abs().max()))
            del ref_y, ref_x, E, Ei, a
    n_y, n_x = y.numel(), xr.numel()
    print(f"{FULL_WORKLOADS[cfg]}: forward {strict_f} of {n_y} coefficients and inverse {strict_i} of {n_x} pixels "
          f"beyond a plain 1 bf16 ulp (all in the cancellation regime); round trip max |err| {rt_max:.3g}")
    assert abs(e_out / e_in - 1.0) < 2e-3       # bf16 rounding of the coefficients only
    assert rt_max < 0.05                        # bf16 coefficients: a few bf16 ulps of the block's range
    del y, xr, xd


def test_image_batch_full():
    """Image batch [16,3,1024,1024] bf16 compared element by element with the oracle."""
    x = synth.haar_input(2)
    y, _ = check_fwd(x, synth.BF16, "image batch [16,3,1024,1024]")
    check_inv(y, 1, 1024, 1024, "image batch inverse")
