"""Shared helpers of the GPU parity tests: dtype plumbing and the tolerances.

Tolerances (derived from the arithmetic of the kernels):
  fp32 Haar      max |gpu - oracle| <= 1e-5.
  bf16 outputs   one bf16 ulp of the oracle value (the path's stated figure), read as
                 follows.  The kernel computes an fp32 value v within E of the exact
                 result r (E bounds its fp32 accumulation error) and rounds it once to
                 bf16 (nearest even), so |gpu - r| <= E + ulp(|r| + E) / 2.  The test
                 bound is max(ulp(r), E + ulp(|r| + E) / 2): one ulp wherever
                 E < ulp(r) / 2, and an output more than one ulp off is accepted only in
                 the cancellation regime 2E >= ulp(r), where the fp32 sums of a block
                 that mixes tiny and large inputs cannot resolve a near-zero result to
                 half a bf16 ulp (check_bf16 asserts both, with no free count).
                 Haar: E = d * 2^-24 * sum|inputs of the block| / scale * 1.01, with
                 d = 6 butterfly stages and scale 8 on video, d = 4 and scale 4 on
                 images (recursive pairwise summation through d rounded stages, then an
                 exact power-of-two scale; 1.01 covers the 1/(1 - d u) factor).
  FSQ indices    bit-exact except tokens the oracle flags as within 1e-5 of a
                 rounding boundary; those mismatches are capped at 1e-6 of tokens.
  FSQ decode     |gpu - oracle| <= 8 * 2^-24 * sum_i |w_ic zhat_i| (fp32 chain of 6 FMAs).
"""
import numpy as np
import torch

import synth

U = 2.0 ** -24


def to_device(a: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    if dtype == synth.BF16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (2^(e-7) in the binade [2^e, 2^(e+1)); 2^-133 below 2^-126)."""
    _, e = np.frexp(np.maximum(np.abs(v), 2.0 ** -126))
    return np.ldexp(1.0, e - 8)


def bf16_tol(ref, E):
    """Largest |gpu - ref| of a bf16 output rounded once from an fp32 value within E of ref."""
    return np.maximum(ulp_bf16(ref), E + 0.5 * ulp_bf16(np.abs(ref) + E))


def check_bf16(got, ref, E, label):
    """Assert the bf16 bound above element by element; return the count of outputs beyond a
    plain 1 ulp (each of them must lie in the cancellation regime 2E >= ulp(ref))."""
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    E = np.broadcast_to(E, err.shape)
    tol = bf16_tol(ref, E)
    bad = err > tol
    assert not bad.any(), f"{label}: {int(bad.sum())} outputs beyond the bf16 bound, worst excess {(err - tol).max():.3g}"
    ulp = ulp_bf16(ref)
    strict = err > ulp
    off = strict & (2.0 * E < ulp)
    assert not off.any(), f"{label}: {int(off.sum())} outputs beyond 1 ulp outside the cancellation regime"
    return int(strict.sum())


def ulp_bf16_t(v: torch.Tensor) -> torch.Tensor:
    """ulp_bf16 for float64 torch tensors (any device)."""
    _, e = torch.frexp(torch.clamp(v.abs(), min=2.0 ** -126))
    return torch.ldexp(torch.ones_like(v), e - 8)


def check_bf16_t(got: torch.Tensor, ref: torch.Tensor, E: torch.Tensor, label: str) -> int:
    """check_bf16 on float64 torch tensors (used on the device for the full-size workloads)."""
    err = (got.double() - ref).abs()
    E = E.expand_as(err)
    tol = torch.maximum(ulp_bf16_t(ref), E + 0.5 * ulp_bf16_t(ref.abs() + E))
    nbad = int((err > tol).sum())
    assert nbad == 0, f"{label}: {nbad} outputs beyond the bf16 bound"
    ulp = ulp_bf16_t(ref)
    strict = err > ulp
    noff = int((strict & (2.0 * E < ulp)).sum())
    assert noff == 0, f"{label}: {noff} outputs beyond 1 ulp outside the cancellation regime"
    return int(strict.sum())


def haar_fp32_bound(block_sum, video: bool):
    """E of the Haar kernels: d rounded add/sub stages, then the exact 1/8 (1/4) scale."""
    depth, scale = (6, 8.0) if video else (4, 4.0)
    return depth * U * block_sum / scale * 1.01


def block_abs_sums(x64: np.ndarray) -> np.ndarray:
    """sum |x| over the input block of each output position: [B, C, Tq, h, w] (video) or [B, C, 1, h, w]."""
    B, C, T, H, W = x64.shape
    a = np.abs(x64)
    sp = a.reshape(B, C, T, H // 4, 4, W // 4, 4).sum(axis=(4, 6))  # [B, C, T, h, w]
    if T == 1:
        return sp
    Tq = 1 + (T - 1) // 4
    out = np.empty((B, C, Tq) + sp.shape[3:])
    out[:, :, 0] = 4.0 * sp[:, :, 0]
    out[:, :, 1:] = sp[:, :, 1:].reshape(B, C, Tq - 1, 4, *sp.shape[3:]).sum(axis=3)
    return out


def expand_to_channels(per_block: np.ndarray, groups: int) -> np.ndarray:
    """[B, C, Tq, h, w] -> [B, groups*C, Tq, h, w], channel g*C + c taking block (b, c)."""
    return np.concatenate([per_block] * groups, axis=1)


def inv_block_abs_sums(y64: np.ndarray, C: int, video: bool) -> np.ndarray:
    """sum |y| over the 64 (16) coefficients of each block: [B, C, Tq, h, w]."""
    B, CC, Tq, h, w = y64.shape
    groups = CC // C
    return np.abs(y64).reshape(B, groups, C, Tq, h, w).sum(axis=1)


def expand_blocks_to_pixels(per_block: np.ndarray, T: int) -> np.ndarray:
    """[B, C, Tq, h, w] -> [B, C, T, H, W]: each pixel takes its block's value."""
    B, C, Tq, h, w = per_block.shape
    sp = np.repeat(np.repeat(per_block, 4, axis=3), 4, axis=4)
    if T == 1:
        return sp
    frames = [0] + [1 + (f - 1) // 4 for f in range(1, T)]
    return sp[:, :, frames]
