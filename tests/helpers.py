"""Shared helpers of the GPU parity tests: dtype plumbing and the tolerances.

Tolerances (derived from the arithmetic of the kernels):
  fp32 Haar      max |gpu - oracle| <= 1e-5.
  bf16 Haar      |gpu - oracle| <= ulp_bf16(oracle) + E, where E bounds the fp32
                 accumulation error of the kernel's butterflies:
                 E = d * 2^-24 * sum|inputs of the block| / scale * 1.01,
                 d = 6 butterfly stages and scale 8 on video, d = 4 and scale 4 on
                 images.  The count of outputs beyond a plain 1 ulp is reported.
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
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


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


def haar_bf16_tolerance(ref: np.ndarray, block_sum: np.ndarray, video: bool) -> np.ndarray:
    depth, scale = (6, 8.0) if video else (4, 4.0)
    return ulp_bf16(ref) + depth * U * block_sum / scale * 1.01


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
