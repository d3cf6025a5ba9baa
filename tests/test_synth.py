"""The seeded input generators: deterministic, counter-based, correctly rounded, with the stated distributions."""
import numpy as np
import torch

import synth


def test_counter_based_and_deterministic():
    a = synth.uniform((1000,), seed=7)
    b = synth.uniform((1000,), seed=7)
    c = synth.uniform((1000,), seed=8)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    # element i does not depend on how many are drawn
    np.testing.assert_array_equal(synth.uniform((10,), seed=7), a[:10])


def test_uniform_and_normal_moments():
    u = synth.uniform((200000,), seed=1, lo=-1, hi=1, dtype=synth.F64)
    assert u.min() >= -1 and u.max() < 1 and abs(u.mean()) < 0.01 and abs(u.var() - 1 / 3) < 0.01
    n = synth.normal((200000,), seed=2, std=1.5, dtype=synth.F64)
    assert abs(n.mean()) < 0.02 and abs(n.std() - 1.5) < 0.02


def test_bf16_rounding_matches_torch_on_fp32_values():
    """On values already exact in fp32 the generator's double->bf16 rounding equals torch's fp32->bf16 (RNE)."""
    # 1 + 2^-8 and 1 + 3*2^-8 are exact ties between bf16 neighbours: they must round to even
    special = [0.0, 1.0, -1.0, 1.00390625, 1.01171875, -0.7421875 - 2 ** -10]
    lib = synth._load()
    ours = np.empty(len(special), np.uint16)
    for i, x in enumerate(special):  # a uniform draw on [x, x] is exactly x
        lib.synth_uniform(ours[i:].ctypes.data, synth.BF16, 1, 0, 0, float(x), float(x))
    ref = torch.tensor(special, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    u16 = synth.uniform((100000,), seed=3, dtype=synth.BF16)
    f32 = synth.uniform((100000,), seed=3, dtype=synth.F64).astype(np.float32)
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # the generator rounds the double once; torch rounds the fp32 copy: they differ only on double-rounding ties
    assert np.count_nonzero(u16 != ref) <= 2


def test_smooth_field_range_and_smoothness():
    x = synth.bf16_bits_to_f64(synth.smooth_field((1, 2, 9, 32, 64), seed=3))
    assert x.min() >= -1 and x.max() <= 1
    # neighbouring pixels differ by little more than the noise amplitude
    assert np.abs(np.diff(x, axis=-1)).max() < 0.1 + 0.05
    assert x.std() > 0.1


def test_workload_shapes():
    assert synth.haar_input(1).shape == (1, 3, 9, 64, 64) and synth.haar_input(1).dtype == np.float32
    assert synth.fsq_input(1).shape == (1, 16, 4096)
    assert synth.fsq_weight().shape == (6, 16)
    assert synth.FSQ_CONFIGS[4]["S"] == 16 * 44 * 80
