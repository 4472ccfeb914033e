"""The seeded input generators both sides of every parity test use (CPU).

The generator must give the same value for (seed, index) however a caller
slices or chunks the stream, or a test could compare the CUDA path and the
oracle on different inputs without noticing.
"""

import math

import torch

from head_split_kv_decode_b200 import synth

MASK64 = (1 << 64) - 1


def _splitmix64_int(z):
    """SplitMix64 finaliser on Python integers (mod 2^64), written from the
    published definition: add the golden-ratio increment, then three
    xor-shift / multiply rounds."""
    z = (z + 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def _normal_at_int(seed, index):
    key = index + (seed << 40)
    acc = 0
    for half in (0, 1):
        h = _splitmix64_int((key * 2 + half) & MASK64)
        acc += sum((h >> sh) & 0xFFFF for sh in (0, 16, 32, 48))
    inv_std = 1.0 / math.sqrt(8.0 * (65536.0 ** 2 - 1.0) / 12.0)
    return float(torch.tensor(float(acc - 4 * 65535), dtype=torch.float32) *
                 torch.tensor(inv_std, dtype=torch.float32))


def test_int64_tensor_generator_matches_big_integer_arithmetic():
    """The torch int64 implementation (signed wrap-around, masked logical
    shifts) equals the same arithmetic on unbounded integers mod 2^64."""
    idx = [0, 1, 2, 12345, (1 << 31) + 7, (1 << 39) - 1, 987654321987]
    for seed in (0, 1, 77, (1 << 22) - 1):
        got = synth.normal_at(seed, torch.tensor(idx, dtype=torch.int64))
        want = [_normal_at_int(seed, i) for i in idx]
        assert got.tolist() == want, seed


def test_any_slice_has_the_same_values():
    full = synth.kv_field(7, [0, 1, 2], range(0, 64), 4, 16)
    part = synth.kv_field(7, [2, 1], range(17, 40), 4, 16, heads=[3, 1])
    assert torch.equal(part, full[[2, 1]][:, 17:40][:, :, [3, 1]])
    chunked = synth.normal(5, (3, 1000), chunk=257)
    whole = synth.normal(5, (3, 1000))
    assert torch.equal(chunked, whole)


def test_moments_and_bounds():
    x = synth.normal(11, (1 << 20,))
    assert abs(x.mean().item()) < 5e-3
    assert abs(x.std().item() - 1.0) < 5e-3
    assert x.abs().max().item() < 5.0  # Irwin-Hall with n = 8 is bounded near 4.9 sigma


def test_head_mask_counts():
    m = synth.head_mask(3, 32, 8, 0.5)
    assert m.shape == (32, 8) and torch.all(m.sum(1) == 4)
    m = synth.head_mask(4, 5, 32, 0.25)
    assert torch.all(m.sum(1) == 8)
    assert not torch.equal(m[0], m[1])  # layers draw their own heads
