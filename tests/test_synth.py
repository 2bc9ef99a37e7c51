"""The input generator's bf16 conversion is round-to-nearest-even.

Every bf16 tensor both sides read (activations, scales) and every bf16
expected value of an exact test goes through synth.f32_to_bf16_bits, so it
is pinned here against torch's own fp32 -> bf16 conversion (round to
nearest, ties to even) on random values, exact ties of both parities,
subnormals, signed zeros, the overflow boundary and infinities.
"""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")


def _torch_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_random_values_round_like_torch():
    rng = np.random.default_rng(0)
    for scale in (1e-30, 1e-3, 1.0, 1e3, 1e30):
        a = (rng.standard_normal(100_000) * scale).astype(np.float32)
        assert np.array_equal(synth.f32_to_bf16_bits(a), _torch_bits(a))


def test_ties_go_to_even():
    rng = np.random.default_rng(1)
    hi = rng.integers(0, 0x7F7F, size=2000, dtype=np.uint32)   # finite bf16 patterns, both parities
    ties = ((hi << 16) | 0x8000).view(np.float32)
    want = np.where(hi & 1, hi + 1, hi).astype(np.uint16)       # odd rounds up, even stays
    assert np.array_equal(synth.f32_to_bf16_bits(ties), want)
    assert np.array_equal(_torch_bits(ties), want)
    # one ulp either side of the tie
    below = (((hi << 16) | 0x7FFF)).view(np.float32)
    above = (((hi << 16) | 0x8001)).view(np.float32)
    assert np.array_equal(synth.f32_to_bf16_bits(below), hi.astype(np.uint16))
    assert np.array_equal(synth.f32_to_bf16_bits(above), (hi + 1).astype(np.uint16))


def test_special_values():
    f32max = np.finfo(np.float32).max
    a = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-39, np.inf, -np.inf, f32max, -f32max, 3.3895314e38],
                 np.float32)
    got = synth.f32_to_bf16_bits(a)
    assert np.array_equal(got, _torch_bits(a))
    assert got[0] == 0x0000 and got[1] == 0x8000
    assert got[5] == 0x7F80 and got[6] == 0xFF80
    assert got[7] == 0x7F80   # the largest fp32 is past bf16's rounding boundary: infinity


def test_bits_round_trip_is_exact():
    b = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    finite = (b & 0x7F80) != 0x7F80
    f = synth.bf16_bits_to_f32(b[finite])
    assert np.array_equal(synth.f32_to_bf16_bits(f), b[finite])
