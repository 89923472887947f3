"""Pins of the oracle's 16-bit conversions against library conversions.

binary16: numpy's float16 cast (round half to even from float64).
bfloat16: torch's float32 -> bfloat16 cast (round half to even) on values
that float32 holds exactly, so no double rounding is involved.
"""
import numpy as np
import pytest
import torch

from oracle.numerics import round_to_storage, storage_to_f64, to_storage_bits


def _sample_doubles(rng, n):
    mant = rng.uniform(-2.0, 2.0, n)
    expo = rng.integers(-30, 18, n)
    x = np.ldexp(mant, expo)
    specials = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 7e4, -7e4, 2.0 ** -14,
                         2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -25, 3 * 2.0 ** -26, 1e-9,
                         1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, np.inf, -np.inf])
    return np.concatenate([x, specials])


def test_f16_round_matches_numpy_cast():
    rng = np.random.default_rng(0)
    x = _sample_doubles(rng, 200_000)
    ours = round_to_storage(x, "f16")
    ref = x.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)


def test_f16_ties_go_to_even():
    # 1 + 2^-11 is halfway between 1 and 1 + 2^-10: even mantissa is 1.0
    assert round_to_storage(np.array([1.0 + 2.0 ** -11]), "f16")[0] == 1.0
    # 1 + 3*2^-11 is halfway between 1+2^-10 and 1+2^-9: even is 1 + 2^-9
    assert round_to_storage(np.array([1.0 + 3 * 2.0 ** -11]), "f16")[0] == 1.0 + 2.0 ** -9


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(1)
    x32 = np.ldexp(rng.uniform(-2, 2, 200_000), rng.integers(-130, 120, 200_000)).astype(np.float32)
    x32 = np.concatenate([x32, np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0e38, -3.4e38,
                                         1e-39, 0.0], dtype=np.float32)])
    ours = round_to_storage(x32.astype(np.float64), "bf16")
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_widening_every_bit_pattern(dtype):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = storage_to_f64(bits, dtype)
    if dtype == "f16":
        ref = bits.view(np.float16).astype(np.float64)
    else:
        ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(ours[finite], ref[finite])
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_round_trip_bits(dtype):
    rng = np.random.default_rng(2)
    x = round_to_storage(rng.normal(0, 3, 10_000), dtype)
    np.testing.assert_array_equal(storage_to_f64(to_storage_bits(x, dtype), dtype), x)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_generator_rounding_agrees(dtype):
    """The input generator's C rounding and the oracle's numpy rounding are
    independent statements of the same definition; they must agree."""
    import synth
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 0.02, 3000), rng.normal(0, 100, 1000),
                        np.ldexp(rng.uniform(-2, 2, 1000), rng.integers(-40, 10, 1000))])
    if dtype == "bf16":
        x = x.astype(np.float32).astype(np.float64)
    gen = np.array([synth.round_to_storage(float(v), dtype) for v in x], dtype=np.uint16)
    np.testing.assert_array_equal(storage_to_f64(gen, dtype), round_to_storage(x, dtype))
