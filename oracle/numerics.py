"""Storage-type conversions of the oracle (IEEE binary16 and bfloat16).

Weights and the KV cache are stored in a 16-bit type (FP16 per the pages'
results table; bfloat16 for the 8B-class workload).  Widening to float64 is
exact.  Narrowing rounds to nearest, ties to even, from the format definition:
a value with binary exponent e (clamped to the format's smallest normal
exponent, so subnormals come out right) is a multiple of 2^(e - p), where p is
the number of fraction bits; beyond the largest finite value it overflows to
infinity.
"""
from __future__ import annotations

import numpy as np

# (fraction bits, smallest normal exponent, largest finite value)
_FORMATS = {
    "f16": (10, -14, 65504.0),
    "bf16": (7, -126, float((2.0 - 2.0 ** -7) * 2.0 ** 127)),
}


def storage_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of raw 16-bit storage words (uint16 array)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest storage-type value (ties to even).

    Returns float64 values that are exactly representable in ``dtype``.
    """
    p, emin, vmax = _FORMATS[dtype]
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e2 = np.frexp(a)                 # a = f * 2**e2, f in [0.5, 1)
    e = np.maximum(e2.astype(np.int64) - 1, emin)
    q = np.ldexp(1.0, (e - p).astype(np.int32))   # spacing of the format at a
    r = np.rint(a / q) * q              # np.rint rounds half to even
    r = np.where(r > vmax, np.inf, r)
    r = np.where(np.isnan(x), np.nan, r)
    return np.copysign(r, x)


def to_storage_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage words of already-representable float64 values."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        return (x.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(dtype)
