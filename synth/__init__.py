"""Seeded synthetic weights and prompts, shared by the oracle tests and the GPU path.

The generator lives in ``synth.c`` (built into ``libsynth.so`` beside this
file); this module only marshals arguments.  It holds no decoder arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .configs import (WORKLOADS, ModelShape, TensorSpec, Workload, kv_bytes_read,  # noqa: F401
                      streamed_weight_bytes, tensor_table, total_elements)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

FNV_OFFSET = 0xCBF29CE484222325
PROMPT_STREAM = 1 << 40      # stream index of prompt tokens (far from tensor indices)
FORCED_STREAM = (1 << 40) + 1  # stream index of forced (teacher) token sequences


def build(force: bool = False) -> str:
    """Compile libsynth.so with gcc (OpenMP) if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC,
                               "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.synth_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_int]
        L.synth_fill_normal.restype = None
        L.synth_fill_tokens.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_int32]
        L.synth_fill_tokens.restype = None
        L.synth_fnv1a64.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64]
        L.synth_fnv1a64.restype = ctypes.c_uint64
        L.synth_round_f16.argtypes = [ctypes.c_double]
        L.synth_round_f16.restype = ctypes.c_uint16
        L.synth_round_bf16.argtypes = [ctypes.c_double]
        L.synth_round_bf16.restype = ctypes.c_uint16
        _lib = L
    return _lib


def generate_weights(m: ModelShape, seed: int, out: np.ndarray | None = None) -> np.ndarray:
    """All weights of model ``m`` in the canonical layout, as raw uint16 storage bits.

    ``out`` may be a preallocated (e.g. pinned) uint16 buffer of the right size.
    """
    n = total_elements(m)
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == n and out.flags.c_contiguous
    L = lib()
    base = out.ctypes.data
    for t in tensor_table(m):
        L.synth_fill_normal(base + 2 * t.offset, t.numel, seed, t.index, t.mean, t.std,
                            m.dtype_code)
    return out


def generate_tokens(n: int, vocab: int, seed: int, stream: int = PROMPT_STREAM) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    if n:
        lib().synth_fill_tokens(out.ctypes.data, n, seed, stream, vocab)
    return out


def prompt(w: Workload) -> np.ndarray:
    return generate_tokens(w.prompt_len, w.model.vocab, w.prompt_seed, PROMPT_STREAM)


def forced_tokens(w: Workload, n: int) -> np.ndarray:
    """A seeded token sequence used to teacher-force decode steps."""
    return generate_tokens(n, w.model.vocab, w.prompt_seed, FORCED_STREAM)


def fnv1a64(buf: np.ndarray, h: int = FNV_OFFSET) -> int:
    buf = np.ascontiguousarray(buf)
    return int(lib().synth_fnv1a64(buf.ctypes.data, buf.nbytes, h))


def round_to_storage(x: float, dtype: str) -> int:
    """The generator's own double -> 16-bit rounding (exposed for its tests)."""
    L = lib()
    return int(L.synth_round_f16(x) if dtype == "f16" else L.synth_round_bf16(x))


def tensor_view(buf: np.ndarray, t: TensorSpec) -> np.ndarray:
    return buf[t.offset:t.offset + t.numel].reshape(t.shape)
