"""Python binding of libkie.so, the persistent batch-1 decode library.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind the C ABI declared in ``include/kie.h``.  PyTorch supplies
device memory and streams.  There is no fallback: if the compiled library is
missing, importing the binding's calls raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkie.so")
PROF_LIB_PATH = os.path.join(HERE, "libkie_prof.so")   # built with -DKIE_PROFILE
HEADER = os.path.join(os.path.dirname(HERE), "include", "kie.h")

KIE_OK = 0
KIE_ERR_INVALID = -1
KIE_ERR_OOM = -2
KIE_ERR_CUDA = -3
KIE_ERR_CAPACITY = -4
KIE_ERR_NOT_RESIDENT = -5
KIE_ERR_DEVICE_TIMEOUT = -6
KIE_ERR_POISONED = -7
KIE_ERR_NONFINITE = -8
KIE_SYNC_DEPENDENCY = 0
KIE_SYNC_GRID = 1
KIE_SUM_FP32_ATOMIC = 0
KIE_SUM_EXACT = 1
KIE_PREFILL_STEPS = 0
KIE_PREFILL_GEMM = 1
KIE_F16 = 0
KIE_BF16 = 1
KIE_MAX_TOP_K = 64


class kie_model_desc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn_dim", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("n_lanes", ctypes.c_int32), ("lane_delay", ctypes.c_int32),
                ("max_seq", ctypes.c_int32)]


class kie_stats(ctypes.Structure):
    _fields_ = [("n_ctas", ctypes.c_int32), ("threads_per_cta", ctypes.c_int32),
                ("ring_slots", ctypes.c_int32), ("slot_bytes", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("pos", ctypes.c_int32),
                ("weight_bytes_per_step", ctypes.c_int64),
                ("kv_bytes_per_position", ctypes.c_int64),
                ("last_kernel_ms", ctypes.c_float), ("last_launch_steps", ctypes.c_int32),
                ("pending_token", ctypes.c_int32), ("last_prefill_ms", ctypes.c_float),
                ("prefill_mode", ctypes.c_int32)]


class kie_sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_k", ctypes.c_int32),
                ("top_p", ctypes.c_float)]


class KieError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{msg} (status {code})")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


_lib_path = None


def load(path: str = None) -> ctypes.CDLL:
    """Load libkie.so (built by ``build.py``), or ``path`` (e.g. the profiling
    build libkie_prof.so); raises if it is not there.  One library per process:
    asking for a different one after the first load raises."""
    global _lib, _lib_path
    if _lib is not None:
        if path is not None and os.path.abspath(path) != _lib_path:
            raise RuntimeError(f"{_lib_path} is already loaded; cannot switch to {path}")
        return _lib
    path = LIB_PATH if path is None else path
    if not os.path.exists(path):
        raise RuntimeError(f"libkie.so not built: {path} is missing (run "
                           "decode_persistent_monokernel_b200/build.py)")
    L = ctypes.CDLL(path)
    sig = {
        "kie_create": ([ctypes.POINTER(kie_model_desc), _P, _P, ctypes.POINTER(_P)], _I),
        "kie_weights_bytes": ([ctypes.POINTER(kie_model_desc), ctypes.POINTER(ctypes.c_int64)], _I),
        "kie_prefill": ([_P, _P, _I, ctypes.POINTER(_I)], _I),
        "kie_prefill_ex": ([_P, _P, _I, ctypes.POINTER(_I), _P], _I),
        "kie_set_prefill_mode": ([_P, _I], _I),
        "kie_decode": ([_P, _I, _P], _I),
        "kie_decode_ex": ([_P, _I, _P, _P, _P], _I),
        "kie_decode_ex_static": ([_P, _I, _P, _P, _P], _I),
        "kie_decode_sample": ([_P, _I, ctypes.POINTER(kie_sampling), _P, _P, _P, _P], _I),
        "kie_destroy": ([_P], _I),
        "kie_strerror": ([_I], ctypes.c_char_p),
        "kie_get_stats": ([_P, ctypes.POINTER(kie_stats)], _I),
        "kie_copy_kv": ([_P, _I, _I, _I, _I, _P, _P], _I),
        "kie_debug_set": ([_P, _I, _I], _I),
        "kie_set_sync_mode": ([_P, _I], _I),
        "kie_set_sum_mode": ([_P, _I], _I),
        "kie_set_max_steps_per_launch": ([_P, _I], _I),
        "kie_trace_request": ([_P, _I, _I], _I),
        "kie_get_trace": ([_P, _P, _I], _I),
        "kie_get_profile": ([_P, _P, _I], _I),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    _lib_path = os.path.abspath(path)
    return L


def header_functions(path: str = HEADER) -> list:
    """Names of every function the C header declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kie_[a-z_]+)\s*\(", text)))


def strerror(code: int) -> str:
    return load().kie_strerror(code).decode()


def _check(code: int) -> None:
    if code != KIE_OK:
        raise KieError(code, strerror(code))


def make_desc(shape, max_seq: int) -> kie_model_desc:
    """A descriptor from any object with the model-shape attributes."""
    return kie_model_desc(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads,
                          shape.head_dim, shape.ffn_dim, shape.vocab, shape.rms_eps,
                          shape.rope_theta, KIE_F16 if shape.dtype == "f16" else KIE_BF16,
                          shape.n_lanes, shape.lane_delay if shape.n_lanes > 1 else 0, max_seq)


def weights_bytes(desc: kie_model_desc) -> int:
    """Bytes of the canonical weights kie_create reads for `desc`."""
    n = ctypes.c_int64()
    _check(load().kie_weights_bytes(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def _ptr(buf):
    """Address of a torch tensor or a numpy array (host buffers must be contiguous)."""
    if buf is None:
        return None
    if hasattr(buf, "data_ptr"):
        return buf.data_ptr()
    return buf.ctypes.data


class Decoder:
    """Owns one kie_ctx.  Host-side token arrays are int32 numpy arrays."""

    def __init__(self, desc: kie_model_desc, weights_dev, stream=None):
        L = load()
        self._h = _P()
        if hasattr(weights_dev, "data_ptr"):
            # the library reads exactly weights_bytes(desc) from the pointer
            need = weights_bytes(desc)
            if not (weights_dev.is_cuda and weights_dev.is_contiguous()
                    and weights_dev.numel() * weights_dev.element_size() == need):
                raise ValueError(f"weights must be a contiguous CUDA tensor of {need} bytes "
                                 f"(the canonical layout of this model)")
        st = None if stream is None else (stream.cuda_stream if hasattr(stream, "cuda_stream")
                                          else stream)
        _check(L.kie_create(ctypes.byref(desc), _ptr(weights_dev), st, ctypes.byref(self._h)))
        self.desc = desc

    def kie_prefill(self, tokens) -> int:
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        nxt = _I()
        _check(load().kie_prefill(self._h, t.ctypes.data, len(t), ctypes.byref(nxt)))
        return nxt.value

    def kie_prefill_ex(self, tokens, logits_out=None) -> int:
        """kie_prefill; logits_out (float32 CUDA tensor of vocab elements, or
        None) receives the logits of the last prompt position."""
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        if logits_out is not None:
            if not (hasattr(logits_out, "data_ptr") and logits_out.is_cuda
                    and str(logits_out.dtype) == "torch.float32" and logits_out.is_contiguous()
                    and logits_out.numel() >= self.desc.vocab):
                raise ValueError(f"logits_out must be a contiguous float32 CUDA tensor of at "
                                 f"least vocab = {self.desc.vocab} elements")
        nxt = _I()
        _check(load().kie_prefill_ex(self._h, t.ctypes.data, len(t), ctypes.byref(nxt),
                                     _ptr(logits_out)))
        return nxt.value

    def kie_set_prefill_mode(self, mode: int) -> None:
        _check(load().kie_set_prefill_mode(self._h, mode))

    def kie_decode(self, n_steps: int):
        import numpy as np
        out = np.empty(n_steps, dtype=np.int32)
        _check(load().kie_decode(self._h, n_steps, out.ctypes.data))
        return out

    def _decode_args(self, n_steps: int, forced, logits_out):
        """The library reads n_steps forced tokens and writes n_steps * vocab
        logits through raw pointers, so their buffers are checked here."""
        import numpy as np
        f = None
        if forced is not None:
            f = np.ascontiguousarray(forced, dtype=np.int32)
            if f.ndim != 1 or f.size != n_steps:
                raise ValueError(f"forced must hold exactly n_steps = {n_steps} token ids")
        if logits_out is not None:
            need = max(n_steps, 0) * self.desc.vocab
            if not (hasattr(logits_out, "data_ptr") and logits_out.is_cuda
                    and str(logits_out.dtype) == "torch.float32" and logits_out.is_contiguous()
                    and logits_out.numel() >= need):
                raise ValueError(f"logits_out must be a contiguous float32 CUDA tensor of at "
                                 f"least n_steps * vocab = {need} elements")
        return (None if f is None else f.ctypes.data), _ptr(logits_out), f

    def kie_decode_ex(self, n_steps: int, forced=None, logits_out=None):
        import numpy as np
        out = np.empty(n_steps, dtype=np.int32)
        fp, lp, _keep = self._decode_args(n_steps, forced, logits_out)
        _check(load().kie_decode_ex(self._h, n_steps, fp, out.ctypes.data, lp))
        return out

    def kie_decode_sample(self, n_steps: int, temperature: float, top_k: int = 0,
                          top_p: float = 1.0, uniforms=None, forced=None, logits_out=None):
        """kie_decode_ex with each step's token drawn (temperature, top-k,
        top-p, inverse CDF at uniforms[k]) instead of the argmax."""
        import numpy as np
        out = np.empty(n_steps, dtype=np.int32)
        fp, lp, _keep = self._decode_args(n_steps, forced, logits_out)
        u = None
        if uniforms is not None:
            u = np.ascontiguousarray(uniforms, dtype=np.float32)
            if u.ndim != 1 or u.size != n_steps:
                raise ValueError(f"uniforms must hold exactly n_steps = {n_steps} values")
        prm = kie_sampling(float(temperature), int(top_k), float(top_p))
        _check(load().kie_decode_sample(self._h, n_steps, ctypes.byref(prm),
                                        None if u is None else u.ctypes.data, fp,
                                        out.ctypes.data, lp))
        return out

    def kie_decode_ex_static(self, n_steps: int, forced=None, logits_out=None):
        """kie_decode_ex with the kernel scratch in the library's fixed device array."""
        import numpy as np
        out = np.empty(n_steps, dtype=np.int32)
        fp, lp, _keep = self._decode_args(n_steps, forced, logits_out)
        _check(load().kie_decode_ex_static(self._h, n_steps, fp, out.ctypes.data, lp))
        return out

    def kie_get_stats(self) -> kie_stats:
        s = kie_stats()
        _check(load().kie_get_stats(self._h, ctypes.byref(s)))
        return s

    def kie_copy_kv(self, layer: int, kv_head: int, pos0: int, n: int):
        import numpy as np
        k = np.empty((n, self.desc.head_dim), dtype=np.uint16)
        v = np.empty((n, self.desc.head_dim), dtype=np.uint16)
        _check(load().kie_copy_kv(self._h, layer, kv_head, pos0, n, k.ctypes.data, v.ctypes.data))
        return k, v

    def kie_get_profile(self):
        """Per-SM activity counters [n_ctas, 32] of the last launch (profiling build)."""
        import numpy as np
        n = self.kie_get_stats().n_ctas
        out = np.zeros((n, 32), dtype=np.uint64)
        _check(load().kie_get_profile(self._h, out.ctypes.data, out.size))
        return out

    def kie_debug_set(self, watchdog_ms: int, skip_signal_cta: int = -1) -> None:
        _check(load().kie_debug_set(self._h, watchdog_ms, skip_signal_cta))

    def kie_trace_request(self, cta: int, step: int) -> None:
        _check(load().kie_trace_request(self._h, cta, step))

    def kie_get_trace(self):
        """(clock, type, argument) triples of the last traced launch."""
        import numpy as np
        out = np.zeros(65537, dtype=np.uint64)
        _check(load().kie_get_trace(self._h, out.ctypes.data, out.size))
        n = int(min(out[0], out.size - 1))
        ev = out[1:1 + n]
        return ev >> np.uint64(8), (ev >> np.uint64(4)) & np.uint64(15), ev & np.uint64(15)

    def kie_set_sync_mode(self, mode: int) -> None:
        _check(load().kie_set_sync_mode(self._h, mode))

    def kie_set_sum_mode(self, mode: int) -> None:
        _check(load().kie_set_sum_mode(self._h, mode))

    def kie_set_max_steps_per_launch(self, n: int) -> None:
        _check(load().kie_set_max_steps_per_launch(self._h, n))

    def kie_destroy(self) -> None:
        if self._h:
            _check(load().kie_destroy(self._h))
            self._h = _P()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.kie_destroy()

    def __del__(self):
        try:
            if self._h:
                load().kie_destroy(self._h)
        except Exception:
            pass
