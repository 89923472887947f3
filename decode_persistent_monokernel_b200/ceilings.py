"""Ceilings for the decode kernel on the local GPU (libkie_ubench.so).

    python -m decode_persistent_monokernel_b200.ceilings

prints one JSON object:
  * launch_us: one empty kernel launch, back to back (what a decode made of
    one kernel per operation pays for each operation);
  * grid_wait_us: one dependency point across all SMs (release-add and
    acquire-poll of one counter), the decode kernel's wait for every SM;
  * stream_*: the decode kernel's weight stream alone -- its 32 KB bulk-copy
    ring with 16 consumer warps -- with and without the row-GEMV arithmetic,
    from HBM (regions far larger than L2) and from L2 (small regions walked
    repeatedly), in GB/s and microseconds per 32 KB tile per SM.
"""
from __future__ import annotations

import ctypes
import json
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkie_ubench.so")
TILE = 32768


def load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run decode_persistent_monokernel_b200.build")
    lib = ctypes.CDLL(path)
    f = ctypes.POINTER(ctypes.c_float)
    lib.kie_ubench_launch_overhead.argtypes = [ctypes.c_int32, f]
    lib.kie_ubench_stream.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, f]
    lib.kie_ubench_barrier.argtypes = [ctypes.c_int32, ctypes.c_int32, f]
    for fn in (lib.kie_ubench_launch_overhead, lib.kie_ubench_stream, lib.kie_ubench_barrier):
        fn.restype = ctypes.c_int32
    return lib


def _call(fn, *args):
    out = ctypes.c_float()
    rc = fn(*args, ctypes.byref(out))
    if rc != 0:
        raise RuntimeError(f"{fn.__name__} failed with status {rc}")
    return float(out.value)


def measure(hbm_mb_per_cta: int = 32, l2_kb_per_cta: int = 256, l2_passes: int = 64):
    import torch
    lib = load()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    out = {"sms": n_sm}
    out["launch_us"] = round(_call(lib.kie_ubench_launch_overhead, 2000), 3)
    out["grid_wait_us"] = round(_call(lib.kie_ubench_barrier, n_sm, 2000), 3)
    region = hbm_mb_per_cta << 20
    buf = torch.full((n_sm * region // 2,), 0.01, dtype=torch.float16, device="cuda")
    for slots in (3, 4, 6):
        for consume in (0, 1):
            ms = _call(lib.kie_ubench_stream, buf.data_ptr(), region, n_sm, 1, slots, consume)
            tiles = region // TILE
            out[f"stream_hbm_ns{slots}_gemv{consume}"] = {
                "GBps": round(n_sm * region / (ms * 1e-3) / 1e9, 1),
                "us_per_tile": round(ms * 1e3 / tiles, 4)}
    small = l2_kb_per_cta << 10
    for consume in (0, 1):
        ms = _call(lib.kie_ubench_stream, buf.data_ptr(), small, n_sm, l2_passes, 6, consume)
        tiles = small // TILE * l2_passes
        out[f"stream_l2_ns6_gemv{consume}"] = {
            "GBps": round(n_sm * small * l2_passes / (ms * 1e-3) / 1e9, 1),
            "us_per_tile": round(ms * 1e3 / tiles, 4)}
    del buf
    return out


if __name__ == "__main__":
    print(json.dumps(measure()))
