"""The C-ABI library loads, exports every function include/kie.h declares, and
rejects bad descriptors on the host (no GPU needed: validation runs before any
CUDA call)."""
import ctypes
import os
import subprocess

import pytest

import synth

import decode_persistent_monokernel_b200 as kie
from decode_persistent_monokernel_b200 import build as kbuild


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kie.load()


def test_exports_every_declared_function(lib):
    names = kie.header_functions()
    assert {"kie_create", "kie_prefill", "kie_decode", "kie_decode_ex", "kie_destroy",
            "kie_strerror"} <= set(names)
    out = subprocess.check_output(["nm", "-D", "--defined-only", kie.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)


def test_ubench_library_exports_its_header(lib):
    from decode_persistent_monokernel_b200 import ceilings
    hdr = os.path.join(os.path.dirname(kie.HEADER), "kie_ubench.h")
    names = kie.header_functions(hdr)
    assert set(names) == {"kie_ubench_launch_overhead", "kie_ubench_stream",
                          "kie_ubench_barrier"}
    out = subprocess.check_output(["nm", "-D", "--defined-only", ceilings.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(names) <= exported
    ub = ceilings.load()
    f = ctypes.c_float()
    # argument checks happen before any device work
    assert ub.kie_ubench_launch_overhead(0, ctypes.byref(f)) == -1
    assert ub.kie_ubench_stream(None, 32768, 1, 1, 6, 1, ctypes.byref(f)) == -1
    assert ub.kie_ubench_stream(ctypes.c_void_p(256), 1000, 1, 1, 6, 1, ctypes.byref(f)) == -1
    assert ub.kie_ubench_stream(ctypes.c_void_p(256), 32768, 1, 1, 7, 1, ctypes.byref(f)) == -1
    assert ub.kie_ubench_barrier(0, 10, ctypes.byref(f)) == -1


def test_build_targets_sm100a_only():
    flags = " ".join(kbuild.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def _desc(**kw):
    base = dict(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn_dim=704,
                vocab=4096, rms_eps=1e-5, rope_theta=1e4, dtype=0, n_lanes=1, lane_delay=0,
                max_seq=64)
    base.update(kw)
    return kie.kie_model_desc(*[base[f] for f, _ in kie.kie_model_desc._fields_])


@pytest.mark.parametrize("bad", [
    dict(head_dim=96, d_model=384),      # head_dim must be 64 or 128
    dict(n_kv_heads=3),                  # heads not a multiple of kv heads
    dict(d_model=264),                   # n_heads * head_dim != d_model
    dict(dtype=7),
    dict(n_lanes=2, lane_delay=1),       # delay must be >= 2
    dict(n_lanes=3),                     # lanes must divide the sizes
    dict(ffn_dim=700),                   # not a multiple of 8
    dict(max_seq=0),
    dict(n_heads=8, n_kv_heads=1, d_model=512),  # more than 4 q heads per kv head
    # rows shared by K/128 lanes of a warp: 128 x a power of two only
    dict(n_heads=6, n_kv_heads=6, head_dim=128, d_model=768),
    dict(n_heads=24, n_kv_heads=8, head_dim=128, d_model=3072, ffn_dim=8192),
    dict(n_lanes=3, lane_delay=2, n_heads=6, n_kv_heads=3, d_model=384, ffn_dim=768),
])
def test_invalid_descriptors_rejected(lib, bad):
    h = ctypes.c_void_p()
    rc = lib.kie_create(ctypes.byref(_desc(**bad)), ctypes.c_void_p(16), None, ctypes.byref(h))
    assert rc == kie.KIE_ERR_INVALID
    assert not h.value


def test_weights_bytes_matches_the_canonical_layout(lib):
    # the library's layout size against the generator's own tensor table
    for w in synth.WORKLOADS.values():
        desc = kie.make_desc(w.model, 64)
        assert kie.weights_bytes(desc) == 2 * synth.total_elements(w.model), w.model
        # a step streams all of it but the V - 1 embedding rows it does not use
        m = w.model
        assert kie.weights_bytes(desc) - 2 * (m.vocab - 1) * m.d_model == \
            synth.streamed_weight_bytes(m)
    n = ctypes.c_int64()
    assert lib.kie_weights_bytes(ctypes.byref(_desc(n_kv_heads=3)), ctypes.byref(n)) == \
        kie.KIE_ERR_INVALID
    assert lib.kie_weights_bytes(ctypes.byref(_desc()), None) == kie.KIE_ERR_INVALID


def test_binding_checks_the_weights_tensor_before_the_library(lib):
    import torch
    desc = _desc()
    with pytest.raises(ValueError):      # a host tensor
        kie.Decoder(desc, torch.zeros(kie.weights_bytes(desc) // 2, dtype=torch.int16))


def test_binding_checks_decode_buffers_before_the_library(lib):
    # a Decoder shell (no context: nothing may reach the library) with a model
    # descriptor, to exercise the argument checks alone
    import numpy as np
    import torch
    dec = kie.Decoder.__new__(kie.Decoder)
    dec._h = ctypes.c_void_p()
    dec.desc = _desc()
    with pytest.raises(ValueError):       # fewer forced tokens than steps
        dec.kie_decode_ex(4, forced=np.zeros(3, dtype=np.int32))
    with pytest.raises(ValueError):       # logits into host memory
        dec.kie_decode_ex(2, logits_out=torch.zeros(2, dec.desc.vocab))
    with pytest.raises(ValueError):       # the static variant checks the same
        dec.kie_decode_ex_static(4, forced=np.zeros(5, dtype=np.int32))
    fp, lp, _ = dec._decode_args(3, np.arange(3), None)
    assert fp is not None and lp is None


_C_CLIENT = r"""
#include <stdio.h>
#include "kie.h"
#include "kie_ubench.h"
int main(void) {
  kie_model_desc d = {0};
  int64_t bytes = 0;
  d.n_layers = 2; d.d_model = 256; d.n_heads = 4; d.n_kv_heads = 4; d.head_dim = 64;
  d.ffn_dim = 704; d.vocab = 4096; d.rms_eps = 1e-5f; d.rope_theta = 1e4f;
  d.dtype = KIE_F16; d.n_lanes = 1; d.lane_delay = 0; d.max_seq = 64;
  int rc = kie_weights_bytes(&d, &bytes);
  printf("%d %lld\n", rc, (long long)bytes);
  d.n_kv_heads = 3;
  const int bad = kie_weights_bytes(&d, &bytes);
  printf("%d %s\n", bad, kie_strerror(KIE_ERR_INVALID));
  return rc;
}
"""


def test_plain_c_client_compiles_links_and_calls_the_library(lib, tmp_path):
    """The headers are plain C (C99, pedantic, warnings as errors) and a C
    program links against libkie.so and calls it (host-only calls here)."""
    src = tmp_path / "client.c"
    src.write_text(_C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(kie.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.dirname(kie.HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-lkie", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    rc, nbytes = out[0].split()
    assert int(rc) == 0 and int(nbytes) == 2 * synth.total_elements(synth.WORKLOADS[0].model)
    assert out[1].startswith(f"{kie.KIE_ERR_INVALID} invalid argument")
    assert "multiple of n_kv_heads" in out[1]


def test_null_and_misaligned_weights_rejected(lib):
    h = ctypes.c_void_p()
    assert lib.kie_create(ctypes.byref(_desc()), None, None, ctypes.byref(h)) == kie.KIE_ERR_INVALID
    assert lib.kie_create(ctypes.byref(_desc()), ctypes.c_void_p(18), None,
                          ctypes.byref(h)) == kie.KIE_ERR_INVALID
    assert lib.kie_create(None, ctypes.c_void_p(16), None, ctypes.byref(h)) == kie.KIE_ERR_INVALID


def test_null_context_calls_rejected(lib):
    assert lib.kie_prefill(None, None, 1, None) == kie.KIE_ERR_INVALID
    assert lib.kie_decode(None, 1, None) == kie.KIE_ERR_INVALID
    assert lib.kie_destroy(None) == kie.KIE_ERR_INVALID
    assert lib.kie_get_stats(None, None) == kie.KIE_ERR_INVALID
    assert "invalid" in kie.strerror(kie.KIE_ERR_INVALID)
    assert "watchdog" in kie.strerror(kie.KIE_ERR_DEVICE_TIMEOUT)
    assert "non-finite" in kie.strerror(kie.KIE_ERR_NONFINITE)
    assert lib.kie_set_sync_mode(None, kie.KIE_SYNC_GRID) == kie.KIE_ERR_INVALID
    assert lib.kie_set_max_steps_per_launch(None, 5) == kie.KIE_ERR_INVALID
    # every other call that takes a context refuses a null one before any device work
    buf = (ctypes.c_uint64 * 8)()
    assert lib.kie_decode_ex(None, 1, None, buf, None) == kie.KIE_ERR_INVALID
    assert lib.kie_decode_ex_static(None, 1, None, buf, None) == kie.KIE_ERR_INVALID
    assert lib.kie_copy_kv(None, 0, 0, 0, 1, buf, buf) == kie.KIE_ERR_INVALID
    assert lib.kie_get_profile(None, buf, 8) == kie.KIE_ERR_INVALID
    assert lib.kie_trace_request(None, 0, 0) == kie.KIE_ERR_INVALID
    assert lib.kie_get_trace(None, buf, 8) == kie.KIE_ERR_INVALID
    assert lib.kie_debug_set(None, 100, -1) == kie.KIE_ERR_INVALID
    assert lib.kie_create(ctypes.byref(_desc()), ctypes.c_void_p(16), None, None) == kie.KIE_ERR_INVALID


def test_binding_loads_one_library_per_process(lib):
    # the library is already loaded by the fixture: asking again returns it,
    # asking for another one raises instead of silently reusing the first
    assert kie.load() is lib
    assert kie.load(kie.LIB_PATH) is lib
    with pytest.raises(RuntimeError):
        kie.load(kie.PROF_LIB_PATH)
