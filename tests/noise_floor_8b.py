"""Noise floor of the full-depth 8B-class parity case (run by hand, ~10 min of CPU).

    python tests/noise_floor_8b.py [eps ...]

The oracle (float64) against itself with its k and v perturbed by a relative
eps before they are rounded to the bf16 cache, on the exact case of
tests/test_gpu_parity.py::test_8b_class_full_model (the 1024-token prompt,
16 teacher-forced steps).  eps of 1e-6 is the size of fp32-versus-float64
differences: any fp32 implementation sees this much logits difference from the
oracle through one-ulp bf16 rounding flips alone.  Measured: rel-L2 1.9e-3,
max-abs 0.012 at eps 1e-6; 6.1e-4 at eps 1e-7.
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle.decoder as od  # noqa: E402
import synth  # noqa: E402
from oracle import Oracle  # noqa: E402


def main(eps_list):
    w = synth.WORKLOADS[4]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, 16)
    P, N = len(prompt), len(forced)
    z_ref = Oracle(m, bits, P + N + 4).teacher_forced_logits(prompt, forced)
    orig = od.round_to_storage
    for eps in eps_list:
        rng = np.random.default_rng(11)
        od.round_to_storage = lambda x, dtype: orig(x * (1 + eps * rng.standard_normal(x.shape)), dtype)
        try:
            z = Oracle(m, bits, P + N + 4).teacher_forced_logits(prompt, forced)
        finally:
            od.round_to_storage = orig
        rel = np.linalg.norm(z_ref - z, axis=1) / np.linalg.norm(z_ref, axis=1)
        print(f"eps {eps:g}: logits rel-L2 max {rel.max():.3g}, max-abs {np.abs(z_ref - z).max():.3g}", flush=True)


if __name__ == "__main__":
    main([float(e) for e in sys.argv[1:]] or [1e-6, 1e-7])
