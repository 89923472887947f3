"""The seeded input generator: reproducible bytes, thread-count invariance,
and the distribution it is asked for."""
import json
import os

import numpy as np

import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "synth_checksums.json")


def test_checksums_of_small_workloads():
    gold = json.load(open(GOLD))
    w = synth.WORKLOADS[0]
    bits = synth.generate_weights(w.model, w.weight_seed)
    assert hex(synth.fnv1a64(bits)) == gold["0"]["weights_fnv1a64"]
    assert hex(synth.fnv1a64(synth.prompt(w))) == gold["0"]["prompt_fnv1a64"]


def test_thread_count_invariance(monkeypatch):
    import subprocess
    import sys
    code = ("import synth,sys;w=synth.WORKLOADS[0];"
            "print(hex(synth.fnv1a64(synth.generate_weights(w.model,w.weight_seed))))")
    outs = set()
    for n in ("1", "3"):
        env = dict(os.environ, OMP_NUM_THREADS=n)
        outs.add(subprocess.check_output([sys.executable, "-c", code], env=env,
                                         cwd=os.path.dirname(os.path.dirname(os.path.dirname(GOLD)))).strip())
    assert len(outs) == 1


def test_distribution_and_tokens():
    m = synth.WORKLOADS[0].model
    bits = synth.generate_weights(m, 1)
    spec = {t.name: t for t in synth.tensor_table(m)}
    t = spec["layers.0.w_gate"]
    v = bits[t.offset:t.offset + t.numel].view(np.float16).astype(np.float64)
    assert abs(v.mean()) < 2e-4 and abs(v.std() - 0.02) < 2e-4
    g = bits[spec["layers.0.attn_norm"].offset:][:256].view(np.float16)
    assert (g == 1.0).all()
    toks = synth.generate_tokens(100000, 4096, 5)
    assert toks.min() >= 0 and toks.max() < 4096
    counts = np.bincount(toks, minlength=4096)
    assert counts.std() < 3 * np.sqrt(100000 / 4096)
