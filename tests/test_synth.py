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


# ---------------------------------------------------------------------------
# The generator against its published definitions, restated in pure Python
# (independent of synth.c): SplitMix64 (Steele, Lea & Flood 2014), the
# Box-Muller cosine branch, IEEE round-to-nearest-even into binary16 (numpy's
# float64 -> float16 cast), Lemire's multiply-shift, FNV-1a 64.
_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def _mix(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _at(key, n):
    return _mix((key + (n + 1) * _GAMMA) & _M64)


def _key(seed, index):
    return _mix((seed * _GAMMA + 0x632BE59BD9B4E019) & _M64) ^ _mix(((index + 1) * 0xD1B54A32D192ED03) & _M64)


def test_splitmix64_restatement_matches_published_outputs():
    # the first outputs of SplitMix64 seeded with 0 (the reference splitmix64.c)
    assert [_at(0, n) for n in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                            0x06C45D188009454F]


def test_fnv1a64_published_vectors():
    assert synth.fnv1a64(np.frombuffer(b"", dtype=np.uint8)) == 0xCBF29CE484222325
    assert synth.fnv1a64(np.frombuffer(b"a", dtype=np.uint8)) == 0xAF63DC4C8601EC8C
    assert synth.fnv1a64(np.frombuffer(b"foobar", dtype=np.uint8)) == 0x85944171F73967E8


def test_tokens_follow_the_definition():
    seed, vocab, n = 77, 32768, 300
    key = _key(seed, synth.PROMPT_STREAM)
    want = [((_at(key, i) >> 32) * vocab) >> 32 for i in range(n)]
    assert synth.generate_tokens(n, vocab, seed).tolist() == want


def test_normal_draws_follow_the_definition():
    import math
    m = synth.WORKLOADS[0].model
    spec = {t.name: t for t in synth.tensor_table(m)}
    t = spec["layers.1.wq"]
    bits = synth.generate_weights(m, 1234)[t.offset:t.offset + 2000]
    key = _key(1234, t.index)
    want = []
    for i in range(2000):
        u1 = ((_at(key, 2 * i) >> 11) + 0.5) / 9007199254740992.0
        u2 = ((_at(key, 2 * i + 1) >> 11) + 0.5) / 9007199254740992.0
        v = t.mean + t.std * (math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2))
        want.append(int(np.float64(v).astype(np.float16).view(np.uint16)))
    # the same libm log/cos on both sides, so the bits agree exactly
    assert bits.tolist() == want
