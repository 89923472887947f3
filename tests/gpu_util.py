"""Helpers shared by the GPU parity tests (acceptance rules, device setup)."""
import numpy as np

from oracle import top2_margin

REL_L2 = 1e-3      # per-step logits: ||z_gpu - z_ora|| / ||z_ora||
MAX_ABS = 2e-2     # per-step logits: max |z_gpu - z_ora|
NEAR_TIE = 2e-2    # oracle top-2 margin below which the greedy token may differ


def make_decoder(shape, bits, max_seq):
    import torch
    import decode_persistent_monokernel_b200 as kie
    w = torch.from_numpy(bits.view(np.int16)).cuda()
    dec = kie.Decoder(kie.make_desc(shape, max_seq), w)
    torch.cuda.synchronize()
    del w   # the library copied what it needs
    return dec


def check_logits(z_gpu, z_ora, label=""):
    """Per-step acceptance: relative L2 and max-abs error of each step's logits."""
    z_gpu = np.asarray(z_gpu, dtype=np.float64)
    z_ora = np.asarray(z_ora, dtype=np.float64)
    assert z_gpu.shape == z_ora.shape
    assert np.isfinite(z_gpu).all(), f"{label}: non-finite logits"
    rel = np.linalg.norm(z_gpu - z_ora, axis=-1) / np.linalg.norm(z_ora, axis=-1)
    mab = np.abs(z_gpu - z_ora).max(axis=-1)
    assert rel.max() <= REL_L2, f"{label}: rel-L2 {rel.max():.3g} at step {rel.argmax()}"
    assert mab.max() <= MAX_ABS, f"{label}: max-abs {mab.max():.3g} at step {mab.argmax()}"
    return float(rel.max()), float(mab.max())


def check_argmax(tok_gpu, z_ora, label=""):
    """The GPU's argmax must equal the oracle's wherever the oracle's top-2
    margin is at least NEAR_TIE; at near ties it must be one of the tied-ish
    candidates (within NEAR_TIE of the oracle's maximum)."""
    z_ora = np.atleast_2d(z_ora)
    tok_gpu = np.atleast_1d(tok_gpu)
    near = 0
    for k, (t, z) in enumerate(zip(tok_gpu, z_ora)):
        best = int(np.argmax(z))
        if top2_margin(z) >= NEAR_TIE:
            assert t == best, f"{label}: step {k}: gpu {t} oracle {best} margin {top2_margin(z):.3g}"
        else:
            near += 1
            assert 0 <= t < z.size and z[t] >= z[best] - NEAR_TIE, f"{label}: step {k}: bad token"
    return near


def free_run_prefix(gpu_toks, ora_toks, ora_logits, label=""):
    """Free-running greedy tokens must match the oracle's until the first step
    where the oracle's top-2 margin is below NEAR_TIE (past it the runs may
    legitimately diverge).  Returns the number of steps compared exactly."""
    n = 0
    for k in range(len(ora_toks)):
        if top2_margin(ora_logits[k]) < NEAR_TIE:
            break
        assert gpu_toks[k] == ora_toks[k], f"{label}: step {k}: gpu {gpu_toks[k]} oracle {ora_toks[k]}"
        n += 1
    return n
