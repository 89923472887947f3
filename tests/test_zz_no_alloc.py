"""kie_decode_ex_static, the decode call that allocates nothing.

It serves callers that may not allocate device memory while they decode; its
kernel scratch is the library's fixed device array.  It must give what
kie_decode_ex gives on the same context state, call after call (the array
keeps the previous call's contents, so two calls in a row are compared).
This file is collected last so that a failure here comes after every other
test has run.
"""
import numpy as np
import pytest

import synth
from oracle import top2_margin
from tests.gpu_util import NEAR_TIE, check_argmax, check_logits, make_decoder

pytestmark = pytest.mark.gpu


def _run(dec, fn, prompt, forced, chunks, vocab):
    import torch
    dec.kie_prefill(prompt)
    toks, zs = [], []
    s = 0
    for n in chunks:
        z = torch.empty((n, vocab), dtype=torch.float32, device="cuda")
        f = None if forced is None else forced[s:s + n]
        toks.append(fn(n, forced=f, logits_out=z))
        torch.cuda.synchronize()
        zs.append(z.cpu().numpy())
        s += n
    return np.concatenate(toks), np.vstack(zs)


_TINY = synth.WORKLOADS[0].model
_SHAPES = {
    "tiny": _TINY,
    # a lane model: its delayed cross-lane sums also live in the fixed array
    "lanes2_d2": _TINY.replace(n_lanes=2, lane_delay=2, n_layers=4, mix_std=0.02, gain_std=0.1),
}


@pytest.mark.parametrize("shape", sorted(_SHAPES))
@pytest.mark.parametrize("cap", [0, 3])
@pytest.mark.parametrize("teacher_forced", [True, False])
def test_static_scratch_is_bit_exact_with_exact_sums(shape, cap, teacher_forced):
    """With fixed-point O / down sums every launch is deterministic, so the
    static-scratch call must give exactly the logits and tokens of
    kie_decode_ex, call after call; also when each call is split into launches
    of at most 3 steps (the keys and tokens of every launch come from the
    fixed array too)."""
    import torch
    import decode_persistent_monokernel_b200 as kie
    assert torch.cuda.is_available()
    m = _SHAPES[shape]
    bits = synth.generate_weights(m, 41)
    prompt = synth.generate_tokens(11, m.vocab, 3)
    forced = synth.generate_tokens(24, m.vocab, 4) if teacher_forced else None
    dec = make_decoder(m, bits, 64)
    dec.kie_set_sum_mode(kie.KIE_SUM_EXACT)
    dec.kie_set_max_steps_per_launch(cap)
    chunks = (10, 14)                       # two calls in a row
    t_ref, z_ref = _run(dec, dec.kie_decode_ex, prompt, forced, chunks, m.vocab)
    t_new, z_new = _run(dec, dec.kie_decode_ex_static, prompt, forced, chunks, m.vocab)
    assert np.array_equal(t_new, t_ref)
    assert np.array_equal(z_new.view(np.uint32), z_ref.view(np.uint32))
    assert dec.kie_get_stats().pos == len(prompt) + sum(chunks)
    dec.kie_destroy()


@pytest.mark.parametrize("teacher_forced", [True, False])
def test_static_scratch_decode_matches_decode_ex(teacher_forced):
    import torch
    assert torch.cuda.is_available()
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, 24) if teacher_forced else None
    dec = make_decoder(m, bits, 64)
    chunks = (10, 14)                       # two calls in a row
    t_ref, z_ref = _run(dec, dec.kie_decode_ex, prompt, forced, chunks, m.vocab)
    t_new, z_new = _run(dec, dec.kie_decode_ex_static, prompt, forced, chunks, m.vocab)
    # the default fp32 atomic sums may differ between two launches in the last
    # bits: compare logits within the tests' tolerance and tokens by the
    # near-tie rule; a free run may part ways only at a near tie
    n = len(t_ref)
    if not teacher_forced:
        for k in range(n):
            if t_new[k] != t_ref[k]:
                assert top2_margin(z_ref[k]) < NEAR_TIE, (k, t_new[k], t_ref[k])
                n = k + 1
                break
    check_logits(z_new[:n], z_ref[:n], "static scratch")
    check_argmax(t_new[:n], z_ref[:n], "static scratch")
    assert dec.kie_get_stats().pos == len(prompt) + sum(chunks)
    dec.kie_destroy()


def test_static_scratch_rejects_oversize():
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    dec = make_decoder(m, bits, 200000)
    dec.kie_prefill(synth.prompt(w))
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode_ex_static(150000)   # argmax keys alone exceed the fixed array
    assert e.value.code == kie.KIE_ERR_CAPACITY
    assert "static scratch" in str(e.value)
    # the context is unharmed: a fitting call still works
    assert len(dec.kie_decode_ex_static(4)) == 4
    dec.kie_destroy()
