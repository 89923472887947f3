"""Sampling at the LM head (temperature, top-k, top-p) vs the oracle's sampler.

Each step's token is an integer decided by float comparisons, so it is
compared with the oracle's sampler applied to the kernel's own logits of
that step (dumped through logits_out): the top-k set then agrees exactly
(the same float32 keys, the same tie rule), and the top-p cut and the draw
may differ only where the oracle puts the cut's mass or the uniform within
1e-5 of a boundary (fp32 against float64 sums).  The logits themselves are
compared with the oracle teacher-forced along the sampled tokens.
"""
import numpy as np
import pytest

import synth
from oracle import Oracle
from oracle.sampling import sample_token, sampling_margins
from synth.configs import ModelShape
from tests.gpu_util import check_logits, make_decoder

pytestmark = pytest.mark.gpu

NEAR = 1e-5


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import decode_persistent_monokernel_b200 as kie
    kie.load()
    return torch


def _sample_run(dec, n, vocab, T, k, p, u, forced=None):
    import torch
    z = torch.empty((n, vocab), dtype=torch.float32, device="cuda")
    toks = dec.kie_decode_sample(n, T, k, p, u, forced=forced, logits_out=z)
    torch.cuda.synchronize()
    return toks, z.cpu().numpy().astype(np.float64)


def check_sampled(toks, z, u, T, k, p, label, max_near=2):
    """Every token equals the oracle sampler's on the same logits, except at
    steps whose cut or draw lies within NEAR of a boundary (at most max_near
    of them may differ).  Returns the number of such differing steps."""
    diff = 0
    for s in range(len(toks)):
        want = sample_token(z[s], float(u[s]), T, k, p)
        if int(toks[s]) == want:
            continue
        _, cut_gap, draw_gap = sampling_margins(z[s], float(u[s]), T, k, p)
        assert min(cut_gap, draw_gap) < NEAR, (
            f"{label}: step {s}: gpu {toks[s]} oracle {want} (cut gap {cut_gap:.3g}, draw gap {draw_gap:.3g})")
        diff += 1
    assert diff <= max_near, f"{label}: {diff} boundary steps differ"
    return diff


MODES = {
    "top_k_top_p": (0.8, 40, 0.9),
    "top_k": (1.0, 20, 1.0),
    "cold_nucleus": (0.3, 64, 0.5),
    "full_vocab": (1.0, 0, 1.0),
}


@pytest.mark.parametrize("mode", sorted(MODES))
def test_tiny_sampling_matches_the_oracle(mode):
    T, k, p = MODES[mode]
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    u = np.random.default_rng(100 + len(mode)).random(N).astype(np.float32)
    dec = make_decoder(m, bits, P + N + 8)
    t0 = dec.kie_prefill(prompt)
    toks, z = _sample_run(dec, N, m.vocab, T, k, p, u)
    st = dec.kie_get_stats()
    assert st.pos == P + N and st.pending_token == toks[-1]
    assert np.all((toks >= 0) & (toks < m.vocab))
    check_sampled(toks, z, u, T, k, p, mode)
    # the logits along the sampled path are the oracle's
    fed = np.concatenate([[t0], toks[:-1]]).astype(np.int32)
    orc = Oracle(m, bits, P + N + 8)
    check_logits(z, orc.teacher_forced_logits(prompt, fed), f"{mode} logits")
    # a sampled run is not a greedy run: at T = 1 most steps leave the argmax
    if mode in ("top_k", "full_vocab"):
        assert np.mean(toks != z.argmax(axis=1)) > 0.5
    dec.kie_destroy()


def test_top_k_one_and_zero_temperature_are_greedy():
    """With order-independent sums the logits repeat exactly, so top-k 1 (any
    uniforms) and temperature 0 give the greedy tokens bit for bit."""
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    runs = []
    for how in ("greedy", "top1", "t0"):
        dec = make_decoder(m, bits, P + N + 8)
        dec.kie_set_sum_mode(kie.KIE_SUM_EXACT)
        dec.kie_prefill(prompt)
        u = np.random.default_rng(5).random(N).astype(np.float32)
        if how == "greedy":
            runs.append(dec.kie_decode(N))
        elif how == "top1":
            runs.append(dec.kie_decode_sample(N, 0.7, 1, 1.0, u))
        else:
            runs.append(dec.kie_decode_sample(N, 0.0, 0, 1.0, None))
        dec.kie_destroy()
    assert np.array_equal(runs[0], runs[1]) and np.array_equal(runs[0], runs[2])


@pytest.mark.parametrize("cap", [1, 5])
def test_sampling_across_launches(cap):
    """Split into launches of at most `cap` steps, each launch reads its own
    run of uniforms: the tokens equal one launch's (order-independent sums)."""
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    u = np.random.default_rng(9).random(N).astype(np.float32)
    out = []
    for c in (0, cap):
        dec = make_decoder(m, bits, P + N + 8)
        dec.kie_set_sum_mode(kie.KIE_SUM_EXACT)
        if c:
            dec.kie_set_max_steps_per_launch(c)
        dec.kie_prefill(prompt)
        out.append(dec.kie_decode_sample(N, 0.9, 30, 0.95, u))
        dec.kie_destroy()
    assert np.array_equal(out[0], out[1])


def test_large_vocabulary_slices():
    """A vocabulary of 150,016 puts 1,014 LM-head rows on each of 148 SMs: the
    per-SM sort of the top-k cut runs at 1,024 keys."""
    m = ModelShape(n_layers=1, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64, ffn_dim=704,
                   vocab=150016)
    bits = synth.generate_weights(m, 77)
    prompt = synth.generate_tokens(8, m.vocab, 78)
    N = 12
    dec = make_decoder(m, bits, 8 + N + 4)
    dec.kie_prefill(prompt)
    for (T, k, p), seed in (((0.9, 50, 0.8), 1), ((1.0, 0, 1.0), 2)):
        u = np.random.default_rng(seed).random(N).astype(np.float32)
        dec.kie_prefill(prompt)
        toks, z = _sample_run(dec, N, m.vocab, T, k, p, u)
        check_sampled(toks, z, u, T, k, p, f"V 150016, k {k}")
    dec.kie_destroy()


@pytest.mark.parametrize("mode", ["top_k_top_p", "full_vocab"])
def test_full_size_sampling(mode, dense_2b):
    """The 2.3B-class model (V 32,768 over 148 SMs), 32 sampled steps after
    the 128-token prompt."""
    T, k, p = MODES[mode]
    w, bits = dense_2b
    m = w.model
    prompt = synth.prompt(w)
    N = 32
    u = np.random.default_rng(31).random(N).astype(np.float32)
    dec = make_decoder(m, bits, len(prompt) + N + 4)
    dec.kie_prefill(prompt)
    toks, z = _sample_run(dec, N, m.vocab, T, k, p, u)
    check_sampled(toks, z, u, T, k, p, f"2.3B {mode}")
    dec.kie_destroy()


def test_8b_class_shapes_sampling():
    """The 8B-class workload's shapes (bf16, 4 query heads per KV head,
    V 128,256: 867 LM-head rows per SM) on two layers, 24 sampled steps
    after a 64-token prompt, in both sampling modes."""
    w = synth.WORKLOADS[4]
    m = w.model.replace(n_layers=2)
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)[:64]
    N = 24
    dec = make_decoder(m, bits, len(prompt) + N + 4)
    for mode, seed in (("top_k_top_p", 41), ("full_vocab", 42)):
        T, k, p = MODES[mode]
        u = np.random.default_rng(seed).random(N).astype(np.float32)
        dec.kie_prefill(prompt)
        toks, z = _sample_run(dec, N, m.vocab, T, k, p, u)
        check_sampled(toks, z, u, T, k, p, f"8b-2L {mode}")
    dec.kie_destroy()


def test_all_logits_equal():
    """A zeroed LM head makes every logit a signed zero (+0 or -0 by the sign of
    the last products): all tie.  Greedy must take token 0 at every step (the
    lowest index of the largest value, g11), and top-k 5 must keep ids 0..4,
    each drawn with probability 1/5: the uniform u picks id floor(5 u)."""
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed).copy()
    lm = {t.name: t for t in synth.tensor_table(m)}["lm_head"]
    bits[lm.offset:lm.offset + lm.numel] = 0
    prompt = synth.prompt(w)
    N = 16
    dec = make_decoder(m, bits, len(prompt) + 2 * N + 8)
    assert dec.kie_prefill(prompt) == 0
    assert np.all(dec.kie_decode(N) == 0)
    u = np.random.default_rng(3).random(N).astype(np.float32)
    dec.kie_prefill(prompt)
    toks, z = _sample_run(dec, N, m.vocab, 1.0, 5, 1.0, u)
    assert np.all(z == 0.0)
    check_sampled(toks, z, u, 1.0, 5, 1.0, "all logits equal", max_near=0)
    assert np.array_equal(toks, np.floor(5 * u.astype(np.float64)).astype(np.int32))
    dec.kie_destroy()


@pytest.fixture(scope="module")
def dense_2b():
    w = synth.WORKLOADS[1]
    return w, synth.generate_weights(w.model, w.weight_seed)


def test_bad_sampling_arguments():
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    dec = make_decoder(m, bits, 64)
    dec.kie_prefill(synth.prompt(w))
    u = np.full(4, 0.5, dtype=np.float32)
    bad = [(-1.0, 10, 1.0, u), (np.inf, 10, 1.0, u), (1.0, 65, 1.0, u), (1.0, -1, 1.0, u),
           (1.0, 10, 0.0, u), (1.0, 10, 1.5, u), (1.0, 0, 0.9, u),
           (1.0, 10, 1.0, np.array([0.1, 1.0, 0.2, 0.3], np.float32)),
           (1.0, 10, 1.0, np.array([0.1, np.nan, 0.2, 0.3], np.float32)),
           (1.0, 10, 1.0, None)]
    pos = dec.kie_get_stats().pos
    for T, k, p, uu in bad:
        with pytest.raises(kie.KieError) as e:
            dec.kie_decode_sample(4, T, k, p, uu)
        assert e.value.code == kie.KIE_ERR_INVALID, (T, k, p)
    assert dec.kie_get_stats().pos == pos       # nothing ran
    toks = dec.kie_decode_sample(4, 1.0, 10, 0.9, u)   # still usable
    assert np.all((toks >= 0) & (toks < m.vocab))
    dec.kie_destroy()
