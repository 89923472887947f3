"""CUDA path vs the float64 oracle, element by element, through the C ABI.

Acceptance (per step): logits relative L2 <= 1e-3 and max-abs <= 2e-2; the
greedy token equal to the oracle's wherever the oracle's top-2 margin is at
least 2e-2 (free runs compare up to the first near tie; teacher-forced runs
compare every step); the KV cache written at exactly positions [0, pos) and
NaN beyond.
"""
import numpy as np
import pytest

import synth
from oracle import Oracle
from oracle.numerics import storage_to_f64
from synth.configs import ModelShape
from tests.gpu_util import (REL_L2_BF16_FULL_DEPTH, check_argmax, check_kv, check_logits,
                            free_run_prefix, make_decoder, storage_ulp)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import decode_persistent_monokernel_b200 as kie
    kie.load()
    return torch


def _gpu_logits(dec, n, vocab, forced):
    import torch
    z = torch.empty((n, vocab), dtype=torch.float32, device="cuda")
    toks = dec.kie_decode_ex(n, forced=forced, logits_out=z)
    torch.cuda.synchronize()
    return toks, z.cpu().numpy()


def _check_kv(dec, orc, m, upto, max_seq):
    check_kv(dec, orc, m, upto, max_seq)


def _teacher_forced(m, bits, prompt, forced, label, cache_f64=False, rel_l2=None):
    """Prefill + teacher-forced decode on the GPU, logits compared every step."""
    P, N = len(prompt), len(forced)
    dec = make_decoder(m, bits, P + N + 4)
    t0 = dec.kie_prefill(prompt)
    toks, z = _gpu_logits(dec, N, m.vocab, forced)
    orc = Oracle(m, bits, P + N + 4, cache_f64=cache_f64)
    z_ora = orc.teacher_forced_logits(prompt, forced)
    rel, mab = check_logits(z, z_ora, label, **({} if rel_l2 is None else {"rel_l2": rel_l2}))
    near = check_argmax(toks, z_ora, label)
    return dec, orc, t0, rel, mab, near


# ------------------------------------------------------------ tiny decoder, full protocol
def test_tiny_free_run_teacher_forced_and_cache():
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    max_seq = P + N + 8
    orc = Oracle(m, bits, max_seq)
    t0, z0 = orc.prefill(prompt)
    toks, zs = orc.decode(N)
    dec = make_decoder(m, bits, max_seq)
    g0 = dec.kie_prefill(prompt)
    check_argmax([g0], z0, "prefill")
    gt = dec.kie_decode(N)
    free_run_prefix(np.concatenate([[g0], gt]), np.concatenate([[t0], toks]),
                    np.vstack([z0, zs]), "tiny free run")
    st = dec.kie_get_stats()
    assert st.pos == P + N and st.pending_token == gt[-1]
    # teacher-forced along the oracle's own greedy path, logits every step
    forced = np.concatenate([[t0], toks[:-1]]).astype(np.int32)
    assert dec.kie_prefill(prompt) == g0
    gt2, z = _gpu_logits(dec, N, m.vocab, forced)
    check_logits(z, zs, "tiny teacher-forced")
    check_argmax(gt2, zs, "tiny teacher-forced")
    orc2 = Oracle(m, bits, max_seq)
    orc2.teacher_forced_logits(prompt, forced)
    _check_kv(dec, orc2, m, P + N, max_seq)
    dec.kie_destroy()


@pytest.mark.parametrize("cap", [1, 5])
def test_calls_split_into_several_launches(cap):
    """A call longer than the per-launch step limit runs as several launches,
    each starting where the previous one stopped: the prompt (16 tokens) and
    32 decode steps with at most `cap` steps per launch give the oracle's
    logits, greedy tokens and cache, as one launch does."""
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    max_seq = P + N + 8
    orc = Oracle(m, bits, max_seq)
    t0, z0 = orc.prefill(prompt)
    toks, zs = orc.decode(N)
    dec = make_decoder(m, bits, max_seq)
    dec.kie_set_max_steps_per_launch(cap)
    g0 = dec.kie_prefill(prompt)
    check_argmax([g0], z0, f"prefill, {cap} steps per launch")
    gt = dec.kie_decode(N)
    free_run_prefix(np.concatenate([[g0], gt]), np.concatenate([[t0], toks]),
                    np.vstack([z0, zs]), f"free run, {cap} steps per launch")
    st = dec.kie_get_stats()
    assert st.pos == P + N and st.pending_token == gt[-1] and st.last_launch_steps == N
    forced = np.concatenate([[t0], toks[:-1]]).astype(np.int32)
    dec.kie_prefill(prompt)
    gt2, z = _gpu_logits(dec, N, m.vocab, forced)
    check_logits(z, zs, f"teacher-forced, {cap} steps per launch")
    check_argmax(gt2, zs, f"teacher-forced, {cap} steps per launch")
    orc2 = Oracle(m, bits, max_seq)
    orc2.teacher_forced_logits(prompt, forced)
    _check_kv(dec, orc2, m, P + N, max_seq)
    import decode_persistent_monokernel_b200 as kie
    with pytest.raises(kie.KieError) as e:
        dec.kie_set_max_steps_per_launch(-1)
    assert e.value.code == kie.KIE_ERR_INVALID
    dec.kie_destroy()


@pytest.mark.parametrize("mode", ["fp32_atomic", "exact"])
def test_tiny_is_repeatable(mode):
    """Two launches on fresh contexts.  With fp32 atomic sums the order in
    which SMs add the O and down projections (and so the last bits) differs
    from run to run: the bound, 5e-5 relative, is a twentieth of the logits
    tolerance against the oracle.  With exact sums the two runs are
    bit-identical: logits, tokens of a free run, and the cache."""
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, 24)
    runs, frees, caches = [], [], []
    for _ in range(2):
        dec = make_decoder(m, bits, 64)
        if mode == "exact":
            dec.kie_set_sum_mode(kie.KIE_SUM_EXACT)
        dec.kie_prefill(prompt)
        runs.append(_gpu_logits(dec, 24, m.vocab, forced)[1])
        dec.kie_prefill(prompt)
        frees.append(dec.kie_decode(24))
        caches.append(dec.kie_copy_kv(m.n_layers - 1, 0, 0, 64))
        dec.kie_destroy()
    a, b = runs[0].astype(np.float64), runs[1].astype(np.float64)
    if mode == "exact":
        assert np.array_equal(runs[0].view(np.uint32), runs[1].view(np.uint32))
        assert np.array_equal(frees[0], frees[1])
        assert all(np.array_equal(x, y) for x, y in zip(caches[0], caches[1]))
    else:
        rel = np.linalg.norm(a - b, axis=1) / np.linalg.norm(a, axis=1)
        assert rel.max() < 5e-5, rel.max()


@pytest.mark.parametrize("shape", ["tiny", "gqa2_gains", "lanes2_d2", "bf16"])
def test_exact_sums_match_oracle(shape):
    """Exact (order-independent) O / down sums give oracle-parity logits and tokens."""
    import decode_persistent_monokernel_b200 as kie
    m = synth.WORKLOADS[0].model if shape == "tiny" else _VARIANTS[shape]
    bits = synth.generate_weights(m, 91)
    prompt = synth.generate_tokens(13, m.vocab, 7)
    forced = synth.generate_tokens(30, m.vocab, 8)
    dec = make_decoder(m, bits, 48)
    dec.kie_set_sum_mode(kie.KIE_SUM_EXACT)
    dec.kie_prefill(prompt)
    toks, z = _gpu_logits(dec, 30, m.vocab, forced)
    z_ora = Oracle(m, bits, 48).teacher_forced_logits(prompt, forced)
    check_logits(z, z_ora, f"{shape} fixed point")
    check_argmax(toks, z_ora, f"{shape} fixed point")
    with pytest.raises(kie.KieError) as e:
        dec.kie_set_sum_mode(7)
    assert e.value.code == kie.KIE_ERR_INVALID
    dec.kie_destroy()


@pytest.mark.parametrize("shape", ["tiny", "lanes2_d2"])
def test_grid_barrier_mode_matches_oracle(shape):
    """The grid-barrier ablation (every dependency wait across all SMs) gives
    the same results as the per-dependency counters."""
    import decode_persistent_monokernel_b200 as kie
    m = synth.WORKLOADS[0].model if shape == "tiny" else _VARIANTS[shape]
    bits = synth.generate_weights(m, 77)
    prompt = synth.prompt(synth.WORKLOADS[0])
    forced = synth.forced_tokens(synth.WORKLOADS[0], 12) % m.vocab
    dec = make_decoder(m, bits, 40)
    dec.kie_set_sync_mode(kie.KIE_SYNC_GRID)
    dec.kie_prefill(prompt)
    toks, z = _gpu_logits(dec, 12, m.vocab, forced.astype(np.int32))
    dec.kie_destroy()
    z_ora = Oracle(m, bits, 40).teacher_forced_logits(prompt, forced)
    check_logits(z, z_ora, f"{shape} grid barriers")
    check_argmax(toks, z_ora, f"{shape} grid barriers")


_TINY = synth.WORKLOADS[0].model
_VARIANTS = {
    "gqa2_gains": _TINY.replace(n_kv_heads=2, gain_std=0.1, n_layers=3),
    "gqa4": _TINY.replace(n_heads=4, n_kv_heads=1, n_layers=2),
    "bf16": _TINY.replace(dtype="bf16", rope_theta=500000.0),
    "lanes2_d2": _TINY.replace(n_lanes=2, lane_delay=2, n_layers=4, mix_std=0.02, gain_std=0.1),
    "lanes4_d3": ModelShape(n_layers=5, d_model=1024, n_heads=8, n_kv_heads=8, head_dim=128,
                            ffn_dim=2048, vocab=5000, dtype="f16", n_lanes=4, lane_delay=3,
                            mix_std=0.02),
    "dh128": ModelShape(n_layers=2, d_model=512, n_heads=4, n_kv_heads=2, head_dim=128,
                        ffn_dim=1376, vocab=5000, dtype="f16"),
}


@pytest.mark.parametrize("name", sorted(_VARIANTS))
def test_small_variants(name):
    m = _VARIANTS[name]
    bits = synth.generate_weights(m, 31)
    prompt = synth.generate_tokens(13, m.vocab, 5)
    forced = synth.generate_tokens(40, m.vocab, 6)
    _teacher_forced(m, bits, prompt, forced, name)
    # free run against the oracle's greedy path
    dec = make_decoder(m, bits, 64)
    orc = Oracle(m, bits, 64)
    t0, z0 = orc.prefill(prompt)
    toks, zs = orc.decode(20)
    g0 = dec.kie_prefill(prompt)
    gt = dec.kie_decode(20)
    free_run_prefix(np.concatenate([[g0], gt]), np.concatenate([[t0], toks]),
                    np.vstack([z0, zs]), name)


# ------------------------------------------------------------ full-size workloads
@pytest.fixture(scope="module")
def dense_2b():
    w = synth.WORKLOADS[1]
    return synth.generate_weights(w.model, w.weight_seed)


@pytest.mark.parametrize("cid", [1, 2])
def test_full_size_teacher_forced(cid, dense_2b):
    """Every step of the benchmarked launch shape (prompt P, N decode steps in
    one launch) compared with the oracle on a seeded forced-token sequence."""
    w = synth.WORKLOADS[cid]
    m = w.model
    bits = dense_2b if cid == 1 else synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, w.decode_len)
    dec, orc, t0, rel, mab, near = _teacher_forced(m, bits, prompt, forced, f"cfg{cid}",
                                                   cache_f64=True)
    print(f"cfg{cid}: rel-L2 {rel:.3g} max-abs {mab:.3g} near ties {near}/{w.decode_len}")
    # every layer's cache: written exactly at positions [0, P + N), NaN beyond
    P, N = len(prompt), len(forced)
    _check_kv(dec, orc, m, P + N, P + N + 4)
    # free run: 64 greedy steps against the oracle's own greedy path, compared
    # up to the first step whose oracle margin is a near tie
    n_free = 64
    g0 = dec.kie_prefill(prompt)
    gt = dec.kie_decode(n_free)
    ot0, oz0 = orc.prefill(prompt)
    otoks, ozs = orc.decode(n_free)
    n_eq = free_run_prefix(np.concatenate([[g0], gt]), np.concatenate([[ot0], otoks]),
                           np.vstack([oz0, ozs]), f"cfg{cid} free run")
    print(f"cfg{cid}: free run equal to the oracle for {n_eq} steps (then a near tie)")
    dec.kie_destroy()


def _first_layers(m: ModelShape, bits: np.ndarray, n_layers: int):
    """Weights of the same model truncated to its first n_layers layers."""
    spec = {t.name: t for t in synth.tensor_table(m)}
    first_after = spec["final_norm"].offset
    sub = m.replace(n_layers=n_layers)
    layer_end = synth.tensor_table(sub)[-3].offset + synth.tensor_table(sub)[-3].numel
    out = np.concatenate([bits[:layer_end], bits[first_after:]])
    assert out.size == synth.total_elements(sub)
    return sub, out


def test_long_context_two_layers(dense_2b):
    """The long-context workload's shapes (8192-token prompt, 256 decode steps)
    on the first two layers of the 2.3B-class model."""
    w = synth.WORKLOADS[3]
    m, bits = _first_layers(w.model, dense_2b, 2)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, w.decode_len)
    _, _, _, rel, mab, near = _teacher_forced(m, bits, prompt, forced, "long-2L")
    print(f"long-2L: rel-L2 {rel:.3g} max-abs {mab:.3g} near ties {near}")


def _check_layer0_kv_and_bounds(dec, m, bits, seq, max_seq):
    """Layer 0's cached K/V depend only on each token and its position, so the
    oracle (the model cut to its first layer) checks them at every position of
    ``seq``; at every layer the cache is written exactly up to len(seq) and
    finite there."""
    L = len(seq)
    m1, b1 = _first_layers(m, bits, 1)
    orc = Oracle(m1, b1, max_seq)
    orc.forward(list(seq), logits="none")
    for g in range(m.n_kv_heads):
        k, v = dec.kie_copy_kv(0, g, 0, max_seq)
        kf, vf = storage_to_f64(k, m.dtype), storage_to_f64(v, m.dtype)
        assert np.isnan(kf[L:]).all() and np.isnan(vf[L:]).all()
        for got, want in ((kf[:L], orc.K[0, g, :L]), (vf[:L], orc.V[0, g, :L])):
            # to one storage ulp (a rounding flip) plus 4e-3 of the head's scale
            tol = 4e-3 * np.abs(want).max() + storage_ulp(want, m.dtype)
            assert (np.abs(got - want) <= tol).all(), g
    for l in (1, m.n_layers // 2, m.n_layers - 1):
        for g in (0, m.n_kv_heads - 1):
            k, v = dec.kie_copy_kv(l, g, 0, max_seq)
            for c in (storage_to_f64(k, m.dtype), storage_to_f64(v, m.dtype)):
                assert np.isfinite(c[:L]).all() and np.isnan(c[L:]).all(), (l, g)


def _greedy_full_model(m, bits, w):
    """Prefill the workload's prompt, then its greedy decode steps in one
    launch with the logits kept.  Every fed-back token must be the lowest index
    of the largest logit the kernel wrote for its step (bit-exact: the same
    fp32 values decide both), and the cache must hold the oracle's layer-0 K/V
    for the prompt followed by exactly the tokens the kernel reported."""
    prompt = synth.prompt(w)
    P, N = w.prompt_len, w.decode_len
    max_seq = P + N + 16
    dec = make_decoder(m, bits, max_seq)
    t0 = dec.kie_prefill(prompt)
    toks, z = _gpu_logits(dec, N, m.vocab, None)
    assert 0 <= t0 < m.vocab and ((toks >= 0) & (toks < m.vocab)).all()
    assert np.isfinite(z).all()
    assert (toks == np.argmax(z, axis=1)).all()
    seq = np.concatenate([prompt, [t0], toks[:-1]])
    _check_layer0_kv_and_bounds(dec, m, bits, seq, max_seq)
    dec.kie_destroy()


def test_long_context_full_model(dense_2b):
    """The full long-context workload, as it is benchmarked: the 8192-token
    prompt, then all 256 steps teacher-forced in one launch; every step's
    logits and argmax against the oracle (float64, prompt in 512-row chunks),
    and every layer's cache checked position by position."""
    w = synth.WORKLOADS[3]
    m = w.model
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, w.decode_len)
    dec, orc, _, rel, mab, near = _teacher_forced(m, dense_2b, prompt, forced, "long-full",
                                                  cache_f64=True)
    print(f"long-full: rel-L2 {rel:.3g} max-abs {mab:.3g} near ties {near}/{w.decode_len}")
    P, N = len(prompt), len(forced)
    _check_kv(dec, orc, m, P + N, P + N + 4)
    dec.kie_destroy()


def test_long_context_full_model_properties(dense_2b):
    """The full long-context workload: 8192-token prefill then 256 greedy steps
    in one launch, checked through the properties that hold at any size."""
    w = synth.WORKLOADS[3]
    _greedy_full_model(w.model, dense_2b, w)


def test_8b_class_full_model_properties():
    """The full 8B-class workload as it is benchmarked (bf16, 32 layers,
    V 128256; 1024-token prefill then 256 greedy steps in one launch), checked
    through the same properties; its logits are compared with the oracle's on
    the first two layers by the test above."""
    w = synth.WORKLOADS[4]
    bits = synth.generate_weights(w.model, w.weight_seed)
    _greedy_full_model(w.model, bits, w)


def test_8b_class_two_layers():
    """The 8B-class workload's shapes (bf16, d 4096, 32x128 / 8 KV heads,
    F 14336, V 128256; prompt 1024 -> 256 steps) on its first two layers."""
    w = synth.WORKLOADS[4]
    m = w.model.replace(n_layers=2)
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, w.decode_len)
    _, _, _, rel, mab, near = _teacher_forced(m, bits, prompt, forced, "8b-2L", cache_f64=True)
    print(f"8b-2L: rel-L2 {rel:.3g} max-abs {mab:.3g} near ties {near}")


def test_8b_class_full_model():
    """The full 8B-class workload (bf16, 32 layers, V 128256): the 1024-token
    prompt, then 16 teacher-forced steps; every step's logits and argmax
    against the oracle (weights kept in their 16-bit words, widened per use),
    and every layer's cache."""
    w = synth.WORKLOADS[4]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, 16)
    # bf16 KV cache at full depth: checked against the oracle's own noise floor
    # (REL_L2_BF16_FULL_DEPTH); max-abs, tokens and cache as everywhere
    dec, orc, _, rel, mab, near = _teacher_forced(m, bits, prompt, forced, "8b-full",
                                                  cache_f64=False, rel_l2=REL_L2_BF16_FULL_DEPTH)
    print(f"8b-full: rel-L2 {rel:.3g} max-abs {mab:.3g} near ties {near}/16")
    P, N = len(prompt), len(forced)
    check_kv(dec, orc, m, P + N, P + N + 4, rel=REL_L2_BF16_FULL_DEPTH)
    dec.kie_destroy()


# ------------------------------------------------------------ host-side errors
def test_errors_and_capacity():
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    dec = make_decoder(m, bits, 20)
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(1)                          # nothing prefilled yet
    assert e.value.code == kie.KIE_ERR_INVALID
    with pytest.raises(kie.KieError) as e:
        dec.kie_prefill(np.array([1, 2, m.vocab], dtype=np.int32))
    assert e.value.code == kie.KIE_ERR_INVALID
    with pytest.raises(kie.KieError) as e:
        dec.kie_prefill(np.zeros(21, dtype=np.int32))
    assert e.value.code == kie.KIE_ERR_CAPACITY
    with pytest.raises(kie.KieError) as e:
        dec.kie_prefill(np.zeros(0, dtype=np.int32))   # empty prompt
    assert e.value.code == kie.KIE_ERR_INVALID
    dec.kie_prefill(np.arange(15, dtype=np.int32))
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(0)                          # no steps
    assert e.value.code == kie.KIE_ERR_INVALID
    dec.kie_decode(5)                              # fills the cache to max_seq exactly
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(1)
    assert e.value.code == kie.KIE_ERR_CAPACITY
    # the context is still usable after host-side rejections
    assert dec.kie_prefill(np.arange(3, dtype=np.int32)) >= 0
    dec.kie_destroy()


def test_nonfinite_logits_stop_the_kernel():
    """A NaN in one LM-head row makes that logit NaN: the kernel reports
    KIE_ERR_NONFINITE (it never turns a NaN argmax into a token id) and the
    context is poisoned afterwards."""
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed).copy()
    head = [t for t in synth.tensor_table(m) if t.name == "lm_head"][0]
    row = m.vocab // 3
    bits[head.offset + row * m.d_model] = 0x7E00           # fp16 quiet NaN
    dec = make_decoder(m, bits, 16)
    with pytest.raises(kie.KieError) as e:
        dec.kie_prefill(np.arange(4, dtype=np.int32))
    assert e.value.code == kie.KIE_ERR_NONFINITE
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(1)
    assert e.value.code == kie.KIE_ERR_POISONED
    dec.kie_destroy()


def test_watchdog_reports_a_missing_signal():
    """Failure detection without a fault: one SM skips its q/k/v signal in the
    first step of a launch, so its KV group's waits run out after the short
    watchdog; the kernel returns KIE_ERR_DEVICE_TIMEOUT (every SM leaves its
    bounded waits, producers drain their copies), the context is poisoned, and
    the device stays usable for a new context."""
    import decode_persistent_monokernel_b200 as kie
    w = synth.WORKLOADS[0]
    m = w.model
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    dec = make_decoder(m, bits, 64)
    dec.kie_prefill(prompt)
    dec.kie_debug_set(200, 5)        # 200 ms limit; SM 5 never signals its group
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(4)
    assert e.value.code == kie.KIE_ERR_DEVICE_TIMEOUT
    with pytest.raises(kie.KieError) as e:
        dec.kie_decode(1)
    assert e.value.code == kie.KIE_ERR_POISONED
    with pytest.raises(kie.KieError) as e:
        dec.kie_prefill(prompt)
    assert e.value.code == kie.KIE_ERR_POISONED
    # the read-back calls still work, so the failed launch can be inspected
    assert dec.kie_get_stats().pos == len(prompt)
    k, _ = dec.kie_copy_kv(0, 0, 0, len(prompt))
    assert np.isfinite(storage_to_f64(k, m.dtype)).all()
    dec.kie_destroy()
    dec = make_decoder(m, bits, 64)
    t0 = dec.kie_prefill(prompt)
    toks = dec.kie_decode(4)
    assert 0 <= t0 < m.vocab and all(0 <= t < m.vocab for t in toks)
    dec.kie_destroy()
