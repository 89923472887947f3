"""The tensor-core prompt pass (KIE_PREFILL_GEMM) against the float64 oracle,
through the C ABI.

Per case: the logits of the last prompt position (kie_prefill_ex) within the
logits tolerances (relative L2 <= 1e-3, max-abs <= 2e-2), the greedy next
token by the near-tie rule, every cached K/V position written exactly once
(values to rounding, NaN beyond), then teacher-forced decode steps from the
state the prompt pass left.  Prompt lengths span several 128-row GEMM tiles
with a ragged last tile; shapes include GQA 2:1 and 4:1, bf16 (three operand
parts), head dim 64 and 128, a hidden size that is not a multiple of the
GEMM's 64-column K step, and a vocabulary that is not a multiple of its
128-column N tile.
"""
import numpy as np
import pytest

import synth
from oracle import Oracle
from synth.configs import ModelShape
from tests.gpu_util import check_argmax, check_kv, check_logits, make_decoder

pytestmark = pytest.mark.gpu

_TINY = synth.WORKLOADS[0].model
_SHAPES = {
    "tiny": _TINY,
    "gqa2_gains": _TINY.replace(n_kv_heads=2, gain_std=0.1, n_layers=3),
    "gqa4": _TINY.replace(n_heads=4, n_kv_heads=1, n_layers=2),
    "bf16": _TINY.replace(dtype="bf16", rope_theta=500000.0),
    "dh128_f1376": ModelShape(n_layers=2, d_model=512, n_heads=4, n_kv_heads=2, head_dim=128,
                              ffn_dim=1376, vocab=5000, dtype="f16"),
}


@pytest.fixture(scope="module", autouse=True)
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import decode_persistent_monokernel_b200 as kie
    kie.load()
    return torch


def _prefill_and_decode(m, bits, prompt, forced, label):
    import torch
    import decode_persistent_monokernel_b200 as kie
    P, N = len(prompt), len(forced)
    max_seq = P + N + 4
    dec = make_decoder(m, bits, max_seq)
    # the default for fp16 models; bf16 models select it
    assert dec.kie_get_stats().prefill_mode == (kie.KIE_PREFILL_GEMM if m.dtype == "f16"
                                                else kie.KIE_PREFILL_STEPS)
    dec.kie_set_prefill_mode(kie.KIE_PREFILL_GEMM)
    z = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
    t0 = dec.kie_prefill_ex(prompt, logits_out=z)
    torch.cuda.synchronize()
    orc = Oracle(m, bits, max_seq)
    o0, z0 = orc.prefill(prompt)
    rel, mab = check_logits(z.cpu().numpy()[None], z0[None], f"{label} prompt logits")
    check_argmax([t0], z0, f"{label} prompt token")
    st = dec.kie_get_stats()
    assert st.pos == P and st.pending_token == t0 and st.last_prefill_ms > 0
    check_kv(dec, orc, m, P, max_seq)
    # decoding continues from the cache and position the prompt pass left
    zs = torch.empty((N, m.vocab), dtype=torch.float32, device="cuda")
    toks = dec.kie_decode_ex(N, forced=forced, logits_out=zs)
    torch.cuda.synchronize()
    _, z_ora = orc.decode(N, forced=forced)
    check_logits(zs.cpu().numpy(), z_ora, f"{label} decode after the prompt pass")
    check_argmax(toks, z_ora, f"{label} decode after the prompt pass")
    dec.kie_destroy()
    return rel, mab


@pytest.mark.parametrize("plen", [1, 150, 300])
@pytest.mark.parametrize("name", sorted(_SHAPES))
def test_gemm_prefill_matches_oracle(name, plen):
    m = _SHAPES[name]
    bits = synth.generate_weights(m, 23)
    prompt = synth.generate_tokens(plen, m.vocab, 11)
    forced = synth.generate_tokens(12, m.vocab, 12)
    _prefill_and_decode(m, bits, prompt, forced, f"{name} P{plen}")


def test_prefill_modes_agree():
    """The prompt pass and the persistent kernel's one-position-per-step prompt
    leave the same state: logits of the last position within a tenth of the
    oracle tolerance of each other, and the same cache to rounding."""
    import torch
    import decode_persistent_monokernel_b200 as kie
    from oracle.numerics import storage_to_f64
    m = _SHAPES["gqa2_gains"]
    bits = synth.generate_weights(m, 29)
    prompt = synth.generate_tokens(200, m.vocab, 13)
    out = []
    for mode in (kie.KIE_PREFILL_GEMM, kie.KIE_PREFILL_STEPS):
        dec = make_decoder(m, bits, 210)
        dec.kie_set_prefill_mode(mode)
        assert dec.kie_get_stats().prefill_mode == mode
        z = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
        t = dec.kie_prefill_ex(prompt, logits_out=z)
        torch.cuda.synchronize()
        kv = [storage_to_f64(c, m.dtype) for l in range(m.n_layers) for c in dec.kie_copy_kv(l, 1, 0, 200)]
        out.append((t, z.cpu().numpy().astype(np.float64), kv))
        dec.kie_destroy()
    (ta, za, kva), (tb, zb, kvb) = out
    assert np.linalg.norm(za - zb) / np.linalg.norm(zb) <= 1e-4
    for a, b in zip(kva, kvb):
        assert np.abs(a - b).max() <= 4e-3 * np.abs(b).max()


def test_prefill_mode_choice():
    """Lane models have no tensor-core prompt pass: they default to the
    per-step prompt and refuse KIE_PREFILL_GEMM; an unknown mode is refused."""
    import decode_persistent_monokernel_b200 as kie
    lanes = _TINY.replace(n_lanes=2, lane_delay=2, n_layers=4, mix_std=0.02)
    dec = make_decoder(lanes, synth.generate_weights(lanes, 3), 32)
    assert dec.kie_get_stats().prefill_mode == kie.KIE_PREFILL_STEPS
    with pytest.raises(kie.KieError) as e:
        dec.kie_set_prefill_mode(kie.KIE_PREFILL_GEMM)
    assert e.value.code == kie.KIE_ERR_INVALID
    with pytest.raises(kie.KieError) as e:
        dec.kie_set_prefill_mode(5)
    assert e.value.code == kie.KIE_ERR_INVALID
    assert dec.kie_prefill(np.arange(5, dtype=np.int32)) >= 0
    dec.kie_destroy()


@pytest.fixture(scope="module")
def dense_2b():
    w = synth.WORKLOADS[1]
    return synth.generate_weights(w.model, w.weight_seed)


def test_gemm_prefill_2b_class(dense_2b):
    """The 2.3B-class model in full: its 128-token prompt through the prompt
    pass, then 8 teacher-forced decode steps."""
    w = synth.WORKLOADS[1]
    rel, mab = _prefill_and_decode(w.model, dense_2b, synth.prompt(w), synth.forced_tokens(w, 8), "2b prompt")
    print(f"2b prompt pass: logits rel-L2 {rel:.3g} max-abs {mab:.3g}")


def test_gemm_prefill_long_context_two_layers(dense_2b):
    """The long-context workload's 8192-token prompt on the first two layers
    of the 2.3B-class model (64 GEMM row tiles, causal attention over 8192
    positions)."""
    from tests.test_gpu_parity import _first_layers
    w = synth.WORKLOADS[3]
    m, bits = _first_layers(w.model, dense_2b, 2)
    rel, mab = _prefill_and_decode(m, bits, synth.prompt(w), synth.forced_tokens(w, 8), "long-2L prompt")
    print(f"long-2L prompt pass: logits rel-L2 {rel:.3g} max-abs {mab:.3g}")


def test_gemm_prefill_8b_class_two_layers():
    """The 8B-class workload's shapes (bf16, d 4096, 32 x 128 / 8 KV heads,
    F 14336, V 128256) on two layers: its 1024-token prompt through the
    tensor-core pass (selected: bf16 models default to the per-position
    prompt), then 8 teacher-forced decode steps."""
    w = synth.WORKLOADS[4]
    m = w.model.replace(n_layers=2)
    bits = synth.generate_weights(m, w.weight_seed)
    rel, mab = _prefill_and_decode(m, bits, synth.prompt(w), synth.forced_tokens(w, 8), "8b-2L prompt")
    print(f"8b-2L prompt pass: logits rel-L2 {rel:.3g} max-abs {mab:.3g}")
