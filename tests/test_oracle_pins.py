"""Pins of the float64 oracle against things other than itself.

* library routines: torch SDPA (causal, grouped-query), torch.nn.functional.silu,
  the ``transformers`` Llama decoder run in float64 (pre-norm RMSNorm,
  rotate-half RoPE, grouped-query attention, SwiGLU, untied head);
* closed forms and invariants: RMSNorm's rms, RoPE at position 0, RoPE's
  relative-position property, attention over one position;
* a pure-Python no-cache brute force (tests/bruteforce.py) on tiny shapes,
  dense and lane-structured with the delayed cross-lane sum;
* the lane-decomposition invariant with the mixing matrices zeroed.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import Oracle, argmax_lowest, rmsnorm, rope, silu, top2_margin
from oracle.decoder import attention
from oracle.numerics import round_to_storage, storage_to_f64
from synth.configs import ModelShape
from tests import bruteforce


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 0.02, (5, 256))
    g = np.ones(256)
    for eps in (1e-5, 0.0):
        y = rmsnorm(x, g, eps)
        ms = np.mean(x * x, axis=1)
        rms_y = np.sqrt(np.mean(y * y, axis=1))
        np.testing.assert_allclose(rms_y, np.sqrt(ms / (ms + eps)), rtol=1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(rmsnorm(x, g, 0.0) ** 2, axis=1)), 1.0, rtol=1e-12)


def test_rmsnorm_gain_is_per_element():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, (3, 64))
    g = rng.normal(1, 0.3, 64)
    np.testing.assert_allclose(rmsnorm(x, g, 1e-5), rmsnorm(x, np.ones(64), 1e-5) * g, rtol=1e-14)


# ---------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 1, (1, 3, 128))
    np.testing.assert_array_equal(rope(x, np.array([0]), 1e4), x)


def test_rope_rotates_dimension_pairs_half_apart():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (4, 2, 64))
    y = rope(x, np.array([1, 7, 100, 8000]), 1e4)
    half = 32
    n_in = x[..., :half] ** 2 + x[..., half:] ** 2
    n_out = y[..., :half] ** 2 + y[..., half:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def test_rope_relative_position():
    rng = np.random.default_rng(4)
    q = rng.normal(0, 1, (1, 1, 128))
    k = rng.normal(0, 1, (1, 1, 128))
    for theta in (1e4, 5e5):
        base = float(np.sum(rope(q, np.array([37]), theta) * rope(k, np.array([5]), theta)))
        for shift in (1, 250, 8000):
            s = float(np.sum(rope(q, np.array([37 + shift]), theta) *
                             rope(k, np.array([5 + shift]), theta)))
            assert abs(s - base) < 1e-9 * max(1.0, abs(base))


def test_rope_matches_transformers():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    dh, theta = 64, 1e4
    rng = np.random.default_rng(5)
    q = rng.normal(0, 1, (6, 2, dh))
    pos = np.array([0, 1, 2, 17, 33, 47])
    inv = 1.0 / (theta ** (np.arange(0, dh, 2) / dh))
    freqs = pos[:, None] * inv[None, :]
    emb = np.concatenate([freqs, freqs], axis=-1)
    cos = torch.from_numpy(np.cos(emb))[None]
    sin = torch.from_numpy(np.sin(emb))[None]
    qt = torch.from_numpy(q.transpose(1, 0, 2).copy())[None]   # [1, H, T, dh]
    ref, _ = apply_rotary_pos_emb(qt, qt, cos, sin)
    ours = rope(q, pos, theta).transpose(1, 0, 2)[None]
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- attention
def test_attention_single_position_returns_v_exactly():
    rng = np.random.default_rng(6)
    q = rng.normal(0, 3, (1, 4, 128))
    K = rng.normal(0, 1, (2, 1, 128))
    V = rng.normal(0, 1, (2, 1, 128))
    o = attention(q, K, V, np.array([0]))
    for h in range(4):
        np.testing.assert_array_equal(o[0, h], V[h // 2, 0])


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (32, 8)])
def test_attention_matches_sdpa(hq, hkv):
    rng = np.random.default_rng(7)
    T, S, dh = 5, 12, 64
    q = rng.normal(0, 1, (T, hq, dh))
    K = rng.normal(0, 1, (hkv, S, dh))
    V = rng.normal(0, 1, (hkv, S, dh))
    qpos = np.arange(S - T, S)
    ours = attention(q, K, V, qpos)
    qt = torch.from_numpy(q.transpose(1, 0, 2).copy())[None]
    Kt = torch.from_numpy(K.copy())[None]
    Vt = torch.from_numpy(V.copy())[None]
    mask = torch.from_numpy(np.arange(S)[None, :] <= qpos[:, None])
    ref = F.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask, enable_gqa=True)
    np.testing.assert_allclose(ours, ref[0].numpy().transpose(1, 0, 2), rtol=1e-11, atol=1e-12)


def test_silu_matches_torch():
    z = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(silu(z), F.silu(torch.from_numpy(z)).numpy(), rtol=1e-14, atol=1e-300)


def test_argmax_lowest_index_on_ties():
    z = np.array([0.1, 0.7, -1.0, 0.7, 0.7])
    assert argmax_lowest(z) == 1
    assert top2_margin(z) == 0.0
    assert top2_margin(np.array([1.0, 3.0, 2.5])) == pytest.approx(0.5)


# ---------------------------------------------------------------- whole decoder
def _hf_model(m: ModelShape, bits: np.ndarray):
    from transformers import LlamaConfig, LlamaForCausalLM
    cfg = LlamaConfig(vocab_size=m.vocab, hidden_size=m.d_model, intermediate_size=m.ffn_dim,
                      num_hidden_layers=m.n_layers, num_attention_heads=m.n_heads,
                      num_key_value_heads=m.n_kv_heads, head_dim=m.head_dim,
                      rms_norm_eps=m.rms_eps, rope_theta=m.rope_theta,
                      tie_word_embeddings=False, attention_bias=False, mlp_bias=False,
                      max_position_embeddings=4096, attn_implementation="eager")
    model = LlamaForCausalLM(cfg).double().eval()
    spec = {t.name: t for t in synth.tensor_table(m)}

    def get(name):
        t = spec[name]
        return torch.from_numpy(storage_to_f64(bits[t.offset:t.offset + t.numel], m.dtype)
                                .reshape(t.shape))
    sd = {"model.embed_tokens.weight": get("embed"), "model.norm.weight": get("final_norm"),
          "lm_head.weight": get("lm_head")}
    for l in range(m.n_layers):
        p = f"model.layers.{l}."
        sd[p + "self_attn.q_proj.weight"] = get(f"layers.{l}.wq")
        sd[p + "self_attn.k_proj.weight"] = get(f"layers.{l}.wk")
        sd[p + "self_attn.v_proj.weight"] = get(f"layers.{l}.wv")
        sd[p + "self_attn.o_proj.weight"] = get(f"layers.{l}.wo")
        sd[p + "mlp.gate_proj.weight"] = get(f"layers.{l}.w_gate")
        sd[p + "mlp.up_proj.weight"] = get(f"layers.{l}.w_up")
        sd[p + "mlp.down_proj.weight"] = get(f"layers.{l}.w_down")
        sd[p + "input_layernorm.weight"] = get(f"layers.{l}.attn_norm")
        sd[p + "post_attention_layernorm.weight"] = get(f"layers.{l}.ffn_norm")
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected and all("rotary" in k for k in missing), (missing, unexpected)
    return model


@pytest.mark.parametrize("variant", ["mha", "gqa_gains"])
def test_decoder_matches_transformers_llama(tiny_weights, variant):
    w, bits = tiny_weights
    m = w.model
    if variant == "gqa_gains":
        m = m.replace(n_kv_heads=2, gain_std=0.1, n_layers=3)
        bits = synth.generate_weights(m, 77)
    prompt = synth.prompt(w)
    forced = synth.forced_tokens(w, 24)
    orc = Oracle(m, bits, max_seq=64, kv_round=False)
    z_or = orc.teacher_forced_logits(prompt, forced)
    seq = torch.from_numpy(np.concatenate([prompt, forced]).astype(np.int64))[None]
    with torch.no_grad():
        z_hf = _hf_model(m, bits)(seq).logits[0].numpy()[len(prompt):]
    # transformers evaluates the RoPE angles in float32; allow for that only
    rel = np.linalg.norm(z_or - z_hf) / np.linalg.norm(z_hf)
    assert rel < 2e-6, rel
    assert orc.pos == len(prompt) + len(forced)


def _micro(lanes=1, layers=2, delay=0, kv=2, dtype="f16"):
    if lanes == 1:
        return ModelShape(n_layers=layers, d_model=16, n_heads=4, n_kv_heads=kv, head_dim=4,
                          ffn_dim=24, vocab=40, rms_eps=1e-5, rope_theta=100.0, dtype=dtype,
                          gain_std=0.2, init_std=0.3)
    return ModelShape(n_layers=layers, d_model=16, n_heads=4, n_kv_heads=4, head_dim=4,
                      ffn_dim=24, vocab=40, rms_eps=1e-5, rope_theta=100.0, dtype=dtype,
                      n_lanes=lanes, lane_delay=delay, gain_std=0.2, init_std=0.3, mix_std=0.3)


@pytest.mark.parametrize("shape", [
    _micro(),
    _micro(kv=1, dtype="bf16"),
    _micro(lanes=2, layers=3, delay=2),
    _micro(lanes=2, layers=4, delay=3),
])
def test_decoder_matches_bruteforce(shape):
    bits = synth.generate_weights(shape, 99)
    prompt = synth.generate_tokens(5, shape.vocab, 3)
    orc = Oracle(shape, bits, max_seq=16)
    t0, z0 = orc.prefill(list(prompt), chunk=2)
    toks, zs = orc.decode(6)
    seq = list(prompt) + [t0] + list(toks[:-1])
    bf = bruteforce.Tiny(shape, bits)
    z_bf, _ = bruteforce.logits_at_every_position(bf, seq)
    np.testing.assert_allclose(z0, z_bf[len(prompt) - 1], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(zs, z_bf[len(prompt):], rtol=1e-10, atol=1e-12)
    assert t0 == argmax_lowest(z_bf[len(prompt) - 1])


def test_kv_cache_holds_rounded_keys(tiny_weights):
    w, bits = tiny_weights
    m = w.model
    prompt = synth.prompt(w)
    a = Oracle(m, bits, 32, kv_round=True)
    b = Oracle(m, bits, 32, kv_round=False)
    a.prefill(prompt)
    b.prefill(prompt)
    P = len(prompt)
    # layer 0's keys depend only on the token: rounding the exact keys gives the cache
    np.testing.assert_array_equal(a.K[0, :, :P], round_to_storage(b.K[0, :, :P], m.dtype))
    np.testing.assert_array_equal(a.V[0, :, :P], round_to_storage(b.V[0, :, :P], m.dtype))
    assert np.isnan(a.K[:, :, P:]).all() and np.isnan(a.V[:, :, P:]).all()
    assert np.isfinite(a.K[:, :, :P]).all()


def test_prefill_chunking_and_teacher_forcing_agree(tiny_weights):
    w, bits = tiny_weights
    m = w.model
    prompt = synth.prompt(w)
    o1 = Oracle(m, bits, 64)
    t_a, z_a = o1.prefill(prompt, chunk=512)
    toks, zs = o1.decode(8)
    o2 = Oracle(m, bits, 64)
    t_b, z_b = o2.prefill(prompt, chunk=3)
    assert t_a == t_b
    np.testing.assert_allclose(z_a, z_b, rtol=1e-12, atol=1e-13)
    forced = [t_a] + list(toks[:-1])
    z_tf = Oracle(m, bits, 64).teacher_forced_logits(prompt, forced, chunk=7)
    np.testing.assert_allclose(z_tf, zs, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- lane variant
def _lane_shape(layers=3):
    return ModelShape(n_layers=layers, d_model=64, n_heads=8, n_kv_heads=8, head_dim=8,
                      ffn_dim=128, vocab=50, rope_theta=1e4, dtype="f16", n_lanes=4,
                      lane_delay=2, out_scale=True, mix_std=0.05, gain_std=0.1)


def _zero_mix(m, bits):
    bits = bits.copy()
    for t in synth.tensor_table(m):
        if t.name.endswith(".mix"):
            bits[t.offset:t.offset + t.numel] = 0
    return bits


def test_zero_mix_decomposes_into_independent_lanes():
    m = _lane_shape()
    bits = _zero_mix(m, synth.generate_weights(m, 5))
    toks = list(synth.generate_tokens(6, m.vocab, 8))
    hidden = _hidden(Oracle(m, bits, 16), toks)
    spec = {t.name: t for t in synth.tensor_table(m)}
    dl = m.lane_width
    for lane in range(m.n_lanes):
        one = m.replace(d_model=dl, n_heads=m.lane_heads, n_kv_heads=m.lane_kv_heads,
                        ffn_dim=m.lane_ffn, n_lanes=1, lane_delay=0)
        parts = []
        # embedding restricted to this lane's columns, then the lane's layers
        E = bits[spec["embed"].offset:spec["embed"].offset + spec["embed"].numel].reshape(m.vocab, -1)
        parts.append(np.ascontiguousarray(E[:, lane * dl:(lane + 1) * dl]).ravel())
        for l in range(m.n_layers):
            for name in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up",
                         "w_down"):
                t = spec[f"layers.{l}.lane{lane}.{name}"]
                parts.append(bits[t.offset:t.offset + t.numel])
        parts.append(np.ones(dl, dtype=np.uint16))            # unused final norm / head
        parts.append(np.zeros(m.vocab * dl, dtype=np.uint16))
        sub = np.concatenate(parts)
        assert sub.size == synth.total_elements(one)
        h1 = _hidden(Oracle(one, sub, 16), toks)
        np.testing.assert_array_equal(hidden[:, lane * dl:(lane + 1) * dl], h1)


def _hidden(orc, toks):
    """Residual stream before the final norm."""
    orc.reset()
    return orc.forward(toks, logits="hidden")


def test_delayed_sum_lands_delta_layers_later():
    """With a single nonzero mixing entry M_0[a, b], layer 0's lane output u_0[b]
    reaches x[a] exactly at the start of layer 2 (delta = 2): layers 0 and 1 are
    unchanged, and with only 2 layers the sum lands in the final flush."""
    m = _lane_shape(layers=2)
    bits = _zero_mix(m, synth.generate_weights(m, 6))
    toks = list(synth.generate_tokens(3, m.vocab, 9))
    base = Oracle(m, bits, 8)
    h0 = _hidden(base, toks)
    x = base.embed_rows(toks)
    u0 = Oracle(m, bits, 8)._layer(0, x.copy(), 0)
    spec = {t.name: t for t in synth.tensor_table(m)}
    a, b = 5, 40
    val_bits = np.array([0.5], dtype=np.float16).view(np.uint16)[0]
    bits2 = bits.copy()
    bits2[spec["layers.0.mix"].offset + a * m.d_model + b] = val_bits
    h1 = _hidden(Oracle(m, bits2, 8), toks)
    diff = h1 - h0
    expect = np.zeros_like(diff)
    expect[:, a] = 0.5 * u0[:, b]
    np.testing.assert_allclose(diff, expect, rtol=1e-12, atol=1e-15)
