"""Shapes and seeds of the five decode workloads, and the canonical weight layout.

Nothing here computes any part of the decoder.  The workloads follow the
pages' subject: a batch-1, single-request decode of a pre-norm decoder
(Kog Inference Engine write-ups: "Laneformer 2B: results shown" table, FP16,
batch 1; the lane-structured transformer bullet, 8 lanes; the Delayed Tensor
Parallelism bullet, delta = 2 layers).

Canonical weight layout (storage dtype, row-major ``[out, in]``, tensors
concatenated in this order with no padding):

* ``embed[V, d]``
* per layer, per lane (one lane for the dense models):
  ``attn_norm[dl]``, ``wq[Hql*dh, dl]``, ``wk[Hkvl*dh, dl]``, ``wv[Hkvl*dh, dl]``,
  ``wo[dl, Hql*dh]``, ``ffn_norm[dl]``, ``w_gate[Fl, dl]``, ``w_up[Fl, dl]``,
  ``w_down[dl, Fl]``; then, for lane models, ``mix[d, d]``
* ``final_norm[d]``, ``lm_head[V, d]``

where ``dl = d / n_lanes``, ``Hql = Hq / n_lanes``, ``Hkvl = Hkv / n_lanes``,
``Fl = F / n_lanes``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0
    dtype: str = "f16"  # "f16" or "bf16": weights and KV cache
    n_lanes: int = 1
    lane_delay: int = 0
    # init: std of every matrix; output projections (wo, w_down) divided by
    # sqrt(2 * n_layers) when out_scale; lane mixing matrix std
    init_std: float = 0.02
    out_scale: bool = False
    mix_std: float = 0.0
    # norm gains: constant 1 unless gain_std > 0 (then 1 + N(0, gain_std))
    gain_std: float = 0.0

    @property
    def lane_width(self) -> int:
        return self.d_model // self.n_lanes

    @property
    def lane_heads(self) -> int:
        return self.n_heads // self.n_lanes

    @property
    def lane_kv_heads(self) -> int:
        return self.n_kv_heads // self.n_lanes

    @property
    def lane_ffn(self) -> int:
        return self.ffn_dim // self.n_lanes

    @property
    def dtype_code(self) -> int:
        return 0 if self.dtype == "f16" else 1

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    model: ModelShape
    prompt_len: int
    decode_len: int
    weight_seed: int
    prompt_seed: int


_DENSE_2B = ModelShape(n_layers=34, d_model=2048, n_heads=16, n_kv_heads=8, head_dim=128,
                       ffn_dim=8192, vocab=32768, rope_theta=10000.0, dtype="f16",
                       out_scale=True)

WORKLOADS = {
    0: Workload(0, "tiny decoder, 2L d256 4x64 MHA F704 V4096 fp16, prompt 16 -> decode 32",
                ModelShape(n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
                           ffn_dim=704, vocab=4096, rope_theta=10000.0, dtype="f16"),
                16, 32, 1234 + 0, 42 + 0),
    1: Workload(1, "2.3B-class dense decoder, 34L d2048 16x128/8kv F8192 V32768 fp16, "
                   "prompt 128 -> decode 512",
                _DENSE_2B, 128, 512, 1234 + 1, 42 + 1),
    2: Workload(2, "lane-structured variant, 34L 8 lanes x 256, lane F1024, per-layer mix "
                   "2048x2048 delayed 2 layers, V32768 fp16, prompt 128 -> decode 512",
                ModelShape(n_layers=34, d_model=2048, n_heads=16, n_kv_heads=16,
                           head_dim=128, ffn_dim=8192, vocab=32768, rope_theta=10000.0,
                           dtype="f16", n_lanes=8, lane_delay=2, out_scale=True,
                           mix_std=0.02 / math.sqrt(8.0)),
                128, 512, 1234 + 2, 42 + 2),
    # the long-context workload decodes with the 2.3B-class model's own weights
    3: Workload(3, "long context on the 2.3B-class model, prompt 8192 -> decode 256",
                _DENSE_2B, 8192, 256, 1234 + 1, 42 + 3),
    4: Workload(4, "8B-class dense decoder, 32L d4096 32x128/8kv F14336 V128256 bf16, "
                   "prompt 1024 -> decode 256",
                ModelShape(n_layers=32, d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                           ffn_dim=14336, vocab=128256, rope_theta=500000.0, dtype="bf16"),
                1024, 256, 1234 + 4, 42 + 4),
}


@dataclasses.dataclass(frozen=True)
class TensorSpec:
    index: int        # tensor index keyed into the generator
    name: str
    shape: tuple
    offset: int       # in elements, into the canonical buffer
    mean: float
    std: float

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n


def tensor_table(m: ModelShape) -> List[TensorSpec]:
    """Canonical order of every weight tensor, with its init distribution."""
    specs: List[TensorSpec] = []
    off = 0

    def add(name, shape, mean, std):
        nonlocal off
        t = TensorSpec(len(specs), name, tuple(shape), off, mean, std)
        specs.append(t)
        off += t.numel

    d, dh, V = m.d_model, m.head_dim, m.vocab
    dl, hq, hkv, fl = m.lane_width, m.lane_heads, m.lane_kv_heads, m.lane_ffn
    std = m.init_std
    ostd = std / math.sqrt(2.0 * m.n_layers) if m.out_scale else std
    gain = (1.0, m.gain_std)
    add("embed", (V, d), 0.0, std)
    for l in range(m.n_layers):
        for ln in range(m.n_lanes):
            p = f"layers.{l}." if m.n_lanes == 1 else f"layers.{l}.lane{ln}."
            add(p + "attn_norm", (dl,), *gain)
            add(p + "wq", (hq * dh, dl), 0.0, std)
            add(p + "wk", (hkv * dh, dl), 0.0, std)
            add(p + "wv", (hkv * dh, dl), 0.0, std)
            add(p + "wo", (dl, hq * dh), 0.0, ostd)
            add(p + "ffn_norm", (dl,), *gain)
            add(p + "w_gate", (fl, dl), 0.0, std)
            add(p + "w_up", (fl, dl), 0.0, std)
            add(p + "w_down", (dl, fl), 0.0, ostd)
        if m.n_lanes > 1:
            add(f"layers.{l}.mix", (d, d), 0.0, m.mix_std)
    add("final_norm", (d,), *gain)
    add("lm_head", (V, d), 0.0, std)
    return specs


def total_elements(m: ModelShape) -> int:
    t = tensor_table(m)
    return t[-1].offset + t[-1].numel


def streamed_weight_bytes(m: ModelShape) -> int:
    """Bytes of weights one decode step must read: every matrix once, the norm
    gains, one embedding row (all of it except the V-1 unused embedding rows)."""
    esz = 2
    total = 0
    for t in tensor_table(m):
        if t.name == "embed":
            total += m.d_model * esz
        else:
            total += t.numel * esz
    return total


def kv_bytes_read(m: ModelShape, context_len: int) -> int:
    """K and V bytes one decode step reads at context length L (incl. the new one)."""
    return 2 * m.n_layers * m.n_kv_heads * context_len * m.head_dim * 2
