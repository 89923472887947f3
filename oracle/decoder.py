"""Float64 statement of the decoder step that the persistent kernel runs.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Every step is the textbook definition, written in the order the step runs
(Kog Inference Engine write-ups, monokernel bullet: the whole decode path,
layer after layer, then "LM-head sampling"):

    x  = E[token]
    per layer l (lane models: first  x += M_{l-delta} u_{l-delta}  if l >= delta):
      per lane (one lane for dense models), on that lane's slice of x:
        y  = rmsnorm(x, g_attn)
        q, k, v = Wq y, Wk y, Wv y             ; rope(q), rope(k) at position p
        K[p], V[p] = round(k), round(v)          ; 16-bit KV cache
        o_h = sum_j softmax_j(q_h . K_g[j] / sqrt(dh)) V_g[j],  j = 0..p,
              g = floor(h * Hkv / Hq)            ; grouped-query attention
        a  = Wo o ;  x += a
        y  = rmsnorm(x, g_ffn) ;  h = silu(Wg y) * (Wu y) ;  m = Wd h ;  x += m
        u  = a + m                               ; lane output (lane models)
    lane models: flush every delayed sum that has not landed yet
    z  = W_lm rmsnorm(x, g_final) ;  token = argmax z (lowest index on ties)

Weights stay in their 16-bit storage words and are widened to float64 (an
exact conversion) when used; all arithmetic is float64.  A sequence of T
tokens runs as one chunk of T rows (prompt processing) or as T one-row steps
(decoding): causal attention makes the two identical by definition.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from synth.configs import ModelShape, tensor_table

from .numerics import round_to_storage, storage_to_f64


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y_i = x_i / sqrt(mean_j x_j^2 + eps) * g_i over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding of x[..., T, H, dh] at integer positions[T].

    Dimension i < dh/2 pairs with i + dh/2 and turns by the angle
    p * theta^(-2i/dh), computed in float64.
    """
    dh = x.shape[-1]
    half = dh // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / dh)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]   # [T, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, qpos: np.ndarray) -> np.ndarray:
    """Causal grouped-query attention.

    q: [T, Hq, dh] queries at positions qpos[T]; K, V: [Hkv, S, dh] cached keys
    and values for positions 0..S-1.  Query head h reads KV head
    floor(h * Hkv / Hq); query t sees keys j <= qpos[t].  Returns [T, Hq, dh].
    """
    T, Hq, dh = q.shape
    Hkv, S, _ = K.shape
    out = np.empty_like(q)
    allowed = np.arange(S)[None, :] <= np.asarray(qpos)[:, None]      # [T, S]
    scale = 1.0 / math.sqrt(dh)
    for h in range(Hq):
        g = (h * Hkv) // Hq
        s = (q[:, h, :] @ K[g].T) * scale                               # [T, S]
        s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        w = np.exp(s)
        w = w / w.sum(axis=1, keepdims=True)
        out[:, h, :] = w @ V[g]
    return out


def argmax_lowest(z: np.ndarray) -> int:
    """Greedy token: index of the largest logit, the lowest index on ties."""
    return int(np.argmax(z))   # numpy returns the first occurrence of the maximum


def top2_margin(z: np.ndarray) -> float:
    """Largest logit minus the second largest (0 on an exact tie)."""
    part = np.partition(np.asarray(z, dtype=np.float64), -2)[-2:]
    return float(part[1] - part[0])


class Oracle:
    """Stateful single-request decoder: a KV cache plus the current position.

    ``kv_round`` stores K (after RoPE) and V rounded to the storage type and
    uses the rounded values for the current token too (the 16-bit KV cache of
    the workloads).  ``cache_f64`` keeps float64 copies of the weights between
    calls instead of widening them on every use.
    """

    def __init__(self, m: ModelShape, weights: np.ndarray, max_seq: int,
                 kv_round: bool = True, cache_f64: bool = False):
        if weights.dtype != np.uint16:
            raise TypeError("weights must be raw uint16 storage words")
        self.m = m
        self.bits = weights
        self.max_seq = max_seq
        self.kv_round = kv_round
        self.cache_f64 = cache_f64
        self._f64: Dict[str, np.ndarray] = {}
        self.spec = {t.name: t for t in tensor_table(m)}
        L, Hkv, dh = m.n_layers, m.n_kv_heads, m.head_dim
        self.K = np.full((L, Hkv, max_seq, dh), np.nan)
        self.V = np.full((L, Hkv, max_seq, dh), np.nan)
        self.pos = 0
        self.pending: Optional[int] = None

    # -- weights -------------------------------------------------------------
    def w(self, name: str) -> np.ndarray:
        if name in self._f64:
            return self._f64[name]
        t = self.spec[name]
        a = storage_to_f64(self.bits[t.offset:t.offset + t.numel], self.m.dtype).reshape(t.shape)
        if self.cache_f64:
            self._f64[name] = a
        return a

    def _lw(self, l: int, lane: int, what: str) -> np.ndarray:
        if self.m.n_lanes == 1:
            return self.w(f"layers.{l}.{what}")
        return self.w(f"layers.{l}.lane{lane}.{what}")

    def embed_rows(self, tokens: Sequence[int]) -> np.ndarray:
        t = self.spec["embed"]
        d = self.m.d_model
        rows = [storage_to_f64(self.bits[t.offset + int(tok) * d: t.offset + (int(tok) + 1) * d],
                               self.m.dtype) for tok in tokens]
        return np.stack(rows)

    # -- one layer -----------------------------------------------------------
    def _layer(self, l: int, x: np.ndarray, pos0: int) -> np.ndarray:
        """Run layer l on rows x[T, d] (positions pos0..pos0+T-1) in place.

        Returns the lane outputs u[T, d] (attention plus MLP sublayer outputs).
        """
        m = self.m
        T = x.shape[0]
        dl, hq, hkv, dh = m.lane_width, m.lane_heads, m.lane_kv_heads, m.head_dim
        positions = np.arange(pos0, pos0 + T)
        u = np.zeros_like(x)
        for lane in range(m.n_lanes):
            sl = slice(lane * dl, (lane + 1) * dl)
            y = rmsnorm(x[:, sl], self._lw(l, lane, "attn_norm"), m.rms_eps)
            q = (y @ self._lw(l, lane, "wq").T).reshape(T, hq, dh)
            k = (y @ self._lw(l, lane, "wk").T).reshape(T, hkv, dh)
            v = (y @ self._lw(l, lane, "wv").T).reshape(T, hkv, dh)
            q = rope(q, positions, m.rope_theta)
            k = rope(k, positions, m.rope_theta)
            if self.kv_round:
                k = round_to_storage(k, m.dtype)
                v = round_to_storage(v, m.dtype)
            heads = slice(lane * hkv, (lane + 1) * hkv)
            self.K[l, heads, pos0:pos0 + T, :] = k.transpose(1, 0, 2)
            self.V[l, heads, pos0:pos0 + T, :] = v.transpose(1, 0, 2)
            S = pos0 + T
            o = attention(q, self.K[l, heads, :S, :], self.V[l, heads, :S, :], positions)
            a = o.reshape(T, hq * dh) @ self._lw(l, lane, "wo").T
            x[:, sl] += a
            y = rmsnorm(x[:, sl], self._lw(l, lane, "ffn_norm"), m.rms_eps)
            h = silu(y @ self._lw(l, lane, "w_gate").T) * (y @ self._lw(l, lane, "w_up").T)
            mo = h @ self._lw(l, lane, "w_down").T
            x[:, sl] += mo
            u[:, sl] = a + mo
        return u

    # -- a chunk of consecutive positions ------------------------------------
    def forward(self, tokens: Sequence[int], logits: str = "all") -> Optional[np.ndarray]:
        """Append ``tokens`` at positions pos..pos+T-1 and return their logits.

        ``logits``: "all" -> [T, V], "last" -> [V], "none" -> None,
        "hidden" -> the residual stream [T, d] before the final norm.
        """
        m = self.m
        T = len(tokens)
        if T == 0:
            raise ValueError("empty chunk")
        if self.pos + T > self.max_seq:
            raise ValueError("KV capacity exceeded")
        pos0 = self.pos
        x = self.embed_rows(tokens)
        delta = m.lane_delay
        pending: List[Tuple[int, np.ndarray]] = []        # (layer i, u_i) not yet landed
        for l in range(m.n_layers):
            if m.n_lanes > 1 and pending and pending[0][0] == l - delta:
                i, ui = pending.pop(0)
                x += ui @ self.w(f"layers.{i}.mix").T
            u = self._layer(l, x, pos0)
            if m.n_lanes > 1:
                pending.append((l, u))
        for i, ui in pending:                              # flush delayed sums
            x += ui @ self.w(f"layers.{i}.mix").T
        self.pos += T
        if logits == "none":
            return None
        if logits == "hidden":
            return x
        rows = x if logits == "all" else x[-1:]
        z = rmsnorm(rows, self.w("final_norm"), m.rms_eps) @ self.w("lm_head").T
        return z if logits == "all" else z[0]

    # -- request-level calls -------------------------------------------------
    def reset(self) -> None:
        self.K.fill(np.nan)
        self.V.fill(np.nan)
        self.pos = 0
        self.pending = None

    def prefill(self, tokens: Sequence[int], chunk: int = 512) -> Tuple[int, np.ndarray]:
        """Process a prompt from position 0; returns (next token, its logits)."""
        self.reset()
        tokens = list(tokens)
        z = None
        for s in range(0, len(tokens), chunk):
            part = tokens[s:s + chunk]
            last = s + chunk >= len(tokens)
            z = self.forward(part, logits="last" if last else "none")
        self.pending = argmax_lowest(z)
        return self.pending, z

    def decode(self, n: int, forced: Optional[Sequence[int]] = None
               ) -> Tuple[np.ndarray, np.ndarray]:
        """n decode steps.  Step k feeds forced[k] (or the pending greedy token)
        at the current position, then the pending token becomes argmax of its
        logits.  Returns (tokens[n], logits[n, V])."""
        if self.pending is None and forced is None:
            raise ValueError("prefill first")
        toks = np.empty(n, dtype=np.int32)
        zs = np.empty((n, self.m.vocab))
        for k in range(n):
            feed = int(forced[k]) if forced is not None else self.pending
            z = self.forward([feed], logits="last")
            self.pending = argmax_lowest(z)
            toks[k] = self.pending
            zs[k] = z
        return toks, zs

    def teacher_forced_logits(self, prompt: Sequence[int], forced: Sequence[int],
                              chunk: int = 512) -> np.ndarray:
        """Logits of every decode step when step k is fed forced[k]: the prompt
        and the forced tokens run as one causal sequence.  Returns [n, V] where
        row k belongs to the step that feeds forced[k]."""
        self.reset()
        seq = list(prompt) + list(forced)
        P, n = len(prompt), len(forced)
        out = np.empty((n, self.m.vocab))
        # logits of rows P..P+n-1 (the forced tokens' positions)
        s = 0
        while s < len(seq):
            part = seq[s:s + chunk]
            z = self.forward(part, logits="all" if s + len(part) > P else "none")
            if z is not None:
                for r in range(len(part)):
                    g = s + r
                    if g >= P:
                        out[g - P] = z[r]
            s += len(part)
        return out
