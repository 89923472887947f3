"""Pure-Python, no-cache brute force of the decoder, for tiny shapes only.

Written independently of the oracle: explicit per-element loops, ``math``
functions, and the input generator's own C rounding for the 16-bit KV cache.
Every step recomputes the whole sequence from position 0, so nothing is
cached between steps.
"""
import math

import numpy as np

import synth


def _widen(bits, dtype):
    if dtype == "f16":
        return [float(v) for v in np.asarray(bits, dtype=np.uint16).view(np.float16)]
    return [float(v) for v in (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16)
            .view(np.float32)]


def _round(v, dtype):
    return _widen([synth.round_to_storage(v, dtype)], dtype)[0]


class Tiny:
    def __init__(self, m, weights):
        self.m = m
        self.t = {}
        for s in synth.tensor_table(m):
            flat = _widen(weights[s.offset:s.offset + s.numel], m.dtype)
            if len(s.shape) == 1:
                self.t[s.name] = flat
            else:
                r, c = s.shape
                self.t[s.name] = [flat[i * c:(i + 1) * c] for i in range(r)]

    def lw(self, l, lane, name):
        if self.m.n_lanes == 1:
            return self.t[f"layers.{l}.{name}"]
        return self.t[f"layers.{l}.lane{lane}.{name}"]


def _matvec(W, x):
    out = []
    for row in W:
        s = 0.0
        for a, b in zip(row, x):
            s += a * b
        out.append(s)
    return out


def _norm(x, g, eps):
    ms = sum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [v * r * gi for v, gi in zip(x, g)]


def _rope(vec, p, theta):
    dh = len(vec)
    half = dh // 2
    out = list(vec)
    for i in range(half):
        ang = p * theta ** (-2.0 * i / dh)
        c, s = math.cos(ang), math.sin(ang)
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def logits_at_every_position(model: Tiny, tokens, kv_round=True):
    """Logits after each token of ``tokens``, recomputing everything."""
    m = model.m
    d, dh = m.d_model, m.head_dim
    dl, hq, hkv, fl = m.lane_width, m.lane_heads, m.lane_kv_heads, m.lane_ffn
    T = len(tokens)
    xs = [list(model.t["embed"][tok]) for tok in tokens]
    keys = {}
    vals = {}
    us = []
    for l in range(m.n_layers):
        if m.n_lanes > 1 and l >= m.lane_delay:
            M = model.t[f"layers.{l - m.lane_delay}.mix"]
            for t in range(T):
                add = _matvec(M, us[l - m.lane_delay][t])
                xs[t] = [a + b for a, b in zip(xs[t], add)]
        u_l = [[0.0] * d for _ in range(T)]
        for lane in range(m.n_lanes):
            lo = lane * dl
            # projections for every position
            qs, ks, vs = [], [], []
            for t in range(T):
                y = _norm(xs[t][lo:lo + dl], model.lw(l, lane, "attn_norm"), m.rms_eps)
                q = _matvec(model.lw(l, lane, "wq"), y)
                k = _matvec(model.lw(l, lane, "wk"), y)
                v = _matvec(model.lw(l, lane, "wv"), y)
                q = sum((_rope(q[h * dh:(h + 1) * dh], t, m.rope_theta) for h in range(hq)), [])
                k = sum((_rope(k[h * dh:(h + 1) * dh], t, m.rope_theta) for h in range(hkv)), [])
                if kv_round:
                    k = [_round(a, m.dtype) for a in k]
                    v = [_round(a, m.dtype) for a in v]
                qs.append(q)
                ks.append(k)
                vs.append(v)
            for t in range(T):
                o = []
                for h in range(hq):
                    g = h * hkv // hq
                    sc = []
                    for j in range(t + 1):
                        dot = 0.0
                        for i in range(dh):
                            dot += qs[t][h * dh + i] * ks[j][g * dh + i]
                        sc.append(dot / math.sqrt(dh))
                    mx = max(sc)
                    e = [math.exp(s - mx) for s in sc]
                    tot = sum(e)
                    for i in range(dh):
                        acc = 0.0
                        for j in range(t + 1):
                            acc += e[j] / tot * vs[j][g * dh + i]
                        o.append(acc)
                a = _matvec(model.lw(l, lane, "wo"), o)
                for i in range(dl):
                    xs[t][lo + i] += a[i]
                y = _norm(xs[t][lo:lo + dl], model.lw(l, lane, "ffn_norm"), m.rms_eps)
                gt = _matvec(model.lw(l, lane, "w_gate"), y)
                up = _matvec(model.lw(l, lane, "w_up"), y)
                hh = [gv / (1.0 + math.exp(-gv)) * uv for gv, uv in zip(gt, up)]
                mo = _matvec(model.lw(l, lane, "w_down"), hh)
                for i in range(dl):
                    xs[t][lo + i] += mo[i]
                    u_l[t][lo + i] = a[i] + mo[i]
        us.append(u_l)
    if m.n_lanes > 1:
        for i in range(max(0, m.n_layers - m.lane_delay), m.n_layers):
            M = model.t[f"layers.{i}.mix"]
            for t in range(T):
                add = _matvec(M, us[i][t])
                xs[t] = [a + b for a, b in zip(xs[t], add)]
    out = []
    for t in range(T):
        y = _norm(xs[t], model.t["final_norm"], m.rms_eps)
        out.append(_matvec(model.t["lm_head"], y))
    return np.array(out), [list(x) for x in xs]
