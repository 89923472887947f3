"""Sampling beyond greedy at the LM head.  TEST INFRASTRUCTURE ONLY.

The pages put "LM-head sampling" inside the one persistent kernel (Kog
Inference Engine write-ups, "Software versus silicon" section: prefill,
decode and LM-head sampling in one go) and report greedy decoding only (the
"Laneformer 2B" results table).  They define no sampler, so this module
states the plain one that serving stacks use, in this order:

1. temperature: T > 0 scales the logits, y = z / T (T == 0 is greedy, the
   argmax with the lowest index on ties);
2. top-k: the k largest logits are kept, ties going to the lower token id
   (the argmax's tie rule); k == 0 keeps every token;
3. top-p (nucleus): of the kept tokens, taken from the most probable down
   (same order as top-k), the smallest leading set whose probability under
   softmax(y) over the top-k set reaches p; p == 1 keeps them all;
4. the draw: with a uniform u in [0, 1) supplied by the caller (the random
   number is an input, not drawn here), the kept tokens are walked in
   increasing token id and the first whose cumulative probability,
   renormalised over the kept set, exceeds u is the token (inverse CDF).

Everything is float64; the caller compares a device result at float32 with
these decisions away from their boundaries (``sampling_margins``).

Pins: ``tests/test_oracle_sampling.py`` checks closed-form token counts over
a grid of u (softmax of log 1, log 2, log 3 and its top-k / top-p / T cuts),
the tie rule, the greedy limits (k = 1, tiny p, tiny T), shift invariance and
monotonicity in u.
"""
from typing import Tuple

import numpy as np

from .decoder import argmax_lowest


def _check(u: float, temperature: float, top_k: int, top_p: float, V: int) -> None:
    if not (temperature >= 0.0) or not np.isfinite(temperature):
        raise ValueError("temperature must be finite and >= 0")
    if top_k < 0:
        raise ValueError("top_k must be >= 0")
    if not (0.0 < top_p <= 1.0):
        raise ValueError("top_p must lie in (0, 1]")
    if not (0.0 <= u < 1.0):
        raise ValueError("u must lie in [0, 1)")
    if V < 1:
        raise ValueError("empty logits")


def descending_order(z: np.ndarray) -> np.ndarray:
    """Token ids by logit, largest first; equal logits by increasing id."""
    z = np.asarray(z, dtype=np.float64)
    return np.lexsort((np.arange(z.size), -z))


def kept_tokens(z: np.ndarray, temperature: float, top_k: int = 0, top_p: float = 1.0
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Steps 1-3: the kept token ids (most probable first) and their
    unnormalised weights exp((z - z_max) / T)."""
    z = np.asarray(z, dtype=np.float64)
    order = descending_order(z)
    if top_k > 0:
        order = order[:min(top_k, z.size)]
    zk = z[order]
    w = np.exp((zk - zk[0]) / temperature)
    if top_p < 1.0:
        c = np.cumsum(w)
        m = int(np.argmax(c >= top_p * c[-1])) + 1   # first prefix reaching p of the mass
        order, w = order[:m], w[:m]
    return order, w


def sample_token(z: np.ndarray, u: float, temperature: float, top_k: int = 0,
                 top_p: float = 1.0) -> int:
    """The sampled token of logits z for the uniform u (steps 1-4)."""
    z = np.asarray(z, dtype=np.float64)
    _check(u, temperature, top_k, top_p, z.size)
    if temperature == 0.0:
        return argmax_lowest(z)
    order, w = kept_tokens(z, temperature, top_k, top_p)
    by_id = np.argsort(order, kind="stable")
    ids, wi = order[by_id], w[by_id]
    c = np.cumsum(wi)
    j = int(np.argmax(c > u * c[-1]))
    return int(ids[j])


def sampling_margins(z: np.ndarray, u: float, temperature: float, top_k: int = 0,
                     top_p: float = 1.0) -> Tuple[float, float, float]:
    """How far each decision of ``sample_token`` is from flipping:
    (top-k gap: the k-th largest logit minus the next one, inf without a cut;
     top-p gap: distance of the cut's cumulative masses from p, relative to
     the top-k mass, inf without a cut;
     draw gap: distance of u from the nearest boundary of the kept tokens'
     cumulative distribution, relative to its total)."""
    z = np.asarray(z, dtype=np.float64)
    _check(u, temperature, top_k, top_p, z.size)
    if temperature == 0.0:
        return np.inf, np.inf, np.inf
    order = descending_order(z)
    topk_gap = np.inf
    if 0 < top_k < z.size:
        topk_gap = float(z[order[top_k - 1]] - z[order[top_k]])
    kk = order[:top_k] if top_k > 0 else order
    zk = z[kk]
    w = np.exp((zk - zk[0]) / temperature)
    c = np.cumsum(w)
    S = c[-1]
    cut_gap = np.inf
    if top_p < 1.0:
        m = int(np.argmax(c >= top_p * S)) + 1
        cut_gap = float(c[m - 1] - top_p * S) / S
        if m >= 2:
            cut_gap = min(cut_gap, float(top_p * S - c[m - 2]) / S)
        kk, w = kk[:m], w[:m]
    by_id = np.argsort(kk, kind="stable")
    ci = np.cumsum(w[by_id])
    draw_gap = float(np.min(np.abs(ci - u * ci[-1])) / ci[-1])
    return topk_gap, cut_gap, draw_gap
