"""Pins of the oracle's sampler (temperature, top-k, top-p, inverse-CDF draw).

The expected token counts are closed forms: for logits z = log(a) the
softmax is a / sum(a), so over the grid u_j = (j + 1/2) / N (j < N) a token
of probability p_i is drawn exactly N p_i times whenever every cumulative
boundary N * C_i falls between grid points (all cases below are chosen so).
"""
import numpy as np
import pytest

from oracle import argmax_lowest
from oracle.sampling import kept_tokens, sample_token, sampling_margins


def counts(z, N, T, k=0, p=1.0):
    out = np.zeros(len(z), dtype=int)
    for j in range(N):
        out[sample_token(z, (j + 0.5) / N, T, k, p)] += 1
    return out.tolist()


Z123 = np.log([1.0, 2.0, 3.0])          # softmax = (1, 2, 3) / 6


@pytest.mark.parametrize("T, k, p, N, want", [
    # plain softmax: (1, 2, 3) / 6
    (1.0, 0, 1.0, 600, [100, 200, 300]),
    # T = 1/2 squares the weights: (1, 4, 9) / 14
    (0.5, 0, 1.0, 1400, [100, 400, 900]),
    # T = 2 takes square roots: weights (1, sqrt 2, sqrt 3) -- boundaries are
    # irrational, so counts are floor/ceil of N p; checked separately below
    # top-k = 2 keeps ids 2 and 1: (0, 2, 3) / 5
    (1.0, 2, 1.0, 500, [0, 200, 300]),
    # top-k = 1 is greedy
    (1.0, 1, 1.0, 100, [0, 0, 100]),
    # top-p: most probable first 3/6 = 0.5 >= 0.45 -> only id 2
    (1.0, 0, 0.45, 100, [0, 0, 100]),
    # top-p 0.55: 0.5 < 0.55 <= 5/6 -> ids 2 and 1, renormalised (0, 2, 3) / 5
    (1.0, 0, 0.55, 500, [0, 200, 300]),
    # top-p 0.9 > 5/6 -> all three
    (1.0, 0, 0.9, 600, [100, 200, 300]),
    # top-k 2 then top-p 0.65 of (2, 3) / 5: 3/5 = 0.6 < 0.65 -> both
    (1.0, 2, 0.65, 500, [0, 200, 300]),
    # top-k 2 then top-p 0.55: 0.6 >= 0.55 -> id 2 only
    (1.0, 2, 0.55, 100, [0, 0, 100]),
])
def test_closed_form_counts(T, k, p, N, want):
    assert counts(Z123, N, T, k, p) == want


def test_irrational_boundaries():
    """T = 2: weights 1, sqrt 2, sqrt 3; each count is within one of N p."""
    N = 1000
    a = np.sqrt([1.0, 2.0, 3.0])
    got = np.array(counts(Z123, N, 2.0))
    assert got.sum() == N
    assert np.all(np.abs(got - N * a / a.sum()) <= 1.0)


def test_ties_go_to_the_lower_id():
    """Three equal logits, top-k 2: ids 0 and 1 are kept, half each; the
    most probable 'first' for top-p is the lowest id too."""
    z = np.array([1.0, 1.0, 1.0, 0.0])
    assert counts(z, 200, 1.0, 2) == [100, 100, 0, 0]
    assert counts(z, 100, 1.0, 0, 0.2) == [100, 0, 0, 0]   # first kept token has 1/(3 + e^-1) > 0.2
    order, w = kept_tokens(z, 1.0, 3)
    assert order.tolist() == [0, 1, 2] and np.all(w == 1.0)


def test_greedy_limits():
    rng = np.random.default_rng(7)
    for _ in range(50):
        z = rng.normal(size=37)
        u = rng.random()
        g = argmax_lowest(z)
        assert sample_token(z, u, 0.0) == g                  # T = 0 is greedy
        assert sample_token(z, u, 0.7, 1) == g               # top-k 1
        assert sample_token(z, u, 0.7, 0, 1e-12) == g        # a vanishing nucleus
        assert sample_token(z, min(u, 1 - 1e-9), 1e-6) == g  # T -> 0


def test_shift_and_scale_invariance_and_monotone_in_u():
    rng = np.random.default_rng(11)
    for _ in range(20):
        z = rng.normal(size=64)
        T, k, p = 0.8, int(rng.integers(0, 20)), float(rng.uniform(0.3, 1.0))
        us = np.sort(rng.random(40))
        a = [sample_token(z, u, T, k, p) for u in us]
        assert a == [sample_token(z + 3.0, u, T, k, p) for u in us]
        assert a == [sample_token(2.0 * z, u, 2.0 * T, k, p) for u in us]
        assert all(x <= y for x, y in zip(a, a[1:]))         # inverse CDF in token order


def test_kept_set_is_a_prefix_of_the_descending_order():
    rng = np.random.default_rng(3)
    z = rng.normal(size=100)
    order, w = kept_tokens(z, 1.0, 10, 0.5)
    full = np.argsort(-z, kind="stable")[:10]
    assert order.tolist() == full[:order.size].tolist()
    assert w[0] == 1.0 and np.all(np.diff(w) <= 0)
    mass = np.exp(z[full] - z[full[0]])
    assert mass[:order.size].sum() >= 0.5 * mass.sum() > mass[:order.size - 1].sum()


def test_margins():
    # draw boundary: u = 0.5 with (1, 2, 3)/6 sits 1/6 from 1/3 and 0 from 1/2
    kg, cg, dg = sampling_margins(Z123, 0.5, 1.0)
    assert kg == np.inf and cg == np.inf and abs(dg) < 1e-12
    kg, cg, dg = sampling_margins(Z123, 0.4, 1.0, 2, 0.55)
    assert abs(kg - (np.log(2.0) - 0.0)) < 1e-12
    assert abs(cg - 0.05) < 1e-12          # 3/5 - 0.55
    assert abs(dg - 0.6) < 1e-12           # one kept token: its only boundary is the total, 1 - u


def test_bad_arguments():
    with pytest.raises(ValueError):
        sample_token(Z123, 1.0, 1.0)
    with pytest.raises(ValueError):
        sample_token(Z123, 0.5, -1.0)
    with pytest.raises(ValueError):
        sample_token(Z123, 0.5, 1.0, 0, 0.0)
    with pytest.raises(ValueError):
        sample_token(Z123, 0.5, 1.0, -1)
