"""Pins for the oracle's seeded sampler (oracle/sampling.py): the counter
generator against its published known-answer vectors, the filter chain
against closed forms, special cases that reduce to greedy selection or to
the plain softmax, and brute force over a grid of uniforms."""

import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle
from oracle import sampling

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(77)


def test_philox_known_answer_vectors():
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        ctr = [int(x, 16) for x in v["counter"]]
        key = [int(x, 16) for x in v["key"]]
        assert [f"{x:08x}" for x in sampling.philox4x32_10(ctr, key)] == v["out"]


def test_uniform_is_24_bits_in_unit_interval():
    us = [sampling.uniform(123, step, row) for step in range(50) for row in range(4)]
    assert all(0.0 <= u < 1.0 for u in us)
    assert all(float(np.float32(u)) == u and (u * 2 ** 24).is_integer() for u in us)
    assert len(set(us)) == len(us)
    # the 64-bit seed reaches both key words
    assert sampling.uniform(1, 0, 0) != sampling.uniform(1 + (1 << 32), 0, 0)


def test_hand_computed_five_logit_example():
    """Logits (2, 1, 0.5, 3, 1): ranking 3, 0, 1, 4, 2 (the tie 1 vs 4 goes to
    the lower id). Top-k 4 drops id 2; top-p 0.8 keeps ids 3 and 0, whose
    renormalised probabilities are sigma(1) and 1 - sigma(1) (their logits
    differ by 1 at temperature 1)."""
    logits = np.array([2.0, 1.0, 0.5, 3.0, 1.0])
    assert sampling.ranking(logits).tolist() == [3, 0, 1, 4, 2]
    ids, probs = sampling.filtered_distribution(logits, 1.0, 4, 1.0)
    assert ids.tolist() == [3, 0, 1, 4]
    e = np.exp([3.0, 2.0, 1.0, 1.0])
    np.testing.assert_allclose(probs, e / e.sum(), rtol=1e-15)
    ids, probs = sampling.filtered_distribution(logits, 1.0, 4, 0.8)
    sig = 1.0 / (1.0 + math.exp(-1.0))
    assert ids.tolist() == [3, 0]
    np.testing.assert_allclose(probs, [sig, 1.0 - sig], rtol=1e-15)
    # draw order is ascending id: id 0 owns [0, 1 - sigma(1)), id 3 the rest
    assert sampling.sample(logits, 1.0, 4, 0.8, 0.0) == 0
    assert sampling.sample(logits, 1.0, 4, 0.8, 1.0 - sig - 1e-9) == 0
    assert sampling.sample(logits, 1.0, 4, 0.8, 1.0 - sig + 1e-9) == 3
    # temperature 2: the pair's probabilities become sigma(1/2), 1 - sigma(1/2)
    ids, probs = sampling.filtered_distribution(logits, 2.0, 2, 1.0)
    np.testing.assert_allclose(probs, [1 / (1 + math.exp(-0.5)), 1 / (1 + math.exp(0.5))],
                               rtol=1e-15)


def test_top_k_one_is_greedy():
    for _ in range(20):
        logits = RNG.standard_normal(300)
        logits[RNG.integers(300)] = logits.max()  # plant an exact tie at the top
        want = oracle.greedy_select(logits)
        for u in (0.0, 0.3, 0.999):
            for t in (0.1, 1.0, 5.0):
                assert sampling.sample(logits, t, 1, 0.9, u) == want


def test_no_filters_is_the_softmax():
    logits = RNG.standard_normal(257) * 3
    for t in (0.5, 1.0, 2.0):
        for k in (0, 257, 1000):
            ids, probs = sampling.filtered_distribution(logits, t, k, 1.0)
            got = np.zeros(257)
            got[ids] = probs
            np.testing.assert_allclose(got, softmax(logits / t), rtol=1e-12, atol=1e-300)


def test_top_p_keeps_the_shortest_prefix_reaching_p():
    for _ in range(30):
        logits = RNG.standard_normal(500) * RNG.uniform(0.2, 4)
        p = RNG.uniform(0.05, 0.99)
        t = RNG.uniform(0.3, 2)
        k = int(RNG.integers(1, 600))
        full = softmax(np.sort(logits)[::-1][: min(k, 500)] / t)
        ids, probs = sampling.filtered_distribution(logits, t, k, p)
        n = ids.size
        assert full[: n].sum() >= p - 1e-12
        assert n == 1 or full[: n - 1].sum() < p
        assert abs(probs.sum() - 1.0) < 1e-12
        assert ids.tolist() == sampling.ranking(logits)[: n].tolist()


def test_draw_is_the_inverse_cdf_on_a_grid():
    """Brute force: over N evenly spaced uniforms each kept token is drawn a
    fraction of times equal to its probability within 1/N."""
    logits = np.array([0.3, -1.2, 2.0, 0.3, 1.1, -0.4])
    ids, probs = sampling.filtered_distribution(logits, 0.7, 5, 0.95)
    N = 20000
    counts = {}
    for i in range(N):
        tok = sampling.sample(logits, 0.7, 5, 0.95, (i + 0.5) / N)
        counts[tok] = counts.get(tok, 0) + 1
    assert set(counts) == set(ids.tolist())
    for tok, pr in zip(ids, probs):
        assert abs(counts[int(tok)] / N - pr) <= 1.0 / N + 1e-12


def test_temperature_scaling_invariance_and_nonfinite_logits():
    logits = RNG.standard_normal(64)
    for u in np.linspace(0, 0.99, 7):
        assert sampling.sample(logits, 0.8, 10, 0.9, u) == sampling.sample(4 * logits, 3.2, 10,
                                                                           0.9, u)
    logits[5] = np.inf
    logits[9] = np.nan
    ids, _ = sampling.filtered_distribution(logits, 1.0, 0, 1.0)
    assert 5 not in ids and 9 not in ids and ids.size == 62
    with pytest.raises(ValueError):
        sampling.filtered_distribution(logits, 0.0, 0, 1.0)
