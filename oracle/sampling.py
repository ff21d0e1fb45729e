"""Seeded sampling after the LM head — TEST INFRASTRUCTURE ONLY (see
``oracle/__init__.py``).

"Coming back to Failed Star", "Next: one complete deterministic generation
arc": after greedy parity, the next arc adds temperature, then top-k, then
top-p, as explicit filters with known-answer tests ("Failed Star / fs —
Milestones", M3 Generation: only then add temperature / top-k / top-p;
ferrite, "What it does": a sampler with temperature, top-k and top-p).

The pages fix the filters and their order but not the arithmetic; the reading
taken here:

* temperature ``T > 0`` divides the logits; ``T == 0`` is greedy selection;
* candidates are ranked by (logit descending, id ascending), which is the
  same order as probability descending with ties to the lowest id;
* top-k keeps the first ``k`` candidates of that ranking (``k >= V`` or
  ``k <= 0`` keeps all);
* top-p keeps the shortest prefix of the ranking whose softmax mass (over
  the top-k survivors, at temperature T) reaches ``p`` (at least one token;
  ``p >= 1`` keeps all survivors);
* the kept probabilities are renormalised to sum to 1;
* the draw takes a uniform ``u`` in [0, 1) and returns the first kept token,
  in ascending id order, whose cumulative renormalised probability exceeds
  ``u`` (the pages give no order for the draw; id order needs no sort of the
  kept set, which top-p alone can leave at most of the vocabulary).

The uniform comes from a counter-based generator so that the GPU and this
oracle draw the same numbers: Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), key = the 64-bit seed
(low word first), counter = (step low word, row, step high word, 0); ``u`` =
the top 24 bits of the first output word times 2^-24, exact in fp32.
"""

from __future__ import annotations

import numpy as np

_M0, _M1 = 0xD2511F53, 0xCD9E8D57   # Philox4x32 round multipliers
_W0, _W1 = 0x9E3779B9, 0xBB67AE85   # key schedule (Weyl) increments
_MASK = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """Ten rounds of Philox4x32 on a 4-word counter with a 2-word key.

    A round multiplies words 0 and 2 by the two multipliers (64-bit
    products), and forms the new words from the high halves xor-ed with the
    other words and the key, and the low halves; the key advances by the two
    Weyl increments between rounds.
    """
    c0, c1, c2, c3 = (int(x) & _MASK for x in counter)
    k0, k1 = (int(x) & _MASK for x in key)
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> 32, p0 & _MASK
        hi1, lo1 = p1 >> 32, p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def uniform(seed: int, step: int, row: int) -> float:
    """The draw's uniform in [0, 1): 24 bits of Philox4x32-10 output."""
    x = philox4x32_10((step & _MASK, row, (step >> 32) & _MASK, 0),
                      (seed & _MASK, (seed >> 32) & _MASK))[0]
    return (x >> 8) * 2.0 ** -24


def ranking(logits: np.ndarray) -> np.ndarray:
    """Token ids by logit descending, ties to the lowest id (finite logits only)."""
    logits = np.asarray(logits, dtype=np.float64)
    ids = np.flatnonzero(np.isfinite(logits))
    order = np.lexsort((ids, -logits[ids]))
    return ids[order]


def filtered_distribution(logits, temperature: float, top_k: int, top_p: float):
    """(kept ids in ranking order, their renormalised probabilities)."""
    logits = np.asarray(logits, dtype=np.float64)
    if temperature <= 0:
        raise ValueError("temperature 0 is greedy selection; use greedy_select")
    ranked = ranking(logits)
    if ranked.size == 0:
        raise ValueError("no finite logit")
    if 0 < top_k < ranked.size:
        ranked = ranked[:top_k]
    z = logits[ranked] / temperature
    w = np.exp(z - z[0])
    probs = w / w.sum()
    if top_p < 1.0:
        cum = np.cumsum(probs)
        n = int(np.searchsorted(cum, top_p, side="left")) + 1
        ranked, probs = ranked[:n], probs[:n]
        probs = probs / probs.sum()
    return ranked, probs


def draw(ids: np.ndarray, probs: np.ndarray, u: float) -> int:
    """The first id, in ascending id order, whose cumulative probability exceeds u."""
    order = np.argsort(ids, kind="stable")
    ids, probs = ids[order], probs[order]
    cum = np.cumsum(probs)
    i = int(np.searchsorted(cum, u, side="right"))
    return int(ids[min(i, ids.size - 1)])


def sample(logits, temperature: float, top_k: int, top_p: float, u: float) -> int:
    """Temperature -> top-k -> top-p -> renormalise -> draw with uniform u."""
    ids, probs = filtered_distribution(logits, temperature, top_k, top_p)
    return draw(ids, probs, u)
