"""CPU oracle for the dense Qwen3-class forward pass — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this module. The library never does, and this module
imports nothing from the library: it receives plain numpy arrays.

What it computes, and where the pages say so:

* "Failed Star (fs)" README, "How it's built": Qwen3-0.6B is a dense model with
  GQA, RoPE, SwiGLU and RMSNorm; the bf16 weights are widened for a clear fp32
  CPU oracle ("Status").
* "Milestones", M2 (Forward pass -> logits): embeddings, N transformer blocks
  (RMSNorm, RoPE, attention, SwiGLU), final norm, logits.
* "Coming back to Failed Star", "Second sitting": a Linear stored ``[out,in]``
  maps ``[S,in]`` to ``[S,out]``; the shape legend (H=1024, 16 q heads, 8 KV
  heads, d=128, so 16*128 = 2048 != H); the data-flow figure: ids -> embedding
  -> blocks -> final norm -> only the last row is projected to logits[V].
* "Coming back to Failed Star", "Next: one complete deterministic generation
  arc": greedy selection is the argmax of the finite logits with the lowest id
  winning an exact tie; stop reasons EOS / budget / context; the first loop
  recomputes the growing prefix (``generate_greedy(..., cached=False)``).
* "Milestones", M4 (KV cache): cache K/V per layer; cached and uncached
  outputs agree.
* "ferrite", "What it does": rotate-half RoPE convention; Q8_0 among the
  dequantised formats (32 int8 codes + one fp16 scale per block).

Precision: every value is fp64. The only roundings are the ones the method
makes on purpose: weights arrive as bf16 (or Q8_0) and are widened exactly;
K and V are rounded to bf16 when they enter the cache (the cache is bf16), in
both the cached and the uncached mode, so the two modes agree exactly.

Readings taken where the pages are silent (each is also checked by a test):
RMSNorm is ``x / sqrt(mean(x^2) + eps) * g``; q/k RMSNorm (over head_dim) comes
before RoPE; RoPE pairs (i, i + d/2) with inv_freq_i = theta^(-2i/d), angles in
fp64; q head h reads kv head ``h // (n_q / n_kv)``; scores are scaled by
1/sqrt(d) with key j visible to query i iff j <= i; no biases; SwiGLU is
``silu(gate) * up``.

Parity pins: tests/test_oracle_pins.py checks every function here against
closed forms, invariants, independent formulations, brute force and the
Qwen3 implementation in ``transformers``.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

# --------------------------------------------------------------------------
# Number formats


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp64.

    A bf16 value is the upper half of an fp32 word ("Failed Star (fs)" README,
    "Status": the bf16 weights are widened for the fp32 CPU oracle).
    """
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value, ties to even, returned as fp64.

    The value is first rounded to fp32 (round-to-nearest-even), then its low 16
    bits are rounded away, again to nearest with ties to the even neighbour.
    """
    f32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f32.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def q8_0_dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Q8_0 blocks to weights: w = q * s ("ferrite", "What it does": Q8_0).

    ``codes`` is int8 ``[N, K]``; ``scales`` is fp16 ``[N, K/32]`` and scale
    ``scales[n, b]`` applies to ``codes[n, 32*b : 32*b+32]``. The product of an
    8-bit integer and an 11-bit fp16 significand is exact in fp32 and fp64.
    """
    codes = np.asarray(codes, dtype=np.int8)
    scales = np.asarray(scales, dtype=np.float16)
    n, k = codes.shape
    if k % 32 or scales.shape != (n, k // 32):
        raise ValueError("Q8_0 needs [N,K] codes and [N,K/32] scales")
    return codes.astype(np.float64) * np.repeat(scales.astype(np.float64), 32, axis=1)


# --------------------------------------------------------------------------
# The pieces of one block


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g.

    "Milestones", M2: each block and the final norm use RMSNorm.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope_cos_sin(positions: np.ndarray, head_dim: int, theta: float):
    """cos/sin tables [len(positions), head_dim/2] for rotary embedding.

    Frequency i (0 <= i < d/2) is theta^(-2i/d); the angle is position times
    frequency, all in fp64.
    """
    half = head_dim // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE ("ferrite", "What it does"): pairs (i, i + d/2).

    ``x`` is ``[S, heads, d]``; ``cos``/``sin`` are ``[S, d/2]``.
    """
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention_probs(q_h: np.ndarray, k_g: np.ndarray, q_pos: np.ndarray,
                    k_pos: np.ndarray) -> np.ndarray:
    """Causal softmax(q k^T / sqrt(d)) for one head: [S, C]; hidden keys get 0."""
    d = q_h.shape[-1]
    scores = (q_h @ k_g.T) / math.sqrt(d)
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    scores = np.where(visible, scores, -np.inf)
    m = scores.max(axis=1, keepdims=True)
    p = np.exp(scores - m)
    return p / p.sum(axis=1, keepdims=True)


def causal_gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                         q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Grouped-query causal attention.

    ``q`` [S, n_q, d]; ``k``, ``v`` [C, n_kv, d]; query head h reads kv head
    h // (n_q / n_kv) ("Coming back to Failed Star": 16 query heads share 8 KV
    heads). Returns [S, n_q, d].
    """
    S, n_q, d = q.shape
    n_kv = k.shape[1]
    if n_q % n_kv:
        raise ValueError("n_q must be a multiple of n_kv")
    group = n_q // n_kv
    out = np.empty((S, n_q, d), dtype=np.float64)
    for h in range(n_q):
        g = h // group
        p = attention_probs(q[:, h, :], k[:, g, :], q_pos, k_pos)
        out[:, h, :] = p @ v[:, g, :]
    return out


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def greedy_select(logits: np.ndarray) -> int:
    """Argmax of the finite logits; the lowest id wins an exact tie.

    "Coming back to Failed Star", "Next: one complete deterministic generation
    arc", Selection. No softmax is needed to rank logits.
    """
    logits = np.asarray(logits, dtype=np.float64)
    finite = np.isfinite(logits)
    if not finite.any():
        raise ValueError("no finite logit")
    vals = np.where(finite, logits, -np.inf)
    return int(np.flatnonzero(vals == vals.max())[0])


# --------------------------------------------------------------------------
# The model


_LINEARS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")
_NORMS = ("attn_norm", "ffn_norm", "q_norm", "k_norm")


def expected_shapes(cfg) -> dict:
    """The tensor set a tied dense Qwen3-class config implies (names -> shapes)."""
    H, I, d = cfg.hidden, cfg.ffn, cfg.head_dim
    qd, kvd = cfg.n_q_heads * d, cfg.n_kv_heads * d
    layer = {"wq": (qd, H), "wk": (kvd, H), "wv": (kvd, H), "wo": (H, qd),
             "wg": (I, H), "wu": (I, H), "wd": (H, I),
             "attn_norm": (H,), "ffn_norm": (H,), "q_norm": (d,), "k_norm": (d,)}
    return {"embed": (cfg.vocab, H), "final_norm": (H,), "layer": layer}


def parameter_count(cfg) -> int:
    """Logical parameters of the tied model: the embedding is the LM head too."""
    shapes = expected_shapes(cfg)
    per_layer = sum(int(np.prod(s)) for s in shapes["layer"].values())
    return (int(np.prod(shapes["embed"])) + cfg.n_layers * per_layer
            + int(np.prod(shapes["final_norm"])))


@dataclasses.dataclass
class KVCache:
    """Flat per-layer cache of one sequence: K and V as bf16 values (fp64 arrays)."""

    k: list
    v: list

    @property
    def length(self) -> int:
        return self.k[0].shape[0]


def _widen_linear(w) -> np.ndarray:
    if isinstance(w, tuple):
        return q8_0_dequant(*w)
    return bf16_bits_to_f64(w)


class Qwen3Oracle:
    """Dense Qwen3-class decoder with a tied LM head, evaluated in fp64.

    ``cfg`` is any object with ``n_layers, hidden, n_q_heads, n_kv_heads,
    head_dim, ffn, vocab, rms_eps, rope_theta, max_pos``. ``weights`` is
    ``{"embed": uint16 [V,H], "final_norm": uint16 [H], "layers": [dict]}``
    with bf16 tensors as uint16 bit patterns and a Q8_0 linear as a
    ``(int8 codes [N,K], float16 scales [N,K/32])`` pair.

    ``kv_bf16=False`` keeps K/V unrounded (only for comparing with an fp64
    library implementation that has no bf16 cache).

    ``dtype=np.float32`` evaluates the same steps in fp32 arithmetic (weights
    widened exactly, K/V still rounded to bf16): an emulation of an ideal
    fp32 implementation, used only to measure how much of a GPU's deviation
    any fp32 forward would show. The oracle proper is fp64.
    """

    def __init__(self, cfg, weights: dict, kv_bf16: bool = True, dtype=np.float64):
        self.cfg = cfg
        self.kv_bf16 = kv_bf16
        self.dtype = np.dtype(dtype)
        shapes = expected_shapes(cfg)
        self.embed = bf16_bits_to_f64(weights["embed"]).astype(self.dtype)
        if self.embed.shape != shapes["embed"]:
            raise ValueError(f"embed shape {self.embed.shape} != {shapes['embed']}")
        self.final_norm = bf16_bits_to_f64(weights["final_norm"]).astype(self.dtype)
        self.layers = []
        for lw in weights["layers"]:
            layer = {}
            for name in _LINEARS:
                layer[name] = _widen_linear(lw[name]).astype(self.dtype)
            for name in _NORMS:
                layer[name] = bf16_bits_to_f64(lw[name]).astype(self.dtype)
            for name, s in shapes["layer"].items():
                if layer[name].shape != s:
                    raise ValueError(f"{name} shape {layer[name].shape} != {s}")
            self.layers.append(layer)
        if len(self.layers) != cfg.n_layers:
            raise ValueError("layer count does not match the config")

    def new_cache(self) -> KVCache:
        c = self.cfg
        z = np.zeros((0, c.n_kv_heads, c.head_dim), dtype=self.dtype)
        return KVCache(k=[z.copy() for _ in range(c.n_layers)],
                       v=[z.copy() for _ in range(c.n_layers)])

    def forward(self, tokens, cache: KVCache | None = None, all_logits: bool = False):
        """Run ``tokens`` at positions cache.length, cache.length+1, ...

        Appends their K/V to ``cache`` (a fresh cache if None) and returns
        ``(logits, hidden, cache)``: ``logits`` of the last row, fp64 [V] (or
        of every row, [S, V], with ``all_logits``); ``hidden`` the residual
        stream before block 0 and after each block, [L+1, S, H].
        """
        c = self.cfg
        tokens = np.asarray(tokens, dtype=np.int64)
        if tokens.ndim != 1 or tokens.size == 0:
            raise ValueError("need a non-empty 1-D token list")
        if tokens.min() < 0 or tokens.max() >= c.vocab:
            raise ValueError("token id out of range")
        cache = self.new_cache() if cache is None else cache
        S, p0 = tokens.size, cache.length
        if p0 + S > c.max_pos:
            raise ValueError("context exhausted")
        pos = np.arange(p0, p0 + S)
        x = self.embed[tokens]
        hidden = [x.copy()]
        for l in range(len(self.layers)):
            x = self.block(l, x, pos, cache)
            hidden.append(x.copy())
        rows = x if all_logits else x[-1:]
        logits = rms_norm(rows, self.final_norm, c.rms_eps) @ self.embed.T
        return (logits if all_logits else logits[0]), np.stack(hidden), cache

    def block(self, l: int, x: np.ndarray, pos: np.ndarray, cache: KVCache) -> np.ndarray:
        """Block ``l`` on rows ``x`` [S, H] at positions ``pos`` (consecutive,
        starting at cache.length): appends the rows' K/V to layer l of the
        cache and returns the block output. "Coming back to Failed Star",
        "Second sitting": RMSNorm in both residual halves; "Milestones", M2."""
        c, W, dt = self.cfg, self.layers[l], self.dtype
        S = x.shape[0]
        d, nq, nkv = c.head_dim, c.n_q_heads, c.n_kv_heads
        cos, sin = rope_cos_sin(pos, d, c.rope_theta)
        cos, sin = cos.astype(dt), sin.astype(dt)
        xn = rms_norm(x, W["attn_norm"], c.rms_eps)
        q = (xn @ W["wq"].T).reshape(S, nq, d)
        k = (xn @ W["wk"].T).reshape(S, nkv, d)
        v = (xn @ W["wv"].T).reshape(S, nkv, d)
        q = apply_rope(rms_norm(q, W["q_norm"], c.rms_eps), cos, sin)
        k = apply_rope(rms_norm(k, W["k_norm"], c.rms_eps), cos, sin)
        if self.kv_bf16:
            k, v = round_to_bf16(k).astype(dt), round_to_bf16(v).astype(dt)
        cache.k[l] = np.concatenate([cache.k[l], k], axis=0)
        cache.v[l] = np.concatenate([cache.v[l], v], axis=0)
        o = causal_gqa_attention(q, cache.k[l], cache.v[l], pos,
                                 np.arange(cache.k[l].shape[0])).astype(dt)
        x = x + o.reshape(S, nq * d) @ W["wo"].T
        xn = rms_norm(x, W["ffn_norm"], c.rms_eps)
        a = silu(xn @ W["wg"].T) * (xn @ W["wu"].T)
        return x + a @ W["wd"].T

    def logits_uncached(self, tokens) -> np.ndarray:
        """Last-row logits recomputed from scratch over the whole prefix."""
        return self.forward(tokens)[0]


STOP_EOS, STOP_BUDGET, STOP_CONTEXT = "eos", "budget", "context"


def generate_greedy(oracle: Qwen3Oracle, prompt, max_new: int, eos_ids=(),
                    max_context: int | None = None, cached: bool = True,
                    forced=None):
    """Greedy continuation under the stop contract of "Coming back to Failed
    Star", "Next: one complete deterministic generation arc".

    * no implicit BOS; an empty prompt is an error; ``max_new`` may be 0, in
      which case nothing is run and the reason is ``budget``;
    * each step selects ``greedy_select(logits)`` and appends it;
    * ``eos``: the selected id is in ``eos_ids`` — it is included in the
      returned ids; ``budget``: ``max_new`` ids produced; ``context``: the next
      forward would need a position >= ``max_context`` (the prediction of the
      last allowed forward is still returned). Checked in that order.
    * ``cached=False`` recomputes the growing prefix at every step (the first
      generation loop of the pages); ``cached=True`` runs one token per step.
    * ``forced``: optional list of ids to append instead of the selection at
      each step (teacher forcing), so a caller can follow another run's tokens.

    Returns ``(ids, reason, logits_per_step)``.
    """
    prompt = [int(t) for t in prompt]
    if not prompt:
        raise ValueError("empty prompt")
    limit = oracle.cfg.max_pos if max_context is None else min(max_context, oracle.cfg.max_pos)
    if len(prompt) > limit:
        raise ValueError("prompt longer than the context")
    ids, logits_seen = [], []
    if max_new <= 0:
        return ids, STOP_BUDGET, logits_seen
    eos = set(int(e) for e in eos_ids)
    cache = None
    prefix = list(prompt)
    step_input = list(prompt)
    while True:
        if cached:
            logits, _, cache = oracle.forward(step_input, cache)
        else:
            logits = oracle.logits_uncached(prefix)
        logits_seen.append(logits)
        tok = greedy_select(logits)
        if forced is not None and len(ids) < len(forced):
            tok = int(forced[len(ids)])
        ids.append(tok)
        if tok in eos:
            return ids, STOP_EOS, logits_seen
        if len(ids) >= max_new:
            return ids, STOP_BUDGET, logits_seen
        if len(prefix) + 1 > limit:
            return ids, STOP_CONTEXT, logits_seen
        prefix.append(tok)
        step_input = [tok]
